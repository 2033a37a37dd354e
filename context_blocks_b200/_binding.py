"""ctypes binding of ``libpa_attn.so`` (the C ABI in ``include/pa_attn.h``).

Argument marshalling only: tensors are checked for dtype, device, layout and
shape, their device pointers and sizes are handed to the C entry points, and
a non-zero status becomes a :class:`PaError`.  Every step of the attention
and the merge runs in the library's CUDA kernels.  There is no fallback: if
the library is missing or does not load, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libpa_attn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_MISALIGNED = -3
PA_ERR_CUDA = -4
PA_ERR_TIMEOUT = -5
PA_ERR_BAD_INPUT = -6
PA_ACCUM_FIRST = 1
PA_ACCUM_FINAL = 2

# (name, restype, argtypes) for every symbol declared in include/pa_attn.h.
_VP, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "pa_attn_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP]),
    "pa_attn_fwd_accum": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP]),
    "pa_attn_fwd_fp8": (_I, [_VP, _VP, _VP, _F, _F, _F, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP]),
    "pa_attn_fwd_fp8_dev": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP]),
    "pa_quantize_e4m3": (_I, [_VP, ctypes.c_longlong, _VP, _VP, _VP]),
    "pa_attn_fwd_chunks": (_I, [_VP, _VP, _VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _F, _VP]),
    "pa_attn_merge": (_I, [_VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _VP]),
    "pa_attn_chunks_noalloc": (_I, [_VP, _VP, _VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _F, _VP]),
    "pa_residual_diff": (_I, [_VP, _VP, ctypes.c_longlong, _VP, _VP]),
    "pa_status_string": (ctypes.c_char_p, [_I]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_poll_device_status": (_I, []),
    "pa_selftest_timeout": (_I, [_I, _VP]),
    "pa_set_wait_limit_ms": (_I, [_I]),
    "pa_version": (_I, []),
}


class PaError(RuntimeError):
    """A non-zero status from the C library."""

    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({detail})" if detail else
                         f"{where}: {status_string(code)}")


_lib = None
_lock = threading.Lock()


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (once) and return the library; raises if it is not built."""
    global _lib
    if path is None and _lib is not None:  # the common case, without the lock
        return _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m context_blocks_b200.build`")
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().pa_status_string(int(code)).decode()


def last_error() -> str:
    return load_library().pa_last_error().decode()


def version() -> int:
    return int(load_library().pa_version())


def _check(rc: int, where: str, check: bool = False) -> None:
    """Raise on a non-zero status.  With ``check`` also wait for the device
    and raise on an error the kernels recorded (a bounded wait that gave up,
    a bad value read on the device): this synchronises, so it is for
    debugging and tests, not for a hot loop."""
    if rc != PA_OK:
        raise PaError(rc, where, last_error())
    if check:
        import torch
        torch.cuda.synchronize()
        code = poll_device_status()
        if code != PA_OK:
            raise PaError(code, where, "reported by the device after the call")


_raw_stream = None  # torch's current-stream handle getter, looked up once


def _stream_handle(stream, device) -> int:
    """cudaStream_t of `stream`, or of torch's current stream on `device`."""
    global _raw_stream
    import torch
    if stream is None:
        if _raw_stream is None:
            _raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", False)
        if _raw_stream:  # the handle alone, without building a Stream object
            index = device.index if isinstance(device, torch.device) else device
            return int(_raw_stream(torch.cuda.current_device() if index is None else int(index)))
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _check_bf16(name, t, ndim):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16 (got {t.dtype})")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def attn_fwd(q, k, v, scale: Optional[float] = None, out=None, lse=None, stream=None, check: bool = False):
    """Attention of q [B,H,Nq,d] against one K/V chunk k, v [B,H,Nk,d].

    Returns (o [B,H,Nq,d] bf16, lse [B,H,Nq] fp32, natural log), written into
    ``out`` / ``lse`` when given.  ``scale`` defaults to 1/sqrt(d).
    ``check=True`` synchronises and raises on a device-side error.
    """
    _check_bf16("q", q, 4)
    _check_bf16("k", k, 4)
    _check_bf16("v", v, 4)
    B, H, Nq, d = q.shape
    kB, kH, Nk, kd = k.shape
    if kB != B or kH != H or kd != d or v.shape != k.shape:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse)
    rc = load_library().pa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     B, H, Nq, Nk, d, float(scale), _stream_handle(stream, q.device))
    _check(rc, "pa_attn_fwd", check)
    return out, lse


def attn_fwd_accum(q, k, v, o_acc, lse_acc, first: bool = False, final: bool = False, out=None,
                   scale: Optional[float] = None, stream=None, check: bool = False):
    """Fold the attention of q over one more K/V chunk into the running state
    (``pa_attn_fwd_accum``): o_acc [B,H,Nq,d] fp32 and lse_acc [B,H,Nq] fp32,
    updated in place.  ``first`` ignores their incoming contents.  With
    ``final`` the result goes to ``out`` (bf16, allocated when None) instead
    of o_acc, and that tensor is returned; otherwise o_acc is returned.
    Returns (o, lse_acc)."""
    import torch
    _check_bf16("q", q, 4)
    _check_bf16("k", k, 4)
    _check_bf16("v", v, 4)
    B, H, Nq, d = q.shape
    if k.shape[:2] != (B, H) or k.shape[3] != d or v.shape != k.shape:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    for name, t, shape in (("o_acc", o_acc, (B, H, Nq, d)), ("lse_acc", lse_acc, (B, H, Nq))):
        if (not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or tuple(t.shape) != shape
                or not t.is_contiguous() or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous float32 tensor of shape {shape} on q's device")
    if final:
        if out is None:
            out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
        else:
            _check_bf16("out", out, 4)
            if tuple(out.shape) != (B, H, Nq, d):
                raise ValueError("out must have q's shape")
    elif out is not None:
        raise ValueError("out is written only by the final fold")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    flags = (PA_ACCUM_FIRST if first else 0) | (PA_ACCUM_FINAL if final else 0)
    rc = load_library().pa_attn_fwd_accum(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_acc.data_ptr(),
                                           lse_acc.data_ptr(), out.data_ptr() if final else None, B, H, Nq,
                                           k.shape[2], d, float(scale), flags, _stream_handle(stream, q.device))
    _check(rc, "pa_attn_fwd_accum", check)
    return (out if final else o_acc), lse_acc


def attn_fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, scale: Optional[float] = None,
                 out=None, lse=None, stream=None, check: bool = False):
    """Attention over e4m3 inputs (``pa_attn_fwd_fp8``): q [B,H,Nq,128],
    k, v [B,H,Nk,128] of dtype torch.float8_e4m3fn, whose real values are the
    tensors times their scales.  Returns (o bf16, lse fp32) like attn_fwd."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float8_e4m3fn:
            raise TypeError(f"{name} must be a torch.float8_e4m3fn tensor")
        if t.device.type != "cuda" or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-d CUDA tensor")
    B, H, Nq, d = q.shape
    if k.shape[:2] != (B, H) or k.shape[3] != d or v.shape != k.shape:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse)
    scales = (q_scale, k_scale, v_scale)
    if all(isinstance(x, torch.Tensor) for x in scales):
        # device-resident scales (as pa_quantize_e4m3 writes them)
        for x in scales:
            if x.dtype != torch.float32 or x.numel() != 1 or x.device != q.device:
                raise ValueError("device scales must be one-element float32 tensors on q's device")
        rc = load_library().pa_attn_fwd_fp8_dev(q.data_ptr(), k.data_ptr(), v.data_ptr(), *[x.data_ptr() for x in scales],
                                                out.data_ptr(), lse.data_ptr(), B, H, Nq, k.shape[2], d, float(scale),
                                                _stream_handle(stream, q.device))
        _check(rc, "pa_attn_fwd_fp8_dev", check)
        return out, lse
    rc = load_library().pa_attn_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_scale), float(k_scale),
                                        float(v_scale), out.data_ptr(), lse.data_ptr(), B, H, Nq, k.shape[2], d,
                                        float(scale), _stream_handle(stream, q.device))
    _check(rc, "pa_attn_fwd_fp8", check)
    return out, lse


def quantize_e4m3(x, out=None, scale=None, stream=None, check: bool = False):
    """Per-tensor e4m3 quantisation of a bf16 tensor on the device
    (``pa_quantize_e4m3``): returns (q torch.float8_e4m3fn of x's shape,
    scale one-element float32 device tensor) with x ~= scale * q."""
    import torch
    if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16 or x.device.type != "cuda" \
            or not x.is_contiguous():
        raise TypeError("x must be a contiguous bfloat16 CUDA tensor")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=x.device)
    elif out.dtype != torch.float8_e4m3fn or out.shape != x.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous float8_e4m3fn tensor of x's shape")
    if scale is None:
        scale = torch.empty((1,), dtype=torch.float32, device=x.device)
    elif scale.dtype != torch.float32 or scale.numel() != 1:
        raise ValueError("scale must be a one-element float32 tensor")
    rc = load_library().pa_quantize_e4m3(x.data_ptr(), x.numel(), out.data_ptr(), scale.data_ptr(),
                                         _stream_handle(stream, x.device))
    _check(rc, "pa_quantize_e4m3", check)
    return out, scale


def residual_diff(cur, prev, out=None, stream=None, check: bool = False):
    """First Block Cache's residual difference (``pa_residual_diff``):
    sum |cur - prev| / sum |prev| over two bf16 CUDA tensors of the same
    shape, as a one-element float32 device tensor (no host synchronisation;
    compare it with the threshold on the device or read it when needed)."""
    import torch
    for name, t in (("cur", cur), ("prev", prev)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.device.type != "cuda" \
                or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous bfloat16 CUDA tensor")
    if cur.shape != prev.shape:
        raise ValueError(f"shape mismatch: cur {tuple(cur.shape)}, prev {tuple(prev.shape)}")
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=cur.device)
    elif out.dtype != torch.float32 or out.numel() != 1 or out.device != cur.device:
        raise ValueError("out must be a one-element float32 tensor on cur's device")
    rc = load_library().pa_residual_diff(cur.data_ptr(), prev.data_ptr(), cur.numel(), out.data_ptr(),
                                         _stream_handle(stream, cur.device))
    _check(rc, "pa_residual_diff", check)
    return out


def attn_merge(o_parts, lse_parts, out=None, lse=None, stream=None, check: bool = False):
    """Merge n partial results o_parts [n,B,H,N,d] bf16, lse_parts [n,B,H,N]
    fp32 (over disjoint key chunks) into (o [B,H,N,d], lse [B,H,N])."""
    import torch
    _check_bf16("o_parts", o_parts, 5)
    n, B, H, N, d = o_parts.shape
    if (lse_parts.dtype != torch.float32 or tuple(lse_parts.shape) != (n, B, H, N)
            or not lse_parts.is_contiguous() or lse_parts.device != o_parts.device):
        raise ValueError("lse_parts must be a contiguous float32 [n,B,H,N] tensor on o_parts' device")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=o_parts.device)
    else:
        _check_bf16("out", out, 4)
        if tuple(out.shape) != (B, H, N, d):
            raise ValueError(f"out must be [B,H,N,d] = {(B, H, N, d)} (got {tuple(out.shape)})")
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=o_parts.device)
    elif lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B,H,N] tensor")
    rc = load_library().pa_attn_merge(o_parts.data_ptr(), lse_parts.data_ptr(), n, out.data_ptr(),
                                      lse.data_ptr(), B, H, N, d,
                                      _stream_handle(stream, o_parts.device))
    _check(rc, "pa_attn_merge", check)
    return out, lse


def _outputs(q, out, lse):
    """(out, lse) for a query tensor q [B,H,Nq,d]: allocated when None,
    otherwise checked for dtype, shape and layout."""
    import torch
    B, H, Nq, d = q.shape
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    else:
        _check_bf16("out", out, 4)
        if tuple(out.shape) != (B, H, Nq, d):
            raise ValueError("out must have q's shape")
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    elif lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Nq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B,H,Nq] tensor")
    return out, lse


def _chunk_arrays(q, k_chunks, v_chunks):
    B, H, Nq, d = q.shape
    n = len(k_chunks)
    if n < 1 or len(v_chunks) != n:
        raise ValueError("need at least one chunk and as many V chunks as K chunks")
    for kc, vc in zip(k_chunks, v_chunks):
        _check_bf16("k chunk", kc, 4)
        _check_bf16("v chunk", vc, 4)
        if kc.shape != vc.shape or kc.shape[:2] != (B, H) or kc.shape[3] != d:
            raise ValueError("chunk shapes must be [B, H, n_c, d] matching q")
    kp = (ctypes.c_void_p * n)(*[kc.data_ptr() for kc in k_chunks])
    vp = (ctypes.c_void_p * n)(*[vc.data_ptr() for vc in v_chunks])
    nk = (ctypes.c_int * n)(*[kc.shape[2] for kc in k_chunks])
    return kp, vp, nk, n


def attn_fwd_chunks(q, k_chunks, v_chunks, scale: Optional[float] = None, out=None, lse=None, stream=None,
                    check: bool = False):
    """Attention of q over the concatenation of the K/V chunks (up to 8) in a
    single launch (``pa_attn_fwd_chunks``); no partial results are written."""
    _check_bf16("q", q, 4)
    B, H, Nq, d = q.shape
    kp, vp, nk, n = _chunk_arrays(q, k_chunks, v_chunks)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse)
    rc = load_library().pa_attn_fwd_chunks(q.data_ptr(), kp, vp, nk, n, out.data_ptr(), lse.data_ptr(),
                                           B, H, Nq, d, float(scale), _stream_handle(stream, q.device))
    _check(rc, "pa_attn_fwd_chunks", check)
    return out, lse


def attn_chunks_noalloc(q, k_chunks, v_chunks, scale: Optional[float] = None, out=None, lse=None, stream=None,
                        check: bool = False):
    """Attention of q over the concatenation of the K/V chunks through
    ``pa_attn_chunks_noalloc``: the library keeps the per-chunk partials in
    its fixed static array instead of allocating them (see the header for the
    size limit and the sharing rules).  Outputs are allocated here only when
    not given."""
    _check_bf16("q", q, 4)
    B, H, Nq, d = q.shape
    kp, vp, nk, n = _chunk_arrays(q, k_chunks, v_chunks)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out, lse = _outputs(q, out, lse)
    rc = load_library().pa_attn_chunks_noalloc(q.data_ptr(), kp, vp, nk, n, out.data_ptr(), lse.data_ptr(),
                                               B, H, Nq, d, float(scale), _stream_handle(stream, q.device))
    _check(rc, "pa_attn_chunks_noalloc", check)
    return out, lse


def poll_device_status() -> int:
    """Read and clear the device status word (synchronising).  Returns the
    status code (0 = no device-side error since the last poll)."""
    return int(load_library().pa_poll_device_status())


def set_wait_limit_ms(ms: int) -> None:
    """Limit of every device-side barrier wait for later launches
    (``pa_set_wait_limit_ms``; default 5000 ms)."""
    _check(load_library().pa_set_wait_limit_ms(int(ms)), "pa_set_wait_limit_ms")


def selftest_timeout(limit_us: int, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see pa_selftest_timeout)."""
    import torch
    rc = load_library().pa_selftest_timeout(int(limit_us),
                                            _stream_handle(stream, torch.cuda.current_device()))
    _check(rc, "pa_selftest_timeout")
