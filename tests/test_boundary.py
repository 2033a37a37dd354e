"""The C ABI on the host: the library builds, loads, exports every symbol of
include/pa_attn.h, and rejects bad arguments with the documented codes.

Every call here returns before any CUDA API is touched (argument checks come
first), so this file runs on a machine without a GPU.
"""

import ctypes
import os
import re

import pytest

from context_blocks_b200 import _binding as B
from context_blocks_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa_attn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_expected_api():
    names = _declared_functions()
    assert "pa_attn_fwd" in names and "pa_attn_merge" in names
    assert names == sorted(B.SIGNATURES), (names, sorted(B.SIGNATURES))


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_codes_match_header():
    text = open(HEADER).read()
    codes = {m.group(1): int(m.group(2)) for m in
             re.finditer(r"#define\s+(PA_\w+)\s+\(?(-?\d+)\)?", text)}
    for name in ("PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_MISALIGNED",
                 "PA_ERR_CUDA", "PA_ERR_TIMEOUT", "PA_ERR_BAD_INPUT", "PA_ACCUM_FIRST", "PA_ACCUM_FINAL"):
        assert codes[name] == getattr(B, name), name


def test_status_strings(lib):
    assert B.status_string(0) == "PA_OK"
    for code in (-1, -2, -3, -4, -5, -6):
        assert B.status_string(code).startswith("PA_ERR_")
    assert B.status_string(12345) == "unknown status code"
    assert B.version() == 200


def test_wait_limit_setter(lib):
    assert lib.pa_set_wait_limit_ms(0) == B.PA_ERR_INVALID_ARG
    assert lib.pa_set_wait_limit_ms(600001) == B.PA_ERR_INVALID_ARG
    assert lib.pa_set_wait_limit_ms(5000) == B.PA_OK


A = 1 << 20          # a 16-byte aligned fake address; never dereferenced
MB = 1 << 24


def _fwd(lib, q=A, k=A + MB, v=A + 2 * MB, o=A + 3 * MB, lse=A + 4 * MB, Bn=1, H=1, Nq=8, Nk=8,
         d=128, scale=0.125):
    return lib.pa_attn_fwd(q, k, v, o, lse, Bn, H, Nq, Nk, d, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), B.PA_ERR_INVALID_ARG), (dict(k=0), B.PA_ERR_INVALID_ARG),
    (dict(v=0), B.PA_ERR_INVALID_ARG), (dict(o=0), B.PA_ERR_INVALID_ARG),
    (dict(lse=0), B.PA_ERR_INVALID_ARG),
    (dict(Bn=0), B.PA_ERR_INVALID_ARG), (dict(H=-1), B.PA_ERR_INVALID_ARG),
    (dict(Nq=-1), B.PA_ERR_INVALID_ARG), (dict(Nk=0), B.PA_ERR_INVALID_ARG),
    (dict(scale=0.0), B.PA_ERR_INVALID_ARG), (dict(scale=-1.0), B.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.PA_ERR_INVALID_ARG), (dict(scale=float("inf")), B.PA_ERR_INVALID_ARG),
    (dict(d=96), B.PA_ERR_UNSUPPORTED), (dict(d=256), B.PA_ERR_UNSUPPORTED),
    (dict(Bn=256, H=256), B.PA_ERR_UNSUPPORTED),
    (dict(q=A + 8), B.PA_ERR_MISALIGNED), (dict(o=A + 3 * MB + 4), B.PA_ERR_MISALIGNED),
    (dict(lse=A + 4 * MB + 2), B.PA_ERR_MISALIGNED),
    (dict(o=A), B.PA_ERR_INVALID_ARG),                        # o aliases q
    (dict(lse=A + MB + 64), B.PA_ERR_INVALID_ARG),            # lse inside k
    (dict(lse=A + 3 * MB + 16), B.PA_ERR_INVALID_ARG),        # lse inside o
])
def test_fwd_argument_checks(lib, kw, code):
    assert _fwd(lib, **kw) == code
    assert B.last_error() != ""


def test_fwd_empty_query_is_noop(lib):
    assert _fwd(lib, Nq=0) == B.PA_OK


def _merge(lib, op=A, lp=A + 8 * MB, n=2, o=A + 12 * MB, lse=A + 14 * MB, Bn=1, H=2, N=16, d=64):
    return lib.pa_attn_merge(op, lp, n, o, lse, Bn, H, N, d, None)


@pytest.mark.parametrize("kw,code", [
    (dict(op=0), B.PA_ERR_INVALID_ARG), (dict(lp=0), B.PA_ERR_INVALID_ARG),
    (dict(o=0), B.PA_ERR_INVALID_ARG), (dict(lse=0), B.PA_ERR_INVALID_ARG),
    (dict(n=0), B.PA_ERR_INVALID_ARG), (dict(Bn=0), B.PA_ERR_INVALID_ARG),
    (dict(N=-3), B.PA_ERR_INVALID_ARG), (dict(d=32), B.PA_ERR_UNSUPPORTED),
    (dict(op=A + 4), B.PA_ERR_MISALIGNED), (dict(lse=A + 14 * MB + 1), B.PA_ERR_MISALIGNED),
    (dict(o=A + 64), B.PA_ERR_INVALID_ARG),                   # o inside o_parts
])
def test_merge_argument_checks(lib, kw, code):
    assert _merge(lib, **kw) == code


def test_merge_empty_is_noop(lib):
    assert _merge(lib, N=0) == B.PA_OK


def test_selftest_limit_checked_first(lib):
    assert lib.pa_selftest_timeout(0, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_selftest_timeout(2_000_000, None) == B.PA_ERR_INVALID_ARG


def test_python_binding_type_checks():
    import torch
    q = torch.zeros((1, 1, 4, 64), dtype=torch.float32)
    with pytest.raises(TypeError):
        B.attn_fwd(q, q, q)
    qb = q.to(torch.bfloat16)
    with pytest.raises(ValueError):
        B.attn_fwd(qb, qb, qb)          # host tensors are refused before the library


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        B.load_library(str(tmp_path / "nope.so"))


def test_build_flags_target_sm100a():
    assert "arch=compute_100a,code=sm_100a" in build_mod.NVCC_FLAGS


def _accum(lib, q=A, k=A + MB, v=A + 2 * MB, oacc=A + 5 * MB, lacc=A + 4 * MB, o=0, Nq=8, Nk=8, d=128,
           flags=0):
    return lib.pa_attn_fwd_accum(q, k, v, oacc, lacc, o or None, 1, 1, Nq, Nk, d, 0.125, flags, None)


def test_accum_argument_checks(lib):
    assert _accum(lib, q=0) == B.PA_ERR_INVALID_ARG
    assert _accum(lib, oacc=0) == B.PA_ERR_INVALID_ARG
    assert _accum(lib, flags=4) == B.PA_ERR_INVALID_ARG                       # unknown flag
    assert _accum(lib, flags=B.PA_ACCUM_FINAL) == B.PA_ERR_INVALID_ARG        # final fold without o
    assert _accum(lib, o=A + 3 * MB) == B.PA_ERR_INVALID_ARG                  # o without the final fold
    assert _accum(lib, d=96) == B.PA_ERR_UNSUPPORTED
    assert _accum(lib, oacc=A + 5 * MB + 8) == B.PA_ERR_MISALIGNED
    assert _accum(lib, oacc=A + 2 * MB + 64) == B.PA_ERR_INVALID_ARG          # state inside v
    # the fp32 state is 4 bytes per element: 8 rows x 128 x 4 = 4 KB past o_acc
    assert _accum(lib, lacc=A + 5 * MB + 4096 - 4) == B.PA_ERR_INVALID_ARG
    assert _accum(lib, o=A + 5 * MB + 1024, flags=B.PA_ACCUM_FINAL) == B.PA_ERR_INVALID_ARG  # o inside the state
    assert _accum(lib, Nq=0, flags=B.PA_ACCUM_FIRST) == B.PA_OK


def _chunks(lib, n=3, nk=(8, 8, 8), kaddr=None, Nq=8, d=128, q=A, o=A + 3 * MB, lse=A + 4 * MB):
    kaddr = kaddr or [A + MB + c * 4096 for c in range(n)]
    kp = (ctypes.c_void_p * max(n, 1))(*kaddr[:n])
    vp = (ctypes.c_void_p * max(n, 1))(*[A + 2 * MB + c * 4096 for c in range(n)])
    nkp = (ctypes.c_int * max(n, 1))(*nk[:n])
    return lib.pa_attn_fwd_chunks(q, kp, vp, nkp, n, o, lse, 1, 1, Nq, d, 0.125, None)


def test_fwd_chunks_argument_checks(lib):
    assert lib.pa_attn_fwd_chunks(A, None, None, None, 1, A + 3 * MB, A + 4 * MB, 1, 1, 8, 128, 0.1,
                                  None) == B.PA_ERR_INVALID_ARG
    assert _chunks(lib, n=0) == B.PA_ERR_INVALID_ARG
    assert _chunks(lib, n=9, nk=(8,) * 9, kaddr=[A + MB + c * 4096 for c in range(9)]) == B.PA_ERR_INVALID_ARG
    assert "n_chunks" in B.last_error()
    assert _chunks(lib, nk=(8, 0, 8)) == B.PA_ERR_INVALID_ARG          # an empty chunk
    assert _chunks(lib, kaddr=[A + MB, A + MB + 4104, A + MB + 8192]) == B.PA_ERR_MISALIGNED
    assert _chunks(lib, kaddr=[A + MB, 0, A + MB + 8192]) == B.PA_ERR_INVALID_ARG
    assert _chunks(lib, d=96) == B.PA_ERR_UNSUPPORTED
    assert _chunks(lib, o=A + MB + 4096) == B.PA_ERR_INVALID_ARG         # o overlaps a K chunk
    assert _chunks(lib, Nq=0) == B.PA_OK                                 # empty query: nothing to do


def test_fwd_fp8_argument_checks(lib):
    f = lib.pa_attn_fwd_fp8
    args = lambda **kw: dict(dict(q=A, k=A + MB, v=A + 2 * MB, sq=1.0, sk=1.0, sv=1.0, o=A + 3 * MB,
                                  lse=A + 4 * MB, Nq=8, Nk=8, d=128), **kw)
    call = lambda a: f(a["q"], a["k"], a["v"], a["sq"], a["sk"], a["sv"], a["o"], a["lse"], 1, 1, a["Nq"],
                       a["Nk"], a["d"], 0.125, None)
    assert call(args(q=0)) == B.PA_ERR_INVALID_ARG
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert call(args(sq=bad)) == B.PA_ERR_INVALID_ARG
        assert call(args(sv=bad)) == B.PA_ERR_INVALID_ARG
    assert call(args(d=64)) == B.PA_ERR_UNSUPPORTED
    assert "d = 128" in B.last_error()
    assert call(args(k=A + MB + 8)) == B.PA_ERR_MISALIGNED
    assert call(args(o=A + 512)) == B.PA_ERR_INVALID_ARG          # o overlaps q (1 KB of e4m3)
    assert call(args(Nq=0)) == B.PA_OK


def test_output_checks_refuse_wrong_shapes(monkeypatch):
    # The C ABI cannot see buffer sizes, so the binding refuses outputs of the
    # wrong shape before any launch.  _check_bf16's device test is relaxed so
    # that CPU tensors stand in for device ones here.
    import torch
    monkeypatch.setattr(B, "_check_bf16", lambda name, t, ndim: None)
    q = torch.zeros((1, 2, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B._outputs(q, torch.zeros((1, 2, 7, 64), dtype=torch.bfloat16), None)
    with pytest.raises(ValueError):
        B._outputs(q, None, torch.zeros((1, 2, 8), dtype=torch.float64))
    o, l = B._outputs(q, None, None)
    assert tuple(o.shape) == (1, 2, 8, 64) and tuple(l.shape) == (1, 2, 8)


def test_quantize_and_fp8_dev_argument_checks(lib):
    qz = lib.pa_quantize_e4m3
    assert qz(0, 16, A + MB, A + 2 * MB, None) == B.PA_ERR_INVALID_ARG
    assert qz(A, 0, A + MB, A + 2 * MB, None) == B.PA_ERR_INVALID_ARG
    assert qz(A + 8, 16, A + MB, A + 2 * MB, None) == B.PA_ERR_MISALIGNED
    assert qz(A, 16, A + MB, A + 2 * MB + 2, None) == B.PA_ERR_MISALIGNED
    assert qz(A, 1024, A + 1024, A + 2 * MB, None) == B.PA_ERR_INVALID_ARG     # q overlaps x (2 KB)
    f = lib.pa_attn_fwd_fp8_dev
    ok = dict(q=A, k=A + MB, v=A + 2 * MB, sq=A + 5 * MB, sk=A + 5 * MB + 4, sv=A + 5 * MB + 8)
    call = lambda **kw: f(*[dict(ok, **kw)[n] for n in ("q", "k", "v", "sq", "sk", "sv")], A + 3 * MB, A + 4 * MB,
                          1, 1, 8, 8, kw.get("d", 128), 0.125, None)
    assert call(sk=0) == B.PA_ERR_INVALID_ARG
    assert call(sv=A + 5 * MB + 9) == B.PA_ERR_MISALIGNED
    assert call(d=64) == B.PA_ERR_UNSUPPORTED


def test_residual_diff_argument_checks(lib):
    rd = lib.pa_residual_diff
    assert rd(0, A + MB, 16, A + 2 * MB, None) == B.PA_ERR_INVALID_ARG
    assert rd(A, A + MB, 0, A + 2 * MB, None) == B.PA_ERR_INVALID_ARG
    assert rd(A + 8, A + MB, 16, A + 2 * MB, None) == B.PA_ERR_MISALIGNED
    assert rd(A, A + MB, 16, A + 2 * MB + 2, None) == B.PA_ERR_MISALIGNED
    assert rd(A, A + MB, 1024, A + 64, None) == B.PA_ERR_INVALID_ARG     # out inside cur (2 KB)


def test_plain_c_caller(lib, tmp_path):
    """A C program compiled with gcc against the header and linked to the
    library gets the documented status codes (no Python in between)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = os.path.join(ROOT, "tests", "c", "abi_smoke.c")
    exe = str(tmp_path / "abi_smoke")
    libdir = os.path.dirname(B.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-O1", f"-I{os.path.join(ROOT, 'include')}", src,
                        "-o", exe, f"-L{libdir}", "-l:libpa_attn.so", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "C ABI checks passed" in r.stdout
