"""pa_attn_chunks_noalloc: multi-chunk attention that allocates nothing.

Some callers cannot allocate device memory on the call path (a fixed budget
under a framework's allocator, loops that cannot afford cudaMalloc's
device-wide synchronisation, plug-ins handed only their inputs and outputs).
For them the library keeps the per-chunk partial results in one static
device array instead of buffers someone allocates.  These tests call that
entry point through the C ABI and hold its output both against the fp64
oracle over the unchunked keys and against the existing entry points
(pa_attn_fwd per chunk into caller-allocated partials, then pa_attn_merge),
within the parity tolerances, on two calls in a row with different inputs:
the shared array still holds the first call's partials when the second call
runs.  A larger call followed by a smaller one with a different chunk count
checks that stale partials at other offsets are never read, and one case goes
through the Python binding with caller-supplied outputs.  A shape whose
partials do not fit is refused.

This file is collected last, so a run that stops at the first failure has
already run every other test.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

LIMIT_BYTES = 32 << 20


@pytest.fixture(scope="module")
def pa():
    from context_blocks_b200 import build
    build.build()
    import context_blocks_b200 as pa_mod
    pa_mod.load_library()
    return pa_mod


def _noalloc_c_abi(pa, q, k_chunks, v_chunks, scale):
    """One call of the C entry point; host arrays of chunk pointers/lengths."""
    lib = pa.load_library()
    B, H, Nq, d = q.shape
    n = len(k_chunks)
    kp = (ctypes.c_void_p * n)(*[k.data_ptr() for k in k_chunks])
    vp = (ctypes.c_void_p * n)(*[v.data_ptr() for v in v_chunks])
    nk = (ctypes.c_int * n)(*[k.shape[2] for k in k_chunks])
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=q.device)
    rc = lib.pa_attn_chunks_noalloc(q.data_ptr(), kp, vp, nk, n, o.data_ptr(), lse.data_ptr(), B, H, Nq, d,
                                    float(scale), torch.cuda.current_stream().cuda_stream)
    return rc, o, lse


def _existing(pa, q, k_chunks, v_chunks, scale):
    o, lse = pa.blockwise_attention(q, list(k_chunks), list(v_chunks), scale=scale)
    return o, lse


def _check_against_existing(pa, w, seed):
    q, k, v = workloads.make_case(w, device="cuda", seed=seed)
    pairs = workloads.split_keys(k, v, w.chunks)
    kc, vc = [p[0] for p in pairs], [p[1] for p in pairs]
    o_ex, l_ex = _existing(pa, q, kc, vc, w.scale)
    rc, o, lse = _noalloc_c_abi(pa, q, kc, vc, w.scale)
    assert rc == pa.PA_OK, pa.last_error()
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    assert_close(o, lse, o_ex.float().cpu().double().numpy(), l_ex.cpu().double().numpy(),
                 f"no-alloc vs existing entry points ({w.name}, seed {seed})")
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_close(o, lse, o_ref, l_ref, f"no-alloc vs oracle over all keys ({w.name}, seed {seed})")
    return o, lse


def test_noalloc_matches_existing_entry_points_two_calls_in_a_row(pa):
    w = workloads.get("ring")        # 4 chunks; partials 28.8 MB, inside the 32 MiB array
    o1, _ = _check_against_existing(pa, w, seed=101)
    o2, _ = _check_against_existing(pa, w, seed=202)
    assert not torch.equal(o1, o2)   # the second call really computed new values


def test_noalloc_uneven_chunks_head_dim_64(pa):
    w = workloads.Workload("noalloc64", B=2, H=3, Nq=300, Nk=517, d=64, rms_qk=False,
                           chunks=(200, 1, 316), seed=7)
    _check_against_existing(pa, w, seed=7)
    _check_against_existing(pa, w, seed=8)


def test_noalloc_larger_call_then_smaller_call(pa):
    """8 chunks fill most of the array; then 3 chunks of another shape place
    their partials at other offsets, over what the first call left."""
    big = workloads.Workload("noalloc_big", B=1, H=8, Nq=1000, Nk=8 * 150, d=128, rms_qk=True,
                             chunks=(150,) * 8, seed=9)
    small = workloads.Workload("noalloc_small", B=2, H=2, Nq=333, Nk=401, d=128, rms_qk=False,
                               chunks=(129, 255, 17), seed=10)
    _check_against_existing(pa, big, seed=11)
    _check_against_existing(pa, small, seed=12)
    _check_against_existing(pa, big, seed=13)


def test_noalloc_through_the_binding(pa):
    """The public binding with caller-supplied outputs, and its shape checks."""
    w = workloads.get("flux1008")
    q, k, v = workloads.make_case(w, device="cuda", seed=14)
    q = q[:, :4].contiguous()                     # 4 heads: partials fit the array
    pairs = workloads.split_keys(k[:, :4].contiguous(), v[:, :4].contiguous(), w.chunks)
    kc, vc = [p[0] for p in pairs], [p[1] for p in pairs]
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    o2, l2 = pa.attn_chunks_noalloc(q, kc, vc, scale=w.scale, out=o, lse=lse, check=True)
    assert o2.data_ptr() == o.data_ptr() and l2.data_ptr() == lse.data_ptr()
    kh = torch.cat([a.cpu() for a in kc], dim=2)
    vh = torch.cat([b.cpu() for b in vc], dim=2)
    o_ref, l_ref = oracle.attention(q.cpu(), kh, vh, w.scale)
    assert_close(o, lse, o_ref, l_ref, "no-alloc through the binding")
    with pytest.raises(ValueError):
        pa.attn_chunks_noalloc(q, kc, vc, out=torch.empty((1, 4, 7, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        pa.attn_chunks_noalloc(q, kc, vc, lse=torch.empty((1, 4, w.Nq), dtype=torch.float64, device="cuda"))


def test_noalloc_single_chunk(pa):
    w = workloads.get("tiny").with_chunks([256])
    _check_against_existing(pa, w, seed=3)


def test_noalloc_refuses_partials_beyond_the_limit(pa):
    B, H, Nq, d = 1, 1, 70000, 128
    n = 2
    need = ((n * B * H * Nq * d * 2 + 255) // 256) * 256 + n * B * H * Nq * 4
    assert need > LIMIT_BYTES
    q = torch.zeros((B, H, Nq, d), dtype=torch.bfloat16, device="cuda")
    k = [torch.zeros((B, H, 64, d), dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    v = [torch.zeros((B, H, 64, d), dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    rc, _, _ = _noalloc_c_abi(pa, q, k, v, 1.0 / math.sqrt(d))
    assert rc == pa.PA_ERR_INVALID_ARG
    assert "scratch" in pa.last_error()
