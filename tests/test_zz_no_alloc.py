"""pa_attn_chunks_noalloc: multi-chunk attention that allocates nothing.

Some callers cannot allocate device memory on the call path (a fixed budget
under a framework's allocator, loops that cannot afford cudaMalloc's
device-wide synchronisation, plug-ins handed only their inputs and outputs).
For them the library keeps the per-chunk partial results in one static
device array instead of buffers someone allocates.  These tests call that
entry point through the C ABI and hold its output against the existing entry
points (pa_attn_fwd per chunk into caller-allocated partials, then
pa_attn_merge), within the parity tolerances, on two calls in a row with
different inputs: the shared array still holds the first call's partials when
the second call runs.  A shape whose partials do not fit is refused.

This file is collected last, so a run that stops at the first failure has
already run every other test.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

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
    o_ref, l_ref = _existing(pa, q, kc, vc, w.scale)
    rc, o, lse = _noalloc_c_abi(pa, q, kc, vc, w.scale)
    assert rc == pa.PA_OK, pa.last_error()
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    assert_close(o, lse, o_ref.float().cpu().double().numpy(), l_ref.cpu().double().numpy(),
                 f"no-alloc vs existing entry points ({w.name}, seed {seed})")
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
