"""Seeded random sweep of small shapes through every bf16 entry point,
against the fp64 oracle over the unchunked key sequence.

Each case draws B, H, Nq, Nk (at least 64), d and a split of the keys into
1..6 chunks (ragged, possibly of a single key), so that query rows end inside a warp's
32 rows and inside a 128-row tile, key tiles end anywhere inside a chunk, and
chunk boundaries fall inside tiles.  The same case runs through

* pa_attn_fwd per chunk + pa_attn_merge (blockwise_attention),
* pa_attn_fwd_chunks (one launch over all chunks, when there are at most 8),
* pa_attn_fwd_accum folds into an fp32 running state, and
* pa_attn_chunks_noalloc,

each held to the same bounds as the fixed parity tests.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests._parity import assert_close

pytestmark = pytest.mark.gpu

CASES = 24


@pytest.fixture(scope="module")
def pa():
    from context_blocks_b200 import build
    build.build()
    import context_blocks_b200 as pa_mod
    pa_mod.load_library()
    return pa_mod


def _case(i):
    r = np.random.default_rng(4242 + i)
    B = int(r.integers(1, 3))
    H = int(r.integers(1, 4))
    Nq = int(r.choice([int(r.integers(1, 40)), int(r.integers(100, 300)), int(r.integers(250, 700))]))
    n_chunks = int(r.integers(1, 7))
    sizes = [int(x) for x in r.integers(1, 400, size=n_chunks)]
    if r.random() < 0.3:
        sizes[int(r.integers(0, n_chunks))] = 1
    # At least 64 keys in all: with only a handful of keys |o| is about 1 and
    # the absolute bars sit at bf16's own rounding of O (the fixed edge-shape
    # tests cover those sequences deterministically).
    if sum(sizes) < 64:
        sizes[-1] += 64 - sum(sizes)
    d = int(r.choice([64, 128]))
    return B, H, Nq, sizes, d, int(r.integers(0, 2**31))


@pytest.mark.parametrize("i", range(CASES))
def test_random_shape(pa, i):
    B, H, Nq, sizes, d, seed = _case(i)
    Nk = sum(sizes)
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda").to(torch.bfloat16)
    ks = [t.contiguous() for t in torch.split(k, sizes, dim=2)]
    vs = [t.contiguous() for t in torch.split(v, sizes, dim=2)]
    scale = 1.0 / math.sqrt(d)
    what = f"B={B} H={H} Nq={Nq} chunks={sizes} d={d}"
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)

    o, lse = pa.blockwise_attention(q, ks, vs, scale=scale)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    assert_close(o, lse, o_ref, l_ref, f"random per-chunk + merge, {what}")

    if len(sizes) <= 8:
        o, lse = pa.attn_fwd_chunks(q, ks, vs, scale=scale)
        torch.cuda.synchronize()
        assert_close(o, lse, o_ref, l_ref, f"random fused, {what}")

    o_acc = torch.full((B, H, Nq, d), float("nan"), dtype=torch.float32, device="cuda")
    lse_acc = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device="cuda")
    for c in range(len(sizes)):
        last = c == len(sizes) - 1
        o, lse = pa.attn_fwd_accum(q, ks[c], vs[c], o_acc, lse_acc, first=(c == 0), final=last, scale=scale)
    torch.cuda.synchronize()
    assert_close(o, lse, o_ref, l_ref, f"random folds, {what}")

    o, lse = pa.attn_chunks_noalloc(q, ks, vs, scale=scale)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    assert_close(o, lse, o_ref, l_ref, f"random no-alloc, {what}")


def _fp8_case(i):
    r = np.random.default_rng(9090 + i)
    return (int(r.integers(1, 3)), int(r.integers(1, 4)), int(r.integers(1, 700)), int(r.integers(64, 1500)),
            int(r.integers(0, 2**31)))


@pytest.mark.parametrize("i", range(8))
def test_random_shape_e4m3(pa, i):
    """The e4m3 forward on random shapes, with the scales made on the device
    by the library's quantiser (pa_attn_fwd_fp8_dev) and given on the host
    (pa_attn_fwd_fp8): both against the oracle on the dequantised codes, with
    the e4m3 bounds."""
    from tests._parity import assert_close_fp8
    B, H, Nq, Nk, seed = _fp8_case(i)
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, H, Nq, 128), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, H, Nk, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, H, Nk, 128), generator=g, device="cuda").to(torch.bfloat16)
    (q8, sq), (k8, sk), (v8, sv) = pa.quantize_e4m3(q), pa.quantize_e4m3(k), pa.quantize_e4m3(v)
    scale = 1.0 / math.sqrt(128)
    o_dev, l_dev = pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=scale)
    o_host, l_host = pa.attn_fwd_fp8(q8, k8, v8, float(sq.item()), float(sk.item()), float(sv.item()), scale=scale)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    deq = [x.cpu().double() * float(s.item()) for x, s in ((q8, sq), (k8, sk), (v8, sv))]
    o_ref, l_ref = oracle.attention(deq[0], deq[1], deq[2], scale)
    what = f"e4m3 B={B} H={H} Nq={Nq} Nk={Nk}"
    v_max = float(deq[2].abs().max())
    assert_close_fp8(o_dev, l_dev, o_ref, l_ref, v_max, f"random {what}, device scales")
    assert_close_fp8(o_host, l_host, o_ref, l_ref, v_max, f"random {what}, host scales")
