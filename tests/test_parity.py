"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Every case draws seeded inputs from ``workloads``, runs ``pa_attn_fwd`` /
``pa_attn_merge`` through the Python binding, and compares element by element
with the oracle on the same bf16 values.  Chunked cases are compared twice:
each partial against the oracle over that chunk alone, and the merged result
against the oracle over the whole, unchunked key sequence (the ring-attention
claim: block-by-block attention combined is exact; diffusers "Context
parallelism", section "Ring Attention").
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_close, assert_close_fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from context_blocks_b200 import build
    build.build()
    import context_blocks_b200 as pa_mod
    pa_mod.load_library()
    return pa_mod


def _run_chunks(pa, q, k, v, chunks, scale):
    pairs = workloads.split_keys(k, v, chunks)
    n = len(pairs)
    B, H, Nq, d = q.shape
    o_parts = torch.full((n, B, H, Nq, d), float("nan"), dtype=torch.bfloat16, device=q.device)
    lse_parts = torch.full((n, B, H, Nq), float("nan"), dtype=torch.float32, device=q.device)
    o, lse = pa.blockwise_attention(q, [p[0] for p in pairs], [p[1] for p in pairs], scale=scale,
                                    o_parts=o_parts if n > 1 else None,
                                    lse_parts=lse_parts if n > 1 else None)
    torch.cuda.synchronize()
    return o, lse, o_parts, lse_parts


def _check_workload(pa, w, rows=None, check_parts=True):
    q, k, v = workloads.make_case(w, device="cuda")
    o, lse, o_parts, lse_parts = _run_chunks(pa, q, k, v, w.chunks, w.scale)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    if rows is None:
        o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale)
        assert_close(o, lse, o_ref, l_ref, f"{w.name} merged vs unchunked oracle")
    else:
        o_ref, l_ref = oracle.attention_rows(qh, kh, vh, w.scale, rows)
        assert_close(o[:, :, rows], lse[:, :, rows], o_ref, l_ref, f"{w.name} sampled rows")
    if check_parts and len(w.chunks) > 1:
        s = 0
        for p, c in enumerate(w.chunks):
            kc, vc = kh[:, :, s:s + c], vh[:, :, s:s + c]
            if rows is None:
                po, pl = oracle.attention(qh, kc, vc, w.scale)
                assert_close(o_parts[p], lse_parts[p], po, pl, f"{w.name} part {p}")
            else:
                po, pl = oracle.attention_rows(qh, kc, vc, w.scale, rows)
                assert_close(o_parts[p][:, :, rows], lse_parts[p][:, :, rows], po, pl,
                             f"{w.name} part {p} sampled rows")
            s += c
    assert pa.poll_device_status() == pa.PA_OK


# ---------------------------------------------------------------- workloads

def test_tiny(pa):
    _check_workload(pa, workloads.get("tiny"))


def test_tiny_single_chunk(pa):
    _check_workload(pa, workloads.get("tiny").with_chunks([256]))


def test_flux(pa):
    _check_workload(pa, workloads.get("flux"))


def test_ring_step(pa):
    _check_workload(pa, workloads.get("ring"))


def test_uneven_tails(pa):
    _check_workload(pa, workloads.get("tails"))


def test_uneven_tails_single_chunk(pa):
    w = workloads.get("tails")
    _check_workload(pa, w.with_chunks([w.Nk]))


def _hunyuan_rows(w):
    rows = workloads.sample_rows(w.Nq, 256, seed=w.seed)
    tail = np.arange((w.Nq // 128) * 128, w.Nq)          # the final partial query tile
    return np.unique(np.concatenate([rows, tail]))


@pytest.mark.slow
def test_hunyuan_single_chunk(pa):
    w = workloads.get("hunyuan")
    _check_workload(pa, w, rows=_hunyuan_rows(w))


@pytest.mark.slow
def test_hunyuan_eight_chunks(pa):
    w = workloads.get("hunyuan").with_chunks(workloads.HUNYUAN_CHUNKS8)
    _check_workload(pa, w, rows=_hunyuan_rows(w), check_parts=False)


# ---------------------------------------------------------------- edge shapes

EDGE = [
    # B, H, Nq, Nk, d
    (1, 1, 1, 1, 64), (1, 1, 1, 1, 128), (1, 1, 2, 2, 128), (1, 3, 127, 129, 128),
    (2, 1, 129, 127, 64), (1, 2, 255, 1, 128), (1, 2, 1, 255, 128), (1, 1, 256, 256, 128),
    (1, 1, 257, 383, 128), (2, 3, 300, 130, 64), (1, 1, 128, 128, 64), (1, 2, 513, 1000, 128),
    (3, 2, 100, 4097, 128), (1, 1, 640, 17, 64),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d", EDGE)
def test_edge_shapes(pa, B, H, Nq, Nk, d):
    g = torch.Generator(device="cuda").manual_seed(1000 + Nq * 7 + Nk * 13 + d)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda").to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), device="cuda")
    pa.attn_fwd(q, k, v, scale=scale, out=o, lse=lse)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)
    assert_close(o, lse, o_ref, l_ref, f"edge {(B, H, Nq, Nk, d)}")


def test_rescale_path_rising_logits(pa):
    """Logits that rise by far more than the lazy-rescale threshold from one
    key tile to the next, so every tile moves the reference maximum."""
    B, H, Nq, Nk, d = 1, 2, 200, 1100, 128
    g = torch.Generator(device="cuda").manual_seed(77)
    q = (torch.randn((B, H, Nq, d), generator=g, device="cuda") * 0.2 + 1.0)
    ramp = torch.linspace(0.0, 1.0, Nk, device="cuda")[None, None, :, None]
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda") * 0.1 + ramp * 6.0
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda")
    q, k, v = (x.to(torch.bfloat16).contiguous() for x in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    o, lse = pa.attn_fwd(q, k, v, scale=scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)
    assert float(np.max(l_ref)) > 60.0          # large logits really were reached
    assert_close(o, lse, o_ref, l_ref, "rising logits")


def test_falling_logits(pa):
    B, H, Nq, Nk, d = 1, 2, 130, 900, 64
    g = torch.Generator(device="cuda").manual_seed(78)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda") * 0.2 + 1.0
    ramp = torch.linspace(1.0, 0.0, Nk, device="cuda")[None, None, :, None]
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda") * 0.1 + ramp * 5.0
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda")
    q, k, v = (x.to(torch.bfloat16).contiguous() for x in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    o, lse = pa.attn_fwd(q, k, v, scale=scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)
    assert_close(o, lse, o_ref, l_ref, "falling logits")


def test_constant_v_closed_form(pa):
    """Constant V: every output row equals that constant (bf16 exactly)."""
    B, H, Nq, Nk, d = 1, 2, 300, 700, 128
    g = torch.Generator(device="cuda").manual_seed(79)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda").to(torch.bfloat16)
    row = torch.randn((d,), generator=g, device="cuda").to(torch.bfloat16)
    v = row.expand(B, H, Nk, d).contiguous()
    o, _ = pa.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    err = (o.float() - row.float()).abs().max().item()
    assert err <= 2 ** -7 * row.float().abs().max().item(), err


# ---------------------------------------------------------------- robustness

def test_no_reads_past_chunk_and_no_writes_past_outputs(pa):
    """K/V chunks followed in memory by NaN garbage, outputs surrounded by
    canaries: results must match, garbage must not leak, canaries intact."""
    B, H, Nq, Nk, d = 1, 2, 200, 333, 128
    g = torch.Generator(device="cuda").manual_seed(80)
    n_in = B * H * Nk * d
    pad = 128 * d * 4
    kbuf = torch.full((n_in + pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    vbuf = torch.full((n_in + pad,), float("nan"), dtype=torch.bfloat16, device="cuda")
    k = kbuf[:n_in].view(B, H, Nk, d)
    v = vbuf[:n_in].view(B, H, Nk, d)
    k.copy_(torch.randn((B, H, Nk, d), generator=g, device="cuda"))
    v.copy_(torch.randn((B, H, Nk, d), generator=g, device="cuda"))
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda").to(torch.bfloat16)
    n_out = B * H * Nq * d
    guard = 4096
    obuf = torch.full((guard + n_out + guard,), 1234.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((guard + B * H * Nq + guard,), -4321.0, dtype=torch.float32, device="cuda")
    o = obuf[guard:guard + n_out].view(B, H, Nq, d)
    lse = lbuf[guard:guard + B * H * Nq].view(B, H, Nq)
    pa.attn_fwd(q, k, v, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(obuf[:guard] == 1234.0) and torch.all(obuf[guard + n_out:] == 1234.0)
    assert torch.all(lbuf[:guard] == -4321.0) and torch.all(lbuf[guard + B * H * Nq:] == -4321.0)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), 1.0 / math.sqrt(d))
    assert_close(o, lse, o_ref, l_ref, "garbage past chunk")


def test_outputs_fully_written(pa):
    w = workloads.get("tails")
    q, k, v = workloads.make_case(w, device="cuda")
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    pa.attn_fwd(q, k[:, :, :1151].contiguous(), v[:, :, :1151].contiguous(), out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_deterministic(pa):
    w = workloads.get("ring")
    q, k, v = workloads.make_case(w, device="cuda")
    o1, l1 = pa.attn_fwd(q, k, v)
    o2, l2 = pa.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ---------------------------------------------------------------- merge

@pytest.mark.parametrize("n,d", [(1, 128), (2, 64), (3, 128), (8, 128), (5, 64)])
def test_merge_vs_oracle(pa, n, d):
    B, H, N = 2, 3, 517
    g = torch.Generator(device="cuda").manual_seed(90 + n)
    # Partial outputs are convex combinations of V rows, so their entries are
    # far below |v| ~ 1 (about 1/sqrt(chunk length)); draw them at that
    # scale.  At |o| ~ 4 the bf16 rounding of the output alone (2^-9
    # relative) would exceed the 1e-2 absolute bar.
    o_parts = (torch.randn((n, B, H, N, d), generator=g, device="cuda") * 0.1).to(torch.bfloat16)
    lse_parts = torch.randn((n, B, H, N), generator=g, device="cuda") * 4.0 + 10.0
    o, lse = pa.attn_merge(o_parts, lse_parts)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.merge(o_parts.cpu(), lse_parts.cpu())
    assert_close(o, lse, o_ref, l_ref, f"merge n={n} d={d}")


def test_merge_single_part_is_exact_copy(pa):
    g = torch.Generator(device="cuda").manual_seed(95)
    o_parts = torch.randn((1, 1, 2, 300, 128), generator=g, device="cuda").to(torch.bfloat16)
    lse_parts = torch.randn((1, 1, 2, 300), generator=g, device="cuda")
    o, lse = pa.attn_merge(o_parts, lse_parts)
    torch.cuda.synchronize()
    assert torch.equal(o, o_parts[0])
    assert torch.allclose(lse, lse_parts[0], rtol=0, atol=1e-6)


def test_merge_neg_inf_parts(pa):
    """-inf parts carry no weight and their (NaN) rows are never read; an
    all -inf row gives o = 0, lse = -inf."""
    n, B, H, N, d = 3, 1, 2, 260, 128
    g = torch.Generator(device="cuda").manual_seed(96)
    o_parts = torch.randn((n, B, H, N, d), generator=g, device="cuda").to(torch.bfloat16)
    lse_parts = torch.randn((n, B, H, N), generator=g, device="cuda")
    o_parts[1] = float("nan")
    lse_parts[1] = float("-inf")
    lse_parts[:, :, :, :7] = float("-inf")     # seven rows with every part empty
    o, lse = pa.attn_merge(o_parts, lse_parts)
    torch.cuda.synchronize()
    assert torch.all(o[:, :, :7] == 0) and torch.all(torch.isneginf(lse[:, :, :7]))
    keep = [0, 2]
    o_ref, l_ref = oracle.merge(o_parts[keep].cpu(), lse_parts[keep].cpu())
    assert_close(o, lse, o_ref, l_ref, "merge with -inf parts")


# ---------------------------------------------------------------- failure path

def test_host_pointer_is_rejected_not_faulted(pa):
    q = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16)           # host memory
    k, v, o = (torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    lse = torch.zeros((1, 1, 8), device="cuda")
    lib = pa.load_library()
    rc = lib.pa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                         lse.data_ptr(), 1, 1, 8, 8, 128, 0.1, None)
    assert rc == pa.PA_ERR_INVALID_ARG
    assert "not device memory" in pa.last_error()


def test_bounded_wait_times_out_and_reports(pa):
    assert pa.poll_device_status() == pa.PA_OK
    pa.selftest_timeout(2000)          # a wait that nothing completes, limited to 2 ms
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_ERR_TIMEOUT
    assert pa.poll_device_status() == pa.PA_OK      # polling clears the word
    # the context is still usable
    w = workloads.get("tiny")
    q, k, v = workloads.make_case(w, device="cuda")
    o, lse = pa.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_close(o, lse, o_ref, l_ref, "after timeout self-test")
    assert pa.poll_device_status() == pa.PA_OK


# ---------------------------------------------------------------- fused chunks

def _fused_check(pa, w, rows=None):
    """pa_attn_fwd_chunks over the workload's chunks vs the oracle over all keys."""
    q, k, v = workloads.make_case(w, device="cuda")
    pairs = workloads.split_keys(k, v, w.chunks)
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    pa.attn_fwd_chunks(q, [a for a, _ in pairs], [b for _, b in pairs], scale=w.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    if rows is None:
        o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale)
        assert_close(o, lse, o_ref, l_ref, f"fused chunks {w.name}")
    else:
        o_ref, l_ref = oracle.attention_rows(qh, kh, vh, w.scale, rows)
        assert_close(o[:, :, rows], lse[:, :, rows], o_ref, l_ref, f"fused chunks {w.name} sampled rows")
    return q, pairs, o, lse


def test_fused_ring_step(pa):
    w = workloads.get("ring")
    q, pairs, o, lse = _fused_check(pa, w)
    # same values as one forward per chunk followed by the merge
    o2, l2 = pa.blockwise_attention(q, [a for a, _ in pairs], [b for _, b in pairs], scale=w.scale)
    torch.cuda.synchronize()
    # the per-chunk path rounds each partial O to bf16 before the merge; the
    # fused launch rounds once, so the two differ by a few bf16 half-ulps at most
    assert (o.float() - o2.float()).abs().max().item() <= 1e-2
    assert (lse - l2).abs().max().item() <= 1e-3


def test_fused_uneven_tails(pa):
    _fused_check(pa, workloads.get("tails"))


def test_fused_tiny_head_dim_64(pa):
    _fused_check(pa, workloads.get("tiny"))


def test_fused_ragged_and_single_key_chunks(pa):
    w = workloads.Workload("ragged", B=1, H=2, Nq=300, Nk=260, d=128, rms_qk=False,
                           chunks=(1, 128, 3, 127, 1), seed=31)
    _fused_check(pa, w)


def test_fused_eight_chunks_of_one_tile(pa):
    w = workloads.Workload("eight", B=1, H=2, Nq=257, Nk=8 * 128, d=128, rms_qk=True,
                           chunks=(128,) * 8, seed=32)
    _fused_check(pa, w)


@pytest.mark.slow
def test_fused_hunyuan_eight_chunks(pa):
    w = workloads.get("hunyuan").with_chunks(workloads.HUNYUAN_CHUNKS8)
    _fused_check(pa, w, rows=_hunyuan_rows(w))


def test_flux_1008_ring_anything(pa):
    # per-chunk forward + merge, and the same chunks in one fused launch
    w = workloads.get("flux1008")
    _check_workload(pa, w)
    _fused_check(pa, w)


def test_fused_rejects_more_than_eight_chunks(pa):
    q = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    ks = [torch.zeros((1, 1, 4, 128), dtype=torch.bfloat16, device="cuda") for _ in range(9)]
    with pytest.raises(pa.PaError) as e:
        pa.attn_fwd_chunks(q, ks, [x.clone() for x in ks])
    assert e.value.code == pa.PA_ERR_INVALID_ARG


# ---------------------------------------------------------------- e4m3 inputs

def _quantize_e4m3(x):
    """Per-tensor scaled e4m3: returns (x8, scale) with x ~= x8 * scale."""
    amax = float(x.float().abs().max())
    scale = max(amax, 1e-12) / 448.0
    return (x.float() / scale).to(torch.float8_e4m3fn).contiguous(), scale


def _dequant(x8, scale):
    return x8.cpu().double() * scale


def _fp8_check(pa, q, k, v, scale, what, rows=None):
    (q8, sq), (k8, sk), (v8, sv) = _quantize_e4m3(q), _quantize_e4m3(k), _quantize_e4m3(v)
    o = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    qd, kd, vd = _dequant(q8, sq), _dequant(k8, sk), _dequant(v8, sv)
    v_max = float(vd.abs().max())
    if rows is None:
        o_ref, l_ref = oracle.attention(qd, kd, vd, scale)
        return assert_close_fp8(o, lse, o_ref, l_ref, v_max, what)
    o_ref, l_ref = oracle.attention_rows(qd, kd, vd, scale, rows)
    return assert_close_fp8(o[:, :, rows], lse[:, :, rows], o_ref, l_ref, v_max, what)


def test_fp8_flux(pa):
    w = workloads.get("flux")
    q, k, v = workloads.make_case(w, device="cuda")
    _fp8_check(pa, q, k, v, w.scale, "fp8 flux")


def test_fp8_ragged_shapes(pa):
    for (B, H, Nq, Nk) in [(1, 2, 300, 517), (2, 1, 1, 1), (1, 1, 129, 255), (1, 3, 256, 4097)]:
        w = workloads.Workload("fp8edge", B=B, H=H, Nq=Nq, Nk=Nk, d=128, rms_qk=True, chunks=(Nk,), seed=40 + Nk)
        q, k, v = workloads.make_case(w, device="cuda")
        _fp8_check(pa, q, k, v, w.scale, f"fp8 edge {(B, H, Nq, Nk)}")


def test_fp8_rising_logits(pa):
    B, H, Nq, Nk, d = 1, 2, 200, 1100, 128
    g = torch.Generator(device="cuda").manual_seed(79)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda") * 0.2 + 1.0
    ramp = torch.linspace(0.0, 1.0, Nk, device="cuda")[None, None, :, None]
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda") * 0.1 + ramp * 6.0
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda")
    _fp8_check(pa, q, k, v, 1.0 / math.sqrt(d), "fp8 rising logits")


def test_fp8_scales_apply(pa):
    # the same e4m3 codes with scales (2, 0.5, 3) equal scales (1, 1, 1) on
    # inputs multiplied out: logits unchanged, output times 3
    w = workloads.Workload("fp8s", B=1, H=2, Nq=256, Nk=384, d=128, rms_qk=True, chunks=(384,), seed=51)
    q, k, v = workloads.make_case(w, device="cuda")
    (q8, _), (k8, _), (v8, _) = _quantize_e4m3(q), _quantize_e4m3(k), _quantize_e4m3(v)
    o1, l1 = pa.attn_fwd_fp8(q8, k8, v8, 1.0, 1.0, 1.0, scale=w.scale)
    o2, l2 = pa.attn_fwd_fp8(q8, k8, v8, 2.0, 0.5, 3.0, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(l1, l2)
    assert (o2.float() - 3.0 * o1.float()).abs().max().item() <= 3.0 * 2 ** -7 * o1.float().abs().max().item()


def test_merge_rejects_wrong_output_shapes(pa):
    op = torch.zeros((2, 1, 2, 16, 64), dtype=torch.bfloat16, device="cuda")
    lp = torch.zeros((2, 1, 2, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        pa.attn_merge(op, lp, out=torch.empty((1, 2, 8, 64), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        pa.attn_merge(op, lp, lse=torch.empty((1, 2, 8), dtype=torch.float32, device="cuda"))


def test_quantize_e4m3_bit_exact(pa):
    from oracle import e4m3 as E
    g = torch.Generator(device="cuda").manual_seed(61)
    for n in (1, 7, 8, 1000, 4099, 1 << 20):
        x = (torch.randn((n,), generator=g, device="cuda") * 3.0).to(torch.bfloat16)
        q8, sc = pa.quantize_e4m3(x)
        torch.cuda.synchronize()
        xs = x.float().cpu().numpy()
        s = np.float32(sc.item())
        # the scale is amax / 448 in fp32; the codes are the oracle's quantisation
        ref, s_ref = E.quantize(xs)
        assert s == s_ref, n
        got = q8.view(torch.uint8).cpu().numpy()
        assert np.array_equal(got, ref), (n, int(np.sum(got != ref)))
    z = torch.zeros((40,), dtype=torch.bfloat16, device="cuda")
    q8, sc = pa.quantize_e4m3(z)
    torch.cuda.synchronize()
    assert sc.item() == 1.0 and not q8.view(torch.uint8).any()


def test_fp8_device_scales_pipeline(pa):
    # bf16 -> pa_quantize_e4m3 -> pa_attn_fwd_fp8_dev, checked against the oracle
    # on the dequantised codes, and equal to the host-scale entry point.
    w = workloads.Workload("fp8dev", B=1, H=3, Nq=700, Nk=1300, d=128, rms_qk=True, chunks=(1300,), seed=62)
    q, k, v = workloads.make_case(w, device="cuda")
    (q8, sq), (k8, sk), (v8, sv) = pa.quantize_e4m3(q), pa.quantize_e4m3(k), pa.quantize_e4m3(v)
    o, lse = pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=w.scale)
    o2, l2 = pa.attn_fwd_fp8(q8, k8, v8, sq.item(), sk.item(), sv.item(), scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
    qd, kd, vd = (_dequant(a, float(b.item())) for a, b in ((q8, sq), (k8, sk), (v8, sv)))
    o_ref, l_ref = oracle.attention(qd, kd, vd, w.scale)
    assert_close_fp8(o, lse, o_ref, l_ref, float(vd.abs().max()), "fp8 device-scale pipeline")


def test_fp8_rejects_bf16(pa):
    q = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        pa.attn_fwd_fp8(q, q, q, 1.0, 1.0, 1.0)


# ---------------------------------------------------------------- values read on the device

def test_fp8_device_scale_that_is_not_positive_is_reported(pa):
    """A dequantisation scale read on the device that is zero, negative, Inf
    or NaN is recorded as PA_ERR_BAD_INPUT in the status word (a normal
    launch: the kernel runs to the end, its outputs are meaningless)."""
    w = workloads.Workload("badscale", B=1, H=1, Nq=128, Nk=256, d=128, rms_qk=True, chunks=(256,), seed=63)
    q, k, v = workloads.make_case(w, device="cuda")
    (q8, sq), (k8, sk), (v8, sv) = pa.quantize_e4m3(q), pa.quantize_e4m3(k), pa.quantize_e4m3(v)
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        for which in range(3):
            scales = [sq.clone(), sk.clone(), sv.clone()]
            scales[which].fill_(bad)
            pa.attn_fwd_fp8(q8, k8, v8, *scales, scale=w.scale)
            torch.cuda.synchronize()
            assert pa.poll_device_status() == pa.PA_ERR_BAD_INPUT, (bad, which)
    # good scales again: clean status, correct result
    o, lse = pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=w.scale, check=True)
    qd, kd, vd = (_dequant(a, float(b.item())) for a, b in ((q8, sq), (k8, sk), (v8, sv)))
    o_ref, l_ref = oracle.attention(qd, kd, vd, w.scale)
    assert_close_fp8(o, lse, o_ref, l_ref, float(vd.abs().max()), "fp8 after bad scales")


def test_quantize_reports_non_finite_input(pa):
    for bad in (float("inf"), float("-inf"), float("nan")):
        x = torch.randn((4099,), device="cuda").to(torch.bfloat16)
        x[1234] = bad
        pa.quantize_e4m3(x)
        torch.cuda.synchronize()
        assert pa.poll_device_status() == pa.PA_ERR_BAD_INPUT, bad
        # the binding's check option raises on the same condition
        with pytest.raises(pa.PaError) as e:
            pa.quantize_e4m3(x, check=True)
        assert e.value.code == pa.PA_ERR_BAD_INPUT
        assert pa.poll_device_status() == pa.PA_OK     # the check consumed the status


def test_check_option_passes_on_good_input(pa):
    w = workloads.get("tiny")
    q, k, v = workloads.make_case(w, device="cuda")
    o, lse = pa.attn_fwd(q, k, v, scale=w.scale, check=True)
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_close(o, lse, o_ref, l_ref, "attn_fwd with check=True")
