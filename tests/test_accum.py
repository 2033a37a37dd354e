"""GPU parity of pa_attn_fwd_accum: chunks folded one at a time into a running
fp32 (O, LSE), the step a ring-attention device takes each time a block
arrives (diffusers "Context parallelism", section "Ring Attention").

The folded result is compared with the fp64 oracle over the whole, unchunked
key sequence; the intermediate fp32 state after some folds is compared with
the oracle over the chunks folded so far.  One case measures how the error
of the merged result grows with the number of parts for bf16 partials
(pa_attn_fwd per chunk + pa_attn_merge) against the fp32 running state.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from context_blocks_b200 import build
    build.build()
    import context_blocks_b200 as pa_mod
    pa_mod.load_library()
    return pa_mod


def _fold(pa, q, pairs, scale, check_every=False, qh=None, kh=None, vh=None, what=""):
    """Fold every (k, v) chunk into a fresh state; return (o bf16, lse)."""
    B, H, Nq, d = q.shape
    o_acc = torch.full((B, H, Nq, d), float("nan"), dtype=torch.float32, device=q.device)
    lse_acc = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device=q.device)
    out = torch.full_like(q, float("nan"))
    n = len(pairs)
    seen = 0
    for c, (k, v) in enumerate(pairs):
        first, final = c == 0, c == n - 1
        pa.attn_fwd_accum(q, k, v, o_acc, lse_acc, first=first, final=final, out=out if final else None,
                          scale=scale)
        seen += k.shape[2]
        if check_every and not final:
            torch.cuda.synchronize()
            o_ref, l_ref = oracle.attention(qh, kh[:, :, :seen], vh[:, :, :seen], scale)
            assert_close(o_acc, lse_acc, o_ref, l_ref, f"{what} state after {c + 1} folds")
    torch.cuda.synchronize()
    assert pa.poll_device_status() == pa.PA_OK
    return out, lse_acc


def _check(pa, w, check_every=True):
    q, k, v = workloads.make_case(w, device="cuda")
    pairs = workloads.split_keys(k, v, w.chunks)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    o, lse = _fold(pa, q, pairs, w.scale, check_every, qh, kh, vh, w.name)
    o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale)
    assert_close(o, lse, o_ref, l_ref, f"fold {w.name} vs unchunked oracle")
    return q, pairs, o, lse


def test_fold_ring_step(pa):
    _check(pa, workloads.get("ring"))


def test_fold_uneven_tails(pa):
    _check(pa, workloads.get("tails"), check_every=False)


def test_fold_ring_anything_1008(pa):
    _check(pa, workloads.get("flux1008"))


def test_fold_head_dim_64_ragged(pa):
    w = workloads.Workload("fold64", B=2, H=3, Nq=300, Nk=517, d=64, rms_qk=False, chunks=(200, 1, 316), seed=41)
    _check(pa, w)


def test_fold_single_key_chunks(pa):
    w = workloads.Workload("fold1", B=1, H=2, Nq=129, Nk=6, d=128, rms_qk=False, chunks=(1, 1, 1, 1, 1, 1), seed=42)
    _check(pa, w)


def test_first_and_final_together_equals_attn_fwd(pa):
    """One fold with both flags is pa_attn_fwd with the LSE written to the
    state: the same arithmetic, so the same bits."""
    w = workloads.get("tails").with_chunks([4603])
    q, k, v = workloads.make_case(w, device="cuda")
    o_acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse_acc = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    o1, l1 = pa.attn_fwd_accum(q, k, v, o_acc, lse_acc, first=True, final=True, scale=w.scale)
    o2, l2 = pa.attn_fwd(q, k, v, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_empty_rows_are_not_read(pa):
    """Rows whose running LSE is -inf are empty: their O (NaN here) is not
    read, and the fold gives the attention over the new chunk alone."""
    w = workloads.Workload("empty", B=1, H=2, Nq=200, Nk=300, d=128, rms_qk=True, chunks=(300,), seed=43)
    q, k, v = workloads.make_case(w, device="cuda")
    o_acc = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    lse_acc = torch.full(q.shape[:3], float("-inf"), dtype=torch.float32, device="cuda")
    pa.attn_fwd_accum(q, k, v, o_acc, lse_acc, scale=w.scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), w.scale)
    assert_close(o_acc, lse_acc, o_ref, l_ref, "fold into empty rows")


def test_fold_rescales_across_chunks(pa):
    """Later chunks hold much larger logits (the running maximum moves by far
    more than the lazy-rescale threshold at every fold), then smaller ones."""
    B, H, Nq, d = 1, 2, 260, 128
    g = torch.Generator(device="cuda").manual_seed(44)
    q = torch.randn((B, H, Nq, d), generator=g, device="cuda") * 0.2 + 1.0
    chunks = (300, 200, 257, 129)
    Nk = sum(chunks)
    ramp = torch.tensor(np.repeat([0.0, 3.0, 6.0, 1.0], chunks), dtype=torch.float32, device="cuda")
    k = torch.randn((B, H, Nk, d), generator=g, device="cuda") * 0.1 + ramp[None, None, :, None]
    v = torch.randn((B, H, Nk, d), generator=g, device="cuda")
    q, k, v = (x.to(torch.bfloat16).contiguous() for x in (q, k, v))
    pairs = workloads.split_keys(k, v, chunks)
    scale = 1.0 / math.sqrt(d)
    o, lse = _fold(pa, q, pairs, scale, True, q.cpu(), k.cpu(), v.cpu(), "rescale")
    o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)
    assert float(np.max(l_ref)) > 50.0
    assert_close(o, lse, o_ref, l_ref, "fold with rescales")


@pytest.mark.parametrize("n_parts", [16, 32])
def test_fp32_state_vs_bf16_partials_error_growth(pa, n_parts):
    """Many parts: bf16 partials rounded before the merge against the fp32
    running state.  Both stay inside the tolerance; the fp32 state's error
    does not grow with the part count, and the two errors are recorded."""
    w = workloads.Workload(f"parts{n_parts}", B=1, H=4, Nq=384, Nk=n_parts * 160, d=128, rms_qk=True,
                           chunks=(160,) * n_parts, seed=45)
    q, k, v = workloads.make_case(w, device="cuda")
    pairs = workloads.split_keys(k, v, w.chunks)
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale)
    o16, l16 = pa.blockwise_attention(q, [a for a, _ in pairs], [b for _, b in pairs], scale=w.scale)
    o32, l32 = _fold(pa, q, pairs, w.scale)
    e16 = assert_close(o16, l16, o_ref, l_ref, f"{n_parts} bf16 partials + merge")
    e32 = assert_close(o32, l32, o_ref, l_ref, f"{n_parts} folds into the fp32 state")
    # the fp32 state rounds once (the final bf16 output); the bf16 partials
    # round every part and then the merged output
    assert e32["o_rel_l2"] <= e16["o_rel_l2"], (e32, e16)
