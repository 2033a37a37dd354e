"""Pins for the fp64 oracle: what ties it to something other than itself.

Every pin below is a fact fixed by the mathematics of softmax attention or by
the ring-attention claim (diffusers "Context parallelism" guide, section
"Ring Attention": attending one K/V block at a time and combining the partial
results gives the exact full-sequence attention):

* a hand-worked fixture with exact answers (tests/golden/hand_closed_form.json);
* closed forms: constant V, zero query, one key, identical keys, two keys
  (logistic weights);
* invariants: permutation of K/V pairs, translation of all keys, linearity in V;
* chunk + merge equals unchunked attention for arbitrary splits, and the merge
  conventions (n = 1, -inf parts);
* a 50-digit ``decimal`` brute force on tiny inputs, written from the
  definition without the max-subtraction guard;
* PyTorch's own float64 SDPA and logsumexp (an independent library routine).

``test_pins_catch_planted_mistakes`` plants plausible mistakes in copies of the
oracle (dropped scale, log base, transposed softmax axis, missing
normalisation, sign error, wrong operand, broken merge) and checks that at
least one pin fails for each.  Everything here runs on the CPU.
"""

import json
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import blockwise as oracle_mod

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_qkv(rng, lead=(2, 3), nq=7, nk=11, d=5, dv=None, scale_q=1.0):
    dv = d if dv is None else dv
    q = rng.standard_normal(lead + (nq, d)) * scale_q
    k = rng.standard_normal(lead + (nk, d))
    v = rng.standard_normal(lead + (nk, dv))
    return q, k, v


# --------------------------------------------------------------------------
# Pins written as predicates over (attention, merge) so that the mutation test
# can run them against deliberately broken oracles.
# --------------------------------------------------------------------------

def _parse(expr: str) -> float:
    expr = expr.strip()
    if expr.startswith("ln(") and expr.endswith(")"):
        return math.log(float(Fraction(expr[3:-1])))
    return float(Fraction(expr))


def _golden():
    with open(os.path.join(HERE, "golden", "hand_closed_form.json")) as f:
        return json.load(f)


def pin_golden(attn, merge):
    ok = True
    for case in _golden()["cases"]:
        q = np.array([[_parse(x) for x in row] for row in case["q"]])
        k = np.array([[_parse(x) for x in row] for row in case["k"]])
        v = np.array([[_parse(x) for x in row] for row in case["v"]])
        o_exp = np.array([[_parse(x) for x in row] for row in case["o"]])
        lse_exp = np.array([_parse(x) for x in case["lse"]])
        o, lse = attn(q[None], k[None], v[None], case["scale"])
        ok &= np.allclose(o[0], o_exp, rtol=0, atol=1e-13)
        ok &= np.allclose(lse[0], lse_exp, rtol=0, atol=1e-13)
        if "chunks" in case:
            s = 0
            o_parts, lse_parts = [], []
            for c, part in zip(case["chunks"], case["parts"]):
                po, pl = attn(q[None], k[None, s:s + c], v[None, s:s + c], case["scale"])
                ok &= np.allclose(po[0], np.array([[_parse(x) for x in r] for r in part["o"]]),
                                  rtol=0, atol=1e-13)
                ok &= np.allclose(pl[0], np.array([_parse(x) for x in part["lse"]]),
                                  rtol=0, atol=1e-13)
                o_parts.append(po)
                lse_parts.append(pl)
                s += c
            mo, ml = merge(np.stack(o_parts), np.stack(lse_parts))
            ok &= np.allclose(mo[0], o_exp, rtol=0, atol=1e-13)
            ok &= np.allclose(ml[0], lse_exp, rtol=0, atol=1e-13)
    return bool(ok)


def pin_constant_v(attn, merge):
    rng = _rng(1)
    q, k, _ = _rand_qkv(rng)
    c = rng.standard_normal(5)
    v = np.broadcast_to(c, (2, 3, 11, 5)).copy()
    o, _ = attn(q, k, v, 0.7)
    return bool(np.allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=TOL))


def pin_rows_sum_to_one(attn, merge):
    rng = _rng(2)
    q, k, _ = _rand_qkv(rng, scale_q=3.0)
    v = np.ones((2, 3, 11, 1))
    o, _ = attn(q, k, v, 1.3)
    return bool(np.allclose(o, 1.0, rtol=0, atol=TOL))


def pin_zero_query(attn, merge):
    rng = _rng(3)
    _, k, v = _rand_qkv(rng)
    q = np.zeros((2, 3, 4, 5))
    o, lse = attn(q, k, v, 0.9)
    ok = np.allclose(o, np.broadcast_to(v.mean(axis=-2, keepdims=True), o.shape), rtol=0, atol=TOL)
    ok &= np.allclose(lse, math.log(11), rtol=0, atol=TOL)
    return bool(ok)


def pin_single_key(attn, merge):
    rng = _rng(4)
    q, k, v = _rand_qkv(rng, nk=1)
    o, lse = attn(q, k, v, 0.45)
    ok = np.allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=TOL)
    ok &= np.allclose(lse, 0.45 * (q @ np.swapaxes(k, -1, -2))[..., 0], rtol=0, atol=TOL)
    return bool(ok)


def pin_identical_keys(attn, merge):
    rng = _rng(5)
    q, k1, v = _rand_qkv(rng, nk=1)
    k = np.repeat(k1, 9, axis=-2)
    v = rng.standard_normal((2, 3, 9, 5))
    o, lse = attn(q, k, v, 0.6)
    s = 0.6 * (q @ np.swapaxes(k1, -1, -2))[..., 0]
    ok = np.allclose(o, np.broadcast_to(v.mean(axis=-2, keepdims=True), o.shape), rtol=0, atol=TOL)
    ok &= np.allclose(lse, s + math.log(9), rtol=0, atol=TOL)
    return bool(ok)


def pin_two_keys_logistic(attn, merge):
    from scipy.special import expit
    rng = _rng(6)
    q, k, v = _rand_qkv(rng, nk=2, d=3, dv=4)
    o, lse = attn(q, k, v, 0.8)
    s = 0.8 * (q @ np.swapaxes(k, -1, -2))          # [..., nq, 2]
    w0 = expit(s[..., 0] - s[..., 1])
    w1 = expit(s[..., 1] - s[..., 0])
    o_exp = w0[..., None] * v[..., None, 0, :] + w1[..., None] * v[..., None, 1, :]
    ok = np.allclose(o, o_exp, rtol=0, atol=TOL)
    ok &= np.allclose(lse, np.logaddexp(s[..., 0], s[..., 1]), rtol=0, atol=TOL)
    return bool(ok)


def pin_permutation(attn, merge):
    rng = _rng(7)
    q, k, v = _rand_qkv(rng, nk=13)
    perm = rng.permutation(13)
    o1, l1 = attn(q, k, v, 0.5)
    o2, l2 = attn(q, k[..., perm, :], v[..., perm, :], 0.5)
    return bool(np.allclose(o1, o2, rtol=0, atol=TOL) and np.allclose(l1, l2, rtol=0, atol=TOL))


def pin_key_translation(attn, merge):
    rng = _rng(8)
    q, k, v = _rand_qkv(rng)
    w = rng.standard_normal(5)
    o1, l1 = attn(q, k, v, 0.5)
    o2, l2 = attn(q, k + w, v, 0.5)
    shift = 0.5 * (q @ w)
    return bool(np.allclose(o1, o2, rtol=0, atol=TOL) and np.allclose(l2, l1 + shift, rtol=0, atol=TOL))


def pin_value_linearity(attn, merge):
    rng = _rng(9)
    q, k, v1 = _rand_qkv(rng)
    v2 = rng.standard_normal(v1.shape)
    a = 2.5
    o1, _ = attn(q, k, v1, 0.4)
    o2, _ = attn(q, k, v2, 0.4)
    o3, _ = attn(q, k, v1 + a * v2, 0.4)
    return bool(np.allclose(o3, o1 + a * o2, rtol=0, atol=TOL))


def _chunk_merge(attn, merge, q, k, v, scale, sizes):
    parts, s = [], 0
    for c in sizes:
        parts.append(attn(q, k[..., s:s + c, :], v[..., s:s + c, :], scale))
        s += c
    return merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))


def pin_chunk_merge_exact(attn, merge):
    rng = _rng(10)
    ok = True
    for sizes in ([5, 6], [1] * 11, [3, 1, 7], [11]):
        q, k, v = _rand_qkv(rng, scale_q=2.0)
        o_full, l_full = attn(q, k, v, 0.9)
        o_cm, l_cm = _chunk_merge(attn, merge, q, k, v, 0.9, sizes)
        ok &= np.allclose(o_cm, o_full, rtol=0, atol=TOL) and np.allclose(l_cm, l_full, rtol=0, atol=TOL)
    return bool(ok)


def pin_merge_conventions(attn, merge):
    rng = _rng(11)
    o = rng.standard_normal((1, 2, 3, 4, 5))
    lse = rng.standard_normal((1, 2, 3, 4))
    mo, ml = merge(o, lse)                       # n = 1 is the identity
    ok = np.allclose(mo, o[0], rtol=0, atol=TOL) and np.allclose(ml, lse[0], rtol=0, atol=TOL)
    o2 = np.concatenate([o, rng.standard_normal(o.shape)])
    lse2 = np.concatenate([lse, np.full(lse.shape, -np.inf)])
    mo, ml = merge(o2, lse2)                     # a -inf part carries no weight
    ok &= np.allclose(mo, o[0], rtol=0, atol=TOL) and np.allclose(ml, lse[0], rtol=0, atol=TOL)
    mo, ml = merge(o2, np.full(lse2.shape, -np.inf))  # all -inf: o = 0, lse = -inf
    ok &= bool(np.all(mo == 0.0)) and bool(np.all(np.isneginf(ml)))
    # equal lse on two parts: the merge is the plain mean and lse grows by ln 2
    o3 = rng.standard_normal((2, 3, 4))
    l3 = np.array([[0.3] * 3, [0.3] * 3])
    mo, ml = merge(o3, l3)
    ok &= np.allclose(mo, o3.mean(axis=0), rtol=0, atol=TOL) and np.allclose(ml, 0.3 + math.log(2), atol=TOL)
    return bool(ok)


def _decimal_attention(q, k, v, scale):
    """The definition at 50 digits, with no max subtraction: o = sum_j
    e^{s_j} v_j / sum_j e^{s_j}, lse = ln sum_j e^{s_j}.  One head."""
    getcontext().prec = 50
    sc = Decimal(repr(float(scale)))
    out_o, out_l = [], []
    for qi in q:
        s = [sc * sum(Decimal(repr(float(a))) * Decimal(repr(float(b))) for a, b in zip(qi, kj))
             for kj in k]
        e = [x.exp() for x in s]
        z = sum(e)
        out_o.append([float(sum(ej * Decimal(repr(float(vj[c]))) for ej, vj in zip(e, v)) / z)
                      for c in range(len(v[0]))])
        out_l.append(float(z.ln()))
    return np.array(out_o), np.array(out_l)


def pin_brute_force(attn, merge):
    rng = _rng(12)
    ok = True
    for (nq, nk, d, sc, mag) in [(3, 1, 2, 0.5, 1.0), (4, 5, 3, 0.7, 1.0), (2, 8, 4, 1.0, 3.0),
                                  (3, 6, 2, 40.0, 4.0)]:   # last: logits of several hundred
        q = rng.standard_normal((nq, d)) * mag
        k = rng.standard_normal((nk, d)) * mag
        v = rng.standard_normal((nk, 3))
        o_ref, l_ref = _decimal_attention(q, k, v, sc)
        o, lse = attn(q[None], k[None], v[None], sc)
        ok &= np.allclose(o[0], o_ref, rtol=1e-12, atol=1e-12)
        ok &= np.allclose(lse[0], l_ref, rtol=1e-13, atol=1e-12)
    return bool(ok)


def pin_torch_sdpa(attn, merge):
    import torch
    rng = _rng(13)
    q, k, v = _rand_qkv(rng, lead=(2, 3), nq=9, nk=17, d=8, dv=6, scale_q=1.5)
    sc = 0.35
    o, lse = attn(q, k, v, sc)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=sc).numpy()
    tl = torch.logsumexp(sc * (tq @ tk.transpose(-1, -2)), dim=-1).numpy()
    return bool(np.allclose(o, to, rtol=0, atol=1e-12) and np.allclose(lse, tl, rtol=0, atol=1e-12))


PINS = [pin_golden, pin_constant_v, pin_rows_sum_to_one, pin_zero_query, pin_single_key,
        pin_identical_keys, pin_two_keys_logistic, pin_permutation, pin_key_translation,
        pin_value_linearity, pin_chunk_merge_exact, pin_merge_conventions, pin_brute_force,
        pin_torch_sdpa]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    assert pin(oracle.attention, oracle.merge)


def test_row_blocking_is_invisible():
    """Blocking over query rows (a memory bound) must not change any value."""
    rng = _rng(14)
    q, k, v = _rand_qkv(rng, nq=37, nk=29, d=6)
    o1, l1 = oracle.attention(q, k, v, 0.3, row_block=5)
    o2, l2 = oracle.attention(q, k, v, 0.3, row_block=1000)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_attention_rows_matches_full():
    rng = _rng(15)
    q, k, v = _rand_qkv(rng, nq=20)
    rows = np.array([0, 3, 19, 7])
    o, l = oracle.attention(q, k, v, 0.5)
    orow, lrow = oracle.attention_rows(q, k, v, 0.5, rows)
    assert np.allclose(orow, o[..., rows, :], rtol=0, atol=TOL)
    assert np.allclose(lrow, l[..., rows], rtol=0, atol=TOL)


def test_chunked_attention_helper():
    rng = _rng(16)
    q, k, v = _rand_qkv(rng, nk=23)
    o, l = oracle.attention(q, k, v, 0.5)
    oc, lc, parts = oracle.chunked_attention(q, k, v, 0.5, [7, 7, 9])
    assert len(parts) == 3
    assert np.allclose(oc, o, rtol=0, atol=TOL) and np.allclose(lc, l, rtol=0, atol=TOL)
    with pytest.raises(ValueError):
        oracle.chunked_attention(q, k, v, 0.5, [7, 7])
    with pytest.raises(ValueError):
        oracle.chunked_attention(q, k, v, 0.5, [0, 23])


def test_input_validation():
    rng = _rng(17)
    q, k, v = _rand_qkv(rng)
    with pytest.raises(ValueError):
        oracle.attention(q, k[..., :0, :], v[..., :0, :], 1.0)
    with pytest.raises(ValueError):
        oracle.attention(q, k[..., :4], v, 1.0)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v[..., :3, :], 1.0)


def test_bf16_inputs_upcast_exactly():
    """bf16 tensors reach the oracle as their exact float64 values."""
    import torch
    t = torch.tensor([1.0 + 2 ** -7, -3.0e-5, 65280.0], dtype=torch.bfloat16)
    x = oracle_mod._f64(t)
    assert x.dtype == np.float64
    assert list(x) == [float(y) for y in t.float().tolist()]


def test_large_magnitude_logits_are_finite():
    q = np.full((1, 1, 2, 4), 30.0)
    k = np.full((1, 1, 3, 4), 30.0)
    v = np.arange(12, dtype=np.float64).reshape(1, 1, 3, 4)
    o, lse = oracle.attention(q, k, v, 1.0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.allclose(lse, 3600.0 + math.log(3), rtol=1e-15)


# --------------------------------------------------------------------------
# Planted mistakes: each mutant must be caught by at least one pin.
# --------------------------------------------------------------------------

def _mutant_attend(kind):
    def attend(q, k, v, scale, row_block):
        s = q @ k.T
        if kind != "no_scale":
            s = scale * s
        if kind == "softmax_over_queries":
            m = s.max(axis=0, keepdims=True)
            e = np.exp(s - m)
            z = e.sum(axis=0, keepdims=True)
            return (e / z) @ v, (m + np.log(z)).max(axis=0).repeat(q.shape[0])[:q.shape[0]]
        if kind == "sign":
            s = -s
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        lse = m + np.log(z)
        if kind == "log2_lse":
            lse = (m + np.log(z)) / math.log(2)
        if kind == "dropped_max":
            lse = np.log(z)
        o = e @ v
        if kind != "unnormalised":
            o = o / z
        if kind == "uses_k_for_v":
            o = (e / z) @ k[:, : v.shape[1]] if k.shape[1] >= v.shape[1] else o
        return o, lse[:, 0]
    return attend


def _broken_merge(kind):
    def merge(o_parts, lse_parts):
        o_parts, lse_parts = np.asarray(o_parts, float), np.asarray(lse_parts, float)
        m = lse_parts.max(axis=0)
        w = np.exp(lse_parts - m)
        if kind == "no_divide":
            o = (w[..., None] * o_parts).sum(axis=0)
            return o, m + np.log(w.sum(axis=0))
        if kind == "plain_mean":
            return o_parts.mean(axis=0), m + np.log(w.sum(axis=0))
        if kind == "lse_is_max":
            return (w[..., None] * o_parts).sum(axis=0) / w.sum(axis=0)[..., None], m
        raise AssertionError(kind)
    return merge


ATTEND_MUTANTS = ["no_scale", "softmax_over_queries", "sign", "log2_lse", "dropped_max",
                  "unnormalised", "uses_k_for_v"]
MERGE_MUTANTS = ["no_divide", "plain_mean", "lse_is_max"]


def _run_pins(attn, merge):
    results = {}
    for pin in PINS:
        try:
            results[pin.__name__] = pin(attn, merge)
        except Exception:
            results[pin.__name__] = False
    return results


@pytest.mark.parametrize("kind", ATTEND_MUTANTS)
def test_pins_catch_planted_attention_mistakes(kind, monkeypatch):
    monkeypatch.setattr(oracle_mod, "_attend_2d", _mutant_attend(kind))
    results = _run_pins(oracle_mod.attention, oracle_mod.merge)
    assert not all(results.values()), f"mutant {kind} passed every pin"


@pytest.mark.parametrize("kind", MERGE_MUTANTS)
def test_pins_catch_planted_merge_mistakes(kind):
    results = _run_pins(oracle.attention, _broken_merge(kind))
    assert not all(results.values()), f"merge mutant {kind} passed every pin"


def test_unmutated_oracle_passes_every_pin():
    results = _run_pins(oracle.attention, oracle.merge)
    assert all(results.values()), results


# ---------------------------------------------------------------- e4m3 rounding

from oracle import e4m3 as E


def test_e4m3_decode_table_fixed_points():
    t = E.decode_table()
    assert t[0x00] == 0.0 and t[0x38] == 1.0 and t[0x40] == 2.0 and t[0x30] == 0.5
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6 and t[0x07] == 7 * 2.0 ** -9
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0)                       # codes 0..0x7E increase
    assert np.array_equal(t[0x80:0xFF], -pos)             # sign bit


def test_e4m3_encode_round_trip_and_ties():
    t = E.decode_table()
    finite = np.array([c for c in range(256) if not np.isnan(t[c])])
    # every finite value encodes to itself (0.0 and -0.0 keep their signs)
    for c in finite:
        assert E.encode_rne(t[c]) == c, hex(c)
    # midpoints go to the even code: between 1.0 (0x38) and 1.125 (0x39) -> 0x38;
    # between 1.125 (0x39) and 1.25 (0x3A) -> 0x3A
    assert E.encode_rne(1.0625) == 0x38 and E.encode_rne(1.1875) == 0x3A
    # just off the midpoint goes to the nearer code
    assert E.encode_rne(np.nextafter(1.0625, 2.0)) == 0x39
    # saturation and the subnormal range
    assert E.encode_rne(1e6) == 0x7E and E.encode_rne(-1e6) == 0xFE and E.encode_rne(449.0) == 0x7E
    assert E.encode_rne(2.0 ** -10) == 0x00                  # halfway 0 .. 2^-9 -> even (0)
    assert E.encode_rne(3 * 2.0 ** -10) == 0x02              # halfway 2^-9 .. 2^-8 -> even (0x02)


def test_e4m3_quantize_matches_torch_cast():
    # an independent implementation of the same rounding (PyTorch's cast)
    import torch
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal(5000).astype(np.float32)).to(torch.bfloat16).float().numpy()
    codes, scale = E.quantize(x)
    y = (x * np.float32(np.float32(448.0) / np.max(np.abs(x)))).astype(np.float32)
    ok = np.abs(y) < 448.0                                   # torch's cast does not saturate
    tc = torch.from_numpy(y[ok]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes[ok], tc)
    assert scale == np.float32(np.max(np.abs(x)) / np.float32(448.0))
    assert E.quantize(np.zeros(7))[1] == 1.0 and not np.any(E.quantize(np.zeros(7))[0])


def test_uneven_ring_split_equals_unchunked():
    # the uneven-tails split of the context-parallel guide's ring-anything
    # case (4603 keys over 4 ranks), at a small width: chunk + merge = whole
    rng = np.random.default_rng(12)
    q = rng.standard_normal((1, 2, 48, 8))
    k = rng.standard_normal((1, 2, 4603, 8))
    v = rng.standard_normal((1, 2, 4603, 8))
    o_full, l_full = oracle.attention(q, k, v, 0.35)
    o_cm, l_cm, parts = oracle.chunked_attention(q, k, v, 0.35, [1151, 1151, 1151, 1150])
    assert len(parts) == 4
    assert np.allclose(o_cm, o_full, rtol=0, atol=1e-12) and np.allclose(l_cm, l_full, rtol=0, atol=1e-12)
