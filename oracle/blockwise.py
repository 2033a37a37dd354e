"""fp64 CPU oracle for blockwise (ring-step) scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: it is used by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline / reference leg of ``bench.py``, and by nothing else.
It shares no code with the CUDA library and imports nothing from this
project.

What it computes, and the passages it follows
---------------------------------------------
* Ring attention, as the diffusers guide "Context parallelism" (Turkish
  edition, section "Ring Attention" / "Halka Dikkat") describes it: every
  device attends with the K/V block it holds, hands the block on, and after a
  full turn every device has seen the K/V of every token.  The claim this
  oracle serves is that attending to one block at a time and combining the
  per-block partial results gives the exact full-sequence attention.
* "Ring Anything Attention" in the same guide: padded blocks are trimmed back
  to their real length before attention is computed, so padding never enters
  the softmax; only inference is supported and ``attn_mask`` must be None.
  Here: no mask, no causal flag, and a chunk is exactly its real keys.
* The guide "Accelerate inference" (``fp16.md``), section "Scaled dot product
  attention": SDPA is named as the attention being computed, and section
  "Model data type" names bf16 as the working type.  Inputs arrive as bf16
  values; the oracle upcasts them exactly to float64.

The pages never write the formula.  The oracle takes the textbook definition
(plain reading, stated once here and used everywhere):

    s_ij   = scale * sum_c q[i, c] * k[j, c]
    lse_i  = log( sum_j exp(s_ij) )                  (natural log)
    o[i,:] = sum_j exp(s_ij - lse_i) * v[j, :]

and, for a set of partial results (o_p, lse_p) over disjoint key chunks p,

    M   = max_p lse_p
    L   = sum_p exp(lse_p - M)
    o   = sum_p exp(lse_p - M) * o_p / L
    lse = M + log L

with the convention that a part whose lse is -inf contributes nothing, and
that if every part is -inf the merged row is o = 0, lse = -inf.  The
subtraction of the row maximum before ``exp`` is the usual overflow guard and
changes nothing mathematically.

Pins (the checks that tie this file to something other than itself) live in
``tests/test_oracle.py``: closed forms, invariants, a 50-digit brute force on
tiny inputs, PyTorch's own float64 SDPA and logsumexp, and a hand-derived
fixture in ``tests/golden/``.
"""

from __future__ import annotations

import numpy as np

__all__ = ["attention", "attention_rows", "merge", "chunked_attention"]

# Query rows per block: bounds the fp64 score matrix to row_block x Nk values.
_DEFAULT_ROW_BLOCK = 512


def _f64(x) -> np.ndarray:
    """Exact upcast to float64 (bf16 and fp32 values are representable)."""
    if hasattr(x, "detach"):  # a torch tensor: go through float64 on the CPU
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _attend_2d(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
               row_block: int):
    """Attention of q [Nq, d] against k [Nk, d], v [Nk, dv], one head."""
    nq = q.shape[0]
    o = np.empty((nq, v.shape[1]), dtype=np.float64)
    lse = np.empty((nq,), dtype=np.float64)
    kt = k.T
    for r0 in range(0, nq, row_block):
        r1 = min(nq, r0 + row_block)
        s = scale * (q[r0:r1] @ kt)                  # s_ij
        m = s.max(axis=1, keepdims=True)             # row maximum (guard)
        e = np.exp(s - m)                            # exp(s_ij - m_i)
        z = e.sum(axis=1, keepdims=True)             # sum_j exp(s_ij - m_i)
        lse_blk = m + np.log(z)                      # log sum_j exp(s_ij)
        w = np.exp(s - lse_blk)                      # exp(s_ij - lse_i)
        o[r0:r1] = w @ v
        lse[r0:r1] = lse_blk[:, 0]
    return o, lse


def attention(q, k, v, scale: float, row_block: int = _DEFAULT_ROW_BLOCK):
    """Full (unchunked) attention.

    q: [..., Nq, d], k: [..., Nk, d], v: [..., Nk, dv]; any matching leading
    dims (here [B, H]).  Returns (o [..., Nq, dv], lse [..., Nq]) in float64,
    lse in natural log of the sum of exp of the *scaled* logits.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if k.shape[-2] < 1:
        raise ValueError("attention needs at least one key")
    lead = q.shape[:-2]
    if k.shape[:-2] != lead or v.shape[:-2] != lead:
        raise ValueError("leading dims of q, k, v differ")
    if k.shape[-1] != q.shape[-1] or v.shape[-2] != k.shape[-2]:
        raise ValueError("inner dims of q, k, v do not match")
    nq, dv = q.shape[-2], v.shape[-1]
    o = np.empty(lead + (nq, dv), dtype=np.float64)
    lse = np.empty(lead + (nq,), dtype=np.float64)
    for idx in np.ndindex(*lead):
        o[idx], lse[idx] = _attend_2d(q[idx], k[idx], v[idx], float(scale), row_block)
    return o, lse


def attention_rows(q, k, v, scale: float, rows, row_block: int = _DEFAULT_ROW_BLOCK):
    """Attention for a subset of query rows (index array along the Nq axis).

    Used for sequences whose full oracle is too slow (the 119056-token case):
    each checked row still attends to every key.
    """
    q = _f64(q)
    rows = np.asarray(rows, dtype=np.int64)
    return attention(q[..., rows, :], k, v, scale, row_block)


def merge(o_parts, lse_parts):
    """Combine partial results over disjoint key chunks into the full result.

    o_parts: [n, ..., N, dv], lse_parts: [n, ..., N].  Returns (o, lse).
    A part with lse = -inf carries no weight; an all -inf row gives o = 0 and
    lse = -inf.
    """
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    if o_parts.shape[0] < 1 or lse_parts.shape[0] != o_parts.shape[0]:
        raise ValueError("merge needs n >= 1 parts of matching count")
    big_m = lse_parts.max(axis=0)                        # M = max_p lse_p
    empty = np.isneginf(big_m)
    m_safe = np.where(empty, 0.0, big_m)
    w = np.exp(lse_parts - m_safe[None])                 # exp(lse_p - M); -inf -> 0
    big_l = w.sum(axis=0)                                # L
    l_safe = np.where(empty, 1.0, big_l)
    o = (w[..., None] * o_parts).sum(axis=0) / l_safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, big_m + np.log(l_safe))
    return o, lse


def chunked_attention(q, k, v, scale: float, chunk_sizes, row_block: int = _DEFAULT_ROW_BLOCK):
    """Ring-step emulation: attend to each key chunk alone, then merge.

    chunk_sizes must sum to Nk.  Returns (o, lse, parts) where parts is the
    list of per-chunk (o_p, lse_p).  By the ring-attention claim this equals
    ``attention(q, k, v, scale)``.
    """
    k, v = _f64(k), _f64(v)
    sizes = [int(c) for c in chunk_sizes]
    if sum(sizes) != k.shape[-2] or any(c < 1 for c in sizes):
        raise ValueError("chunk sizes must be >= 1 and sum to Nk")
    parts = []
    start = 0
    for c in sizes:
        parts.append(attention(q, k[..., start:start + c, :], v[..., start:start + c, :],
                               scale, row_block))
        start += c
    o, lse = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    return o, lse, parts
