"""The ring-attention step on one GPU: attend to each K/V chunk, then merge.

This is the local loop of Ring Attention as the diffusers guide "Context
parallelism" describes it (section "Ring Attention"): each step attends to
the K/V block held at that moment, and after all blocks have been seen the
per-block results are combined into the exact full-sequence attention.  Here
the blocks are chunks already resident in local HBM.  Both steps are calls
into the C library; this function only arranges buffers.
"""

from __future__ import annotations

from typing import Optional, Sequence

from ._binding import attn_fwd, attn_merge


def blockwise_attention(q, k_chunks: Sequence, v_chunks: Sequence, scale: Optional[float] = None,
                        o_parts=None, lse_parts=None, out=None, lse=None, stream=None):
    """Attention of q [B,H,Nq,d] over the concatenation of the key chunks.

    k_chunks / v_chunks are lists of contiguous [B,H,n_p,d] bf16 tensors (the
    chunks may have different lengths n_p >= 1).  One chunk is a single
    ``attn_fwd``; several chunks are one ``attn_fwd`` per chunk into packed
    partial buffers ``o_parts`` [n,B,H,Nq,d] / ``lse_parts`` [n,B,H,Nq]
    (allocated if not given) followed by one ``attn_merge``.
    Returns (o, lse).
    """
    import torch
    n = len(k_chunks)
    if n < 1 or len(v_chunks) != n:
        raise ValueError("need at least one chunk and as many V chunks as K chunks")
    if n == 1:
        return attn_fwd(q, k_chunks[0], v_chunks[0], scale=scale, out=out, lse=lse, stream=stream)
    B, H, Nq, d = q.shape
    if o_parts is None:
        o_parts = torch.empty((n, B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse_parts is None:
        lse_parts = torch.empty((n, B, H, Nq), dtype=torch.float32, device=q.device)
    for p in range(n):
        attn_fwd(q, k_chunks[p], v_chunks[p], scale=scale, out=o_parts[p], lse=lse_parts[p],
                 stream=stream)
    return attn_merge(o_parts, lse_parts, out=out, lse=lse, stream=stream)
