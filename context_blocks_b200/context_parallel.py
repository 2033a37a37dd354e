"""Context parallelism across GPUs: the ring of K/V blocks and the Ulysses
all-to-all, each around the library's single-GPU kernels.

Both follow the diffusers guide "Context parallelism":

* section "Ring Attention": every device holds one block of the sequence's
  queries, keys and values.  At each step it attends with the K/V block it
  currently holds and passes that block to the next device, receiving the
  previous device's; after as many steps as there are devices it has seen
  every block, and its queries' attention is exact.  Here each step folds
  the block into a running fp32 (O, LSE) with ``pa_attn_fwd_accum``, and the
  transfer of the next block runs on a separate CUDA stream while the fold
  runs, into one of two receive buffers in local HBM (a remote block is
  always copied into this GPU's memory before a kernel reads it).
  Blocks may differ in length (section "Ring Anything Attention": each block
  keeps its real length; padding never enters the softmax).
* section "Ulysses Attention": an all-to-all turns sequence-sharded Q, K, V
  into head-sharded tensors over the whole sequence, each device attends for
  its heads with ``pa_attn_fwd``, and a second all-to-all turns the output
  back.  It needs the head count, and the per-device sequence length, to be
  the same on every device and the heads to divide by the device count.
* section "Unified Attention" (USP): the devices form a grid of
  ulysses_degree x ring_degree.  Within each group of ulysses_degree
  consecutive ranks the Ulysses all-to-all turns sequence shards into head
  shards over the group's part of the sequence; the ring then runs across
  the groups (ranks holding the same heads), and a second all-to-all turns
  the result back.

The functions take a ``torch.distributed`` process group (NCCL for CUDA
tensors).  The arithmetic of a step is passed in as ``attend`` /
``attend_full`` so that the exchange schedule can be exercised with CPU
tensors and the gloo backend; by default it is the library's kernels.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence

__all__ = ["ring_schedule", "ring_attention", "ring_anything_attention", "ulysses_attention",
           "ulysses_anything_attention", "head_split", "usp_groups", "usp_attention"]


def ring_schedule(rank: int, world: int) -> List[dict]:
    """Which block rank `rank` attends to at each step, and who it sends to
    and receives from (blocks are named by the rank that owns them).

    Step s: attend to the block of rank (rank - s) mod world, send it to
    (rank + 1) mod world and, except on the last step, receive the block of
    rank (rank - s - 1) mod world from (rank - 1) mod world into receive
    buffer s mod 2.  Step s + 1 attends to that buffer; the block of step 0
    is the rank's own."""
    out = []
    for s in range(world):
        ent = {"step": s, "block": (rank - s) % world, "buffer": None if s == 0 else (s - 1) % 2}
        if s < world - 1:
            ent.update(send_to=(rank + 1) % world, recv_from=(rank - 1) % world,
                       recv_block=(rank - s - 1) % world, recv_buffer=s % 2)
        out.append(ent)
    return out


def _default_attend(q, k, v, o_acc, lse_acc, first, final, out, scale):
    from ._binding import attn_fwd_accum
    attn_fwd_accum(q, k, v, o_acc, lse_acc, first=first, final=final, out=out, scale=scale)


def _default_attend_part(q, k, v, o_part, lse_part, scale):
    from ._binding import attn_fwd
    attn_fwd(q, k, v, scale=scale, out=o_part, lse=lse_part)


def _default_merge(o_parts, lse_parts, out, lse):
    from ._binding import attn_merge
    attn_merge(o_parts, lse_parts, out=out, lse=lse)


def ring_attention(q, k, v, group=None, kv_lens: Optional[Sequence[int]] = None, scale: Optional[float] = None,
                   out=None, attend: Optional[Callable] = None, comm_stream=None, trace: Optional[list] = None,
                   partials: bool = False, attend_part: Optional[Callable] = None, merge: Optional[Callable] = None):
    """Ring attention of this rank's queries over every rank's K/V block.

    q [B,H,n_q,d] and k, v [B,H,n_kv,d] are this rank's blocks (bf16 CUDA
    tensors for the library's kernels).  ``kv_lens`` lists every rank's K/V
    block length (gathered from the ranks when not given).  Returns
    (o [B,H,n_q,d], lse [B,H,n_q] fp32): this rank's queries attended over
    the whole sequence.  ``trace``, if a list, receives one entry per step
    (the schedule as executed).

    Each step folds the block it holds into an fp32 running (O, LSE)
    (``attend``: the accumulate launch).  With ``partials`` each step instead
    writes the block's own partial (O in q's dtype, LSE) with the plain
    forward (``attend_part``), and one LSE merge (``merge``) combines the
    world-size partials after the last step: the per-step launches skip the
    state's read and write, at the price of one partial per rank held until
    the end and O rounded once per block (the same result up to that
    rounding; the merge is exact in the pages' sense)."""
    import math

    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_q, d = q.shape
    if k.shape != v.shape or tuple(k.shape[:2]) != (B, H) or k.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attend = attend or _default_attend
    if kv_lens is None:
        n = torch.tensor([k.shape[2]], dtype=torch.int64, device=q.device)
        lens = [torch.zeros_like(n) for _ in range(world)]
        dist.all_gather(lens, n, group=group)
        kv_lens = [int(x.item()) for x in lens]
    kv_lens = [int(x) for x in kv_lens]
    if len(kv_lens) != world or kv_lens[rank] != k.shape[2] or min(kv_lens) < 1:
        raise ValueError(f"kv_lens {kv_lens} does not match the group ({world} ranks, own block {k.shape[2]})")

    cuda = q.is_cuda
    # The running state is fp32 for the library's kernels; CPU tensors (the
    # exchange tests) keep at least their own precision.
    state_dtype = torch.float32 if cuda else torch.promote_types(q.dtype, torch.float32)
    lse_acc = torch.empty((B, H, n_q), dtype=state_dtype, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if partials:
        attend_part = attend_part or _default_attend_part
        merge = merge or _default_merge
        o_parts = torch.empty((world, B, H, n_q, d), dtype=q.dtype, device=q.device)
        lse_parts = torch.empty((world, B, H, n_q), dtype=state_dtype, device=q.device)
        o_acc = None
    else:
        o_acc = torch.empty((B, H, n_q, d), dtype=state_dtype, device=q.device)

    def step_attend(s, kk, vv):
        if partials:
            if world == 1:
                attend_part(q, kk, vv, out, lse_acc, scale)
            else:
                attend_part(q, kk, vv, o_parts[s], lse_parts[s], scale)
        else:
            attend(q, kk, vv, o_acc, lse_acc, s == 0, s == world - 1, out if s == world - 1 else None, scale)

    if world == 1:
        step_attend(0, k, v)
        if trace is not None:
            trace.append({"step": 0, "block": 0})
        return out, lse_acc

    # Two receive buffers, each big enough for the longest block.
    m = max(kv_lens)
    bufs = [(torch.empty(B * H * m * d, dtype=k.dtype, device=k.device),
             torch.empty(B * H * m * d, dtype=v.dtype, device=v.device)) for _ in range(2)]

    def view(buf, n):
        return buf[:B * H * n * d].view(B, H, n, d)

    compute = torch.cuda.current_stream(q.device) if cuda else None
    comm = (comm_stream or torch.cuda.Stream(device=q.device)) if cuda else None
    if cuda:
        comm.wait_stream(compute)          # the own block (and q) are ready
    cur_k, cur_v = k, v
    recv_done = None
    prev_compute_done = None
    sched = ring_schedule(rank, world)
    for s, ent in enumerate(sched):
        reqs = []
        nxt = None
        if s < world - 1:
            nb = kv_lens[ent["recv_block"]]
            nxt = (view(bufs[ent["recv_buffer"]][0], nb), view(bufs[ent["recv_buffer"]][1], nb))
            # P2POp takes global ranks; the schedule is in ranks of the group.
            to_rank = ent["send_to"] if group is None else dist.get_global_rank(group, ent["send_to"])
            from_rank = ent["recv_from"] if group is None else dist.get_global_rank(group, ent["recv_from"])
            ops = [dist.P2POp(dist.isend, cur_k, to_rank, group),
                   dist.P2POp(dist.isend, cur_v, to_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], from_rank, group),
                   dist.P2POp(dist.irecv, nxt[1], from_rank, group)]
            if cuda:
                with torch.cuda.stream(comm):
                    # The buffer being received into held the block of step
                    # s - 1: its fold must be done before it is overwritten.
                    if prev_compute_done is not None:
                        comm.wait_event(prev_compute_done)
                    reqs = dist.batch_isend_irecv(ops)
                    for r in reqs:
                        r.wait()           # makes the comm stream wait for the transfer
                    recv_done = torch.cuda.Event()
                    recv_done.record(comm)
            else:
                reqs = dist.batch_isend_irecv(ops)
        step_attend(s, cur_k, cur_v)
        if trace is not None:
            trace.append({"step": s, "block": ent["block"], "n_keys": int(cur_k.shape[2])})
        if s < world - 1:
            if cuda:
                prev_compute_done = torch.cuda.Event()
                prev_compute_done.record(compute)
                compute.wait_event(recv_done)
            else:
                for r in reqs:
                    r.wait()
            cur_k, cur_v = nxt
    if partials:
        merge(o_parts, lse_parts, out, lse_acc)
    if cuda:
        # Work after this call (and the receive buffers' release) comes after
        # everything the comm stream did.
        compute.wait_stream(comm)
    return out, lse_acc


def _default_attend_chunks(q, k_chunks, v_chunks, scale):
    from ._binding import attn_fwd_chunks
    from .ring import blockwise_attention
    if len(k_chunks) <= 8:
        return attn_fwd_chunks(q, k_chunks, v_chunks, scale=scale)
    return blockwise_attention(q, k_chunks, v_chunks, scale=scale)


def ring_anything_attention(q, k, v, group=None, kv_lens: Optional[Sequence[int]] = None,
                            scale: Optional[float] = None, attend_chunks: Optional[Callable] = None):
    """Ring Anything (diffusers "Context parallelism", section "Ring Anything
    Attention"): every rank pads its K/V block to the longest block, the
    padded blocks are all-gathered, and each is trimmed back to its real
    length before attention, so padding never enters the softmax.  Here the
    trimmed blocks are the chunks of one launch (``attend_chunks``; by
    default pa_attn_fwd_chunks for up to 8 ranks, per-block forwards + merge
    beyond).  Returns (o [B,H,n_q,d], lse [B,H,n_q]) like ring_attention."""
    import math

    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_q, d = q.shape
    if k.shape != v.shape or tuple(k.shape[:2]) != (B, H) or k.shape[3] != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if kv_lens is None:
        t = torch.tensor([k.shape[2]], dtype=torch.int64, device=q.device)
        lens = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(lens, t, group=group)
        kv_lens = [int(x.item()) for x in lens]
    kv_lens = [int(x) for x in kv_lens]
    if len(kv_lens) != world or kv_lens[rank] != k.shape[2] or min(kv_lens) < 1:
        raise ValueError(f"kv_lens {kv_lens} does not match the group ({world} ranks, own block {k.shape[2]})")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attend_chunks = attend_chunks or _default_attend_chunks
    if world == 1:
        return attend_chunks(q, [k], [v], scale)
    m = max(kv_lens)
    kv = torch.zeros((2, B, H, m, d), dtype=k.dtype, device=k.device)
    kv[0, :, :, :k.shape[2]] = k
    kv[1, :, :, :k.shape[2]] = v
    gathered = [torch.empty_like(kv) for _ in range(world)]
    dist.all_gather(gathered, kv, group=group)
    # trimmed to each block's real length, as contiguous chunks
    ks = [g[0, :, :, :n].contiguous() for g, n in zip(gathered, kv_lens)]
    vs = [g[1, :, :, :n].contiguous() for g, n in zip(gathered, kv_lens)]
    del gathered
    return attend_chunks(q, ks, vs, scale)


def _a2a(x, group):
    """all_to_all over dim 0 of a contiguous tensor (one slice per rank)."""
    import torch
    import torch.distributed as dist
    y = torch.empty_like(x)
    dist.all_to_all_single(y, x, group=group)
    return y


def _seq_to_heads(x, group):
    """[B, H, n, ...] sequence shard -> [B, H/P, P*n, ...]: head group j goes to
    rank j of `group`, and the P shards of the group's ranks line up along
    the sequence in rank order."""
    import torch.distributed as dist
    P = dist.get_world_size(group)
    B, H, n = x.shape[:3]
    rest = tuple(x.shape[3:])
    xs = x.reshape(B, P, H // P, n, *rest).transpose(0, 1).contiguous()
    y = _a2a(xs, group)                                      # [P(src rank), B, H/P, n, ...]
    return y.permute(1, 2, 0, *range(3, y.dim())).reshape(B, H // P, P * n, *rest).contiguous()


def _heads_to_seq(y, group):
    """The inverse of _seq_to_heads: [B, H/P, P*n, ...] -> [B, H, n, ...]."""
    import torch.distributed as dist
    P = dist.get_world_size(group)
    B, Hp, Pn = y.shape[:3]
    n = Pn // P
    rest = tuple(y.shape[3:])
    ys = y.reshape(B, Hp, P, n, *rest).permute(2, 0, 1, *range(3, y.dim() + 1)).contiguous()
    z = _a2a(ys, group)                                      # [P(src head group), B, H/P, n, ...]
    return z.transpose(0, 1).reshape(B, Hp * P, n, *rest).contiguous()


def _default_attend_full(q, k, v, scale):
    from ._binding import attn_fwd
    return attn_fwd(q, k, v, scale=scale)


def ulysses_attention(q, k, v, group=None, scale: Optional[float] = None, attend_full: Optional[Callable] = None):
    """Ulysses attention: this rank's sequence shard q, k, v [B,H,n,d] (the
    same n and H on every rank, H divisible by the rank count) in, this
    rank's shard of the output (o [B,H,n,d], lse [B,H,n] fp32) out."""
    import math

    import torch.distributed as dist

    P = dist.get_world_size(group)
    B, H, n, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("Ulysses needs q, k, v of one shape [B,H,n,d] on every rank")
    if H % P:
        raise ValueError(f"{H} heads do not divide over {P} ranks")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attend_full = attend_full or _default_attend_full
    qh, kh, vh = _seq_to_heads(q, group), _seq_to_heads(k, group), _seq_to_heads(v, group)
    o_h, lse_h = attend_full(qh, kh, vh, scale)
    return _heads_to_seq(o_h, group), _heads_to_seq(lse_h, group)


def head_split(H: int, P: int):
    """Heads per rank for Ulysses Anything: contiguous groups in rank order,
    the first H mod P ranks taking one more head (some ranks get none when
    H < P).  Returns (sizes, starts)."""
    base, extra = divmod(H, P)
    sizes = [base + (1 if r < extra else 0) for r in range(P)]
    starts = [sum(sizes[:r]) for r in range(P)]
    return sizes, starts


def _a2a_var(send_parts, recv_numels, group, like):
    """all_to_all with a flat piece per peer: send_parts[s] goes to rank s,
    and the piece from rank s has recv_numels[s] elements."""
    import torch
    import torch.distributed as dist
    send = torch.cat([x.reshape(-1) for x in send_parts]) if send_parts else like.new_empty(0)
    recv = like.new_empty(sum(recv_numels))
    dist.all_to_all_single(recv, send, output_split_sizes=list(recv_numels),
                           input_split_sizes=[x.numel() for x in send_parts], group=group)
    return torch.split(recv, list(recv_numels))


def _seq_to_heads_any(x, group, seq_lens, sizes, starts):
    """[B, H, n_r, ...] sequence shard -> [B, h_r, sum(seq_lens), ...]: rank
    s's head group goes to rank s; the shards line up along the sequence in
    rank order."""
    import torch
    import torch.distributed as dist
    r = dist.get_rank(group)
    B = x.shape[0]
    rest = tuple(x.shape[3:])
    e = 1
    for t in rest:
        e *= t
    send = [x[:, h0:h0 + hs] for h0, hs in zip(starts, sizes)]
    pieces = _a2a_var(send, [B * sizes[r] * n_s * e for n_s in seq_lens], group, x)
    parts = [pc.view(B, sizes[r], n_s, *rest) for pc, n_s in zip(pieces, seq_lens)]
    return torch.cat(parts, dim=2).contiguous()


def _heads_to_seq_any(y, group, seq_lens, sizes):
    """The inverse of _seq_to_heads_any: [B, h_r, sum(seq_lens), ...] ->
    [B, H, n_r, ...]."""
    import torch
    import torch.distributed as dist
    r = dist.get_rank(group)
    B = y.shape[0]
    rest = tuple(y.shape[3:])
    e = 1
    for t in rest:
        e *= t
    offs = [sum(seq_lens[:s]) for s in range(len(seq_lens))]
    send = [y[:, :, o:o + n_s] for o, n_s in zip(offs, seq_lens)]
    pieces = _a2a_var(send, [B * h_s * seq_lens[r] * e for h_s in sizes], group, y)
    parts = [pc.view(B, h_s, seq_lens[r], *rest) for pc, h_s in zip(pieces, sizes)]
    return torch.cat(parts, dim=1).contiguous()


def ulysses_anything_attention(q, k, v, group=None, seq_lens: Optional[Sequence[int]] = None,
                               scale: Optional[float] = None, attend_full: Optional[Callable] = None):
    """Ulysses attention without divisibility (diffusers "Context
    parallelism", section "Ulysses Anything"): this rank's sequence shard q,
    k, v [B,H,n_r,d] in, where the shard lengths may differ between ranks
    (``seq_lens``, gathered when not given) and H need not divide by the rank
    count (head_split); this rank's shard of the output (o [B,H,n_r,d],
    lse [B,H,n_r]) out.  The two all-to-alls carry per-peer pieces of
    different sizes; a rank that holds no head computes nothing."""
    import math

    import torch
    import torch.distributed as dist

    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    B, H, n, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("Ulysses needs q, k, v of one shape [B,H,n,d] on each rank")
    if seq_lens is None:
        t = torch.tensor([n], dtype=torch.int64, device=q.device)
        lens = [torch.zeros_like(t) for _ in range(P)]
        dist.all_gather(lens, t, group=group)
        seq_lens = [int(x.item()) for x in lens]
    seq_lens = [int(x) for x in seq_lens]
    if len(seq_lens) != P or seq_lens[r] != n or min(seq_lens) < 1:
        raise ValueError(f"seq_lens {seq_lens} does not match the group ({P} ranks, own shard {n})")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attend_full = attend_full or _default_attend_full
    sizes, starts = head_split(H, P)
    qh, kh, vh = (_seq_to_heads_any(x, group, seq_lens, sizes, starts) for x in (q, k, v))
    if sizes[r] > 0:
        o_h, lse_h = attend_full(qh, kh, vh, scale)
    else:
        lse_dtype = torch.float32 if q.is_cuda else torch.promote_types(q.dtype, torch.float32)
        o_h = qh.new_empty((B, 0, sum(seq_lens), d))
        lse_h = torch.empty((B, 0, sum(seq_lens)), dtype=lse_dtype, device=q.device)
    return _heads_to_seq_any(o_h, group, seq_lens, sizes), _heads_to_seq_any(lse_h, group, seq_lens, sizes)


def usp_groups(ulysses_degree: int, group=None):
    """The process groups of a ulysses_degree x ring_degree grid over `group`
    (default: the whole world; its size must divide by ulysses_degree).
    Returns (ulysses_group, ring_group) of the calling rank.  Group rank r
    has Ulysses index r % ulysses_degree and ring index r // ulysses_degree:
    a Ulysses group is ulysses_degree consecutive ranks, a ring group the
    ranks with the same Ulysses index.  Every rank of `group` must call this
    (the groups are created collectively, in the same order everywhere)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    U = int(ulysses_degree)
    if U < 1 or world % U:
        raise ValueError(f"ulysses_degree {U} does not divide {world} ranks")
    R = world // U
    glob = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    mine_u = mine_r = None
    for g in range(R):
        ranks = [glob(g * U + u) for u in range(U)]
        pg = dist.new_group(ranks)
        if rank // U == g:
            mine_u = pg
    for u in range(U):
        ranks = [glob(g * U + u) for g in range(R)]
        pg = dist.new_group(ranks)
        if rank % U == u:
            mine_r = pg
    return mine_u, mine_r


def usp_attention(q, k, v, ulysses_group, ring_group, scale: Optional[float] = None, attend: Optional[Callable] = None,
                  comm_stream=None, trace: Optional[list] = None, partials: bool = False,
                  attend_part: Optional[Callable] = None, merge: Optional[Callable] = None):
    """Unified (Ulysses x ring) attention of this rank's sequence shard q, k, v
    [B,H,n,d] (the same n and H on every rank; H divisible by the Ulysses
    degree) over the whole sequence, which is sharded over the ranks in
    group-rank order (see usp_groups).  Returns (o [B,H,n,d], lse [B,H,n]).
    ``attend``, ``partials``, ``attend_part`` and ``merge`` are passed to
    ring_attention."""
    import math

    import torch.distributed as dist

    U = dist.get_world_size(ulysses_group)
    R = dist.get_world_size(ring_group)
    B, H, n, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("USP needs q, k, v of one shape [B,H,n,d] on every rank")
    if H % U:
        raise ValueError(f"{H} heads do not divide over a Ulysses degree of {U}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qh, kh, vh = (_seq_to_heads(t, ulysses_group) for t in (q, k, v))   # [B, H/U, U*n, d]
    out = qh.new_empty(qh.shape)
    o_h, lse_h = ring_attention(qh, kh, vh, group=ring_group, kv_lens=[U * n] * R, scale=scale, out=out,
                                attend=attend, comm_stream=comm_stream, trace=trace, partials=partials,
                                attend_part=attend_part, merge=merge)
    return _heads_to_seq(o_h, ulysses_group), _heads_to_seq(lse_h, ulysses_group)
