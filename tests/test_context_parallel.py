"""The multi-rank exchange schedules of context_parallel on the CPU: gloo
process groups of 2 and 3 ranks, float64 tensors, and the attention step
injected by the test (the fp64 oracle), so that what is checked here is the
exchange itself: which block each rank folds at each step, from which
buffer, that the ring's blocks may differ in length, and that both the ring
and the Ulysses all-to-all give every rank exactly the attention of its
queries over the whole sequence (diffusers "Context parallelism", sections
"Ring Attention", "Ring Anything Attention" and "Ulysses Attention")."""

import socket

import numpy as np
import pytest
import torch

import oracle
from context_blocks_b200.context_parallel import ring_schedule

SCALE = 0.3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_case(seed, B, H, n_total, d):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, n_total, d), generator=g, dtype=torch.float64)
    k = torch.randn((B, H, n_total, d), generator=g, dtype=torch.float64)
    v = torch.randn((B, H, n_total, d), generator=g, dtype=torch.float64)
    return q, k, v


def _oracle_fold(q, k, v, o_acc, lse_acc, first, final, out, scale):
    """The fold of one block, from the oracle: merge the running state with
    the attention over this block."""
    o_b, l_b = oracle.attention(q, k, v, scale)
    if first:
        o_new, l_new = o_b, l_b
    else:
        o_new, l_new = oracle.merge(np.stack([o_acc.numpy(), o_b]), np.stack([lse_acc.numpy(), l_b]))
    lse_acc.copy_(torch.from_numpy(l_new))
    (out if final else o_acc).copy_(torch.from_numpy(o_new))


def _ring_rank(rank, world, port, q_lens, kv_lens, gather, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ring_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        q, k, v = _global_case(5, 2, 3, max(sum(q_lens), sum(kv_lens)), 8)
        qs = np.cumsum([0] + list(q_lens))
        ks = np.cumsum([0] + list(kv_lens))
        q_r = q[:, :, qs[rank]:qs[rank + 1]].contiguous()
        k_r = k[:, :, ks[rank]:ks[rank + 1]].contiguous()
        v_r = v[:, :, ks[rank]:ks[rank + 1]].contiguous()
        trace = []
        passed = None if gather else kv_lens   # None: the ranks gather the lengths themselves
        o = torch.empty(q_r.shape, dtype=torch.float64)
        lse = torch.empty(q_r.shape[:3], dtype=torch.float64)

        def attend(qq, kk, vv, o_acc, lse_acc, first, final, out, scale):
            # the driver's running state is float32 for the kernels; here it is
            # replaced by float64 buffers of the same shape
            _oracle_fold(qq, kk, vv, o, lse, first, final, out, scale)

        out, _ = ring_attention(q_r, k_r, v_r, kv_lens=passed, scale=SCALE, out=torch.empty_like(q_r),
                                attend=attend, trace=trace)
        o_ref, l_ref = oracle.attention(q_r, k[:, :, :ks[-1]], v[:, :, :ks[-1]], SCALE)
        out_q.put((rank, float(np.abs(out.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()),
                   trace))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _oracle_part(q, k, v, o_part, lse_part, scale):
    """One block's partial (O, LSE), from the oracle."""
    o_b, l_b = oracle.attention(q, k, v, scale)
    o_part.copy_(torch.from_numpy(o_b))
    lse_part.copy_(torch.from_numpy(l_b))


def _ring_partials_rank(rank, world, port, q_lens, kv_lens, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ring_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        q, k, v = _global_case(6, 2, 3, max(sum(q_lens), sum(kv_lens)), 8)
        qs = np.cumsum([0] + list(q_lens))
        ks = np.cumsum([0] + list(kv_lens))
        q_r = q[:, :, qs[rank]:qs[rank + 1]].contiguous()
        k_r = k[:, :, ks[rank]:ks[rank + 1]].contiguous()
        v_r = v[:, :, ks[rank]:ks[rank + 1]].contiguous()
        trace, merged = [], []

        def merge(o_parts, lse_parts, out, lse):
            merged.append(o_parts.shape[0])
            o_m, l_m = oracle.merge(o_parts.numpy(), lse_parts.numpy())
            out.copy_(torch.from_numpy(o_m))
            lse.copy_(torch.from_numpy(l_m))

        out, lse = ring_attention(q_r, k_r, v_r, scale=SCALE, out=torch.empty_like(q_r), partials=True,
                                  attend_part=_oracle_part, merge=merge, trace=trace)
        o_ref, l_ref = oracle.attention(q_r, k[:, :, :ks[-1]], v[:, :, :ks[-1]], SCALE)
        out_q.put((rank, float(np.abs(out.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()),
                   trace, merged))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("q_lens,kv_lens", [((6, 6), (6, 6)), ((5, 9, 4), (7, 3, 11))])
def test_ring_attention_partials_gloo(q_lens, kv_lens):
    """The partials form of the ring (diffusers "Context parallelism", section
    "Ring Attention": once the ring has gone round, the blocks' partials
    combine into the exact result): every block's partial once, one merge of
    world-size parts, the whole-sequence attention on every rank."""
    world = len(q_lens)
    got = _run(_ring_partials_rank, world, q_lens, kv_lens)
    for rank in range(world):
        err_o, err_l, trace, merged = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert [t["block"] for t in trace] == [(rank - s) % world for s in range(world)]
        assert [t["n_keys"] for t in trace] == [kv_lens[(rank - s) % world] for s in range(world)]
        assert merged == [world]


def _subgroup_rank(rank, world, port, out_q):
    """Ranks 0 and 2 of a 3-rank world run the ring in a subgroup; rank 1 only
    joins the group creation (a collective over the world)."""
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ring_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        sub = dist.new_group([0, 2])
        if rank == 1:
            out_q.put((rank, 0.0, 0.0, []))
            return
        me = 0 if rank == 0 else 1
        q, k, v = _global_case(7, 1, 2, 10, 8)
        lens = (4, 6)
        s0 = 0 if me == 0 else 4
        sl = slice(s0, s0 + lens[me])
        o = torch.empty((1, 2, lens[me], 8), dtype=torch.float64)
        lse = torch.empty((1, 2, lens[me]), dtype=torch.float64)

        def attend(qq, kk, vv, o_acc, lse_acc, first, final, out, scale):
            _oracle_fold(qq, kk, vv, o, lse, first, final, out, scale)

        trace = []
        out, _ = ring_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), group=sub,
                                scale=SCALE, out=torch.empty_like(o), attend=attend, trace=trace)
        o_ref, l_ref = oracle.attention(q[:, :, sl], k, v, SCALE)
        out_q.put((rank, float(np.abs(out.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()), trace))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_ring_attention_in_a_subgroup():
    got = _run(_subgroup_rank, 3)
    for rank in (0, 2):
        err_o, err_l, trace = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert len(trace) == 2


def _run(target, world, *args):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r = q.get(timeout=180)
        got[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return got


def test_ring_schedule_visits_every_block_once():
    for world in (1, 2, 3, 4, 8):
        for rank in range(world):
            sched = ring_schedule(rank, world)
            assert [e["block"] for e in sched] == [(rank - s) % world for s in range(world)]
            assert sorted(e["block"] for e in sched) == list(range(world))
            for s, e in enumerate(sched[:-1]):
                # what is received at step s is what step s + 1 folds, from
                # the buffer the receive wrote
                assert e["recv_block"] == sched[s + 1]["block"]
                assert e["recv_buffer"] == sched[s + 1]["buffer"]
                # the previous rank holds that block at step s
                assert ring_schedule(e["recv_from"], world)[s]["block"] == e["recv_block"]
                assert ring_schedule(e["send_to"], world)[s]["recv_from"] == rank
            # a receive never overwrites the buffer folded at the same step
            for e in sched[1:-1]:
                assert e["recv_buffer"] != e["buffer"]


@pytest.mark.parametrize("q_lens,kv_lens,gather", [((6, 6), (6, 6), False), ((5, 9, 4), (7, 3, 11), True)])
def test_ring_attention_gloo(q_lens, kv_lens, gather):
    world = len(q_lens)
    got = _run(_ring_rank, world, q_lens, kv_lens, gather)
    for rank in range(world):
        err_o, err_l, trace = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert [t["block"] for t in trace] == [(rank - s) % world for s in range(world)]
        assert [t["n_keys"] for t in trace] == [kv_lens[(rank - s) % world] for s in range(world)]


def _ulysses_rank(rank, world, port, n, H, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ulysses_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        q, k, v = _global_case(6, 2, H, n * world, 8)
        sl = slice(rank * n, (rank + 1) * n)
        seen = []

        def attend_full(qh, kh, vh, scale):
            seen.append(tuple(qh.shape))
            o, l = oracle.attention(qh, kh, vh, scale)
            return torch.from_numpy(o), torch.from_numpy(l)

        o, lse = ulysses_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                   scale=SCALE, attend_full=attend_full)
        o_ref, l_ref = oracle.attention(q[:, :, sl], k, v, SCALE)
        out_q.put((rank, float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()), seen))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,H", [(2, 4), (3, 6)])
def test_ulysses_attention_gloo(world, H):
    n = 5
    got = _run(_ulysses_rank, world, n, H)
    for rank in range(world):
        err_o, err_l, seen = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert seen == [(2, H // world, n * world, 8)]     # its heads, the whole sequence


def _ulysses_anything_rank(rank, world, port, lens, H, gather, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import head_split, ulysses_anything_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        q, k, v = _global_case(8, 2, H, sum(lens), 8)
        off = np.cumsum([0] + list(lens))
        sl = slice(int(off[rank]), int(off[rank + 1]))
        seen = []

        def attend_full(qh, kh, vh, scale):
            seen.append(tuple(qh.shape))
            o, l = oracle.attention(qh, kh, vh, scale)
            return torch.from_numpy(o), torch.from_numpy(l)

        o, lse = ulysses_anything_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                            v[:, :, sl].contiguous(), seq_lens=None if gather else lens,
                                            scale=SCALE, attend_full=attend_full)
        o_ref, l_ref = oracle.attention(q[:, :, sl], k, v, SCALE)
        out_q.put((rank, float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()),
                   tuple(o.shape), seen, head_split(H, world)[0][rank]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("lens,H,gather", [((5, 9), 3, False), ((5, 9, 4), 5, True), ((4, 1, 7), 2, False),
                                           ((6, 6), 4, True)])
def test_ulysses_anything_attention_gloo(lens, H, gather):
    """diffusers "Context parallelism", section "Ulysses Anything": shards of
    different lengths and a head count that need not divide by the ranks
    (with 3 ranks and 2 heads one rank holds none); every rank gets its own
    queries attended over the whole sequence."""
    world = len(lens)
    got = _run(_ulysses_anything_rank, world, lens, H, gather)
    for rank in range(world):
        err_o, err_l, shape, seen, heads = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert shape == (2, H, lens[rank], 8)
        assert seen == ([(2, heads, sum(lens), 8)] if heads else [])


def _ring_anything_rank(rank, world, port, q_lens, kv_lens, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ring_anything_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        q, k, v = _global_case(10, 2, 3, max(sum(q_lens), sum(kv_lens)), 8)
        qs = np.cumsum([0] + list(q_lens))
        ks = np.cumsum([0] + list(kv_lens))
        q_r = q[:, :, qs[rank]:qs[rank + 1]].contiguous()
        k_r = k[:, :, ks[rank]:ks[rank + 1]].contiguous()
        v_r = v[:, :, ks[rank]:ks[rank + 1]].contiguous()
        seen = []

        def attend_chunks(qq, k_chunks, v_chunks, scale):
            seen.append([int(c.shape[2]) for c in k_chunks])
            assert all(c.is_contiguous() for c in k_chunks + v_chunks)
            o, l = oracle.attention(qq, torch.cat(k_chunks, dim=2), torch.cat(v_chunks, dim=2), scale)
            return torch.from_numpy(o), torch.from_numpy(l)

        o, lse = ring_anything_attention(q_r, k_r, v_r, scale=SCALE, attend_chunks=attend_chunks)
        o_ref, l_ref = oracle.attention(q_r, k[:, :, :ks[-1]], v[:, :, :ks[-1]], SCALE)
        out_q.put((rank, float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()), seen))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("q_lens,kv_lens", [((6, 6), (6, 6)), ((5, 9, 4), (7, 3, 11))])
def test_ring_anything_attention_gloo(q_lens, kv_lens):
    """diffusers "Context parallelism", section "Ring Anything Attention":
    blocks padded to the longest, all-gathered, trimmed back to their real
    lengths (padding never enters the softmax), attended as one set of
    chunks in rank order."""
    world = len(q_lens)
    got = _run(_ring_anything_rank, world, q_lens, kv_lens)
    for rank in range(world):
        err_o, err_l, seen = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)
        assert seen == [list(kv_lens)]


def _usp_rank(rank, world, port, U, n, H, partials, out_q):
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import usp_attention, usp_groups
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ug, rg = usp_groups(U)
        q, k, v = _global_case(9, 2, H, n * world, 8)
        sl = slice(rank * n, (rank + 1) * n)
        trace = []
        if partials:
            def merge(o_parts, lse_parts, out, lse):
                o_m, l_m = oracle.merge(o_parts.numpy(), lse_parts.numpy())
                out.copy_(torch.from_numpy(o_m))
                lse.copy_(torch.from_numpy(l_m))
            o, lse = usp_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                   ug, rg, scale=SCALE, trace=trace, partials=True, attend_part=_oracle_part,
                                   merge=merge)
        else:
            o, lse = usp_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                   ug, rg, scale=SCALE, attend=_oracle_fold, trace=trace)
        o_ref, l_ref = oracle.attention(q[:, :, sl], k, v, SCALE)
        out_q.put((rank, float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()),
                   [t["block"] for t in trace], dist.get_world_size(ug), dist.get_world_size(rg)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("U,partials", [(1, False), (2, False), (4, False), (2, True)])
def test_usp_attention_gloo(U, partials):
    """diffusers "Context parallelism", section "Unified Attention": 4 ranks
    as a Ulysses x ring grid (4 x 1, 2 x 2, 1 x 4); every rank gets the
    attention of its queries over the whole sequence."""
    world, n, H = 4, 3, 4
    got = _run(_usp_rank, world, U, n, H, partials)
    R = world // U
    for rank in range(world):
        err_o, err_l, blocks, u_size, r_size = got[rank]
        assert err_o < 1e-12 and err_l < 1e-12, (U, rank, err_o, err_l)
        assert (u_size, r_size) == (U, R)
        g = rank // U
        assert blocks == [(g - s) % R for s in range(R)]     # the ring runs across the groups


@pytest.mark.gpu
@pytest.mark.parametrize("partials", [False, True, "anything"])
def test_ring_attention_one_rank_library_kernels(partials):
    """A one-rank group on the GPU: ring_attention with the library's own
    step (the fp32 fold, or a block partial), and ring_anything_attention
    with the fused chunk launch, against the oracle."""
    import torch.distributed as dist
    from context_blocks_b200.context_parallel import ring_anything_attention, ring_attention
    from tests._parity import assert_close
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        g = torch.Generator(device="cuda").manual_seed(31)
        q, k, v = (torch.randn((1, 3, n, 128), generator=g, device="cuda").to(torch.bfloat16)
                   for n in (300, 517, 517))
        scale = 128 ** -0.5   # the bars of the GPU parity tests are set for 1/sqrt(d)
        if partials == "anything":
            o, lse = ring_anything_attention(q, k, v, kv_lens=[517], scale=scale)
        else:
            o, lse = ring_attention(q, k, v, kv_lens=[517], scale=scale, partials=partials)
        torch.cuda.synchronize()
        o_ref, l_ref = oracle.attention(q.cpu(), k.cpu(), v.cpu(), scale)
        assert_close(o, lse, o_ref, l_ref, f"ring one rank, partials={partials}")
    finally:
        dist.destroy_process_group()


def test_head_split_covers_every_head_once():
    from context_blocks_b200.context_parallel import head_split
    for H in range(1, 30):
        for P in range(1, 9):
            sizes, starts = head_split(H, P)
            assert sum(sizes) == H and len(sizes) == P
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
            assert starts == [sum(sizes[:r]) for r in range(P)]
