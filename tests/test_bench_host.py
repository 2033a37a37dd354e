"""Host-side logic of bench.py on the CPU: aggregation, the max over ranks
on a two-rank gloo group, the workloads, and the reference (oracle) arm."""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_aggregate_throughput():
    # 2 ranks, 10 steps of 1e12 FLOPs each, slowest rank 20 ms -> 1000 TFLOPS
    assert bench.aggregate_throughput(1e12, 10, 2, 20.0) == pytest.approx(1000.0)


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    v = bench.max_over_ranks(10.0 + rank)
    out_q.put((rank, v))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 11.0, 1: 11.0}


def test_workloads_shapes_and_determinism():
    w = workloads.get("tiny")
    q1, k1, v1 = workloads.make_case(w)
    q2, k2, v2 = workloads.make_case(w)
    assert q1.shape == (1, 2, 256, 64) and q1.dtype == torch.bfloat16 and q1.is_contiguous()
    assert torch.equal(q1, q2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    q3, _, _ = workloads.make_case(w, seed=99)
    assert not torch.equal(q1, q3)


def test_workloads_rms_normalised():
    w = workloads.Workload("t", B=1, H=2, Nq=50, Nk=40, d=128, rms_qk=True, chunks=(40,), seed=5)
    q, k, v = workloads.make_case(w)
    rq = q.float().pow(2).mean(-1).sqrt()
    rk = k.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rq, torch.ones_like(rq), atol=1e-2)
    assert torch.allclose(rk, torch.ones_like(rk), atol=1e-2)
    rv = v.float().pow(2).mean(-1).sqrt()
    assert rv.std() > 0.02                     # V is not normalised


def test_workload_table_matches_spec():
    f = workloads.get("flux")
    assert (f.B, f.H, f.Nq, f.Nk, f.d, f.chunks) == (1, 24, 4608, 4608, 128, (4608,))
    r = workloads.get("ring")
    assert (r.Nq, r.Nk, r.chunks) == (1152, 4608, (1152,) * 4)
    t = workloads.get("tails")
    assert (t.B, t.Nq, sum(t.chunks), t.chunks) == (2, 4603, 4603, (1151, 1151, 1151, 1150))
    h = workloads.get("hunyuan")
    assert h.Nq == 33 * 45 * 80 + 256 and sum(workloads.HUNYUAN_CHUNKS8) == h.Nk
    h8 = workloads.get("hunyuan8")
    assert h8.chunks == workloads.HUNYUAN_CHUNKS8 and (h8.Nq, h8.seed) == (h.Nq, h.seed)
    a = workloads.get("flux1008")
    assert a.Nq == 63 * 63 + 512 and a.chunks == (1121, 1121, 1121, 1118)
    for w in workloads.WORKLOADS.values():
        assert sum(w.chunks) == w.Nk


def test_split_keys_and_rows():
    k = torch.arange(2 * 3 * 10 * 4, dtype=torch.float32).view(2, 3, 10, 4)
    parts = workloads.split_keys(k, k + 1, [3, 7])
    assert [p[0].shape[2] for p in parts] == [3, 7]
    assert all(p[0].is_contiguous() for p in parts)
    assert torch.equal(torch.cat([p[0] for p in parts], dim=2), k)
    with pytest.raises(ValueError):
        workloads.split_keys(k, k, [3, 3])
    rows = workloads.sample_rows(1000, 256, seed=4)
    assert len(np.unique(rows)) == 256 and rows.min() >= 0 and rows.max() < 1000
    assert np.array_equal(rows, workloads.sample_rows(1000, 256, seed=4))


def test_flop_and_byte_counts():
    assert workloads.flops(1, 24, 4608, 4608, 128) == pytest.approx(2.609e11, rel=1e-3)
    assert workloads.fwd_bytes(1, 24, 4608, 4608, 128) == pytest.approx(113.7e6, rel=1e-2)


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600, cwd=ROOT)


def test_reference_arm_prints_contract_line():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3",
                    "--cpu-budget", "2"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOPS"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_nonzero_rank_exits_quietly():
    r = _run_bench(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_heads_override_keeps_the_sequence_shape():
    import argparse
    import bench
    w = bench._workload(argparse.Namespace(workload="hunyuan", heads=4))
    h = workloads.get("hunyuan")
    assert (w.H, w.Nq, w.Nk, w.d, w.chunks) == (4, h.Nq, h.Nk, h.d, h.chunks)
    assert bench._workload(argparse.Namespace(workload="flux", heads=None)) == workloads.get("flux")


def test_ring_shard_sizes_cover_the_sequence():
    for n, world in ((119056, 8), (4608, 3), (4481, 4), (5, 8), (7, 1)):
        sizes = bench.shard_sizes(n, world)
        assert len(sizes) == world and sum(sizes) == n
        assert max(sizes) - min(sizes) <= 1
        assert sizes == sorted(sizes, reverse=True)


def test_peaks_file_nested_missing_and_absent(tmp_path, monkeypatch):
    """The peak figures come from MEASURED_PEAKS.json at any nesting; a file
    without them, or no file, falls back to the recipe's figures and says so."""
    import json
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench._peaks()
    assert p["source"] == "fallback" and p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert "absent" in bench._basis(p)
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"box": {"hbm_gbs": 6547.5, "gemm": {"bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4}}}))
    p = bench._peaks()
    assert p == {"hbm_gbs": 6547.5, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4, "source": "measured"}
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6547.5}))
    p = bench._peaks()
    assert p["source"] == "unreadable" and "present" in bench._basis(p)
