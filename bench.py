"""Benchmark of the blockwise attention library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload hunyuan] [--no-extra] [--no-cpu-baseline]

One step is one pass of the hot path over one batch of the named workload:
``pa_attn_fwd`` over each K/V chunk, then ``pa_attn_merge`` when the workload
has more than one chunk.  The default workload is the largest one-GPU
configuration, the HunyuanVideo-shaped attention (B=1, H=24,
Nq=Nk=119056, d=128, one chunk); the FLUX-shaped one is reported among the
extras.  The metric is attention forward TFLOPS, 4*B*H*Nq*Nk*d per step over
the device time.

Multi-GPU: one process per GPU (torchrun).  By default (``--parallel ring``)
the ranks run Ring Attention over the named workload (diffusers "Context
parallelism", section "Ring Attention"): each rank holds 1/N of the query
rows and of the K/V rows and attends to each K/V block while the next one
arrives from the previous rank over NCCL on a second stream: with the default
``--mode chunks`` each block's partial comes from ``pa_attn_fwd`` and one
``pa_attn_merge`` combines them after the last block; with ``--mode fold``
each block is folded into an fp32 running state by ``pa_attn_fwd_accum``.
The whole problem is fixed as N grows, so scaling is strong.  ``--parallel replicas`` runs an independent copy of the
single-GPU step on every rank instead (weak scaling, no data-path
collective).  Either way the process group provides the barrier and the max
over ranks of the timed region.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
on a bounded sample of the same workload instead (the reference arm).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "attention fwd TFLOPS (4·B·H·Nq·Nk·d/s) on 1 B200 and % of bf16 dense peak"
UNIT = "TFLOPS"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of one attn_fwd launch (dram__bytes_read.sum +
# dram__bytes_write.sum) from ncu captures, valid only for the kernel source
# whose digest is recorded with them.  The HunyuanVideo figure is a 4-head
# capture of the same sequence shape scaled to 24 heads (every head's items
# are alike, so traffic grows in proportion to heads).  See profiles/.
NCU_TRAFFIC = {
    "source_sha256": "4f469c18af13c656294c5af86d9ef3facfc6f018fbf1d7c157a1d0fd32d30cbc",
    "bytes_per_launch": {
        "hunyuan": (967502080 + 120467712) * 24 // 4,
        "flux": 84987904 + 5317632,
    },
    "capture": {
        "hunyuan": "ncu --set full, bench.py --heads 4 --steps 3 --warmup 3 --no-extra --no-cpu-baseline, x 24/4",
        "flux": "ncu --set full, bench.py --workload flux --steps 20 --warmup 5 --no-extra --no-cpu-baseline",
    },
}


def _kernel_digest() -> str:
    """SHA-256 of the forward kernel's code (comments and whitespace removed),
    so that a recorded ncu traffic figure is used only for the code it was
    measured on."""
    import re
    h = hashlib.sha256()
    for f in ("ptx.cuh", "fwd_common.cuh", "attn_fwd.cuh"):
        with open(os.path.join(ROOT, "context_blocks_b200", "csrc", f)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("".join(src.split()).encode())
    return h.hexdigest()


def _workload(args):
    """The named workload, with H replaced by --heads when given (a smaller
    case of the same sequence shape, for profiler captures)."""
    import dataclasses
    w = workloads.get(args.workload)
    if getattr(args, "heads", None):
        w = dataclasses.replace(w, H=int(args.heads))
    return w


def _basis(peaks) -> str:
    """Where the peak figures came from, for the JSON line."""
    if peaks["source"] == "measured":
        return "measured burst bf16 (MEASURED_PEAKS.json bf16_tflops)"
    if peaks["source"] == "unreadable":
        return "fallback burst bf16 of the profiling recipe (MEASURED_PEAKS.json present, without hbm_gbs / bf16_tflops)"
    return "fallback burst bf16 of the profiling recipe (MEASURED_PEAKS.json absent on this machine)"


def _find_key(d, key):
    """The first value stored under `key` in a JSON object, searching nested
    objects breadth-first (the file's exact nesting is not fixed here)."""
    todo = [d]
    while todo:
        x = todo.pop(0)
        if isinstance(x, dict):
            if key in x and isinstance(x[key], (int, float)):
                return float(x[key])
            todo.extend(x.values())
        elif isinstance(x, list):
            todo.extend(x)
    return None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return dict(FALLBACK_PEAKS, source="fallback")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return dict(FALLBACK_PEAKS, source="unreadable")
    hbm, bf16 = _find_key(d, "hbm_gbs"), _find_key(d, "bf16_tflops")
    if hbm is None or bf16 is None or hbm <= 0 or bf16 <= 0:
        return dict(FALLBACK_PEAKS, source="unreadable")
    sus = _find_key(d, "bf16_tflops_sustained")
    return {"hbm_gbs": hbm, "bf16_tflops": bf16, "bf16_tflops_sustained": sus if sus and sus > 0 else bf16,
            "source": "measured"}


# --------------------------------------------------------------------- clocks

_REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
            (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
            (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
            (0x100, "display_clock_setting")]


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)
    from a thread while the timed region runs."""

    def __init__(self, torch_device: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            # NVML counts physical GPUs; match torch's device by UUID.
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML here
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, int(reasons)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [name for bit, name in _REASONS if mask & bit]
        mhz = [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# --------------------------------------------------------------- distributed

def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the default process group (identity
    when no group is initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(flops_per_step_per_rank: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOPS: the FLOPs all ranks processed over the slowest
    rank's timed region."""
    return flops_per_step_per_rank * steps * world / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ our arm

class Step:
    """Buffers and launches of one hot-path step on one workload.  A chunked
    workload runs in `mode`: ``chunks`` (pa_attn_fwd per chunk, then
    pa_attn_merge), ``fused`` (one pa_attn_fwd_chunks launch) or ``fold``
    (pa_attn_fwd_accum per chunk into an fp32 running state)."""

    def __init__(self, w: workloads.Workload, sets: int, device, fp8: bool = False, pa=None, mode: str = "chunks"):
        import torch
        self.w = w
        self.fp8 = fp8
        self.mode = mode
        self.sets = []
        n = len(w.chunks)
        if fp8 and n != 1:
            raise SystemExit("--fp8 times the single-chunk e4m3 forward: pick a one-chunk workload")
        if mode == "fused" and n > 8:
            raise SystemExit("--mode fused takes at most 8 chunks")
        for s in range(sets):
            q, k, v = workloads.make_case(w, device=device, seed=w.seed + 1000 * s)
            if fp8:
                # per-tensor e4m3 inputs made by the library's own quantiser
                # (outside the timed region), scales left in device memory
                qs, ks, vs = pa.quantize_e4m3(q), pa.quantize_e4m3(k), pa.quantize_e4m3(v)
                o = torch.empty_like(q)
                lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
                self.sets.append((qs, [(ks, vs)], o, lse, None, None))
                del q, k, v
                continue
            pairs = workloads.split_keys(k, v, w.chunks)
            del k, v
            o = torch.empty_like(q)
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=device)
            o_parts = lse_parts = None
            if n > 1 and mode == "chunks":
                o_parts = torch.empty((n,) + tuple(q.shape), dtype=torch.bfloat16, device=device)
                lse_parts = torch.empty((n,) + tuple(q.shape[:3]), dtype=torch.float32, device=device)
            if mode == "fold":  # the fp32 running state (O; LSE goes to `lse`)
                o_parts = torch.empty(q.shape, dtype=torch.float32, device=device)
            self.sets.append((q, pairs, o, lse, o_parts, lse_parts))
        self.launches_per_step = {"chunks": n + (1 if n > 1 else 0), "fused": 1, "fold": n}[mode]

    def bytes_resident(self) -> int:
        tot = 0
        if self.fp8:
            for (q8, _), [((k8, _), (v8, _))], o, lse, _, _ in self.sets:
                tot += q8.numel() + k8.numel() + v8.numel() + o.numel() * 2 + lse.numel() * 4
            return tot
        for q, pairs, o, lse, op, lp in self.sets:
            tot += q.numel() * 2 + sum(k.numel() * 4 for k, _ in pairs) + o.numel() * 2 + lse.numel() * 4
            if op is not None:
                tot += op.numel() * op.element_size() + (lp.numel() * 4 if lp is not None else 0)
        return tot

    def run(self, i: int, pa, fwd_events=None, merge_events=None):
        if self.fp8:
            (q8, sq), [((k8, sk), (v8, sv))], o, lse, _, _ = self.sets[i % len(self.sets)]
            if fwd_events is not None:
                fwd_events[0].append(_record())
            pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=self.w.scale, out=o, lse=lse)
            if fwd_events is not None:
                fwd_events[1].append(_record())
            return
        q, pairs, o, lse, o_parts, lse_parts = self.sets[i % len(self.sets)]
        n = len(pairs)
        if self.mode == "fused":
            if fwd_events is not None:
                fwd_events[0].append(_record())
            pa.attn_fwd_chunks(q, [k for k, _ in pairs], [v for _, v in pairs], scale=self.w.scale, out=o, lse=lse)
            if fwd_events is not None:
                fwd_events[1].append(_record())
            return
        if self.mode == "fold":
            for p, (k, v) in enumerate(pairs):
                if fwd_events is not None:
                    fwd_events[0].append(_record())
                pa.attn_fwd_accum(q, k, v, o_parts, lse, first=(p == 0), final=(p == n - 1),
                                  out=o if p == n - 1 else None, scale=self.w.scale)
                if fwd_events is not None:
                    fwd_events[1].append(_record())
            return
        for p, (k, v) in enumerate(pairs):
            out = o if n == 1 else o_parts[p]
            ls = lse if n == 1 else lse_parts[p]
            if fwd_events is not None:
                fwd_events[0].append(_record())
            pa.attn_fwd(q, k, v, scale=self.w.scale, out=out, lse=ls)
            if fwd_events is not None:
                fwd_events[1].append(_record())
        if n > 1:
            if merge_events is not None:
                merge_events[0].append(_record())
            pa.attn_merge(o_parts, lse_parts, out=o, lse=lse)
            if merge_events is not None:
                merge_events[1].append(_record())


_EVENT_POOL = []


def _record():
    """Record a timing event on the current stream.  Events come from a pool
    made before the timed region (_event_pool), so that creating them does
    not add host time between the launches being timed."""
    import torch
    e = _EVENT_POOL.pop() if _EVENT_POOL else torch.cuda.Event(enable_timing=True)
    e.record()
    return e


def _event_pool(n: int) -> None:
    import torch
    _EVENT_POOL[:] = [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _sets_for(w: workloads.Workload, fp8: bool = False) -> int:
    per_set = workloads.fwd_bytes(w.B, w.H, w.Nq, w.Nk, w.d)
    if fp8:  # Q, K, V at one byte per element
        per_set -= (w.Nq + 2 * w.Nk) * w.d * w.B * w.H
    return max(1, min(8, math.ceil(2.5 * L2_BYTES / per_set)))


def time_workload(pa, w, steps, warmup, device, sampler=None, barrier=None, fp8=False, mode="chunks"):
    """Device time of `steps` steps (CUDA events on the launching stream,
    synchronised on both sides).  Returns a dict of timings."""
    import torch
    st = Step(w, _sets_for(w, fp8), device, fp8=fp8, pa=pa, mode=mode)
    for i in range(warmup):
        st.run(i, pa)
    torch.cuda.synchronize()
    fwd_ev = ([], [])
    mrg_ev = ([], [])
    _event_pool(2 * steps * st.launches_per_step)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        start.record()
        for i in range(steps):
            st.run(i, pa, fwd_ev, mrg_ev)
        end.record()
        torch.cuda.synchronize()
    if barrier:
        barrier()
    total_ms = start.elapsed_time(end)
    fwd_ms = [a.elapsed_time(b) for a, b in zip(*fwd_ev)]
    mrg_ms = [a.elapsed_time(b) for a, b in zip(*mrg_ev)]
    status = pa.poll_device_status()
    res = {"total_ms": total_ms, "fwd_ms": fwd_ms, "merge_ms": mrg_ms,
           "launches": steps * st.launches_per_step, "sets": len(st.sets),
           "resident_mb": st.bytes_resident() / 1e6, "status": status}
    del st
    torch.cuda.empty_cache()
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def e2e_throughput(pa, w, steps, device, fp8: bool = False, mode: str = "chunks"):
    """Same metric through the public API from pinned HOST buffers: every
    step copies q and the K/V chunks host->device, runs the step, and copies
    o and lse device->host; all inside the timed region.

    Steps alternate between two CUDA streams, each with its own device and
    output buffers, so one step's host->device copy overlaps the previous
    step's attention and device->host copy (the copy engines of the two
    directions and the SMs work at the same time).  Each step still moves
    all of its own bytes.  With fp8 the host holds e4m3 codes (quantised once
    by the library, scales kept on the device) and each step uploads those.
    A chunked workload runs in `mode`, as the device-timed step does."""
    import torch
    q, k, v = workloads.make_case(w, device=device)
    B, H, Nq, d = q.shape
    if fp8:
        quant = [pa.quantize_e4m3(x) for x in (q, k, v)]
        host_in = [x8.view(torch.uint8).cpu().pin_memory() for x8, _ in quant]
        scales = [sc for _, sc in quant]
        del quant
    else:
        pairs = workloads.split_keys(k, v, w.chunks)
        host_in = [q.cpu().pin_memory()] + [t.cpu().pin_memory() for pr in pairs for t in pr]
        del pairs
    n = len(w.chunks)
    del k, v

    class Lane:
        def __init__(self):
            self.stream = torch.cuda.Stream(device=device)
            self.dev_in = [torch.empty(h.shape, dtype=h.dtype, device=device) for h in host_in]
            self.o_parts = (torch.empty((n, B, H, Nq, d), dtype=torch.bfloat16, device=device)
                            if n > 1 and mode == "chunks" else None)
            self.lse_parts = (torch.empty((n, B, H, Nq), dtype=torch.float32, device=device)
                              if n > 1 and mode == "chunks" else None)
            self.o_acc = torch.empty((B, H, Nq, d), dtype=torch.float32, device=device) if mode == "fold" else None
            self.o = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=device)
            self.lse = torch.empty((B, H, Nq), dtype=torch.float32, device=device)
            self.ho = torch.empty(self.o.shape, dtype=self.o.dtype, pin_memory=True)
            self.hl = torch.empty(self.lse.shape, dtype=self.lse.dtype, pin_memory=True)

        def step(self):
            with torch.cuda.stream(self.stream):
                for dv, hv in zip(self.dev_in, host_in):
                    dv.copy_(hv, non_blocking=True)
                if fp8:
                    q8, k8, v8 = (t.view(torch.float8_e4m3fn) for t in self.dev_in)
                    pa.attn_fwd_fp8(q8, k8, v8, *scales, scale=w.scale, out=self.o, lse=self.lse,
                                    stream=self.stream)
                else:
                    dq, rest = self.dev_in[0], self.dev_in[1:]
                    ks, vs = rest[0::2], rest[1::2]
                    if mode == "fused":
                        pa.attn_fwd_chunks(dq, ks, vs, scale=w.scale, out=self.o, lse=self.lse, stream=self.stream)
                    elif mode == "fold":
                        for c in range(n):
                            pa.attn_fwd_accum(dq, ks[c], vs[c], self.o_acc, self.lse, first=(c == 0),
                                              final=(c == n - 1), out=self.o if c == n - 1 else None,
                                              scale=w.scale, stream=self.stream)
                    else:
                        pa.blockwise_attention(dq, ks, vs, scale=w.scale, o_parts=self.o_parts,
                                               lse_parts=self.lse_parts, out=self.o, lse=self.lse,
                                               stream=self.stream)
                self.ho.copy_(self.o, non_blocking=True)
                self.hl.copy_(self.lse, non_blocking=True)

    lanes = [Lane(), Lane()]
    del q
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = lanes[0].ho.numel() * 2 + lanes[0].hl.numel() * 4

    for i in range(2):
        lanes[i % 2].step()
    torch.cuda.synchronize()
    main = torch.cuda.current_stream(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(main)
    for ln in lanes:
        ln.stream.wait_event(t0)
    for i in range(steps):
        lanes[i % 2].step()
    for ln in lanes:
        main.wait_stream(ln.stream)
    t1.record(main)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    fl = workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d)
    return {"value": fl * steps / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps, "ms_per_step": ms / steps,
            "pipelining": "2 streams, double-buffered device tensors", "mode": mode}


# ------------------------------------------------------------ CPU (oracle) leg

def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 0) for i in info), default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(w, seconds: float, seed_rows: int = 0):
    """Time the oracle on a bounded sample of workload `w`: all heads and
    batches, a prefix of `rows` query rows, every key of every chunk, chunks
    merged as the GPU path does.  Rows are chosen from a short calibration
    so that the sample takes about `seconds`.  Returns (tflops, seconds,
    rows, description)."""
    import numpy as np
    import oracle
    q, k, v = workloads.make_case(w, device="cpu", nq=min(w.Nq, 4096))
    qn = q.double().numpy()
    kn, vn = k.double().numpy(), v.double().numpy()

    def run(rows):
        t0 = time.perf_counter()
        qq = np.ascontiguousarray(np.resize(qn, (w.B, w.H, rows, w.d))) if rows > qn.shape[2] else qn[:, :, :rows]
        if len(w.chunks) == 1:
            oracle.attention(qq, kn, vn, w.scale)
        else:
            oracle.chunked_attention(qq, kn, vn, w.scale, w.chunks)
        return time.perf_counter() - t0

    # Two calibration passes: a short one, then one of about a tenth of the
    # budget, so per-call overhead does not skew the row count.
    rows = min(w.Nq, 8)
    for frac in (0.01, 0.1):
        t_cal = max(run(rows), 1e-4)
        rows = int(max(1, min(w.Nq, rows * frac * seconds / t_cal)))
    t_cal = max(run(rows), 1e-4)
    rows = int(max(1, min(w.Nq, rows * seconds / t_cal)))
    t = run(rows)
    while t < 0.6 * seconds and rows < w.Nq:     # time is not quite linear in rows
        rows = int(min(w.Nq, rows * seconds / max(t, 1e-4)))
        t = run(rows)
    fl = workloads.flops(w.B, w.H, rows, w.Nk, w.d)
    desc = (f"{w.name}: all {w.B}x{w.H} (batch x head) of {rows} query rows x {w.Nk} keys"
            f"{' in ' + str(len(w.chunks)) + ' chunks + merge' if len(w.chunks) > 1 else ''}, fp64 NumPy")
    return fl / t / 1e12, t, rows, desc


# --------------------------------------------------------------------- main

def _config(w, sets=None, resident_mb=None, parallelism="one GPU"):
    c = {"workload": f"{w.name}: B={w.B} H={w.H} Nq={w.Nq} Nk={w.Nk} d={w.d}, "
                     f"{len(w.chunks)} K/V chunk(s) {list(w.chunks) if len(w.chunks) > 1 else ''}".strip(),
         "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d, "chunks": list(w.chunks),
         "parallelism": parallelism}
    if sets is not None:
        c["l2"] = (f"inputs rotate over {sets} seeded sets, {resident_mb:.0f} MB resident "
                   f"> 126 MB L2, so no step reads the previous step's inputs from L2")
    return c


def run_reference(args):
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    w = _workload(args)
    total_budget = args.cpu_budget
    per_step = max(0.02, total_budget / max(1, args.steps + args.warmup))
    tflops_cal, t_cal, rows, desc = oracle_sample(w, per_step)
    fl_step = workloads.flops(w.B, w.H, rows, w.Nk, w.d)
    import numpy as np
    import oracle
    q, k, v = workloads.make_case(w, device="cpu", nq=min(w.Nq, max(rows, 1)))
    qn, kn, vn = q.double().numpy(), k.double().numpy(), v.double().numpy()
    qn = np.ascontiguousarray(np.resize(qn, (w.B, w.H, rows, w.d))) if rows > qn.shape[2] else qn[:, :, :rows]

    def step():
        if len(w.chunks) == 1:
            oracle.attention(qn, kn, vn, w.scale)
        else:
            oracle.chunked_attention(qn, kn, vn, w.scale, w.chunks)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = fl_step * args.steps / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    ws, rank, local = _dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    barrier = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        barrier = lambda: dist.barrier(device_ids=[local])  # noqa: E731
    from context_blocks_b200 import build
    if rank == 0:
        build.build()
    if barrier:
        barrier()
    import context_blocks_b200 as pa
    pa.load_library()

    w = _workload(args)
    peaks = _peaks()
    sampler = ClockSampler(local)
    fp8 = bool(getattr(args, "fp8", False))
    if ws > 1 and args.parallel in ("ring", "ulysses", "usp", "ring_anything"):
        return run_ring(args, pa, w, peaks, sampler, device, barrier, ulysses=(args.parallel == "ulysses"),
                        usp_degree=(args.ulysses_degree if args.parallel == "usp" else 0),
                        gather=(args.parallel == "ring_anything"))
    mode = args.mode if len(w.chunks) > 1 else "chunks"
    res = time_workload(pa, w, args.steps, args.warmup, device, sampler=sampler, barrier=barrier, fp8=fp8, mode=mode)
    if res["status"] != 0:
        raise SystemExit(f"device status {res['status']} after the timed region")
    max_ms = max_over_ranks(res["total_ms"], device)
    fl = workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d)
    value = aggregate_throughput(fl, args.steps, ws, max_ms)

    # Roofline of the dominant kernel (attn_fwd): algorithmic FLOPs per launch
    # over its mean launch duration, against the measured bf16 dense peak.
    fwd_mean_ms = statistics.fmean(res["fwd_ms"])
    fl_launch = fl if mode == "fused" else fl / len(w.chunks)
    achieved = fl_launch / (fwd_mean_ms * 1e-3) / 1e12
    traffic = None
    if (not fp8 and len(w.chunks) == 1 and w.name in NCU_TRAFFIC["bytes_per_launch"]
            and w.H == workloads.get(w.name).H and NCU_TRAFFIC["source_sha256"] == _kernel_digest()):
        traffic = NCU_TRAFFIC["bytes_per_launch"][w.name]
    # e4m3 contractions: the measured bf16 peak times the nominal e4m3/bf16 ratio of 2
    peak = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
    alg_bytes = workloads.fwd_bytes(w.B, w.H, w.Nq, w.Nk if mode == "fused" else w.Nk // len(w.chunks), w.d)
    if mode == "fold":  # the fp32 running state read and written
        alg_bytes += 8 * w.B * w.H * w.Nq * w.d
    if fp8:
        alg_bytes -= (w.Nq + 2 * (w.Nk // len(w.chunks))) * w.d * w.B * w.H
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic,
            "kernel": (f"attn_fwd_kernel<{w.d}, {'true' if fp8 else 'false'}, {'true' if mode == 'fold' else 'false'}>"
                       + {"chunks": "", "fused": f" over a table of {len(w.chunks)} chunks",
                          "fold": " (accumulate mode)"}[mode]), "launch_ms": fwd_mean_ms,
            "peak_basis": (_basis(peaks)
                           + (" x 2, the nominal e4m3/bf16 ratio" if fp8 else "")
                           + f"; frac of sustained {achieved / (peak * peaks['bf16_tflops_sustained'] / peaks['bf16_tflops']):.3f}"),
            "algorithmic_bytes_per_launch": alg_bytes}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": dict(_config(w, res["sets"], res["resident_mb"], "replicas (one independent step per GPU)"
                                   if ws > 1 else "one GPU"), mode=mode),
            ("pct_of_e4m3_peak" if fp8 else "pct_of_bf16_peak"): 100.0 * (value / ws) / peak,
            "roofline": roof, "clocks": sampler.summary(), "gpu_launches": res["launches"]}
    if res["merge_ms"]:
        mb = workloads.merge_bytes(len(w.chunks), w.B, w.H, w.Nq, w.d)
        line["merge"] = {"launch_ms": statistics.fmean(res["merge_ms"]),
                         "gbs": mb / (statistics.fmean(res["merge_ms"]) * 1e-3) / 1e9,
                         "peak_gbs": peaks["hbm_gbs"]}

    if rank == 0 or ws > 1:
        line["e2e"] = e2e_throughput(pa, w, steps=max(3, min(args.steps, 20)), device=device, fp8=fp8, mode=mode)
        if ws > 1:
            line["e2e"]["value"] = max_over_ranks(-line["e2e"]["value"], device) * -1 * ws

    if ws == 1 and not args.no_extra:
        line["extra"] = extra_measurements(pa, device, peaks)
    if ws == 1 and not args.no_cpu_baseline:
        tf, t, rows, desc = oracle_sample(w, seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
                                "sample": desc, "seconds": t}
    if barrier:
        barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def shard_sizes(n: int, world: int):
    """Sequence shard lengths of n rows over `world` ranks (the first n %
    world ranks take one row more)."""
    return [n // world + (1 if r < n % world else 0) for r in range(world)]


def _ring_how(partials: bool) -> str:
    return ("; per-block partials (pa_attn_fwd) + one pa_attn_merge" if partials
            else "; per-block folds into an fp32 state (pa_attn_fwd_accum)")


def run_ring(args, pa, w, peaks, sampler, device, barrier, ulysses=False, usp_degree=0, gather=False):
    """Context parallelism over the process group: rank r holds shard r of
    the query rows and of the K/V rows of workload `w` and runs
    context_parallel.ring_attention (or, with ``ulysses``, the all-to-all
    form, which needs equal shards and heads divisible by the rank count; or,
    with ``usp_degree`` U > 0, the Ulysses x ring grid of usp_attention, which
    needs equal shards and heads divisible by U).  Value = the whole
    problem's FLOPs per step over the slowest rank's time (strong scaling)."""
    import dataclasses

    import torch
    import torch.distributed as dist
    from context_blocks_b200 import context_parallel as cp

    ws, rank = dist.get_world_size(), dist.get_rank()
    nq_all, nk_all = shard_sizes(w.Nq, ws), shard_sizes(w.Nk, ws)
    if ulysses and nq_all != nk_all:
        raise SystemExit("--parallel ulysses needs Nq = Nk: each rank holds the same tokens of q, k and v")
    # Shards of different lengths or heads that do not divide over the ranks:
    # Ulysses Anything (per-peer pieces of different sizes in the all-to-alls).
    anything = ulysses and (len(set(nq_all)) > 1 or w.H % ws != 0)
    if usp_degree and (len(set(nq_all)) > 1 or nq_all != nk_all or w.H % usp_degree or ws % usp_degree):
        raise SystemExit(f"--parallel usp needs Nq = Nk divisible by {ws}, and heads and {ws} ranks divisible by "
                         f"the Ulysses degree {usp_degree}")
    if args.mode == "fused" and not ulysses and not gather:
        raise SystemExit("--mode fused is a one-GPU mode: the ring's blocks arrive one at a time")
    partials = not ulysses and not gather and args.mode == "chunks"
    groups = cp.usp_groups(usp_degree) if usp_degree else None
    ring_len = ws // usp_degree if usp_degree else ws
    wr = dataclasses.replace(w, Nq=nq_all[rank], Nk=nk_all[rank], chunks=(nk_all[rank],), seed=w.seed + 100 * rank)
    q, k, v = workloads.make_case(wr, device=device)
    out = torch.empty_like(q)
    comm = torch.cuda.Stream(device=device)
    fwd_ev = ([], [])

    def attend_timed(qq, kk, vv, o_acc, lse_acc, first, final, o, scale):
        fwd_ev[0].append(_record())
        pa.attn_fwd_accum(qq, kk, vv, o_acc, lse_acc, first=first, final=final, out=o, scale=scale)
        fwd_ev[1].append(_record())

    def attend_part_timed(qq, kk, vv, o_part, lse_part, scale):
        fwd_ev[0].append(_record())
        pa.attn_fwd(qq, kk, vv, scale=scale, out=o_part, lse=lse_part)
        fwd_ev[1].append(_record())

    def attend_chunks_timed(qq, kcs, vcs, scale):
        fwd_ev[0].append(_record())
        res = cp._default_attend_chunks(qq, kcs, vcs, scale)
        fwd_ev[1].append(_record())
        return res

    def attend_full_timed(qq, kk, vv, scale):
        fwd_ev[0].append(_record())
        res = pa.attn_fwd(qq, kk, vv, scale=scale)
        fwd_ev[1].append(_record())
        return res

    def step(timed=False):
        if gather:
            return cp.ring_anything_attention(q, k, v, kv_lens=nk_all, scale=w.scale,
                                              attend_chunks=attend_chunks_timed if timed else None)
        if anything:
            return cp.ulysses_anything_attention(q, k, v, seq_lens=nq_all, scale=w.scale,
                                                 attend_full=attend_full_timed if timed else None)
        if ulysses:
            return cp.ulysses_attention(q, k, v, scale=w.scale, attend_full=attend_full_timed if timed else None)
        if usp_degree:
            return cp.usp_attention(q, k, v, groups[0], groups[1], scale=w.scale, comm_stream=comm,
                                    attend=attend_timed if timed else None, partials=partials,
                                    attend_part=attend_part_timed if timed else None)
        return cp.ring_attention(q, k, v, kv_lens=nk_all, scale=w.scale, out=out, comm_stream=comm,
                                 attend=attend_timed if timed else None, partials=partials,
                                 attend_part=attend_part_timed if timed else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        t0.record()
        for _ in range(args.steps):
            step(timed=True)
        t1.record()
        torch.cuda.synchronize()
    barrier()
    status = pa.poll_device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the timed region")
    max_ms = max_over_ranks(t0.elapsed_time(t1), device)
    fl = workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d)
    value = fl * args.steps / (max_ms * 1e-3) / 1e12
    fwd_ms = [a.elapsed_time(b) for a, b in zip(*fwd_ev)]
    # the forward kernel (the fold, or the plain forward of a block's partial):
    # this rank's FLOPs per ring pass over its launches; with Ulysses, its
    # heads over the whole sequence
    fl_rank = (workloads.flops(w.B, cp.head_split(w.H, ws)[0][rank], w.Nq, w.Nk, w.d) if ulysses
               else workloads.flops(w.B, w.H, nq_all[rank], w.Nk, w.d))
    # (a Ulysses Anything rank that holds no head launches nothing)
    launch_ms = statistics.fmean(fwd_ms) if fwd_ms else 0.0
    # ring: one fold launch per block, 1/ws of the rank's FLOPs each; Ulysses:
    # one launch over the rank's heads and the whole sequence; USP: one fold
    # per ring step, 1/ring_len of the rank's FLOPs each
    achieved = ((fl_rank if ulysses or gather else fl_rank / ring_len) / (launch_ms * 1e-3) / 1e12
                if launch_ms > 0 else 0.0)
    peak = peaks["bf16_tflops"]
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": None,
            "kernel": f"attn_fwd_kernel<{w.d}, false, {'false' if ulysses or partials or gather else 'true'}>",
            "launch_ms": launch_ms,
            "peak_basis": f"{_basis(peaks)}, rank {rank}"}
    # End to end: each step uploads this rank's shards from pinned host
    # memory, runs the ring, downloads this rank's output and LSE.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hl = torch.empty(out.shape[:3], dtype=torch.float32, pin_memory=True)
    e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        o, lse = step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(_config(w, parallelism=(f"Ulysses Anything attention over {ws} ranks (two NCCL all-to-alls "
                                                   f"with per-peer pieces; uneven shards or heads)" if anything
                                                   else f"Ulysses attention over {ws} ranks (two NCCL all-to-alls)"
                                                   if ulysses
                                                   else f"Ring Anything over {ws} ranks (padded K/V blocks all-gathered, "
                                                        f"trimmed, one fused pa_attn_fwd_chunks launch)" if gather
                                                   else f"USP over {ws} ranks: Ulysses degree {usp_degree} x ring "
                                                        f"degree {ring_len}" + _ring_how(partials) if usp_degree
                                                   else f"ring attention over {ws} ranks (NCCL P2P on a second "
                                                        f"stream)" + _ring_how(partials))),
                           q_shards=nq_all, kv_shards=nk_all,
                           l2="each rank's K/V blocks rotate through the ring; inputs far larger than L2"),
            "pct_of_bf16_peak": 100.0 * (value / ws) / peak, "roofline": roof, "clocks": sampler.summary(),
            "gpu_launches": args.steps * (1 if ulysses or (gather and ws <= 8)
                                          else ws + 1 if gather else ring_len + (1 if partials else 0)),
            "e2e": {"value": fl * e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": int((q.numel() + k.numel() + v.numel()) * 2),
                    "d2h_bytes_per_step": int(out.numel() * 2 + out.numel() // w.d * 4), "steps": e_steps,
                    "note": "per rank; every rank moves its own shards"}}
    barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()
    return 0


class ModeSets:
    """Rotating input sets for one way of running a chunked workload:
    ``chunks`` = pa_attn_fwd per chunk, then pa_attn_merge; ``fused`` = one
    pa_attn_fwd_chunks launch; ``fold`` = pa_attn_fwd_accum per chunk into an
    fp32 running state, the last fold writing the bf16 output.  Enough sets
    that consecutive steps read inputs totalling more than L2."""

    def __init__(self, pa, w, mode, device):
        import torch
        self.pa, self.w, self.mode = pa, w, mode
        self.sets = []
        n = len(w.chunks)
        for s in range(_sets_for(w)):
            q, k, v = workloads.make_case(w, device=device, seed=w.seed + 1000 * s)
            pairs = workloads.split_keys(k, v, w.chunks)
            del k, v
            st = {"q": q, "k": [a for a, _ in pairs], "v": [b for _, b in pairs], "o": torch.empty_like(q),
                  "lse": torch.empty(q.shape[:3], dtype=torch.float32, device=device)}
            if mode in ("chunks", "fwds") and n > 1:
                st["o_parts"] = torch.empty((n,) + tuple(q.shape), dtype=torch.bfloat16, device=device)
                st["lse_parts"] = torch.empty((n,) + tuple(q.shape[:3]), dtype=torch.float32, device=device)
            if mode == "fold":
                st["o_acc"] = torch.empty(q.shape, dtype=torch.float32, device=device)
            self.sets.append(st)
        self.launches = {"chunks": n + (1 if n > 1 else 0), "fwds": n, "fused": 1, "fold": n}[mode]

    def run(self, i):
        pa, w, st = self.pa, self.w, self.sets[i % len(self.sets)]
        if self.mode == "chunks":
            pa.blockwise_attention(st["q"], st["k"], st["v"], scale=w.scale, o_parts=st.get("o_parts"),
                                   lse_parts=st.get("lse_parts"), out=st["o"], lse=st["lse"])
        elif self.mode == "fwds":  # the per-chunk forwards alone, into the partial buffers
            for c in range(len(st["k"])):
                pa.attn_fwd(st["q"], st["k"][c], st["v"][c], scale=w.scale, out=st["o_parts"][c],
                            lse=st["lse_parts"][c])
        elif self.mode == "fused":
            pa.attn_fwd_chunks(st["q"], st["k"], st["v"], scale=w.scale, out=st["o"], lse=st["lse"])
        else:
            n = len(st["k"])
            for c in range(n):
                pa.attn_fwd_accum(st["q"], st["k"][c], st["v"][c], st["o_acc"], st["lse"], first=(c == 0),
                                  final=(c == n - 1), out=st["o"] if c == n - 1 else None, scale=w.scale)


def mode_timing(pa, w, mode, steps, warmup, device, graph=False):
    """Device time per step of `mode` on workload `w` (CUDA events on the
    launching stream).  With ``graph`` the steps are captured once in a CUDA
    graph (one pass over the rotating sets) and replayed, so the host-side
    cost of each library call (argument checks, tensor-map encoding, Python)
    drops out and what remains is the GPU's own time."""
    import torch
    ms_sets = ModeSets(pa, w, mode, device)
    nsets = len(ms_sets.sets)
    side = torch.cuda.Stream(device=device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        for i in range(max(warmup, nsets)):
            ms_sets.run(i)
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for i in range(nsets):
                ms_sets.run(i)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, steps // nsets)
        t0.record()
        for _ in range(reps):
            g.replay()
        t1.record()
        torch.cuda.synchronize()
        n_steps = reps * nsets
        del g
    else:
        t0.record()
        for i in range(steps):
            ms_sets.run(i)
        t1.record()
        torch.cuda.synchronize()
        n_steps = steps
    ms = t0.elapsed_time(t1) / n_steps
    status = pa.poll_device_status()
    if status != 0:
        raise SystemExit(f"device status {status} after timing {w.name} {mode}")
    del ms_sets
    torch.cuda.empty_cache()
    fl = workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d)
    return {"step_ms": ms, "tflops_step": fl / (ms * 1e-3) / 1e12, "launches_per_step":
            {"chunks": len(w.chunks) + (1 if len(w.chunks) > 1 else 0), "fwds": len(w.chunks), "fused": 1,
             "fold": len(w.chunks)}[mode],
            "timing": "CUDA graph replay" if graph else "eager launches"}


def fp8_timing(pa, w, steps, warmup, device):
    """Device time of pa_attn_fwd_fp8 on the workload's inputs quantised to
    per-tensor scaled e4m3 (the quantisation is outside the timed region)."""
    import torch
    q, k, v = workloads.make_case(w, device=device)
    qs = []
    for x in (q, k, v):
        sc = max(float(x.float().abs().max()), 1e-12) / 448.0
        qs.append(((x.float() / sc).to(torch.float8_e4m3fn).contiguous(), sc))
    del q, k, v
    (q8, sq), (k8, sk), (v8, sv) = qs
    o = torch.empty(q8.shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty(q8.shape[:3], dtype=torch.float32, device=device)
    for _ in range(warmup):
        pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=w.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        pa.attn_fwd_fp8(q8, k8, v8, sq, sk, sv, scale=w.scale, out=o, lse=lse)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return ms, workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d) / (ms * 1e-3) / 1e12


def extra_measurements(pa, device, peaks):
    """Secondary lines: the other workloads' device throughput (not the
    headline value).  Bounded repetitions each."""
    out = {}
    # The FLUX.1-dev 1024^2 shape, per launch, as the headline is timed.
    wf = workloads.get("flux")
    r = time_workload(pa, wf, 200, 10, device)
    fl = workloads.flops(wf.B, wf.H, wf.Nq, wf.Nk, wf.d)
    out["flux"] = {"step_ms": r["total_ms"] / 200, "fwd_ms_per_launch": statistics.fmean(r["fwd_ms"]),
                   "fwd_tflops": fl / (statistics.fmean(r["fwd_ms"]) * 1e-3) / 1e12}
    out["flux"]["frac_of_bf16_peak"] = out["flux"]["fwd_tflops"] / peaks["bf16_tflops"]
    # Chunked workloads: per-chunk forward + merge with per-launch events
    # (eager), then every mode timed from CUDA-graph replays (device time).
    for name, steps in (("ring", 20), ("tails", 10), ("flux1008", 10)):
        w = workloads.get(name)
        r = time_workload(pa, w, steps, 3, device)
        fl = workloads.flops(w.B, w.H, w.Nq, w.Nk, w.d)
        ent = {"step_ms": r["total_ms"] / steps, "tflops_step": fl * steps / (r["total_ms"] * 1e-3) / 1e12,
               "fwd_ms_per_launch": statistics.fmean(r["fwd_ms"]),
               "fwd_tflops": (fl / len(w.chunks)) / (statistics.fmean(r["fwd_ms"]) * 1e-3) / 1e12,
               "timing": "eager launches, events around each launch"}
        if r["merge_ms"]:
            mb = workloads.merge_bytes(len(w.chunks), w.B, w.H, w.Nq, w.d)
            ent["merge_ms"] = statistics.fmean(r["merge_ms"])
            ent["merge_gbs"] = mb / (ent["merge_ms"] * 1e-3) / 1e9
        ent["pct_of_bf16_peak"] = 100.0 * ent["fwd_tflops"] / peaks["bf16_tflops"]
        out[name] = ent
        for mode in ("fwds", "chunks", "fused", "fold"):
            g = mode_timing(pa, w, mode, 200, 3, device, graph=True)
            g["frac_of_bf16_peak"] = g["tflops_step"] / peaks["bf16_tflops"]
            out[f"{name}_{mode}_graph"] = g
        out[name + "_fused"] = mode_timing(pa, w, "fused", 20, 3, device)
    w8 = workloads.get("hunyuan").with_chunks(workloads.HUNYUAN_CHUNKS8)
    for mode in ("fused", "fold"):
        out[f"hunyuan_8chunks_{mode}"] = mode_timing(pa, w8, mode, 2, 1, device)
    # The e4m3 forward on the FLUX and HunyuanVideo shapes; its peak is the
    # measured bf16 burst figure times the nominal fp8/bf16 ratio of 2.
    # 200 FLUX launches (≈ 40 ms), like the bf16 FLUX line: a few milliseconds
    # of launches only show the clock state the previous phase left behind.
    for name, steps, warm in (("flux", 200, 10), ("hunyuan", 2, 2)):
        ms, tf = fp8_timing(pa, workloads.get(name), steps=steps, warmup=warm, device=device)
        out[name + "_fp8"] = {"fwd_ms_per_launch": ms, "fwd_tflops": tf,
                              "frac_of_fp8_peak": tf / (2.0 * peaks["bf16_tflops"]),
                              "peak_basis": "2 x " + _basis(peaks) + " (nominal e4m3/bf16 ratio)"}
    # e4m3 quantisation (pa_quantize_e4m3) of a HunyuanVideo-sized Q tensor
    # (0.73 GB bf16, far above L2): algorithmic bytes = 2 read + 1 written per
    # element (the kernel streams x twice: amax, then convert).
    import torch
    h = workloads.get("hunyuan")
    x = torch.randn((h.B * h.H * h.Nq * h.d,), device=device).to(torch.bfloat16)
    q8 = torch.empty(x.shape, dtype=torch.float8_e4m3fn, device=device)
    sc = torch.empty((1,), dtype=torch.float32, device=device)
    for _ in range(3):
        pa.quantize_e4m3(x, out=q8, scale=sc)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(10):
        pa.quantize_e4m3(x, out=q8, scale=sc)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / 10
    out["quantize_e4m3"] = {"elements": int(x.numel()), "ms": ms,
                            "gbs": 3.0 * x.numel() / (ms * 1e-3) / 1e9,
                            "frac_of_hbm": 3.0 * x.numel() / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del x, q8
    # First Block Cache's residual difference (pa_residual_diff) between two
    # HunyuanVideo-sized first-block residuals (119056 tokens x 3072 channels
    # bf16, 0.73 GB each, far above L2): algorithmic bytes = 4 per element
    # (both read once); two inputs alternate so no call finds its data in L2.
    n_res = 119056 * 3072
    res = [torch.randn((n_res,), device=device).to(torch.bfloat16) for _ in range(3)]
    rd_out = torch.empty((1,), dtype=torch.float32, device=device)
    for i in range(3):
        pa.residual_diff(res[i % 3], res[(i + 1) % 3], out=rd_out)
    torch.cuda.synchronize()
    t0.record()
    for i in range(12):
        pa.residual_diff(res[i % 3], res[(i + 1) % 3], out=rd_out)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / 12
    out["residual_diff"] = {"elements": n_res, "ms": ms, "gbs": 4.0 * n_res / (ms * 1e-3) / 1e9,
                            "frac_of_hbm": 4.0 * n_res / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del res
    w8 = workloads.get("hunyuan").with_chunks(workloads.HUNYUAN_CHUNKS8)
    r = time_workload(pa, w8, 2, 1, device)
    fl = workloads.flops(w8.B, w8.H, w8.Nq, w8.Nk, w8.d)
    mb = workloads.merge_bytes(8, w8.B, w8.H, w8.Nq, w8.d)
    out["hunyuan_8chunks"] = {"step_ms": r["total_ms"] / 2,
                              "tflops_step": fl * 2 / (r["total_ms"] * 1e-3) / 1e12,
                              "fwd_tflops": (fl / 8) / (statistics.fmean(r["fwd_ms"]) * 1e-3) / 1e12,
                              "merge_ms": statistics.fmean(r["merge_ms"]),
                              "merge_gbs": mb / (statistics.fmean(r["merge_ms"]) * 1e-3) / 1e9}
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="hunyuan", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--parallel", choices=["ring", "ulysses", "usp", "ring_anything", "replicas"], default="ring",
                    help="with more than one GPU: ring, Ulysses or USP (Ulysses x ring) attention over the ranks, "
                         "Ring Anything (padded all-gather + one fused launch), or independent replicas")
    ap.add_argument("--ulysses-degree", type=int, default=2,
                    help="with --parallel usp: ranks per Ulysses group (the ring runs across the groups)")
    ap.add_argument("--mode", choices=["chunks", "fused", "fold"], default="chunks",
                    help="how a chunked workload's step runs: pa_attn_fwd per chunk + pa_attn_merge, one "
                         "pa_attn_fwd_chunks launch, or pa_attn_fwd_accum folds; with the ring or USP over "
                         "several GPUs, chunks = per-block partials + one merge, fold = the fp32 running state")
    ap.add_argument("--fp8", action="store_true",
                    help="time the e4m3 forward (pa_attn_fwd_fp8) instead of bf16; one-chunk workloads")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count (same sequence shape, smaller case; for profiling)")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU seconds of the oracle sample in the cpu_baseline leg")
    ap.add_argument("--cpu-budget", type=float, default=120.0,
                    help="total CPU seconds of the reference arm's timed steps")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
