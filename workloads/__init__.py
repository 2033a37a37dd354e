"""Seeded synthetic workloads shared by the tests, the bench and the oracle checks.

This module holds shapes, seeds and random draws only: none of the attention
arithmetic lives here, so both the CUDA path and the oracle can take their
inputs from it without sharing any of the method.

The workloads stand in for the attention calls of the two models the
diffusers "ParaAttention" guide times (FLUX.1-dev at 1024x1024: 512 text +
4096 image tokens, 24 heads of 128; HunyuanVideo at 720p, 129 frames:
33 x 45 x 80 latent tokens + 256 text tokens) and for the ring-attention
split of the "Context parallelism" guide (section "Ring Attention"; uneven
chunks as in "Ring Anything Attention").  No dataset, prompt or trained weight
is used: every tensor is drawn from a seeded generator.

Value recipe: Q, K, V are standard normal float32 draws; where a workload says
``rms_qk`` the Q and K rows are RMS-normalised over the head dimension
(x / sqrt(mean(x^2) + 1e-6), no learnable weight), as DiT blocks do before
attention; everything is then rounded to bf16 (round to nearest even).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get", "make_case", "split_keys", "sample_rows",
           "flops", "fwd_bytes", "merge_bytes"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    rms_qk: bool
    chunks: Tuple[int, ...]
    seed: int
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_chunks(self, chunks: Sequence[int]) -> "Workload":
        return dataclasses.replace(self, chunks=tuple(int(c) for c in chunks))


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, H=2, Nq=256, Nk=256, d=64, rms_qk=False,
                     chunks=(128, 128), seed=0,
                     note="iid N(0,1) Q/K/V; two key chunks of 128 merged"),
    "flux": Workload("flux", B=1, H=24, Nq=4608, Nk=4608, d=128, rms_qk=True,
                     chunks=(4608,), seed=1,
                     note="FLUX.1-dev 1024^2 joint attention: 512 text + 4096 image tokens"),
    "ring": Workload("ring", B=1, H=24, Nq=1152, Nk=4608, d=128, rms_qk=False,
                     chunks=(1152, 1152, 1152, 1152), seed=2,
                     note="ring_degree=4 step on one GPU: rank-0 query slice vs 4 K/V chunks"),
    "tails": Workload("tails", B=2, H=24, Nq=4603, Nk=4603, d=128, rms_qk=True,
                      chunks=(1151, 1151, 1151, 1150), seed=3,
                      note="uneven chunks, none a multiple of the 128-row tile"),
    "hunyuan": Workload("hunyuan", B=1, H=24, Nq=119056, Nk=119056, d=128, rms_qk=True,
                        chunks=(119056,), seed=4,
                        note="HunyuanVideo 720p x 129 frames: 33*45*80 video + 256 text tokens"),
    # FLUX.1-dev at 1008 x 1008: 63 * 63 = 3969 image tokens + 512 text tokens
    # = 4481, a length that does not divide by 4 ranks.  Split the way
    # "Ring Anything Attention" of the "Context parallelism" guide does it:
    # each rank holds ceil(4481 / 4) = 1121 tokens, the last one 1118 once the
    # padding is trimmed before attention.
    "flux1008": Workload("flux1008", B=1, H=24, Nq=4481, Nk=4481, d=128, rms_qk=True,
                         chunks=(1121, 1121, 1121, 1118), seed=5,
                         note="FLUX.1-dev 1008^2: 512 text + 3969 image tokens, ring-anything split over 4"),
}

# The 8-chunk split of the HunyuanVideo-shaped workload (ring_degree = 8).
HUNYUAN_CHUNKS8 = (14882,) * 8
WORKLOADS["hunyuan8"] = dataclasses.replace(WORKLOADS["hunyuan"], name="hunyuan8", chunks=HUNYUAN_CHUNKS8,
                                            note="HunyuanVideo shape split over 8 ranks: 8 chunks of 14882")


def get(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; choose from {sorted(WORKLOADS)}") from None


def _rms_rows(x):
    import torch
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + 1e-6)


def make_case(w: Workload, device="cpu", seed: int | None = None, nq: int | None = None):
    """Draw (q, k, v) as contiguous bf16 tensors [B, H, N, d] on ``device``.

    The draws are made in float32 by a torch generator living on ``device``
    and seeded with the workload's seed, so a given (workload, device type)
    always yields the same values.  ``nq`` overrides the number of query rows
    (used to cut a bounded CPU sample; the rows are a prefix of the same
    distribution, not of the same draw).
    """
    import torch
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed if seed is None else int(seed))
    n_q = w.Nq if nq is None else int(nq)
    q = torch.randn((w.B, w.H, n_q, w.d), generator=g, device=dev, dtype=torch.float32)
    k = torch.randn((w.B, w.H, w.Nk, w.d), generator=g, device=dev, dtype=torch.float32)
    v = torch.randn((w.B, w.H, w.Nk, w.d), generator=g, device=dev, dtype=torch.float32)
    if w.rms_qk:
        q = _rms_rows(q)
        k = _rms_rows(k)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def split_keys(k, v, chunks: Sequence[int]):
    """Materialise each key chunk as its own contiguous [B, H, n_p, d] buffer,
    the way a ring step receives a neighbour's block into local memory."""
    sizes = [int(c) for c in chunks]
    if sum(sizes) != k.shape[-2]:
        raise ValueError("chunk sizes must sum to Nk")
    out: List[tuple] = []
    s = 0
    for c in sizes:
        out.append((k[..., s:s + c, :].contiguous(), v[..., s:s + c, :].contiguous()))
        s += c
    return out


def sample_rows(n_rows: int, count: int, seed: int) -> np.ndarray:
    """``count`` distinct query-row indices in [0, n_rows), sorted, seeded."""
    rng = np.random.default_rng(seed)
    count = min(count, n_rows)
    return np.sort(rng.choice(n_rows, size=count, replace=False)).astype(np.int64)


def flops(B: int, H: int, Nq: int, Nk: int, d: int) -> float:
    """Attention forward FLOPs counted as 4*B*H*Nq*Nk*d (two contractions)."""
    return 4.0 * B * H * Nq * Nk * d


def fwd_bytes(B: int, H: int, Nq: int, Nk: int, d: int) -> float:
    """Algorithmic HBM bytes of one forward call: Q, K, V read once (bf16),
    O written once (bf16) and LSE written once (fp32)."""
    return 2.0 * B * H * (2 * Nq * d + 2 * Nk * d) + 4.0 * B * H * Nq


def merge_bytes(n_parts: int, B: int, H: int, N: int, d: int) -> float:
    """Algorithmic HBM bytes of one merge: n partial O (bf16) and LSE (fp32)
    read, one O (bf16) and LSE (fp32) written."""
    rows = B * H * N
    return rows * (n_parts * (2.0 * d + 4.0) + 2.0 * d + 4.0)
