"""Seeded synthetic inputs for fused linear cross-entropy (FLCE) workloads.

This module is shared by the CUDA path's tests/bench and by the float64
oracle.  It holds no FLCE arithmetic: it only draws random numbers, rounds
them to bf16 (round-to-nearest-even from fp32) and places ignore_index
markers.  Both sides consume the very same quantised arrays.

Workload shapes follow the pages:
  * `[2, 8192]` tokens at vocab 131072 and the 8 GiB fp32 logits figure
    (Modalities PR #464, "Memory note for large-vocabulary training");
  * vocab 131072 in the float64 comparison (Modalities PR #464, "Measured");
  * ignore_index = -100 (NeMo AutoModel `FusedLinearCrossEntropy` API,
    constructor default; inclusionAI/Ling-3.1-flash discussion #7 example);
  * softcap applied as softcap*tanh(logits/softcap) (modelscope/twinkle
    PR #335, "PR information" item 3);
  * 'sum' / 'mean' reductions and the micro-batch token-weighted scale
    (modelscope/twinkle PR #335, items 1 and 2).
No public dataset is named by the pages; every input here is synthetic.

Random streams: each tensor is drawn in row chunks; chunk i of stream k uses
`PCG64(SeedSequence([seed, k, i]))`, so the values do not depend on how many
threads generate them.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Tuple

import numpy as np

IGNORE_INDEX = -100

_STREAM_HIDDEN = 0
_STREAM_WEIGHT = 1
_STREAM_LABELS = 2
_CHUNK_ROWS = 2048


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic FLCE problem (tokens flattened to N rows)."""

    name: str
    N: int
    H: int
    V: int
    batch_shape: Tuple[int, ...]
    w_std: float
    labels: str  # "uniform" | "zipf1.1"
    ignore_rule: str  # "count" | "tail" | "microbatch"
    ignore_count: int  # rows ignored (per micro-batch for "microbatch")
    softcap: float
    reduction: str  # "sum" | "mean"
    seed: int
    microbatches: int = 1
    empty_microbatch: int = -1  # index of the all-ignored micro-batch
    description: str = ""

    @property
    def flops_per_step(self) -> float:
        """Credited work of one forward+backward: 2NHV + 6NHV."""
        return 8.0 * self.N * self.H * self.V


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        name="tiny", N=64, H=64, V=512, batch_shape=(1, 64), w_std=0.02,
        labels="uniform", ignore_rule="count", ignore_count=16, softcap=0.0,
        reduction="sum", seed=1,
        description="N=64 H=64 V=512, 25% ignored, sum"),
    "v32k_mean": Workload(
        name="v32k_mean", N=4096, H=2048, V=32000, batch_shape=(2, 2048),
        w_std=0.02, labels="uniform", ignore_rule="count", ignore_count=409,
        softcap=0.0, reduction="mean", seed=2,
        description="N=4096 H=2048 V=32000, 10% ignored, mean"),
    "v131k_zipf": Workload(
        name="v131k_zipf", N=16384, H=4096, V=131072, batch_shape=(2, 8192),
        w_std=0.02, labels="zipf1.1", ignore_rule="count", ignore_count=819,
        softcap=0.0, reduction="sum", seed=3,
        description="N=16384 ([2,8192]) H=4096 V=131072, Zipf(1.1) labels, 5% ignored, sum"),
    "v256k_softcap": Workload(
        name="v256k_softcap", N=8192, H=3584, V=256000, batch_shape=(1, 8192),
        w_std=0.03, labels="uniform", ignore_rule="tail", ignore_count=1638,
        softcap=30.0, reduction="sum", seed=4,
        description="N=8192 H=3584 V=256000, softcap 30, last 20% of the sequence ignored, sum"),
    "microbatch": Workload(
        name="microbatch", N=16384, H=4096, V=131072, batch_shape=(4, 4096),
        w_std=0.02, labels="uniform", ignore_rule="microbatch", ignore_count=1228,
        softcap=0.0, reduction="sum", seed=5, microbatches=4, empty_microbatch=1,
        description="N=16384 as 4 micro-batches of 4096, micro-batch 1 all ignored, "
                    "others 30% ignored, sum with token-weighted grad scale"),
    # A smaller problem whose backward launches have exactly the per-launch
    # shapes of v131k_zipf (N=16384, H=4096; 16384-token x 16384-vocab backward
    # chunks) and whose forward is a quarter of its forward (V=32768), used for
    # profiler captures that must stay small on the device (about 2 GB).
    "profile_16k": Workload(
        name="profile_16k", N=16384, H=4096, V=32768, batch_shape=(2, 8192), w_std=0.02,
        labels="zipf1.1", ignore_rule="count", ignore_count=819, softcap=0.0,
        reduction="sum", seed=6,
        description="N=16384 H=4096 V=32768, Zipf(1.1) labels, 5% ignored, sum "
                    "(profiling size)"),
}

# The order of the five problems as they are listed for this workload family.
WORKLOAD_ORDER: List[str] = ["tiny", "v32k_mean", "v131k_zipf", "v256k_softcap", "microbatch"]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Inputs must be finite (the generators never produce NaN/Inf).
    """
    a = np.ascontiguousarray(x, dtype=np.float32)
    b = a.view(np.uint32).copy()
    b += np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return (b >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exactly equal fp32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, stream: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, chunk])))


def _normal_rows(seed: int, stream: int, rows: int, cols: int, std: float,
                 threads: int) -> np.ndarray:
    """fp32 N(0, std^2) matrix drawn in independent row chunks."""
    out = np.empty((rows, cols), dtype=np.float32)
    n_chunks = (rows + _CHUNK_ROWS - 1) // _CHUNK_ROWS

    def fill(i: int) -> None:
        r0 = i * _CHUNK_ROWS
        r1 = min(rows, r0 + _CHUNK_ROWS)
        g = _rng(seed, stream, i)
        blk = g.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            blk *= np.float32(std)
        out[r0:r1] = blk

    if threads <= 1 or n_chunks == 1:
        for i in range(n_chunks):
            fill(i)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out


def _draw_labels(w: Workload) -> np.ndarray:
    g = _rng(w.seed, _STREAM_LABELS, 0)
    if w.labels == "uniform":
        y = g.integers(0, w.V, size=w.N, dtype=np.int64)
    elif w.labels == "zipf1.1":
        # Zipf(1.1) truncated to ranks 1..V; token id = rank - 1.
        ranks = np.arange(1, w.V + 1, dtype=np.float64)
        cdf = np.cumsum(ranks ** -1.1)
        cdf /= cdf[-1]
        u = g.random(w.N)
        y = np.searchsorted(cdf, u, side="right").astype(np.int64)
        np.minimum(y, w.V - 1, out=y)
    else:
        raise ValueError(f"unknown label distribution {w.labels!r}")

    if w.ignore_rule == "count":
        pos = g.choice(w.N, size=w.ignore_count, replace=False)
        y[pos] = IGNORE_INDEX
    elif w.ignore_rule == "tail":
        seq = w.batch_shape[-1]
        for b in range(w.N // seq):
            y[b * seq + seq - w.ignore_count:(b + 1) * seq] = IGNORE_INDEX
    elif w.ignore_rule == "microbatch":
        mb = w.N // w.microbatches
        for k in range(w.microbatches):
            if k == w.empty_microbatch:
                y[k * mb:(k + 1) * mb] = IGNORE_INDEX
            else:
                pos = g.choice(mb, size=w.ignore_count, replace=False)
                y[k * mb + pos] = IGNORE_INDEX
    else:
        raise ValueError(f"unknown ignore rule {w.ignore_rule!r}")
    return y


@dataclasses.dataclass
class Inputs:
    """Quantised inputs of one workload.

    hidden_bits/weight_bits are bf16 bit patterns (uint16); hidden/weight are
    the same values as exact fp32.  hidden_raw/weight_raw hold the fp32 draws
    before rounding (only kept when requested: the fp32 reading of the tiny
    problem uses them).
    """

    workload: Workload
    hidden_bits: np.ndarray
    weight_bits: np.ndarray
    labels: np.ndarray
    hidden_raw: Optional[np.ndarray] = None
    weight_raw: Optional[np.ndarray] = None

    @property
    def hidden(self) -> np.ndarray:
        return bf16_to_f32(self.hidden_bits)

    @property
    def weight(self) -> np.ndarray:
        return bf16_to_f32(self.weight_bits)

    def microbatch_slices(self) -> List[slice]:
        w = self.workload
        mb = w.N // w.microbatches
        return [slice(k * mb, (k + 1) * mb) for k in range(w.microbatches)]


def make_inputs(w: Workload | str, keep_raw: bool = False,
                threads: Optional[int] = None) -> Inputs:
    """Draw the inputs of workload `w` (deterministic in `w.seed`)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if threads is None:
        threads = min(16, os.cpu_count() or 1)
    h = _normal_rows(w.seed, _STREAM_HIDDEN, w.N, w.H, 1.0, threads)
    wt = _normal_rows(w.seed, _STREAM_WEIGHT, w.V, w.H, w.w_std, threads)
    y = _draw_labels(w)
    hb = bf16_round(h)
    wb = bf16_round(wt)
    return Inputs(w, hb, wb, y,
                  h if keep_raw else None,
                  wt if keep_raw else None)


def custom_workload(N: int, H: int, V: int, *, seed: int = 0, w_std: float = 0.02,
                    softcap: float = 0.0, reduction: str = "sum",
                    ignore_count: int = 0, labels: str = "uniform") -> Workload:
    """A small ad-hoc problem with the same recipe (for ragged/edge tests)."""
    return Workload(name=f"custom_{N}x{H}x{V}", N=N, H=H, V=V, batch_shape=(1, N),
                    w_std=w_std, labels=labels, ignore_rule="count",
                    ignore_count=ignore_count, softcap=softcap, reduction=reduction,
                    seed=seed)
