"""Calibration loop around the counting kernel: counts -> fit points -> fit.

The counting itself runs in ``ssa_calibrate`` (dense attention plus, per
(head, q-block) unit, how many KV tiles each trial threshold would skip) and
the log-space fit in ``ssa_fit_logspace``; this module only sums counts per
sequence, pairs each sum with its scale factor and, when heads are sharded
over ranks, adds the per-rank sums with one all-reduce before the fit.

Sources:
  * Model-Optimizer PR #1166 page, "Usage": the sixteen raw-lambda
    ``threshold_trials``; the README "Calibrated threshold" and "Threshold
    Modes": scale_factor = lambda * seq_len_kv and
    scale_factor = a * exp(b * target_sparsity).
  * Model-Optimizer commit page, "Calibration": the fit minimises relative
    error in log space and records the observed sparsity range, outside of
    which a resolved target is an extrapolation (warned about).
Reading: one fit point per (sequence, trial): its sparsity is that
sequence's skipped-tile fraction over all heads, its scale factor
lambda * S_kv of that sequence; points with sparsity 0 or 1 carry no
information and the C fit drops them.
"""
from __future__ import annotations

import warnings
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence

import numpy as np

from . import calibrate as _calibrate
from . import calibrate_fp8 as _calibrate_fp8
from . import fit_logspace as _fit_logspace
from . import resolve as _resolve

TILE = 128
DEFAULT_TRIALS = (1e-6, 5e-6, 1e-5, 5e-5, 1e-4, 5e-4, 1e-3, 5e-3, 1e-2, 2e-2, 5e-2, 1e-1, 2e-1, 3e-1, 5e-1, 7e-1)


@dataclass
class Calibration:
    a: float
    b: float
    s_min: float
    s_max: float
    points: List[tuple] = field(default_factory=list)  # (sparsity, scale_factor)

    def threshold_scale_factor(self, target_sparsity: float) -> float:
        """a * exp(b * s); warns when s lies outside the observed range."""
        if not (self.s_min <= target_sparsity <= self.s_max):
            warnings.warn(f"target_sparsity {target_sparsity} is outside the calibrated range "
                          f"[{self.s_min:.4f}, {self.s_max:.4f}]: extrapolating the fit", RuntimeWarning)
        return _resolve(self.a, self.b, target_sparsity)


def _sequences(cu_seqlens_host):
    cu = np.asarray(cu_seqlens_host, dtype=np.int64)
    lens = np.diff(cu)
    if np.any(lens < 0) or cu[0] < 0:
        raise ValueError("cu_seqlens must be non-decreasing from >= 0")
    nq = (lens + TILE - 1) // TILE
    first = np.concatenate([[0], np.cumsum(nq)[:-1]])
    return lens, nq, first


def sequence_counts(counts_host, cu_seqlens_host) -> np.ndarray:
    """Sum per-unit counts [H, Q, N] over each sequence's units: int64 [B, N]."""
    c = np.asarray(counts_host)
    if c.ndim != 3:
        raise ValueError("counts must be [heads, q-blocks, thresholds]")
    lens, nq, first = _sequences(cu_seqlens_host)
    if int(nq.sum()) != c.shape[1]:
        raise ValueError("counts and cu_seqlens disagree on the number of q-blocks")
    out = np.zeros((len(lens), c.shape[2]), dtype=np.int64)
    for b, (f, n) in enumerate(zip(first, nq)):
        out[b] = c[:, f:f + n, :].astype(np.int64).sum(axis=(0, 1))
    return out


def fit_points(seq_counts, cu_seqlens_host, trials: Sequence[float], total_heads: int):
    """(sparsity, scale_factor) per (sequence, trial) from summed counts."""
    lens, nq, _ = _sequences(cu_seqlens_host)
    sc = np.asarray(seq_counts, dtype=np.int64)
    pts = []
    for b, S in enumerate(lens):
        if S == 0:
            continue
        tiles = total_heads * int(nq[b]) * int(nq[b])
        for k, lam in enumerate(trials):
            pts.append((float(sc[b, k]) / tiles, float(lam) * float(S)))
    return pts


def fit(points) -> Calibration:
    s = [p[0] for p in points]
    y = [p[1] for p in points]
    a, b, smin, smax = _fit_logspace(s, y)
    return Calibration(a, b, smin, smax, list(points))


def torch_allreduce(group=None) -> Callable[[np.ndarray], np.ndarray]:
    """Sum an int64 array over the ranks of a torch.distributed group (NCCL
    sums a CUDA copy, gloo a CPU one)."""
    import torch
    import torch.distributed as dist

    def reduce(a: np.ndarray) -> np.ndarray:
        dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(group) == "nccl" else "cpu"
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.int64)).to(dev)
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        return t.cpu().numpy()

    return reduce


def calibrate(q, k, v, cu_seqlens, max_seqlen: int, trials: Sequence[float] = DEFAULT_TRIALS,
              softmax_scale: float = 0.0, total_heads: Optional[int] = None,
              allreduce: Optional[Callable[[np.ndarray], np.ndarray]] = None, descales=None,
              stream=None) -> Calibration:
    """Count on the GPU, sum per sequence, optionally add the other ranks'
    sums (heads sharded: q, k, v hold this rank's heads, total_heads counts
    all ranks'), and fit. Every rank that takes part gets the same result.
    With ``descales = (q_descale, k_descale)``, q and k are E4M3 codes and the
    counts come from ssa_calibrate_fp8."""
    if descales is None:
        _, counts = _calibrate(q, k, v, cu_seqlens, max_seqlen, list(trials), softmax_scale=softmax_scale,
                               stream=stream)
    else:
        _, counts = _calibrate_fp8(q, k, v, cu_seqlens, max_seqlen, float(descales[0]), float(descales[1]),
                                   list(trials), softmax_scale=softmax_scale, stream=stream)
    cu_host = cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else np.asarray(cu_seqlens)
    seq = sequence_counts(counts.cpu().numpy(), cu_host)
    if allreduce is not None:
        seq = allreduce(seq)
    heads = q.shape[1] if total_heads is None else int(total_heads)
    return fit(fit_points(seq, cu_host, trials, heads))


def shard_heads(num_heads: int, world: int, rank: int) -> range:
    """Contiguous head range of `rank` when heads are split over `world` ranks."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad world/rank")
    base, extra = divmod(num_heads, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
