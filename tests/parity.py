"""GPU-vs-oracle comparison helpers for the parity tests.

The acceptance rule (tolerances fixed for the skip-softmax path: bf16 inputs
and output, fp32 accumulation):
  * outputs: max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3;
  * skip decisions: identical on every tile whose oracle statistic is more
    than 1e-3 away from the threshold ("margin tiles" may go either way);
  * calibration counts: identical up to the number of margin tiles.
For lambda <= 1 the running-max trajectory does not depend on decisions, so
every non-margin tile is compared. For lambda > 1 a margin tile decided the
other way legitimately changes the rest of the unit's walk; such a unit is
compared with the oracle up to that tile, then walked again by the oracle
with every decision forced to the GPU's (the oracle's replay mode): along
that trajectory every non-margin decision must be the one the oracle's own
statistic gives, and the output is held to the same tolerances.
"""
from __future__ import annotations

import math

import numpy as np

import synth

TILE = 128
MARGIN = 1e-3
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_device(q, k, v, cu):
    import torch

    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return t(q), t(k), t(v), torch.from_numpy(np.ascontiguousarray(cu, dtype=np.int32)).to(dev)


def bf16_host(t):
    import torch

    return synth.bf16_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))


def global_qblock(cu, units):
    """Global q-block index of each (sequence, head, qb) unit."""
    cu = np.asarray(cu)
    nq = [(int(cu[b + 1] - cu[b]) + TILE - 1) // TILE for b in range(len(cu) - 1)]
    off = np.concatenate([[0], np.cumsum(nq)]).astype(np.int64)
    return np.array([off[b] + qb for b, _, qb in units], dtype=np.int64)


def unit_rows(cu, unit):
    b, h, qb = unit
    s0 = int(cu[b]) + qb * TILE
    n = min(TILE, int(cu[b + 1] - cu[b]) - qb * TILE)
    return s0, n


class Stats:
    def __init__(self):
        self.max_abs = 0.0
        self.sum_abs = 0.0
        self.count = 0
        self.tiles = 0
        self.margin_tiles = 0
        self.divergent_units = 0
        self.replayed_units = 0

    def add(self, got, exp):
        d = np.abs(got.astype(np.float64) - exp.astype(np.float64))
        self.max_abs = max(self.max_abs, float(d.max()) if d.size else 0.0)
        self.sum_abs += float(d.sum())
        self.count += d.size

    @property
    def mean_abs(self):
        return self.sum_abs / max(self.count, 1)

    def check(self, what=""):
        assert self.max_abs <= MAX_ABS, f"{what}: max abs err {self.max_abs}"
        assert self.mean_abs <= MEAN_ABS, f"{what}: mean abs err {self.mean_abs}"


def decisions_of(words, nt):
    """Per-tile decisions (True = skipped) from one unit's bitmap words."""
    return np.array([(int(words[j >> 5]) >> (j & 31)) & 1 for j in range(nt)], dtype=bool)


def compare_forward(res, cu, L_seq, out_gpu, skip_gpu, bitmap_gpu, stat_gpu, stats: Stats, what="", replay=None):
    """Compare oracle result ``res`` (from oracle.walk with per-sequence
    thresholds ``L_seq``) with the GPU's outputs (host arrays: out [total,H,D]
    fp32, skip [H,Q], bitmap [H,Q,W], stat [H,Q,T]). ``replay(i, forced)``
    walks unit i again in the oracle with decisions forced ([max_tiles] int8,
    1 skip / 0 keep / -1 decide); without it a diverged unit is only checked
    for finite output."""
    units = res["units"]
    gq = global_qblock(cu, units)
    for i, u in enumerate(units):
        b, h, qb = (int(x) for x in u)
        S = int(cu[b + 1] - cu[b])
        nt = (S + TILE - 1) // TILE
        L = float(L_seq[b])
        d_or = res["dstat"][i, :nt].astype(np.float64)
        dec_or = res["decision"][i, :nt].astype(bool)
        dec_gpu = decisions_of(bitmap_gpu[h, gq[i]], nt)
        margin = np.isfinite(d_or) & (np.abs(d_or - L) <= MARGIN) if math.isfinite(L) else np.zeros(nt, bool)
        stats.tiles += nt
        stats.margin_tiles += int(margin.sum())
        diverged_at = nt
        if L > 0:  # lambda > 1: the walk may branch at a margin tile
            diff_m = np.nonzero(margin & (dec_gpu != dec_or))[0]
            if diff_m.size:
                diverged_at = int(diff_m[0])
        cmp = ~margin
        cmp[diverged_at:] = False
        bad = np.nonzero(cmp & (dec_gpu != dec_or))[0]
        assert bad.size == 0, (f"{what}: unit {u}: decisions differ at tiles {bad[:10]} "
                               f"(oracle d {d_or[bad[:3]]}, L {L})")
        # the statistic itself, while the trajectories agree
        st = stat_gpu[h, gq[i], :diverged_at].astype(np.float64)
        fin = np.isfinite(d_or[:diverged_at])
        assert np.all(np.isinf(st[~fin])), f"{what}: unit {u}: tile-0 statistic not +inf"
        if fin.any():
            err = np.abs(st[fin] - d_or[:diverged_at][fin]).max()
            assert err <= 5e-3, f"{what}: unit {u}: tile statistic differs by {err}"
        assert int(skip_gpu[h, gq[i]]) == int(dec_gpu.sum()), f"{what}: unit {u}: counter != bitmap"
        s0, n = unit_rows(cu, u)
        got = out_gpu[s0:s0 + n, h]
        if diverged_at < nt:
            stats.divergent_units += 1
            if replay is None:
                assert np.all(np.isfinite(got))
                continue
            forced = np.full(res["dstat"].shape[1], -1, dtype=np.int8)
            forced[:nt] = dec_gpu
            rep = replay(i, forced)
            d_rep = rep["dstat"][0, :nt].astype(np.float64)
            free = np.isfinite(d_rep) & (np.abs(d_rep - L) > MARGIN)
            bad = np.nonzero(free & (dec_gpu != (d_rep < L)))[0]
            assert bad.size == 0, f"{what}: unit {u}: replayed decisions differ at tiles {bad[:10]}"
            stats.replayed_units += 1
            stats.add(got, rep["out"][0, :n])
            continue
        if not margin.any():
            assert int(skip_gpu[h, gq[i]]) == int(res["skips"][i]), f"{what}: unit {u}: skip count"
        stats.add(got, res["out"][i, :n])


def compare_calibration(res, cu, cal_L, out_gpu, counts_gpu, stats: Stats, what="", stat_gpu=None):
    """Calibration counts (and output) against the oracle's calibration walk.
    With the GPU's per-tile statistic ``stat_gpu`` [H,Q,T] (ssa_calibrate_ex)
    the comparison is tile by tile: each count must equal the number of tiles
    whose GPU statistic lies below the threshold, and that statistic must give
    the oracle's decision on every tile more than the margin away from it, so
    a right count made of two wrong tiles cannot pass."""
    units = res["units"]
    gq = global_qblock(cu, units)
    for i, u in enumerate(units):
        b, h, qb = (int(x) for x in u)
        S = int(cu[b + 1] - cu[b])
        nt = (S + TILE - 1) // TILE
        d_or = res["dstat"][i, :nt].astype(np.float64)
        if stat_gpu is not None:
            d_gpu = stat_gpu[h, gq[i], :nt].astype(np.float64)
            fin = np.isfinite(d_or)
            assert np.all(np.isinf(d_gpu[~fin])), f"{what}: unit {u}: tile-0 statistic not +inf"
            if fin.any():
                err = np.abs(d_gpu[fin] - d_or[fin]).max()
                assert err <= 5e-3, f"{what}: unit {u}: tile statistic differs by {err}"
        for kk, L in enumerate(cal_L):
            near_mask = np.isfinite(d_or) & (np.abs(d_or - L) <= MARGIN)
            near = int(near_mask.sum())
            stats.margin_tiles += near
            diff = abs(int(counts_gpu[h, gq[i], kk]) - int(res["counts"][i, kk]))
            assert diff <= near, f"{what}: unit {u} threshold {kk}: count differs by {diff} ({near} margin tiles)"
            if stat_gpu is not None:
                dec_gpu = d_gpu < np.float32(L)
                assert int(counts_gpu[h, gq[i], kk]) == int(dec_gpu.sum()), f"{what}: unit {u}: count != statistic"
                bad = np.nonzero(~near_mask & (dec_gpu != (d_or < L)))[0]
                assert bad.size == 0, f"{what}: unit {u} threshold {kk}: tiles {bad[:10]} decided differently"
        stats.tiles += nt
        s0, n = unit_rows(cu, u)
        stats.add(out_gpu[s0:s0 + n, h], res["out"][i, :n])
