"""CPU oracle for BLASST skip-softmax attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package; the product library never does. The arithmetic
lives in ``oracle.cpp`` (plain C++, compiled here with gcc); this module only
builds it and marshals arguments.

Every function is pinned by ``tests/test_oracle.py`` against something other
than itself: closed forms, library routines (numpy/torch softmax, polyfit),
hand-built inputs with a known skip set, and invariants the mathematics fixes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None
TILE = 128


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "oracle.cpp")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-o", _SO, src, "-lpthread"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_threshold_log2.restype = ctypes.c_float
        L.oracle_threshold_log2.argtypes = [f64, ctypes.c_int64]
        L.oracle_lambda_log2.restype = ctypes.c_float
        L.oracle_lambda_log2.argtypes = [f64]
        L.oracle_score_scale.restype = ctypes.c_float
        L.oracle_score_scale.argtypes = [f64, i32]
        L.oracle_resolve.restype = f64
        L.oracle_resolve.argtypes = [f64, f64, f64]
        L.oracle_fit_logspace.restype = i32
        L.oracle_fit_logspace.argtypes = [vp, vp, i32, vp, vp, vp, vp]
        L.oracle_walk.restype = i32
        L.oracle_walk.argtypes = [vp, vp, vp, vp, i32, i32, i32, f64, i32, vp, vp, i32, i32, vp, i32, vp,
                                  vp, vp, vp, vp, vp, i32, f64, f64, f64, i32]
        L.oracle_e4m3_nearest.restype = f64
        L.oracle_e4m3_nearest.argtypes = [f64]
        _lib = L
    return _lib


def threshold_log2(tsf: float, s_kv: int) -> float:
    """L = fp32(log2(tsf / S_kv)); -inf for tsf <= 0 (dense)."""
    return float(_load().oracle_threshold_log2(float(tsf), int(s_kv)))


def lambda_log2(lam: float) -> float:
    return float(_load().oracle_lambda_log2(float(lam)))


def score_scale(softmax_scale: float, D: int) -> float:
    return float(_load().oracle_score_scale(float(softmax_scale), int(D)))


def resolve(a: float, b: float, s: float) -> float:
    return float(_load().oracle_resolve(a, b, s))


def fit_logspace(s, sf):
    """Return (a, b, s_min, s_max); raises ValueError if the fit is undetermined."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    sf = np.ascontiguousarray(sf, dtype=np.float64)
    out = [ctypes.c_double() for _ in range(4)]
    rc = _load().oracle_fit_logspace(s.ctypes.data, sf.ctypes.data, len(s), *[ctypes.byref(o) for o in out])
    if rc != 0:
        raise ValueError("fit_logspace: fewer than two distinct usable sparsity points")
    return tuple(o.value for o in out)


def all_units(cu_seqlens, H):
    """Every (sequence, head, q-block) unit, head-major, then sequence, then q-block."""
    cu = np.asarray(cu_seqlens)
    units = []
    for h in range(H):
        for b in range(len(cu) - 1):
            S = int(cu[b + 1] - cu[b])
            for qb in range((S + TILE - 1) // TILE):
                units.append((b, h, qb))
    return np.asarray(units, dtype=np.int32).reshape(-1, 3)


def sample_units(cu_seqlens, H, n, seed=0):
    """A seeded sample of n units that always holds q-block 0 and the tail
    q-block of every sequence (on head 0 and the last head)."""
    cu = np.asarray(cu_seqlens)
    rng = np.random.default_rng(seed)
    must = []
    for b in range(len(cu) - 1):
        S = int(cu[b + 1] - cu[b])
        if S == 0:
            continue
        nq = (S + TILE - 1) // TILE
        for h in sorted({0, H - 1}):
            must += [(b, h, 0), (b, h, nq - 1)]
    chosen = list(dict.fromkeys(must))
    seqs = [b for b in range(len(cu) - 1) if cu[b + 1] > cu[b]]
    tries = 0
    while len(chosen) < n and tries < 100 * n:
        tries += 1
        b = int(rng.choice(seqs))
        S = int(cu[b + 1] - cu[b])
        u = (b, int(rng.integers(H)), int(rng.integers((S + TILE - 1) // TILE)))
        if u not in chosen:
            chosen.append(u)
    return np.asarray(chosen, dtype=np.int32).reshape(-1, 3)


def e4m3_nearest(x: float) -> float:
    """Nearest E4M3 value of x >= 0 (ties to even, saturating at 448)."""
    return float(_load().oracle_e4m3_nearest(float(x)))


P_SHIFT = 8.0  # sigma of the 8-bit P.V reading: P = 2^(s2 - r + sigma) <= 256
P_LAG = 0.0    # tau: the integer reference r follows ceil(m) as soon as m exceeds it


def walk(q, k, v, cu_seqlens, H, D, *, softmax_scale=0.0, units=None, tsf=None, L_seq=None,
         cal_lambdas=None, forced=None, max_tiles=None, nthreads=None, p_e4m3=False, p_shift=P_SHIFT,
         p_lag=P_LAG, out_scale=1.0):
    """Run the tiled skip-softmax walk on CPU.

    q, k, v: uint16 bf16 patterns [total_tokens, H, D]. Either ``tsf`` (one
    threshold_scale_factor for every sequence), ``L_seq`` (per-sequence log2
    thresholds) or ``cal_lambdas`` (calibration mode: raw lambda trials).
    ``p_e4m3`` selects the 8-bit P.V reading (P rounded to E4M3 against a
    per-row integer reference, see oracle.cpp); ``out_scale`` multiplies
    the outputs (the V descale when v holds decoded E4M3 values).
    Returns a dict with ``out`` [n_units, 128, D] fp32, ``dstat`` and
    ``decision`` [n_units, max_tiles], ``skips`` [n_units] and, in calibration
    mode, ``counts`` [n_units, n_cal].
    """
    L = _load()
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    batch = len(cu) - 1
    seqlens = np.diff(cu)
    if units is None:
        units = all_units(cu, H)
    units = np.ascontiguousarray(units, dtype=np.int32).reshape(-1, 3)
    n = units.shape[0]
    if max_tiles is None:
        max_tiles = int((seqlens.max() + TILE - 1) // TILE)
    mode = 1 if cal_lambdas is not None else 0
    if mode == 0:
        if L_seq is None:
            L_seq = [threshold_log2(tsf or 0.0, int(s)) for s in seqlens]
        L_seq = np.ascontiguousarray(L_seq, dtype=np.float32)
        L_cal, n_cal = None, 0
    else:
        L_cal = np.ascontiguousarray([lambda_log2(x) for x in cal_lambdas], dtype=np.float32)
        n_cal = len(L_cal)
    out = np.zeros((n, TILE, D), dtype=np.float32)
    dstat = np.zeros((n, max_tiles), dtype=np.float32)
    decision = np.zeros((n, max_tiles), dtype=np.uint8)
    skips = np.zeros(n, dtype=np.int32)
    counts = np.zeros((n, max(n_cal, 1)), dtype=np.int32)
    if forced is not None:
        forced = np.ascontiguousarray(forced, dtype=np.int8).reshape(n, max_tiles)
    for a in (q, k, v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    ptr = lambda a: a.ctypes.data if a is not None else None
    rc = L.oracle_walk(q.ctypes.data, k.ctypes.data, v.ctypes.data, cu.ctypes.data, batch, H, D,
                       float(softmax_scale), mode, ptr(L_seq) if mode == 0 else None,
                       ptr(L_cal) if mode == 1 else None, n_cal, n, units.ctypes.data, max_tiles,
                       ptr(forced), out.ctypes.data, dstat.ctypes.data, decision.ctypes.data, skips.ctypes.data,
                       counts.ctypes.data if mode == 1 else None, 1 if p_e4m3 else 0, float(p_shift),
                       float(p_lag), float(out_scale), nthreads or min(64, os.cpu_count() or 1))
    if rc != 0:
        raise ValueError("oracle_walk: bad arguments")
    res = dict(out=out, dstat=dstat, decision=decision, skips=skips, units=units, max_tiles=max_tiles)
    if mode == 1:
        res["counts"] = counts[:, :n_cal]
    return res
