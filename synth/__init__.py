"""Seeded synthetic Q/K/V for video-diffusion self-attention (shared test and
benchmark fixture).

Holds no attention arithmetic: it draws the packed ``[total_tokens, H, D]``
bf16 inputs (as uint16 bit patterns) that both the CPU oracle and the GPU
path consume, and names the workloads they are drawn for. The recipe is in
``synth.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", _SO, src, "-lm", "-lpthread"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_qkv.restype = ctypes.c_int64
        lib.synth_qkv.argtypes = [ctypes.c_uint64, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_uint64]
        lib.synth_pe.restype = ctypes.c_double
        lib.synth_pe.argtypes = [ctypes.c_int] * 5
        lib.synth_bf16_rne.restype = ctypes.c_uint16
        lib.synth_bf16_rne.argtypes = [ctypes.c_float]
        lib.synth_splitmix64.restype = ctypes.c_uint64
        lib.synth_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        _lib = lib
    return _lib


def lib():
    return _load()


@dataclass
class Workload:
    """One synthetic self-attention problem: a batch of video token grids."""

    name: str
    grids: list  # [(T, Hh, Ww)] per sequence
    H: int
    D: int
    seed: int = 0
    amp: float = 3.0
    tsf: list = field(default_factory=list)  # threshold_scale_factor values to run

    @property
    def seqlens(self):
        return [t * h * w for (t, h, w) in self.grids]

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens))

    def num_qblocks(self, block: int = 128) -> int:
        return int(sum((s + block - 1) // block for s in self.seqlens))

    def dense_flop(self) -> float:
        """4 * S^2 * D * H summed over sequences (QK^T and PV, every tile)."""
        return float(sum(4.0 * s * s * self.D * self.H for s in self.seqlens))


def generate(w: Workload, nthreads: int | None = None, tensors=("q", "k", "v")):
    """Return (q, k, v) uint16 arrays of shape [total_tokens, H, D] (bf16 bits)."""
    L = _load()
    n = w.total_tokens
    out = {}
    for name in ("q", "k", "v"):
        out[name] = np.empty((n, w.H, w.D), dtype=np.uint16) if name in tensors else None
    grids = np.asarray(w.grids, dtype=np.int32).reshape(-1, 3)
    nt = nthreads or min(64, os.cpu_count() or 1)
    ptr = lambda a: a.ctypes.data if a is not None else None
    got = L.synth_qkv(w.seed, w.amp, w.H, w.D, len(w.grids), grids.ctypes.data,
                      ptr(out["q"]), ptr(out["k"]), ptr(out["v"]), nt)
    if got != n:
        raise RuntimeError(f"synth_qkv failed ({got})")
    return out["q"], out["k"], out["v"]


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bit patterns, nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


# --- E4M3 (OCP 8-bit floating point, the variant without infinities) -------
# 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 holds the
# subnormals m * 2^-9; S.1111.111 is NaN; the largest finite value is 448.
# Used to prepare 8-bit Q/K inputs: every E4M3 value is exact in bf16.
E4M3_MAX = 448.0


def e4m3_to_f32(codes: np.ndarray) -> np.ndarray:
    """Exact value of E4M3 codes (uint8) as float32 (NaN for the NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int32)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * mag
    return np.where((e == 15) & (m == 7), np.nan, val).astype(np.float32)


_E4M3_POS = e4m3_to_f32(np.arange(127, dtype=np.uint8)).astype(np.float64)  # codes 0..126, increasing


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to E4M3 codes: nearest, ties to the even
    code, magnitudes beyond 448 saturate to 448, the sign is kept (-0 -> 0x80)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 126)  # first value >= a
    lo = np.clip(hi - 1, 0, 126)
    d_hi = _E4M3_POS[hi] - a
    d_lo = a - _E4M3_POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= _E4M3_POS[126], 126, code)
    code = np.where(a <= 0.0, 0, code)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def quantize_e4m3(bf16_codes: np.ndarray):
    """Per-tensor E4M3 quantisation of a bf16 tensor: inv_scale = fp32(448 / amax),
    codes = E4M3(fp32(x * inv_scale)). Returns (codes, inv_scale as float32,
    descale = 1 / inv_scale as float32)."""
    x = bf16_to_f32(bf16_codes)
    amax = float(np.max(np.abs(x)))
    inv = np.float32(E4M3_MAX / amax)
    codes = f32_to_e4m3(x * inv)  # float32 product, rounded once
    return codes, inv, np.float32(1.0 / np.float64(inv))


# Workloads: the tiny case the oracle finishes whole, the WAN-5B-like and the
# WAN-14B 720p self-attention shapes, the calibration sweep and a varlen batch.
TINY = Workload("tiny B1 H2 D64 S1024 grid 4x16x16", [(4, 16, 16)], H=2, D=64, seed=0, tsf=[0.0, 100.0, 1000.0])
WAN5B = Workload("WAN-5B-like B1 H24 D128 S8192 grid 8x32x32", [(8, 32, 32)], H=24, D=128, seed=0,
                 tsf=[0.0, 1e2, 1e3, 5e3, 2e4])
WAN14B = Workload("WAN-14B 720p B1 H40 D128 S75600 grid 21x45x80", [(21, 45, 80)], H=40, D=128, seed=0)
VARLEN = Workload("varlen 4 seqs S=32760/46800/5120/75600 H40 D128",
                  [(21, 30, 52), (13, 45, 80), (5, 32, 32), (21, 45, 80)], H=40, D=128, seed=7, tsf=[5000.0])
CALIB_THRESHOLDS = [1e-6, 5e-6, 1e-5, 5e-5, 1e-4, 5e-4, 1e-3, 5e-3, 1e-2, 2e-2, 5e-2, 1e-1, 2e-1, 3e-1, 5e-1, 7e-1]
CALIB_SEEDS = [0, 1, 2, 3]
CALIB_AMPS = [2.0, 3.0, 4.0, 5.0]
# threshold_scale_factor = a * exp(b * s) example coefficients (TRT-LLM PR #12947, "Use Cases", case 1c)
EXAMPLE_FORMULA = (0.0003, 7.5)
TARGET_SPARSITIES = [0.5, 0.7, 0.9]
