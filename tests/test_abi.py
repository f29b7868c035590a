"""The C-ABI library on a machine without a GPU: it loads, exports every
entry point include/ssa.h declares, rejects bad arguments on the host before
touching CUDA, and its host-side math agrees with the oracle."""
import ctypes
import math
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from tests.golden import first

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    text = open(os.path.join(ROOT, "include", "ssa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|double|const char\*)\s+(ssa_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def ssa():
    import __graft_entry__

    __graft_entry__._library_builder().build()
    import block_sparse_flashattention_ssa_b200 as m

    return m


def test_library_exports_every_declared_symbol(ssa):
    names = declared_entry_points()
    assert {"ssa_fwd", "ssa_fwd_ex", "ssa_calibrate", "ssa_resolve", "ssa_fit_logspace"} <= set(names)
    out = subprocess.check_output(["nm", "-D", "--defined-only", ssa.library_path()], text=True)
    exported = set(re.findall(r" T (ssa_\w+)$", out, re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(ssa.lib(), n)


def test_library_is_built_for_sm100a(ssa):
    out = subprocess.run(["cuobjdump", "--list-elf", ssa.library_path()], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_host_argument_validation(ssa):
    L = ssa.lib()
    fake = ctypes.c_void_p(0x10000)
    mis = ctypes.c_void_p(0x10008)
    none = None
    args = dict(q=fake, k=fake, v=fake, cu=fake, batch=1, total=256, maxs=256, H=2, D=128, scale=0.0, tsf=0.0,
                out=fake, sc=None, nq=2, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return L.ssa_fwd(a["q"], a["k"], a["v"], a["cu"], a["batch"], a["total"], a["maxs"], a["H"], a["D"],
                         a["scale"], a["tsf"], a["out"], a["sc"], a["nq"], a["stream"])

    assert call(q=none) == ssa.SSA_ERR_INVALID_ARG
    assert call(out=none) == ssa.SSA_ERR_INVALID_ARG
    assert call(batch=0) == ssa.SSA_ERR_INVALID_ARG
    assert call(total=-1) == ssa.SSA_ERR_INVALID_ARG
    assert call(H=0) == ssa.SSA_ERR_INVALID_ARG
    assert call(D=96) == ssa.SSA_ERR_UNSUPPORTED
    assert call(D=256) == ssa.SSA_ERR_UNSUPPORTED
    assert call(k=mis) == ssa.SSA_ERR_UNSUPPORTED
    assert call(tsf=float("nan")) == ssa.SSA_ERR_INVALID_ARG
    assert call(tsf=float("inf")) == ssa.SSA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == ssa.SSA_ERR_INVALID_ARG
    assert call(total=0) == ssa.SSA_OK  # nothing to do, nothing launched
    assert call(sc=fake, nq=-1) == ssa.SSA_ERR_INVALID_ARG  # a per-unit output needs its q-block count
    th = np.array([1e-3, 0.5], dtype=np.float32)
    cal = lambda th, n, counts=fake, nq=2: L.ssa_calibrate(fake, fake, fake, fake, 1, 256, 256, 2, 128, 0.0,
                                                           th.ctypes.data if th is not None else None, n, fake,
                                                           counts, nq, None)
    assert cal(th, 0) == ssa.SSA_ERR_INVALID_ARG
    assert cal(th, 33) == ssa.SSA_ERR_INVALID_ARG
    assert cal(None, 2) == ssa.SSA_ERR_INVALID_ARG
    assert cal(th, 2, counts=None) == ssa.SSA_ERR_INVALID_ARG
    assert cal(th, 2, nq=-1) == ssa.SSA_ERR_INVALID_ARG
    assert cal(np.array([1e-3, 0.0], dtype=np.float32), 2) == ssa.SSA_ERR_INVALID_ARG
    ex = L.ssa_fwd_ex(fake, fake, fake, fake, 1, 256, 0, 2, 128, 0.0, 10.0, fake, None, 2, fake, None, None)
    assert ex == ssa.SSA_ERR_INVALID_ARG  # diagnostics need max_seqlen >= 1
    cex = L.ssa_calibrate_ex(fake, fake, fake, fake, 1, 256, 0, 2, 128, 0.0, th.ctypes.data, 2, fake, fake, 2,
                             fake, None)
    assert cex == ssa.SSA_ERR_INVALID_ARG  # so does the calibration statistic
    assert ssa.lib().ssa_status_string(ssa.SSA_ERR_TIMEOUT)


def test_num_qblocks(ssa):
    assert ssa.num_qblocks([0, 1, 129, 129, 385]) == 1 + 1 + 0 + 2  # lengths 1, 128, 0, 256
    assert ssa.num_qblocks([0, 75600]) == 591
    with pytest.raises(ssa.SSAError):
        ssa.num_qblocks([0, 10, 5])


def test_resolve_and_fit_match_oracle(ssa):
    for a, b in first("page_constants.txt", "formula"):
        for s in [0.0, 0.25, 0.5, 0.7, 0.9, 1.0]:
            assert ssa.resolve(a, b, s) == oracle.resolve(a, b, s)
    assert math.isnan(ssa.resolve(0.0, 1.0, 0.5)) and math.isnan(ssa.resolve(1.0, 1.0, -0.1))
    rng = np.random.default_rng(1)
    s = rng.uniform(0.0, 1.0, 50)
    s[:3] = [0.0, 1.0, 0.0]
    sf = 3e-4 * np.exp(7.5 * s) * np.exp(rng.normal(0, 0.2, 50))
    got = ssa.fit_logspace(s, sf)
    ref = oracle.fit_logspace(s, sf)
    np.testing.assert_allclose(got, ref, rtol=1e-12)
    with pytest.raises(ssa.SSAError):
        ssa.fit_logspace([0.5, 0.5], [1.0, 1.0])


def test_fp8_entry_points_validate_on_the_host(ssa):
    L = ssa.lib()
    fake = ctypes.c_void_p(0x10000)
    mis = ctypes.c_void_p(0x10008)

    def f8(D=128, qd=1.0, kd=1.0, total=256, q=fake, tsf=0.0):
        return L.ssa_fwd_fp8(q, fake, fake, fake, 1, total, 256, 2, D, 0.0, qd, kd, tsf, fake, None, 0, None, None,
                             None)

    assert f8(D=64) == ssa.SSA_ERR_UNSUPPORTED  # E4M3 rows must be 128 bytes
    assert f8(qd=0.0) == ssa.SSA_ERR_INVALID_ARG
    assert f8(kd=-1.0) == ssa.SSA_ERR_INVALID_ARG
    assert f8(qd=float("inf")) == ssa.SSA_ERR_INVALID_ARG
    assert f8(q=None) == ssa.SSA_ERR_INVALID_ARG
    assert f8(q=mis) == ssa.SSA_ERR_UNSUPPORTED
    assert f8(tsf=float("nan")) == ssa.SSA_ERR_INVALID_ARG
    assert f8(total=0) == ssa.SSA_OK
    def f8v(vd=1.0, D=128, total=256):
        return L.ssa_fwd_fp8_qkv(fake, fake, fake, fake, 1, total, 256, 2, D, 0.0, 1.0, 1.0, vd, 0.0, fake, None, 0,
                                 None, None, None)

    assert f8v(vd=0.0) == ssa.SSA_ERR_INVALID_ARG
    assert f8v(vd=float("inf")) == ssa.SSA_ERR_INVALID_ARG
    assert f8v(D=64) == ssa.SSA_ERR_UNSUPPORTED
    assert f8v(total=0) == ssa.SSA_OK
    th = np.array([1e-3], dtype=np.float32)
    assert L.ssa_calibrate_fp8_qkv(fake, fake, fake, fake, 1, 256, 256, 2, 128, 0.0, 1.0, 1.0, -1.0, th.ctypes.data,
                                   1, fake, fake, 2, None) == ssa.SSA_ERR_INVALID_ARG
    qz = lambda x, y, n, s: L.ssa_quantize_fp8(x, y, n, s, None)
    assert qz(fake, fake, -1, 1.0) == ssa.SSA_ERR_INVALID_ARG
    assert qz(fake, fake, 16, 0.0) == ssa.SSA_ERR_INVALID_ARG
    assert qz(fake, fake, 16, float("inf")) == ssa.SSA_ERR_INVALID_ARG
    assert qz(None, fake, 16, 1.0) == ssa.SSA_ERR_INVALID_ARG
    assert qz(mis, fake, 16, 1.0) == ssa.SSA_ERR_UNSUPPORTED
    assert qz(fake, ctypes.c_void_p(0x10004), 16, 1.0) == ssa.SSA_ERR_UNSUPPORTED
    assert qz(fake, fake, 0, 1.0) == ssa.SSA_OK


def test_per_unit_outputs_are_checked_before_the_library_is_called(ssa):
    """Every per-unit output must be [H, Q, inner] with the inner size that
    max_seqlen (or the threshold count) fixes and one Q shared by all of
    them; an undersized or misshapen buffer of any of the four kinds is a
    ValueError before any call. (The exact Q is checked by the kernels
    against the device copy of cu_seqlens.)"""
    import torch

    cpu = torch.device("cpu")
    H, total, batch, max_seqlen = 3, 1000, 2, 700  # T = 6 tiles, 1 bitmap word
    z = lambda *shape, dt=torch.int32: torch.zeros(shape, dtype=dt)
    good = ssa._forward_outputs(z(H, 9), z(H, 9, 1), z(H, 9, 6, dt=torch.float32), max_seqlen)
    assert ssa._per_unit_qblocks(cpu, H, total, batch, good) == 9
    assert ssa._per_unit_qblocks(cpu, H, total, batch, ssa._forward_outputs(None, None, None, max_seqlen)) == -1
    bad_forward = [
        (z(H - 1, 9), None, None),                          # skip_counter: too few heads
        (z(H, 9, 2), None, None),                           # skip_counter: an inner dimension
        (None, z(H, 9, 0), None),                           # decision_bitmap: no word per unit
        (None, z(H, 9), None),                              # decision_bitmap: missing its word axis
        (None, None, z(H, 9, 5, dt=torch.float32)),         # tile_stat: one tile short
        (None, None, z(H, 9, 6)),                           # tile_stat: wrong dtype
        (z(H, 9), z(H, 8, 1), None),                        # two outputs, two q-block counts
        (z(H, 100), None, None),                            # more q-blocks than 1000 tokens in 2 sequences
    ]
    for sc, bm, ts in bad_forward:
        with pytest.raises((ValueError, TypeError)):
            ssa._per_unit_qblocks(cpu, H, total, batch, ssa._forward_outputs(sc, bm, ts, max_seqlen))
    counts = lambda q, n: [(z(H, q, n), "counts", torch.int32, (4,))]
    assert ssa._per_unit_qblocks(cpu, H, total, batch, counts(9, 4)) == 9
    for q, n in [(9, 3), (9, 5)]:                           # counts: wrong number of thresholds
        with pytest.raises(ValueError):
            ssa._per_unit_qblocks(cpu, H, total, batch, counts(q, n))


def test_package_refuses_to_import_without_its_library(tmp_path):
    """No CPU fallback: a copy of the package without libssa.so fails at
    import with a message naming the missing library."""
    import shutil
    import sys

    src = os.path.join(ROOT, "block_sparse_flashattention_ssa_b200")
    shutil.copytree(src, tmp_path / "block_sparse_flashattention_ssa_b200",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import block_sparse_flashattention_ssa_b200"], cwd=str(tmp_path),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libssa.so is not built" in r.stderr
