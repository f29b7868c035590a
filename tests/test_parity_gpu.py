"""GPU parity: the sm_100a kernels through the C ABI against the CPU oracle on
the same seeded inputs (tolerances and the margin rule in tests/parity.py).

Small cases are compared whole; the long-sequence workloads (S = 8192 and
75,600, the varlen batch) on a seeded sample of (sequence, head, q-block)
units that always holds q-block 0 and the tail q-block of every sequence:
each unit's decisions and output rows depend on nothing outside it.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_ssa_b200 as m

    assert m.get_error() == m.SSA_OK
    return m


class Case:
    """Host inputs, their device copies and the GPU runs of one workload."""

    def __init__(self, ssa, w: synth.Workload, q=None, k=None, v=None):
        self.ssa, self.w = ssa, w
        if q is None:
            q, k, v = synth.generate(w)
        self.q, self.k, self.v = q, k, v
        self.cu = w.cu_seqlens
        self.dq, self.dk, self.dv, self.dcu = parity.to_device(q, k, v, self.cu)
        self.Q = ssa.num_qblocks(self.cu)
        self.T = ssa.max_tiles(w.max_seqlen)

    def fwd(self, tsf, ex=True):
        H = self.w.H
        skip = torch.full((H, self.Q), -1, dtype=torch.int32, device="cuda")
        bitmap = torch.zeros((H, self.Q, self.ssa.bitmap_words(self.w.max_seqlen)), dtype=torch.int32, device="cuda")
        stat = torch.full((H, self.Q, self.T), float("nan"), dtype=torch.float32, device="cuda")
        out = torch.full_like(self.dq, float("nan"))
        self.ssa.fwd(self.dq, self.dk, self.dv, self.dcu, self.w.max_seqlen, tsf, out=out, skip_counter=skip,
                     decision_bitmap=bitmap if ex else None, tile_stat=stat if ex else None)
        self.ssa.check_device()
        return (parity.bf16_host(out), skip.cpu().numpy(), bitmap.cpu().numpy().view(np.uint32),
                stat.cpu().numpy())

    def L_seq(self, tsf):
        return [oracle.threshold_log2(tsf, s) for s in self.w.seqlens]


def check_forward(case, tsf, units=None, what=""):
    out, skip, bitmap, stat = case.fwd(tsf)
    res = oracle.walk(case.q, case.k, case.v, case.cu, case.w.H, case.w.D, tsf=tsf, units=units, max_tiles=case.T)
    st = parity.Stats()
    parity.compare_forward(res, case.cu, case.L_seq(tsf), out, skip, bitmap, stat, st, what=f"{what} tsf={tsf}")
    st.check(f"{what} tsf={tsf}")
    assert st.divergent_units <= max(1, len(res["units"]) // 50), st.divergent_units
    return st, skip


def test_tiny_full(ssa):
    """B1 H2 D64 S1024 (grid 4x16x16), every unit, tsf in {0, 100, 1000}."""
    case = Case(ssa, synth.TINY)
    ratios = []
    for tsf in synth.TINY.tsf:
        st, skip = check_forward(case, tsf, what="tiny")
        ratios.append(skip.sum() / st.tiles)
    assert ratios[0] == 0 and ratios[2] >= ratios[1]


@pytest.mark.parametrize("D", [64, 128])
def test_ragged_varlen(ssa, D):
    """Ragged lengths (1, short, one tile +- 1, an empty sequence, several
    tiles) in one packed batch; thresholds giving lambda both below and
    above 1."""
    lengths = [1, 5, 127, 128, 129, 300, 0, 1000]
    w = synth.Workload("ragged", [(1, 1, s) for s in lengths], H=3, D=D, seed=12, amp=3.0)
    q, k, v = synth.generate(w)
    cu = w.cu_seqlens
    case = Case(ssa, w, q, k, v)
    for tsf in [0.0, 50.0, 300.0, 2000.0]:
        check_forward(case, tsf, what=f"ragged D={D}")


def test_skip_path_without_skips_is_bitwise_dense(ssa):
    """A threshold so small that no tile can be skipped runs the skipping
    kernel yet must give the dense kernel's output bit for bit."""
    case = Case(ssa, synth.TINY)
    dense = case.fwd(0.0, ex=False)
    tiny = case.fwd(1e-30, ex=False)
    np.testing.assert_array_equal(dense[0], tiny[0])
    assert tiny[1].sum() == 0


def test_wan5b_threshold_sweep(ssa):
    """S = 8192, H = 24, D = 128 (grid 8x32x32); tsf in {0, 1e2, 1e3, 5e3, 2e4}
    (lambda up to 2.4 > 1), 32 sampled units each."""
    case = Case(ssa, synth.WAN5B)
    units = oracle.sample_units(case.cu, case.w.H, 32, seed=1)
    for tsf in synth.WAN5B.tsf:
        check_forward(case, tsf, units=units, what="wan5b")


def test_wan14b_resolved_thresholds(ssa):
    """S = 75,600, H = 40, D = 128 (grid 21x45x80): dense and tsf resolved from
    a*exp(b*s) with the pages' example (a, b) = (0.0003, 7.5) at s = 0.5, 0.7, 0.9."""
    case = Case(ssa, synth.WAN14B)
    units = oracle.sample_units(case.cu, case.w.H, 12, seed=2)
    a, b = synth.EXAMPLE_FORMULA
    for tsf in [0.0] + [ssa.resolve(a, b, s) for s in synth.TARGET_SPARSITIES]:
        check_forward(case, tsf, units=units, what="wan14b")


def test_varlen_batch(ssa):
    """Four packed sequences (S = 32,760 / 46,800 / 5,120 / 75,600), H = 40,
    tsf = 5000 with lambda per sequence, 16 sampled units."""
    case = Case(ssa, synth.VARLEN)
    units = oracle.sample_units(case.cu, case.w.H, 16, seed=3)
    check_forward(case, 5000.0, units=units, what="varlen")


def check_calibration(case, units=None, what=""):
    lams = synth.CALIB_THRESHOLDS
    out, counts = case.ssa.calibrate(case.dq, case.dk, case.dv, case.dcu, case.w.max_seqlen, lams)
    case.ssa.check_device()
    res = oracle.walk(case.q, case.k, case.v, case.cu, case.w.H, case.w.D, cal_lambdas=lams, units=units,
                      max_tiles=case.T)
    st = parity.Stats()
    cal_L = [oracle.lambda_log2(x) for x in lams]
    parity.compare_calibration(res, case.cu, cal_L, parity.bf16_host(out), counts.cpu().numpy(), st, what=what)
    st.check(what)
    return counts.cpu().numpy()


def test_calibration_tiny_and_equivalence_with_forward(ssa):
    """16 raw-lambda trials at once; for every lambda_k <= 1 the count equals
    the forward pass's skip count at tsf = lambda_k * S (up to margin tiles);
    the calibration output is the dense output."""
    case = Case(ssa, synth.TINY)
    counts = check_calibration(case, what="calib tiny")
    S = synth.TINY.seqlens[0]
    res_dense = case.fwd(0.0)
    for kk, lam in enumerate(synth.CALIB_THRESHOLDS):
        _, skip, _, stat = case.fwd(lam * S)
        d = stat[:, :, 1:]
        near = int((np.abs(d - oracle.lambda_log2(lam)) <= 2e-3).sum())
        assert abs(int(skip.sum()) - int(counts[:, :, kk].sum())) <= near, lam
    out_cal, _ = ssa.calibrate(case.dq, case.dk, case.dv, case.dcu, case.w.max_seqlen, [0.5])
    np.testing.assert_array_equal(parity.bf16_host(out_cal), res_dense[0])


def test_calibration_wan5b_sampled(ssa):
    case = Case(ssa, synth.WAN5B)
    units = oracle.sample_units(case.cu, case.w.H, 24, seed=4)
    check_calibration(case, units=units, what="calib wan5b")


def test_calibration_varlen_sampled(ssa):
    """Calibration counts over a packed batch of sequences of different
    lengths (each unit counts against its own sequence's tiles)."""
    case = Case(ssa, synth.VARLEN)
    units = oracle.sample_units(case.cu, case.w.H, 16, seed=5)
    check_calibration(case, units=units, what="calib varlen")


def test_d64_long_sequence_sampled(ssa):
    """D = 64 at S = 8192 (the WAN-5B-like grid, 16 heads): dense and two
    thresholds (lambda below and above 1), 24 sampled units each."""
    w = synth.Workload("D64 S8192", [(8, 32, 32)], H=16, D=64, seed=11, amp=3.0)
    case = Case(ssa, w)
    units = oracle.sample_units(case.cu, w.H, 24, seed=6)
    for tsf in [0.0, 3000.0, 12000.0]:
        check_forward(case, tsf, units=units, what="d64 s8192")


def test_empty_inputs_and_device_side_argument_check(ssa):
    w = synth.Workload("one", [(1, 1, 200)], H=2, D=64, seed=0)
    case = Case(ssa, w)
    # total_tokens = 0: a no-op
    e = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    cu0 = torch.zeros(2, dtype=torch.int32, device="cuda")
    ssa.fwd(e, e, e, cu0, 0, 10.0, out=e)
    # a batch of empty sequences: nothing written
    out = torch.full_like(case.dq, 7.0)
    cu_empty = torch.tensor([0, 0, 0], dtype=torch.int32, device="cuda")
    ssa.fwd(case.dq, case.dk, case.dv, cu_empty, 0, 10.0, out=out)
    assert ssa.get_error() == ssa.SSA_OK
    assert bool((out == 7.0).all())
    # decreasing cu_seqlens: the kernel refuses it and reports it; no row is written
    bad = torch.tensor([0, 150, 100], dtype=torch.int32, device="cuda")
    ssa.fwd(case.dq, case.dk, case.dv, bad, 200, 10.0, out=out)
    assert ssa.get_error() == ssa.SSA_ERR_DEVICE_ARG
    assert bool((out == 7.0).all())
    assert ssa.get_error() == ssa.SSA_OK  # the status word was cleared


def test_host_memory_is_refused_before_any_launch(ssa):
    """Arguments that are not device memory of the current device never
    reach a kernel: the binding rejects host tensors, and the C entry points
    reject host pointers (checked here with pinned, device-mapped host
    memory, which a kernel could read without faulting, so the test cannot
    fault the GPU even if the check were missing)."""
    import ctypes

    w = synth.Workload("one", [(1, 1, 200)], H=2, D=64, seed=0)
    case = Case(ssa, w)
    with pytest.raises(ValueError):
        ssa.fwd(case.dq.cpu(), case.dk, case.dv, case.dcu, 200, 10.0)
    with pytest.raises(ValueError):
        ssa.fwd(case.dq, case.dk, case.dv, case.dcu.cpu(), 200, 10.0)
    with pytest.raises(ValueError):
        ssa.fwd(case.dq, case.dk, case.dv, case.dcu, 200, 10.0,
                skip_counter=torch.zeros((2, 2), dtype=torch.int32).pin_memory())
    L = ssa.lib()
    vp = ctypes.c_void_p
    out = torch.full_like(case.dq, 7.0)
    host_cu = torch.tensor([0, 200], dtype=torch.int32).pin_memory()
    host_skip = torch.full((2, 2), -1, dtype=torch.int32).pin_memory()
    stream = vp(torch.cuda.current_stream().cuda_stream)
    rc = L.ssa_fwd(vp(case.dq.data_ptr()), vp(case.dk.data_ptr()), vp(case.dv.data_ptr()), vp(host_cu.data_ptr()),
                   1, 200, 200, 2, 64, 0.0, 10.0, vp(out.data_ptr()), None, stream)
    assert rc == ssa.SSA_ERR_INVALID_ARG
    rc = L.ssa_fwd(vp(case.dq.data_ptr()), vp(case.dk.data_ptr()), vp(case.dv.data_ptr()), vp(case.dcu.data_ptr()),
                   1, 200, 200, 2, 64, 0.0, 10.0, vp(out.data_ptr()), vp(host_skip.data_ptr()), stream)
    assert rc == ssa.SSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert ssa.get_error() == ssa.SSA_OK
    assert bool((out == 7.0).all()) and bool((host_skip == -1).all())  # nothing ran
