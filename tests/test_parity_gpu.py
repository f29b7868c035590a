"""GPU parity: the sm_100a kernels through the C ABI against the CPU oracle on
the same seeded inputs (tolerances and the margin rule in tests/parity.py).

Small cases are compared whole; the long-sequence workloads (S = 8192 and
75,600, the varlen batch) on a seeded sample of (sequence, head, q-block)
units that always holds q-block 0 and the tail q-block of every sequence:
each unit's decisions and output rows depend on nothing outside it.
"""
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

    oracle_scale = 0.0  # softmax_scale the oracle is given (0: 1/sqrt(D))
    oracle_kw = {}      # further oracle arguments of the variant (the 8-bit P.V reading)

    def __init__(self, ssa, w: synth.Workload, q=None, k=None, v=None):
        self.ssa, self.w = ssa, w
        if q is None:
            q, k, v = synth.generate(w)
        self.q, self.k, self.v = q, k, v
        self.cu = w.cu_seqlens
        self.dq, self.dk, self.dv, self.dcu = parity.to_device(q, k, v, self.cu)
        self.Q = ssa.num_qblocks(self.cu)
        self.T = ssa.max_tiles(w.max_seqlen)

    def call(self, tsf, out, skip, bitmap, stat):
        self.ssa.fwd(self.dq, self.dk, self.dv, self.dcu, self.w.max_seqlen, tsf, out=out, skip_counter=skip,
                     decision_bitmap=bitmap, tile_stat=stat)

    def fwd(self, tsf, ex=True):
        """One forward; ex=False runs the call without diagnostics (the
        kernels the benchmark times)."""
        H = self.w.H
        skip = torch.full((H, self.Q), -1, dtype=torch.int32, device="cuda")
        bitmap = torch.zeros((H, self.Q, self.ssa.bitmap_words(self.w.max_seqlen)), dtype=torch.int32, device="cuda")
        stat = torch.full((H, self.Q, self.T), float("nan"), dtype=torch.float32, device="cuda")
        out = torch.full_like(self.dv, float("nan"))
        self.call(tsf, out, skip, bitmap if ex else None, stat if ex else None)
        self.ssa.check_device()
        return (parity.bf16_host(out), skip.cpu().numpy(), bitmap.cpu().numpy().view(np.uint32),
                stat.cpu().numpy())

    def walk(self, **kw):
        return oracle.walk(self.q, self.k, self.v, self.cu, self.w.H, self.w.D, softmax_scale=self.oracle_scale,
                           max_tiles=self.T, **self.oracle_kw, **kw)

    def L_seq(self, tsf):
        return [oracle.threshold_log2(tsf, s) for s in self.w.seqlens]


def check_forward(case, tsf, units=None, what="", plain=False):
    """The diagnostic forward against the oracle (decisions, statistics,
    skip counts, outputs; diverged units replayed). With ``plain`` the call
    without diagnostics runs too and must give the same output bit for bit
    and the same skip counts, so the benchmarked kernels are held to the
    same check."""
    out, skip, bitmap, stat = case.fwd(tsf)
    if plain:
        out_p, skip_p, _, _ = case.fwd(tsf, ex=False)
        np.testing.assert_array_equal(out_p.view(np.uint32), out.view(np.uint32), err_msg=f"{what} tsf={tsf}")
        np.testing.assert_array_equal(skip_p, skip, err_msg=f"{what} tsf={tsf}")
    res = case.walk(tsf=tsf, units=units)
    replay = lambda i, forced: case.walk(tsf=tsf, units=res["units"][i:i + 1], forced=forced[None, :])
    st = parity.Stats()
    parity.compare_forward(res, case.cu, case.L_seq(tsf), out, skip, bitmap, stat, st, what=f"{what} tsf={tsf}",
                           replay=replay)
    st.check(f"{what} tsf={tsf}")
    assert st.divergent_units <= max(1, len(res["units"]) // 10), st.divergent_units
    return st, skip


def test_tiny_full(ssa):
    """B1 H2 D64 S1024 (grid 4x16x16), every unit, tsf in {0, 100, 1000}."""
    case = Case(ssa, synth.TINY)
    ratios = []
    for tsf in synth.TINY.tsf:
        st, skip = check_forward(case, tsf, what="tiny", plain=True)
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
        check_forward(case, tsf, what=f"ragged D={D}", plain=True)


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
        check_forward(case, tsf, units=units, what="wan5b", plain=True)


def test_wan14b_resolved_thresholds(ssa):
    """S = 75,600, H = 40, D = 128 (grid 21x45x80): dense and tsf resolved from
    a*exp(b*s) with the pages' example (a, b) = (0.0003, 7.5) at s = 0.5, 0.7, 0.9."""
    case = Case(ssa, synth.WAN14B)
    units = oracle.sample_units(case.cu, case.w.H, 12, seed=2)
    a, b = synth.EXAMPLE_FORMULA
    for tsf in [0.0] + [ssa.resolve(a, b, s) for s in synth.TARGET_SPARSITIES]:
        check_forward(case, tsf, units=units, what="wan14b", plain=True)


def test_wan14b_at_the_benchmarked_thresholds(ssa):
    """The benchmark's own step: S = 75,600, H = 40, D = 128 at the
    thresholds it resolves (ssa_calibrate on this input, one fit point per
    trial, the log-space fit, a*exp(b*s) at s = 0.5, 0.7, 0.9; lambda reaches
    about 5 at 0.9) and dense. The call without diagnostics (the timed
    kernels) must equal the diagnostic call bit for bit, which is compared
    with the oracle on 16 sampled units; skip ratios land near the targets."""
    from block_sparse_flashattention_ssa_b200 import calibration as cal

    case = Case(ssa, synth.WAN14B)
    c = cal.calibrate(case.dq, case.dk, case.dv, case.dcu, case.w.max_seqlen)
    ssa.check_device()
    units = oracle.sample_units(case.cu, case.w.H, 16, seed=21)
    tiles = case.w.H * case.T * case.T
    check_forward(case, 0.0, units=units, what="wan14b bench dense", plain=True)
    for target in synth.TARGET_SPARSITIES:
        tsf = ssa.resolve(c.a, c.b, target)
        st, skip = check_forward(case, tsf, units=units, what=f"wan14b bench target {target}", plain=True)
        assert abs(skip.sum() / tiles - target) < 0.15, (target, tsf, skip.sum() / tiles)


def test_varlen_batch(ssa):
    """Four packed sequences (S = 32,760 / 46,800 / 5,120 / 75,600), H = 40,
    tsf = 5000 with lambda per sequence, 16 sampled units."""
    case = Case(ssa, synth.VARLEN)
    units = oracle.sample_units(case.cu, case.w.H, 16, seed=3)
    check_forward(case, 5000.0, units=units, what="varlen", plain=True)


def check_calibration(case, units=None, what="", lams=None):
    """ssa_calibrate_ex (counts and every tile's statistic) against the
    oracle's calibration walk, tile by tile; plain ssa_calibrate must give
    the same output and counts bit for bit."""
    lams = synth.CALIB_THRESHOLDS if lams is None else lams
    stat = torch.full((case.w.H, case.Q, case.T), float("nan"), dtype=torch.float32, device="cuda")
    out, counts = case.ssa.calibrate(case.dq, case.dk, case.dv, case.dcu, case.w.max_seqlen, lams, tile_stat=stat)
    case.ssa.check_device()
    out_p, counts_p = case.ssa.calibrate(case.dq, case.dk, case.dv, case.dcu, case.w.max_seqlen, lams)
    case.ssa.check_device()
    assert torch.equal(out.view(torch.int16), out_p.view(torch.int16)) and torch.equal(counts, counts_p)
    res = case.walk(cal_lambdas=lams, units=units)
    st = parity.Stats()
    cal_L = [oracle.lambda_log2(x) for x in lams]
    parity.compare_calibration(res, case.cu, cal_L, parity.bf16_host(out), counts.cpu().numpy(), st, what=what,
                               stat_gpu=stat.cpu().numpy())
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


@pytest.mark.parametrize("D", [64, 128])
def test_more_than_32_sequences(ssa, D):
    """A packed batch of 40 ragged sequences (empty, single-token, partial
    and multi-tile ones): past 32 sequences the kernels map their CTAs to
    (sequence, q-block pairs) in sequence order instead of longest first.
    Forward at three thresholds and a calibration with the largest number of
    trials one call takes (32), every unit against the oracle."""
    rng = np.random.default_rng(40 + D)
    lengths = [int(x) for x in rng.integers(0, 420, size=40)]
    lengths[3], lengths[17], lengths[29] = 0, 1, 128
    w = synth.Workload("40 sequences", [(1, 1, s) for s in lengths], H=2, D=D, seed=17, amp=3.0)
    case = Case(ssa, w)
    assert len(w.seqlens) > 32
    for tsf in [0.0, 60.0, 400.0]:
        check_forward(case, tsf, what=f"40 seqs D={D}", plain=True)
    lams = [float(x) for x in np.geomspace(1e-6, 8.0, ssa.MAX_THRESHOLDS)]
    check_calibration(case, what=f"calib 40 seqs D={D}", lams=lams)


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
                   1, 200, 200, 2, 64, 0.0, 10.0, vp(out.data_ptr()), None, 0, stream)
    assert rc == ssa.SSA_ERR_INVALID_ARG
    rc = L.ssa_fwd(vp(case.dq.data_ptr()), vp(case.dk.data_ptr()), vp(case.dv.data_ptr()), vp(case.dcu.data_ptr()),
                   1, 200, 200, 2, 64, 0.0, 10.0, vp(out.data_ptr()), vp(host_skip.data_ptr()), 2, stream)
    assert rc == ssa.SSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert ssa.get_error() == ssa.SSA_OK
    assert bool((out == 7.0).all()) and bool((host_skip == -1).all())  # nothing ran


def test_per_unit_outputs_sized_for_another_batch_are_never_written(ssa):
    """Per-unit outputs whose q-block count differs from the one cu_seqlens
    gives (too few or too many rows, or a sequence longer than max_seqlen for
    the diagnostics) make every kernel write nothing and report
    SSA_ERR_DEVICE_ARG; the right count works on the same buffers' sizes."""
    w = synth.Workload("two", [(1, 1, 300), (1, 1, 700)], H=2, D=64, seed=0)  # Q = 3 + 6
    case = Case(ssa, w)
    assert case.Q == 9
    lams = [1e-3, 0.5]
    for q_rows in (case.Q - 1, case.Q + 1):
        out = torch.full_like(case.dq, 7.0)
        skip = torch.full((w.H, q_rows), -1, dtype=torch.int32, device="cuda")
        ssa.fwd(case.dq, case.dk, case.dv, case.dcu, w.max_seqlen, 10.0, out=out, skip_counter=skip)
        assert ssa.get_error() == ssa.SSA_ERR_DEVICE_ARG
        counts = torch.full((w.H, q_rows, 2), -1, dtype=torch.int32, device="cuda")
        ssa.calibrate(case.dq, case.dk, case.dv, case.dcu, w.max_seqlen, lams, out=out, counts=counts)
        assert ssa.get_error() == ssa.SSA_ERR_DEVICE_ARG
        assert bool((out == 7.0).all()) and bool((skip == -1).all()) and bool((counts == -1).all())
    # diagnostics sized for a shorter max_seqlen than the batch holds
    short = 300
    bitmap = torch.zeros((w.H, case.Q, ssa.bitmap_words(short)), dtype=torch.int32, device="cuda")
    stat = torch.full((w.H, case.Q, ssa.max_tiles(short)), -1.0, dtype=torch.float32, device="cuda")
    out = torch.full_like(case.dq, 7.0)
    ssa.fwd(case.dq, case.dk, case.dv, case.dcu, short, 10.0, out=out, decision_bitmap=bitmap, tile_stat=stat)
    assert ssa.get_error() == ssa.SSA_ERR_DEVICE_ARG
    assert bool((out == 7.0).all()) and bool((bitmap == 0).all()) and bool((stat == -1.0).all())
    # the right count: written, no error
    skip = torch.full((w.H, case.Q), -1, dtype=torch.int32, device="cuda")
    ssa.fwd(case.dq, case.dk, case.dv, case.dcu, w.max_seqlen, 10.0, out=out, skip_counter=skip)
    assert ssa.get_error() == ssa.SSA_OK and bool((skip >= 0).all())
