"""GPU parity of the 8-bit Q/K forward (ssa_fwd_fp8) and of the E4M3
quantiser (ssa_quantize_fp8). The oracle runs the same walk on the exactly
decoded E4M3 values (each is exact in bf16) with the per-tensor descales
folded into the softmax scale, which is how the scores are defined for this
variant; outputs, decisions and skip counts are held to the same rules as
the bf16 forward."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import parity
from tests.test_parity_gpu import Case, check_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_ssa_b200 as m

    assert m.get_error() == m.SSA_OK
    return m


def _device_codes(ssa, bf16_codes, inv):
    x = torch.from_numpy(bf16_codes.view(np.int16)).to("cuda").view(torch.bfloat16)
    return ssa.quantize_fp8(x, float(inv))


class Fp8Case(Case):
    """Q and K quantised per tensor on the GPU; the oracle sees their exact
    decoded values and the descales inside the softmax scale."""

    def __init__(self, ssa, w):
        q, k, v = synth.generate(w)
        self.q8, self.q_inv, self.q_ds = synth.quantize_e4m3(q)
        self.k8, self.k_inv, self.k_ds = synth.quantize_e4m3(k)
        dec = lambda c: synth.f32_to_bf16(synth.e4m3_to_f32(c))
        super().__init__(ssa, w, dec(self.q8), dec(self.k8), v)
        self.dq8 = _device_codes(ssa, q, self.q_inv)
        self.dk8 = _device_codes(ssa, k, self.k_inv)
        torch.cuda.synchronize()
        assert np.array_equal(self.dq8.cpu().numpy(), self.q8) and np.array_equal(self.dk8.cpu().numpy(), self.k8)
        # oracle softmax scale: 1/sqrt(D) * q_descale * k_descale, in the order the library forms it
        self.oracle_scale = 1.0 / math.sqrt(w.D) * (float(self.q_ds) * float(self.k_ds))

    def call(self, tsf, out, skip, bitmap, stat):
        self.ssa.fwd_fp8(self.dq8, self.dk8, self.dv, self.dcu, self.w.max_seqlen, float(self.q_ds),
                         float(self.k_ds), tsf, out=out, skip_counter=skip, decision_bitmap=bitmap, tile_stat=stat)


def _check(case, tsf, units=None, what=""):
    return check_forward(case, tsf, units=units, what=what, plain=True)


def test_quantiser_matches_the_format_definition_bit_for_bit(ssa):
    rng = np.random.default_rng(9)
    n = 1_000_003  # not a multiple of 8: the scalar tail runs too
    x = (rng.standard_normal(n) * np.exp2(rng.uniform(-14, 12, n))).astype(np.float32)
    xb = synth.f32_to_bf16(x)
    for inv in [1.0, 0.37, 61.5]:
        got = _device_codes(ssa, xb, inv).cpu().numpy()
        want = synth.f32_to_e4m3(synth.bf16_to_f32(xb) * np.float32(inv))
        assert np.array_equal(got, want), inv


def test_fp8_ragged_varlen(ssa):
    lengths = [1, 5, 127, 128, 129, 300, 0, 1000]
    w = synth.Workload("ragged fp8", [(1, 1, s) for s in lengths], H=3, D=128, seed=12, amp=3.0)
    case = Fp8Case(ssa, w)
    for tsf in [0.0, 50.0, 300.0, 2000.0]:
        _check(case, tsf, what="ragged fp8")


def test_fp8_wan5b_sampled(ssa):
    case = Fp8Case(ssa, synth.WAN5B)
    units = oracle.sample_units(case.cu, case.w.H, 24, seed=4)
    for tsf in [0.0, 5e3, 2e4]:
        _check(case, tsf, units=units, what="wan5b fp8")


def test_fp8_skip_path_without_skips_is_bitwise_dense(ssa):
    w = synth.Workload("fp8 bitwise", [(2, 16, 32)], H=2, D=128, seed=3, amp=3.0)
    case = Fp8Case(ssa, w)
    dense = case.fwd(0.0, ex=False)
    tiny = case.fwd(1e-30, ex=False)
    np.testing.assert_array_equal(dense[0], tiny[0])
    assert tiny[1].sum() == 0


def test_fp8_calibration_counts_and_forward_equivalence(ssa):
    """ssa_calibrate_fp8 against the oracle's calibration walk on the decoded
    values; its output is the dense E4M3 output; for lambda <= 1 its counts
    equal ssa_fwd_fp8's skip counts at tsf = lambda * S (S = 1024, so the
    threshold is the same float on both paths)."""
    lams = synth.CALIB_THRESHOLDS
    w = synth.Workload("calib fp8", [(1, 1, 300), (1, 1, 129), (1, 1, 1000)], H=2, D=128, seed=13, amp=3.0)
    case = Fp8Case(ssa, w)
    out, counts = ssa.calibrate_fp8(case.dq8, case.dk8, case.dv, case.dcu, w.max_seqlen, float(case.q_ds),
                                    float(case.k_ds), lams)
    ssa.check_device()
    res = case.walk(cal_lambdas=lams)
    st = parity.Stats()
    parity.compare_calibration(res, case.cu, [oracle.lambda_log2(x) for x in lams], parity.bf16_host(out),
                               counts.cpu().numpy(), st, what="calib fp8")
    st.check("calib fp8")
    np.testing.assert_array_equal(parity.bf16_host(out), case.fwd(0.0, ex=False)[0])

    w1 = synth.Workload("calib fp8 S1024", [(4, 16, 16)], H=2, D=128, seed=14, amp=3.0)
    one = Fp8Case(ssa, w1)
    _, c1 = ssa.calibrate_fp8(one.dq8, one.dk8, one.dv, one.dcu, w1.max_seqlen, float(one.q_ds), float(one.k_ds),
                              lams)
    ssa.check_device()
    c1 = c1.cpu().numpy()
    for kk, lam in enumerate(lams):
        _, skip, _, _ = one.fwd(lam * 1024)
        assert np.array_equal(skip, c1[:, :, kk]), lam


def test_fp8_wan14b_at_the_benchmarked_threshold(ssa):
    """The benchmark's E4M3 row: S = 75,600, H = 40, D = 128 at the threshold
    it uses for target 0.7 (resolved from the bf16 calibration and fit on the
    same input) and dense, 12 sampled units; the call without diagnostics
    equals the diagnostic one bit for bit."""
    from block_sparse_flashattention_ssa_b200 import calibration as cal

    w = synth.WAN14B
    bf = Case(ssa, w)
    c = cal.calibrate(bf.dq, bf.dk, bf.dv, bf.dcu, w.max_seqlen)
    ssa.check_device()
    tsf = ssa.resolve(c.a, c.b, 0.7)
    del bf
    torch.cuda.empty_cache()
    case = Fp8Case(ssa, w)
    units = oracle.sample_units(case.cu, w.H, 12, seed=22)
    _check(case, 0.0, units=units, what="wan14b fp8 dense")
    _, skip = _check(case, tsf, units=units, what="wan14b fp8 target 0.7")
    assert skip.sum() > 0


class Fp8QkvCase(Case):
    """Q, K and V quantised per tensor on the GPU (ssa_fwd_fp8_qkv): the
    oracle walks the exactly decoded values with the Q/K descales in its
    softmax scale, the 8-bit P.V reading (P rounded to E4M3 against the
    per-row integer reference) and the V descale on its output."""

    def __init__(self, ssa, w):
        q, k, v = synth.generate(w)
        self.q8, self.q_inv, self.q_ds = synth.quantize_e4m3(q)
        self.k8, self.k_inv, self.k_ds = synth.quantize_e4m3(k)
        self.v8, self.v_inv, self.v_ds = synth.quantize_e4m3(v)
        dec = lambda c: synth.f32_to_bf16(synth.e4m3_to_f32(c))
        super().__init__(ssa, w, dec(self.q8), dec(self.k8), dec(self.v8))
        self.dq8 = _device_codes(ssa, q, self.q_inv)
        self.dk8 = _device_codes(ssa, k, self.k_inv)
        self.dv8 = _device_codes(ssa, v, self.v_inv)
        torch.cuda.synchronize()
        for dev_codes, host_codes in ((self.dq8, self.q8), (self.dk8, self.k8), (self.dv8, self.v8)):
            assert np.array_equal(dev_codes.cpu().numpy(), host_codes)
        self.oracle_scale = 1.0 / math.sqrt(w.D) * (float(self.q_ds) * float(self.k_ds))
        self.oracle_kw = dict(p_e4m3=True, out_scale=float(self.v_ds))

    def call(self, tsf, out, skip, bitmap, stat):
        self.ssa.fwd_fp8(self.dq8, self.dk8, self.dv8, self.dcu, self.w.max_seqlen, float(self.q_ds),
                         float(self.k_ds), tsf, out=out, skip_counter=skip, decision_bitmap=bitmap, tile_stat=stat,
                         v_descale=float(self.v_ds))


def test_fp8_qkv_ragged_varlen(ssa):
    """E4M3 Q, K, V and P on ragged lengths (1 .. 1000, an empty sequence),
    dense and lambda below and above 1: outputs, decisions, statistics and
    skip counts against the oracle; the call without diagnostics equals the
    diagnostic one bit for bit."""
    lengths = [1, 5, 127, 128, 129, 300, 0, 1000]
    w = synth.Workload("ragged fp8 qkv", [(1, 1, s) for s in lengths], H=3, D=128, seed=12, amp=3.0)
    case = Fp8QkvCase(ssa, w)
    for tsf in [0.0, 50.0, 300.0, 2000.0]:
        _check(case, tsf, what="ragged fp8 qkv")


def test_fp8_qkv_wan5b_sampled(ssa):
    case = Fp8QkvCase(ssa, synth.WAN5B)
    units = oracle.sample_units(case.cu, case.w.H, 24, seed=4)
    for tsf in [0.0, 5e3, 2e4]:
        _check(case, tsf, units=units, what="wan5b fp8 qkv")


def test_fp8_qkv_calibration(ssa):
    """ssa_calibrate_fp8_qkv: its output is the dense E4M3 Q/K/V output (the
    oracle's dense walk with the 8-bit P.V reading, and ssa_fwd_fp8_qkv at
    tsf = 0 bit for bit); its counts depend on Q and K only, so they equal
    ssa_calibrate_fp8's on the same E4M3 Q and K."""
    lams = synth.CALIB_THRESHOLDS
    w = synth.Workload("calib fp8 qkv", [(1, 1, 300), (1, 1, 129), (1, 1, 1000)], H=2, D=128, seed=13, amp=3.0)
    case = Fp8QkvCase(ssa, w)
    out, counts = ssa.calibrate_fp8(case.dq8, case.dk8, case.dv8, case.dcu, w.max_seqlen, float(case.q_ds),
                                    float(case.k_ds), lams, v_descale=float(case.v_ds))
    ssa.check_device()
    v_bf16 = torch.from_numpy(synth.generate(w)[2].view(np.int16)).cuda().view(torch.bfloat16)
    _, counts_qk = ssa.calibrate_fp8(case.dq8, case.dk8, v_bf16, case.dcu, w.max_seqlen, float(case.q_ds),
                                     float(case.k_ds), lams)
    ssa.check_device()
    assert torch.equal(counts, counts_qk)
    res = case.walk(cal_lambdas=lams)
    st = parity.Stats()
    parity.compare_calibration(res, case.cu, [oracle.lambda_log2(x) for x in lams], parity.bf16_host(out),
                               counts.cpu().numpy(), st, what="calib fp8 qkv")
    st.check("calib fp8 qkv")
    np.testing.assert_array_equal(parity.bf16_host(out), case.fwd(0.0, ex=False)[0])
