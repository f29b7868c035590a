"""Failure detection on the GPU without a fault: the kernels' bounded
mbarrier wait gives up on a barrier nothing arrives on, reports
SSA_ERR_TIMEOUT through the device status word, and the context stays
usable (a forward afterwards still matches the oracle)."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_bounded_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_ssa_b200 as ssa
    from tests import parity

    assert ssa.get_error() == ssa.SSA_OK
    completed, abort_flag, waited_us = ssa.wait_timeout_check(20_000_000)  # 20 ms limit
    assert completed == 0 and abort_flag == 1
    assert 20_000 <= waited_us < 2_000_000
    assert ssa.get_error() == ssa.SSA_ERR_TIMEOUT
    assert ssa.get_error() == ssa.SSA_OK  # cleared

    w = synth.Workload("after-timeout", [(1, 1, 300)], H=2, D=64, seed=3)
    q, k, v = synth.generate(w)
    dq, dk, dv, dcu = parity.to_device(q, k, v, w.cu_seqlens)
    out = ssa.fwd(dq, dk, dv, dcu, w.max_seqlen, 50.0)
    ssa.check_device()
    res = oracle.walk(q, k, v, w.cu_seqlens, w.H, w.D, tsf=50.0)
    got = parity.bf16_host(out)
    for i, (b, h, qb) in enumerate(res["units"]):
        n = min(128, 300 - qb * 128)
        assert np.abs(got[qb * 128: qb * 128 + n, h] - res["out"][i, :n]).max() <= parity.MAX_ABS
