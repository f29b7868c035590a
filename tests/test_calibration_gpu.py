"""The calibrated loop on the GPU: count on the kernel, fit, resolve a target
sparsity, run the forward at it (README "Calibrated threshold"; commit page
"Calibration"). The fit is empirical, so the achieved sparsity is held to a
band around the target; at a trial threshold lambda <= 1 the forward's skip
count equals the calibration count exactly (the skipping forward follows the
dense running max when lambda <= 1)."""
import warnings

import numpy as np
import pytest

import synth
from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_flashattention_ssa_b200 as m

    return m


def _skip_ratio(ssa, dq, dk, dv, dcu, w, tsf):
    Q = ssa.num_qblocks(w.cu_seqlens)
    skip = torch.zeros((w.H, Q), dtype=torch.int32, device="cuda")
    ssa.fwd(dq, dk, dv, dcu, w.max_seqlen, tsf, skip_counter=skip)
    ssa.check_device()
    tiles = w.H * sum(((s + 127) // 128) ** 2 for s in w.seqlens)
    return int(skip.sum()) / tiles, skip


# Targets inside each input's observed range: at S = 8192 the largest trial
# (lambda = 0.7) skips about half the tiles, the long varlen batch more.
@pytest.mark.parametrize("wname,targets", [("WAN5B", (0.3, 0.45)), ("VARLEN", (0.5, 0.7))])
def test_calibrate_fit_resolve_forward(ssa, wname, targets):
    from block_sparse_flashattention_ssa_b200 import calibration as cal

    w = getattr(synth, wname)
    q, k, v = synth.generate(w)
    dq, dk, dv, dcu = parity.to_device(q, k, v, w.cu_seqlens)
    c = cal.calibrate(dq, dk, dv, dcu, w.max_seqlen)
    ssa.check_device()
    assert c.b > 0 and c.s_min < min(targets) and max(targets) < c.s_max, (c.s_min, c.s_max)
    for target in targets:
        with warnings.catch_warnings():
            warnings.simplefilter("error")
            tsf = c.threshold_scale_factor(target)
        achieved, _ = _skip_ratio(ssa, dq, dk, dv, dcu, w, tsf)
        assert abs(achieved - target) < 0.12, (wname, target, tsf, achieved)


def test_forward_at_a_trial_threshold_matches_the_calibration_count(ssa):
    from block_sparse_flashattention_ssa_b200 import calibration as cal

    w = synth.WAN5B
    q, k, v = synth.generate(w)
    dq, dk, dv, dcu = parity.to_device(q, k, v, w.cu_seqlens)
    trials = [0.05, 0.2, 0.7]
    _, counts = ssa.calibrate(dq, dk, dv, dcu, w.max_seqlen, trials)
    ssa.check_device()
    S = w.seqlens[0]
    for i, lam in enumerate(trials):
        _, skip = _skip_ratio(ssa, dq, dk, dv, dcu, w, lam * S)
        assert np.array_equal(skip.cpu().numpy(), counts[:, :, i].cpu().numpy()), lam
