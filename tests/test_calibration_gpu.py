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


def test_head_sharded_calibration_equals_the_unsharded_one(ssa):
    """Heads split over two ranks (contiguous head slices, each copied into
    its own [T, H/2, D] tensors as a rank would hold them): each shard counts
    with ssa_calibrate, the per-sequence count sums are added (the all-reduce
    of a head-sharded run, here the other shard's sums added in place of the
    collective) and every shard fits. Counts, sums and (a, b) must equal the
    single-call calibration over all heads bit for bit."""
    from block_sparse_flashattention_ssa_b200 import calibration as cal

    w = synth.VARLEN
    q, k, v = synth.generate(w)
    cu = w.cu_seqlens
    dq, dk, dv, dcu = parity.to_device(q, k, v, cu)
    trials = cal.DEFAULT_TRIALS
    _, counts_all = ssa.calibrate(dq, dk, dv, dcu, w.max_seqlen, list(trials))
    ssa.check_device()
    whole = cal.calibrate(dq, dk, dv, dcu, w.max_seqlen, trials)
    ssa.check_device()
    world = 2
    shards = [cal.shard_heads(w.H, world, r) for r in range(world)]
    per_rank, seq_sums = [], []
    for hr in shards:
        sl = slice(hr.start, hr.stop)
        sq, sk, sv = (t[:, sl].contiguous() for t in (dq, dk, dv))
        _, c = ssa.calibrate(sq, sk, sv, dcu, w.max_seqlen, list(trials))
        ssa.check_device()
        assert torch.equal(c, counts_all[sl]), hr  # a head's counts do not depend on the other heads
        per_rank.append((sq, sk, sv))
        seq_sums.append(cal.sequence_counts(c.cpu().numpy(), cu))
    assert np.array_equal(seq_sums[0] + seq_sums[1], cal.sequence_counts(counts_all.cpu().numpy(), cu))
    for r, (sq, sk, sv) in enumerate(per_rank):
        other = seq_sums[1 - r]
        got = cal.calibrate(sq, sk, sv, dcu, w.max_seqlen, trials, total_heads=w.H, allreduce=lambda s: s + other)
        ssa.check_device()
        assert (got.a, got.b, got.s_min, got.s_max) == (whole.a, whole.b, whole.s_min, whole.s_max), r
        assert got.points == whole.points
