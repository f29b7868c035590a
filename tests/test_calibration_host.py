"""Calibration loop host logic (Model-Optimizer PR #1166 page "Usage";
README "Calibrated threshold"; commit page "Calibration"): per-sequence
count sums, fit points (sparsity, lambda * S_kv), the extrapolation warning,
the head partition, and a two-rank gloo run whose all-reduced fit equals the
single-process fit over all heads. No GPU: counts are synthetic."""
import math
import os
import socket
import warnings

import numpy as np
import pytest
import torch.multiprocessing as mp

from block_sparse_flashattention_ssa_b200 import calibration as cal
from tests.golden import first


def test_default_trials_are_the_pages_list():
    (trials,) = first("page_constants.txt", "trials")
    assert list(cal.DEFAULT_TRIALS) == pytest.approx(trials, rel=0, abs=0)


def test_sequence_sums_and_points_by_hand():
    # two sequences: 200 tokens (2 q-blocks) and 128 tokens (1 q-block); 2 heads; 2 trials
    cu = np.array([0, 200, 328], dtype=np.int32)
    counts = np.zeros((2, 3, 2), dtype=np.int32)
    counts[0, 0] = [0, 1]; counts[0, 1] = [1, 1]; counts[1, 0] = [0, 0]; counts[1, 1] = [1, 2]  # sequence 0
    counts[0, 2] = [0, 0]; counts[1, 2] = [0, 0]                                                # sequence 1
    seq = cal.sequence_counts(counts, cu)
    assert seq.tolist() == [[2, 4], [0, 0]]
    pts = cal.fit_points(seq, cu, [1e-3, 1e-2], total_heads=2)
    # sequence 0: 2 heads x 2 x 2 tiles = 8; sequence 1: 2 x 1 x 1 = 2
    assert pts == [(2 / 8, 1e-3 * 200), (4 / 8, 1e-2 * 200), (0.0, 1e-3 * 128), (0.0, 1e-2 * 128)]
    with pytest.raises(ValueError):
        cal.sequence_counts(counts[:, :2], cu)  # q-block count mismatch


def test_fit_recovers_a_log_linear_model():
    a, b = 7.93, 8.61  # TRT-LLM PR page, "Use Cases", case 2
    s = np.linspace(0.1, 0.8, 9)
    pts = [(float(x), a * math.exp(b * x)) for x in s] + [(0.0, 1.0), (1.0, 5.0)]  # s in {0, 1} carry nothing
    c = cal.fit(pts)
    assert c.a == pytest.approx(a, rel=1e-10) and c.b == pytest.approx(b, rel=1e-10)
    assert (c.s_min, c.s_max) == pytest.approx((0.1, 0.8))
    with warnings.catch_warnings():
        warnings.simplefilter("error")
        assert c.threshold_scale_factor(0.5) == pytest.approx(a * math.exp(b * 0.5), rel=1e-12)
    with pytest.warns(RuntimeWarning, match="extrapolating"):
        c.threshold_scale_factor(0.9)


@pytest.mark.parametrize("H,world", [(40, 1), (40, 2), (40, 3), (24, 8), (5, 8)])
def test_head_shards_partition_the_heads(H, world):
    seen = [h for r in range(world) for h in cal.shard_heads(H, world, r)]
    assert seen == list(range(H))
    sizes = [len(cal.shard_heads(H, world, r)) for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _synthetic_counts(H=6, seed=3):
    cu = np.array([0, 700, 1000, 1900], dtype=np.int32)
    nq = [6, 3, 8]
    rng = np.random.default_rng(seed)
    trials = cal.DEFAULT_TRIALS
    # counts grow with the trial threshold, bounded by the tiles of a unit (nkv - 1 skippable)
    per_unit_max = np.concatenate([[n - 1] * n for n in nq])
    frac = np.sort(rng.uniform(0, 1, size=(H, sum(nq), len(trials))), axis=2)
    counts = np.floor(frac * per_unit_max[None, :, None]).astype(np.int32)
    return cu, counts, trials


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cu, counts, trials = _synthetic_counts()
        heads = cal.shard_heads(counts.shape[0], world, rank)
        local = cal.sequence_counts(counts[heads.start:heads.stop], cu)
        total = cal.torch_allreduce()(local)
        c = cal.fit(cal.fit_points(total, cu, trials, total_heads=counts.shape[0]))
        q.put((rank, c.a, c.b, c.s_min, c.s_max, total.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharded_fit_equals_single_process_fit():
    cu, counts, trials = _synthetic_counts()
    ref_seq = cal.sequence_counts(counts, cu)
    ref = cal.fit(cal.fit_points(ref_seq, cu, trials, total_heads=counts.shape[0]))
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, a, b, smin, smax, total in got:
        assert total == ref_seq.tolist()
        assert (a, b, smin, smax) == (ref.a, ref.b, ref.s_min, ref.s_max)  # bit-identical on every rank
