"""Host policy around the forward: threshold resolution, per-timestep
gating and the CUDA-graph phase key (TRT-LLM docs, "VisualGen Sparse
Attention (Beta)": "User Configuration", "Checkpoint Config", "Mapping
disabled_until_timestep to Actual Denoising Steps", "CUDA Graphs").
No GPU needed: graph capture is replaced by a counting fake."""
import math

import numpy as np
import pytest

from block_sparse_flashattention_ssa_b200.policy import DENSE, SKIP, GraphedAttention, SkipSoftmaxPolicy, dense_steps

from tests import golden


def unipc40(norm):
    """The page's 40-step schedule: linear unshifted sigmas, flow shift 3,
    times a runtime normalisation factor `norm` (1.0 = the printed closed form)."""
    (steps, train, shift), = golden.first("unipc40_gating.txt", "schedule")
    i = np.arange(int(steps))
    s = 1.0 - i * (1.0 - 1.0 / train) / steps
    return shift * s / (1.0 + (shift - 1.0) * s) * norm


ROWS = golden.first("unipc40_gating.txt", "row")
QUOTED_T = golden.first("unipc40_gating.txt", "t")


@pytest.mark.parametrize("norm", [0.99939, 0.9995, 0.99955])
def test_dense_steps_reproduce_the_printed_table(norm):
    # The printed closed form puts t[0] at exactly 1.0 and t[10] at 0.90012,
    # which would make the 1.00 and 0.90 rows 1 and 11 dense steps. Any runtime
    # normalisation in [0.99938, 0.99956) reproduces all six rows and both
    # quoted values; the policy itself only ever sees the actual sequence.
    t = unipc40(norm)
    for cutoff, dense, skip in ROWS:
        assert dense_steps(t, cutoff) == int(dense), cutoff
        assert len(t) - dense_steps(t, cutoff) == int(skip)
    for idx, val in QUOTED_T:
        assert round(float(t[int(idx)]), 3) == pytest.approx(val, abs=1e-9)


def test_closed_form_as_printed_differs_only_at_the_two_boundary_rows():
    t = unipc40(1.0)
    got = {cutoff: dense_steps(t, cutoff) for cutoff, _, _ in ROWS}
    assert got == {1.00: 1, 0.97: 4, 0.94: 7, 0.93: 8, 0.90: 11, 0.86: 14}


def test_equality_belongs_to_the_dense_phase():
    p = SkipSoftmaxPolicy(threshold_scale_factor=5000.0, disabled_until_timestep=0.8)
    assert p.phase(0.8) == DENSE and p.threshold_scale_factor_at(0.8) == 0.0
    assert p.phase(math.nextafter(0.8, 0.0)) == SKIP
    assert p.threshold_scale_factor_at(0.5) == 5000.0
    assert p.phase(1.0) == DENSE
    assert SkipSoftmaxPolicy(threshold_scale_factor=5000.0).phase(1.0) == SKIP  # no cutoff: never dense


def test_threshold_resolution_precedence():
    # the concrete scalar wins over a target
    p = SkipSoftmaxPolicy(threshold_scale_factor=5000.0, target_sparsity=0.5, a=1000.0, b=5.0)
    assert p.resolved_threshold_scale_factor() == 5000.0
    # target through the checkpoint formula a * exp(b * s) (docs "Checkpoint Config" example)
    (a, b), = [v for v in golden.first("page_constants.txt", "formula") if v == [1000.0, 5.0]]
    p = SkipSoftmaxPolicy(target_sparsity=0.5, a=a, b=b)
    assert p.resolved_threshold_scale_factor() == pytest.approx(1000.0 * math.exp(2.5), rel=1e-12)
    # log_a spelling gives the same scalar
    q = SkipSoftmaxPolicy(target_sparsity=0.5, log_a=math.log(a), b=b)
    assert q.resolved_threshold_scale_factor() == pytest.approx(p.resolved_threshold_scale_factor(), rel=1e-12)
    # a target without the formula is an error; nothing requested is dense
    with pytest.raises(ValueError):
        SkipSoftmaxPolicy(target_sparsity=0.5).resolved_threshold_scale_factor()
    assert SkipSoftmaxPolicy().resolved_threshold_scale_factor() == 0.0
    with pytest.raises(ValueError):
        SkipSoftmaxPolicy(a=2.0, log_a=0.0)
    with pytest.raises(ValueError):
        SkipSoftmaxPolicy(target_sparsity=1.5)


class _Buf:
    def __init__(self, shape, ptr, dtype="bf16"):
        self.shape, self._ptr, self.dtype = shape, ptr, dtype

    def data_ptr(self):
        return self._ptr


class _FakeGraph:
    def __init__(self, step):
        self.step, self.replays = step, 0

    def replay(self):
        self.replays += 1


def test_graph_key_changes_only_when_the_phase_does():
    p = SkipSoftmaxPolicy(threshold_scale_factor=5000.0, disabled_until_timestep=0.86)
    g = GraphedAttention(p, capture=_FakeGraph)
    q, k, v = _Buf((1024, 2, 64), 1), _Buf((1024, 2, 64), 2), _Buf((1024, 2, 64), 3)
    cu, out = _Buf((2,), 4, "int32"), _Buf((1024, 2, 64), 5)
    t = unipc40(0.9995)
    for ti in t:
        g(q, k, v, cu, 1024, float(ti), out)
    assert g.captures == 2  # one graph per phase
    replays = sorted(gr.replays for gr in g.graphs.values())
    assert replays == sorted([dense_steps(t, 0.86), len(t) - dense_steps(t, 0.86)])
    # new buffers or shapes capture again
    g(q, k, v, cu, 1024, 0.1, _Buf((1024, 2, 64), 6))
    assert g.captures == 3
