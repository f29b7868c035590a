"""Per-timestep gating with CUDA-graph capture on the GPU (TRT-LLM docs,
"VisualGen Sparse Attention (Beta)", "Mapping disabled_until_timestep to
Actual Denoising Steps" and "CUDA Graphs"): a denoising loop whose buffers
are rewritten in place captures one graph per phase; every replayed step
equals an eager forward at that step's threshold bit for bit, and matches the
oracle walked at the threshold the policy gives for that timestep."""
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

    return m


def test_graphed_denoising_loop_matches_eager_steps(ssa):
    from block_sparse_flashattention_ssa_b200.policy import DENSE, GraphedAttention, SkipSoftmaxPolicy

    w = synth.TINY
    q0, k0, v0 = synth.generate(w)
    dq, dk, dv, dcu = parity.to_device(q0, k0, v0, w.cu_seqlens)
    q_base = dq.clone()
    Q = ssa.num_qblocks(w.cu_seqlens)
    out = torch.empty_like(dq)
    skip = torch.zeros((w.H, Q), dtype=torch.int32, device="cuda")
    policy = SkipSoftmaxPolicy(threshold_scale_factor=1000.0, disabled_until_timestep=0.5)
    graphed = GraphedAttention(policy)
    ts = [1.0, 0.8, 0.6, 0.5, 0.4, 0.3, 0.2, 0.1]
    for step, t in enumerate(ts):
        dq.copy_(q_base * (1.0 + 0.25 * step))  # the denoising state changes in place
        graphed(dq, dk, dv, dcu, w.max_seqlen, t, out, skip_counter=skip)
        torch.cuda.synchronize()
        ref_out = torch.empty_like(dq)
        ref_skip = torch.zeros_like(skip)
        ssa.fwd(dq, dk, dv, dcu, w.max_seqlen, policy.threshold_scale_factor_at(t), out=ref_out, skip_counter=ref_skip)
        ssa.check_device()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), (step, t)
        assert torch.equal(skip, ref_skip), (step, t)
        # the step against the oracle on this step's input, at the policy's threshold
        tsf = policy.threshold_scale_factor_at(t)
        q_step = dq.view(torch.int16).cpu().numpy().view(np.uint16)
        res = oracle.walk(q_step, k0, v0, w.cu_seqlens, w.H, w.D, tsf=tsf)
        got = parity.bf16_host(out)
        st = parity.Stats()
        for i, u in enumerate(res["units"]):
            s0, n = parity.unit_rows(w.cu_seqlens, u)
            st.add(got[s0:s0 + n, u[1]], res["out"][i, :n])
            margin = np.abs(res["dstat"][i] - oracle.threshold_log2(tsf, w.seqlens[0])) <= parity.MARGIN
            if not margin.any():  # lambda <= 1 here: no margin tile, no legitimate difference
                assert int(skip[u[1], u[2]]) == int(res["skips"][i]), (step, t, tuple(u))
        st.check(f"policy step {step} t={t} tsf={tsf}")
        if policy.phase(t) == DENSE:
            assert int(skip.sum()) == 0
    assert graphed.captures == 2
    assert int(skip.sum()) > 0  # the enabled phase skips tiles on this input
