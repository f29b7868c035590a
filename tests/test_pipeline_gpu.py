"""The overlapped host -> device -> host forward (pipeline.PipelinedForward):
every problem of a series, uploaded from pinned host memory while its
neighbours compute and download, gives exactly the output and skip counts
of a plain ssa_fwd on the same inputs."""
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


def test_pipelined_series_equals_plain_calls(ssa):
    from block_sparse_flashattention_ssa_b200.pipeline import PipelinedForward

    w = synth.Workload("pipeline", [(2, 16, 32), (1, 9, 15)], H=3, D=128, seed=21, amp=3.0)
    q, k, v = synth.generate(w)
    Q = ssa.num_qblocks(w.cu_seqlens)
    dq, dk, dv, dcu = parity.to_device(q, k, v, w.cu_seqlens)
    tsf = 800.0
    problems, refs = [], []
    for n in range(5):
        s = 1.0 + 0.3 * n
        hq = (torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).float() * s).to(torch.bfloat16)
        hk = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16)
        hv = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
        problems.append(tuple(t.contiguous().pin_memory() for t in (hq, hk, hv)))
        skip = torch.zeros((w.H, Q), dtype=torch.int32, device="cuda")
        o = ssa.fwd(problems[-1][0].cuda(), dk, dv, dcu, w.max_seqlen, tsf, skip_counter=skip)
        refs.append((o.cpu(), skip.cpu()))
    ssa.check_device()
    outs = [(torch.empty(dq.shape, dtype=torch.bfloat16).pin_memory(),
             torch.full((w.H, Q), -1, dtype=torch.int32).pin_memory()) for _ in problems]
    pf = PipelinedForward(tuple(dq.shape), dcu, w.max_seqlen, Q, tsf)
    pf.run(problems, outs)
    torch.cuda.synchronize()
    ssa.check_device()
    for (o, sk), (ro, rsk) in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), ro.view(torch.int16))
        assert torch.equal(sk, rsk)
    assert sum(int(r[1].sum()) for r in refs) > 0  # the threshold skips tiles on these inputs
