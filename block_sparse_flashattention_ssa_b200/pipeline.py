"""Forward over a series of host-resident problems with the copies overlapped.

Each problem's Q, K, V go host -> device, ``ssa_fwd`` runs, and its output
and skip counters come back device -> host. Three CUDA streams and two
device buffer sets let problem i+1 upload while problem i computes and
problem i-1 downloads; every problem still moves all of its own bytes. The
host buffers should be pinned for the copies to be asynchronous. Plumbing
only: the attention itself is the library's kernel.
"""
from __future__ import annotations

from typing import Sequence, Tuple

from . import fwd as _fwd


class PipelinedForward:
    def __init__(self, shape: Tuple[int, int, int], cu_seqlens, max_seqlen: int, num_qblocks: int,
                 threshold_scale_factor: float, softmax_scale: float = 0.0, device=None):
        import torch

        self.device = device or torch.device("cuda", torch.cuda.current_device())
        total, H, D = shape
        mk = lambda: torch.empty((total, H, D), dtype=torch.bfloat16, device=self.device)
        self.bufs = [dict(q=mk(), k=mk(), v=mk(), out=mk(),
                          skip=torch.empty((H, num_qblocks), dtype=torch.int32, device=self.device))
                     for _ in range(2)]
        self.cu = cu_seqlens
        self.max_seqlen = int(max_seqlen)
        self.tsf = float(threshold_scale_factor)
        self.scale = float(softmax_scale)
        self.s_up = torch.cuda.Stream(self.device)
        self.s_comp = torch.cuda.Stream(self.device)
        self.s_down = torch.cuda.Stream(self.device)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        self.ev_up, self.ev_comp, self.ev_down = ev(), ev(), ev()

    def run(self, inputs: Sequence[tuple], outputs: Sequence[tuple]):
        """inputs[i] = (q, k, v) host bf16 tensors; outputs[i] = (out, skip)
        host tensors that receive problem i's output and per-unit skip counts.
        Enqueues everything and returns; synchronise before reading outputs."""
        import torch

        if len(inputs) != len(outputs):
            raise ValueError("one output slot per input problem")
        for i, ((hq, hk, hv), (hout, hskip)) in enumerate(zip(inputs, outputs)):
            b = i % 2
            d = self.bufs[b]
            if i >= 2:
                self.s_up.wait_event(self.ev_comp[b])  # problem i-2 has finished reading these inputs
            with torch.cuda.stream(self.s_up):
                d["q"].copy_(hq, non_blocking=True)
                d["k"].copy_(hk, non_blocking=True)
                d["v"].copy_(hv, non_blocking=True)
                self.ev_up[b].record(self.s_up)
            self.s_comp.wait_event(self.ev_up[b])
            if i >= 2:
                self.s_comp.wait_event(self.ev_down[b])  # problem i-2's output has left these buffers
            _fwd(d["q"], d["k"], d["v"], self.cu, self.max_seqlen, self.tsf, softmax_scale=self.scale,
                 out=d["out"], skip_counter=d["skip"], stream=self.s_comp)
            self.ev_comp[b].record(self.s_comp)
            self.s_down.wait_event(self.ev_comp[b])
            with torch.cuda.stream(self.s_down):
                hout.copy_(d["out"], non_blocking=True)
                hskip.copy_(d["skip"], non_blocking=True)
                self.ev_down[b].record(self.s_down)
