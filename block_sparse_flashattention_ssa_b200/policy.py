"""Host-side policy around the skip-softmax forward.

Which threshold a call uses, when a denoising loop is still in its dense
phase, and one captured CUDA graph per (shapes, buffers, phase). Nothing here
computes attention: every call lands in ``ssa_fwd`` through the binding.

Sources (TensorRT-LLM docs, "VisualGen Sparse Attention (Beta)"):
  * "User Configuration": ``threshold_scale_factor`` and ``target_sparsity``
    are alternatives and the concrete ``threshold_scale_factor`` wins; a
    ``target_sparsity`` without the checkpoint's calibration formula is an
    error; the kernel consumes the scale factor and forms the threshold with
    the sequence length itself.
  * "Checkpoint Config": the formula ``a * exp(b * target_sparsity)`` and
    ``disabled_until_timestep``, a normalized [0, 1] cutoff.
  * "Mapping disabled_until_timestep to Actual Denoising Steps": denoising
    runs from t near 1 towards 0; skipping is off while
    t >= disabled_until_timestep (equality is dense) and the number of dense
    steps is the count of schedule entries at or above the cutoff.
  * "CUDA Graphs": the phase is part of the graph key, graphs are captured
    lazily on the first step of a (shape, phase) and replayed afterwards, so a
    graph captured in the dense phase is never replayed after the cutoff.
The TensorRT-LLM pull request page ("Accept both ... log_a ... and ... a
coefficients") gives the two spellings of the formula's scale coefficient.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Dict, Optional, Sequence, Tuple

from . import resolve as _resolve
from . import fwd as _fwd

DENSE = "dense"
SKIP = "skip"


@dataclass(frozen=True)
class SkipSoftmaxPolicy:
    """User/checkpoint settings of one attention layer.

    threshold_scale_factor  concrete kernel scalar (lambda * S_kv); wins when set
    target_sparsity         [0, 1], resolved through a * exp(b * s)
    a, log_a, b             calibration formula coefficients (give a or log_a)
    disabled_until_timestep optional cutoff: dense while t >= cutoff
    """

    threshold_scale_factor: Optional[float] = None
    target_sparsity: Optional[float] = None
    a: Optional[float] = None
    log_a: Optional[float] = None
    b: Optional[float] = None
    disabled_until_timestep: Optional[float] = None

    def __post_init__(self):
        if self.a is not None and self.log_a is not None:
            if not math.isclose(math.log(self.a), self.log_a, rel_tol=1e-12, abs_tol=1e-12):
                raise ValueError("a and log_a disagree")
        if self.target_sparsity is not None and not (0.0 <= self.target_sparsity <= 1.0):
            raise ValueError("target_sparsity must lie in [0, 1]")
        if self.disabled_until_timestep is not None and not (0.0 <= self.disabled_until_timestep <= 1.0):
            raise ValueError("disabled_until_timestep must lie in [0, 1]")

    def scale_coefficient(self) -> Optional[float]:
        if self.a is not None:
            return float(self.a)
        if self.log_a is not None:
            return math.exp(self.log_a)
        return None

    def resolved_threshold_scale_factor(self) -> float:
        """The scalar the kernel consumes once skipping is enabled."""
        if self.threshold_scale_factor is not None:
            return float(self.threshold_scale_factor)
        if self.target_sparsity is None:
            return 0.0  # nothing requested: dense
        a = self.scale_coefficient()
        if a is None or self.b is None:
            raise ValueError("target_sparsity needs the calibration formula's coefficients (a or log_a, and b)")
        tsf = _resolve(a, float(self.b), float(self.target_sparsity))
        if not math.isfinite(tsf):
            raise ValueError("calibration formula gave a non-finite threshold_scale_factor")
        return tsf

    def phase(self, t: Optional[float]) -> str:
        """DENSE while t >= disabled_until_timestep (equality included), else SKIP."""
        if self.disabled_until_timestep is not None and t is not None and t >= self.disabled_until_timestep:
            return DENSE
        return SKIP

    def threshold_scale_factor_at(self, t: Optional[float]) -> float:
        return 0.0 if self.phase(t) == DENSE else self.resolved_threshold_scale_factor()


def dense_steps(timesteps: Sequence[float], disabled_until_timestep: float) -> int:
    """Initial dense-attention steps of a schedule: entries with t >= cutoff."""
    return sum(1 for t in timesteps if t >= disabled_until_timestep)


GraphKey = Tuple


class GraphedAttention:
    """Replays one captured CUDA graph of ``fwd`` per (shapes, buffers, phase).

    The caller keeps its q/k/v/cu_seqlens/out (and optional skip_counter)
    buffers at fixed addresses across denoising steps and rewrites them in
    place, as a captured step requires. The first step seen for a key
    captures; later steps with the same key replay; crossing the cutoff
    changes the phase and so the key.
    """

    def __init__(self, policy: SkipSoftmaxPolicy, capture: Optional[Callable] = None):
        self.policy = policy
        self.graphs: Dict[GraphKey, object] = {}
        self.captures = 0
        self._capture = capture or _capture_cuda_graph

    def key(self, q, k, v, cu_seqlens, out, skip_counter, max_seqlen: int, t: Optional[float]) -> GraphKey:
        def sig(x):
            return None if x is None else (tuple(x.shape), str(x.dtype), int(x.data_ptr()))

        return (sig(q), sig(k), sig(v), sig(cu_seqlens), sig(out), sig(skip_counter), int(max_seqlen),
                self.policy.phase(t))

    def __call__(self, q, k, v, cu_seqlens, max_seqlen: int, t: Optional[float], out, skip_counter=None):
        key = self.key(q, k, v, cu_seqlens, out, skip_counter, max_seqlen, t)
        graph = self.graphs.get(key)
        if graph is None:
            tsf = self.policy.threshold_scale_factor_at(t)

            def step():
                _fwd(q, k, v, cu_seqlens, max_seqlen, tsf, out=out, skip_counter=skip_counter)

            graph = self._capture(step)
            self.graphs[key] = graph
            self.captures += 1
        graph.replay()
        return out


def _capture_cuda_graph(step: Callable):
    import torch

    step()  # eager run first: sets the kernel attributes outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    return graph
