"""BLASST skip-softmax attention for B200 (sm_100a): Python binding.

Argument marshalling over the C ABI declared in ``include/ssa.h`` and
implemented in ``libssa.so`` (built in-tree by ``build.py``). Every step of
the computation runs in the library's CUDA kernels; torch only provides
device memory and streams. There is no CPU fallback: importing this package
fails loudly when the library is missing.

Entry points (same names as the C ABI, without the ``ssa_`` prefix):
  fwd          skip-softmax attention forward (optionally with per-tile
               diagnostics, the ``ssa_fwd_ex`` call)
  fwd_fp8      the forward with E4M3 Q and K, or Q, K and V (per-tensor
               descales; ssa_fwd_fp8 / ssa_fwd_fp8_qkv)
  quantize_fp8 bf16 -> E4M3 per-tensor quantisation for fwd_fp8
  calibrate    dense attention + skip counts at N thresholds at once
               (optionally with the per-tile statistic, ``ssa_calibrate_ex``)
  calibrate_fp8  the same with E4M3 Q and K
  resolve      threshold_scale_factor = a * exp(b * target_sparsity)
  fit_logspace log-space least-squares fit of (a, b)
  num_qblocks  number of 128-row query blocks of a batch
  get_error    synchronise and read/clear the device status word
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_PKG, "libssa.so")
TILE = 128
MAX_THRESHOLDS = 32

SSA_OK = 0
SSA_ERR_INVALID_ARG = -1
SSA_ERR_UNSUPPORTED = -2
SSA_ERR_CUDA = -3
SSA_ERR_TIMEOUT = -4
SSA_ERR_DEVICE_ARG = -5


class SSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = ""
        if status == SSA_ERR_CUDA:
            detail = f": {_lib.ssa_last_cuda_error().decode()}"
        super().__init__(f"{what}: {status} ({_lib.ssa_status_string(status).decode()}{detail})")


def _load():
    if not os.path.exists(_SO):
        raise ImportError(f"libssa.so is not built ({_SO}); run block_sparse_flashattention_ssa_b200/build.py")
    L = ctypes.CDLL(_SO)
    vp, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double
    L.ssa_fwd.restype = i32
    L.ssa_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp, i32, vp]
    L.ssa_fwd_ex.restype = i32
    L.ssa_fwd_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp, i32, vp, vp, vp]
    L.ssa_fwd_fp8.restype = i32
    L.ssa_fwd_fp8.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32, f32, vp, vp, i32, vp, vp, vp]
    L.ssa_calibrate_fp8.restype = i32
    L.ssa_calibrate_fp8.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32, vp, i32, vp, vp, i32,
                                    vp]
    L.ssa_fwd_fp8_qkv.restype = i32
    L.ssa_fwd_fp8_qkv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32, f32, f32, vp, vp, i32,
                                  vp, vp, vp]
    L.ssa_calibrate_fp8_qkv.restype = i32
    L.ssa_calibrate_fp8_qkv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32, f32, vp, i32, vp,
                                        vp, i32, vp]
    L.ssa_quantize_fp8.restype = i32
    L.ssa_quantize_fp8.argtypes = [vp, vp, ctypes.c_int64, f32, vp]
    L.ssa_calibrate.restype = i32
    L.ssa_calibrate.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32, vp, vp, i32, vp]
    L.ssa_calibrate_ex.restype = i32
    L.ssa_calibrate_ex.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32, vp, vp, i32, vp, vp]
    L.ssa_resolve.restype = f64
    L.ssa_resolve.argtypes = [f64, f64, f64]
    L.ssa_fit_logspace.restype = i32
    L.ssa_fit_logspace.argtypes = [vp, vp, i32, vp, vp, vp, vp]
    L.ssa_num_qblocks.restype = i32
    L.ssa_num_qblocks.argtypes = [vp, i32]
    L.ssa_get_error.restype = i32
    L.ssa_get_error.argtypes = [vp]
    L.ssa_status_string.restype = ctypes.c_char_p
    L.ssa_status_string.argtypes = [i32]
    L.ssa_last_cuda_error.restype = ctypes.c_char_p
    L.ssa_last_cuda_error.argtypes = []
    L.ssa_wait_timeout_check.restype = i32
    L.ssa_wait_timeout_check.argtypes = [vp, ctypes.c_int64, vp]
    return L


_lib = _load()


def lib():
    """The loaded ctypes library (for callers that marshal raw pointers)."""
    return _lib


def library_path() -> str:
    return _SO


def _check(rc: int, what: str):
    if rc != SSA_OK:
        raise SSAError(rc, what)


def _stream_handle(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape(q):
    if q.dim() != 3:
        raise ValueError("q, k, v must be [total_tokens, H, D]")
    return q.shape[0], q.shape[1], q.shape[2]


def _require(t, name, dtype, device, shape=None, allow_none=False):
    """Host-side check of a tensor argument: on the device of q, contiguous,
    of the expected dtype (and shape). A host tensor handed to the kernels
    would fault the GPU, so this is checked before the library is called."""
    import torch

    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _check_attention_args(q, k, v, cu_seqlens, out, qk_dtype, v_dtype=None):
    import torch

    if not (isinstance(q, torch.Tensor) and q.is_cuda):
        raise ValueError("q must be a CUDA tensor")
    dev = q.device
    shape = tuple(q.shape)
    _require(q, "q", qk_dtype, dev)
    _require(k, "k", qk_dtype, dev, shape)
    _require(v, "v", v_dtype or torch.bfloat16, dev, shape)
    _require(cu_seqlens, "cu_seqlens", torch.int32, dev)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D tensor of batch + 1 offsets")
    _require(out, "out", torch.bfloat16, dev, shape, allow_none=True)
    return dev


def _per_unit_qblocks(dev, H, total, batch, outputs) -> int:
    """Check the per-unit outputs ``(tensor, name, dtypes, inner_shape)``:
    each must be [H, Q, *inner_shape] on ``dev``, all with the same Q, and Q
    no larger than any batch of ``total`` tokens can have. Returns that Q
    (-1 when every output is None). The library counts the q-blocks again
    from the device copy of cu_seqlens and writes nothing when they differ,
    so a wrong Q cannot overrun a buffer either way."""
    q_dim = None
    for t, name, dtype, inner in outputs:
        _require(t, name, dtype, dev, allow_none=True)
        if t is None:
            continue
        if t.dim() != 2 + len(inner) or t.shape[0] != H or tuple(t.shape[2:]) != tuple(inner):
            want = ", ".join([str(H), "num_qblocks"] + [str(i) for i in inner])
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected [{want}]")
        if q_dim is None:
            q_dim = int(t.shape[1])
        elif int(t.shape[1]) != q_dim:
            raise ValueError(f"{name} has {t.shape[1]} q-blocks, another per-unit output {q_dim}")
    if q_dim is None:
        return -1
    if q_dim > (total + TILE - 1) // TILE + batch:
        raise ValueError(f"{q_dim} q-blocks is more than {total} tokens in {batch} sequences can have")
    return q_dim


def num_qblocks(cu_seqlens) -> int:
    """Total 128-row query blocks over the batch (from a host copy of cu_seqlens)."""
    cu = np.ascontiguousarray(np.asarray(cu_seqlens if not hasattr(cu_seqlens, "cpu") else cu_seqlens.cpu()),
                              dtype=np.int32)
    n = _lib.ssa_num_qblocks(cu.ctypes.data, len(cu) - 1)
    if n < 0:
        raise SSAError(n, "ssa_num_qblocks")
    return n


def fwd(q, k, v, cu_seqlens, max_seqlen: int, threshold_scale_factor: float = 0.0, softmax_scale: float = 0.0,
        out=None, skip_counter=None, decision_bitmap=None, tile_stat=None, stream=None):
    """Skip-softmax attention forward. q, k, v: CUDA bf16 [total_tokens, H, D];
    cu_seqlens: CUDA int32 [B+1]. Returns ``out`` (allocated when None).
    ``skip_counter`` (int32 [H, Q]), ``decision_bitmap`` (int32/uint32
    [H, Q, ceil(T/32)]) and ``tile_stat`` (float32 [H, Q, T]) are optional
    caller-allocated outputs; passing either of the last two selects the
    diagnostic call ``ssa_fwd_ex``."""
    import torch

    total, H, D = _shape(q)
    dev = _check_attention_args(q, k, v, cu_seqlens, out, torch.bfloat16)
    batch = cu_seqlens.numel() - 1
    nq = _per_unit_qblocks(dev, H, total, batch, _forward_outputs(skip_counter, decision_bitmap, tile_stat,
                                                                  max_seqlen))
    if out is None:
        out = torch.empty_like(q)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, total, int(max_seqlen), H, D,
            float(softmax_scale), float(threshold_scale_factor), _ptr(out), _ptr(skip_counter), nq]
    if decision_bitmap is not None or tile_stat is not None:
        rc = _lib.ssa_fwd_ex(*args, _ptr(decision_bitmap), _ptr(tile_stat), _stream_handle(stream))
        _check(rc, "ssa_fwd_ex")
    else:
        _check(_lib.ssa_fwd(*args, _stream_handle(stream)), "ssa_fwd")
    return out


def fwd_fp8(q8, k8, v, cu_seqlens, max_seqlen: int, q_descale: float, k_descale: float,
            threshold_scale_factor: float = 0.0, softmax_scale: float = 0.0, out=None, skip_counter=None,
            decision_bitmap=None, tile_stat=None, v_descale=None, stream=None):
    """Forward with E4M3 Q and K (CUDA uint8 [total_tokens, H, 128], values
    q_descale * decode(q8)); returns bf16 ``out``. V is bf16 (ssa_fwd_fp8) or,
    with ``v_descale``, E4M3 codes as well, P then rounded to E4M3 for the
    P.V product (ssa_fwd_fp8_qkv)."""
    import torch

    total, H, D = _shape(q8)
    qkv = v_descale is not None
    dev = _check_attention_args(q8, k8, v, cu_seqlens, out, torch.uint8, torch.uint8 if qkv else None)
    batch = cu_seqlens.numel() - 1
    nq = _per_unit_qblocks(dev, H, total, batch, _forward_outputs(skip_counter, decision_bitmap, tile_stat,
                                                                  max_seqlen))
    if out is None:
        out = torch.empty(v.shape, dtype=torch.bfloat16, device=v.device)
    head = [_ptr(q8), _ptr(k8), _ptr(v), _ptr(cu_seqlens), batch, total, int(max_seqlen), H, D,
            float(softmax_scale), float(q_descale), float(k_descale)]
    tail = [float(threshold_scale_factor), _ptr(out), _ptr(skip_counter), nq, _ptr(decision_bitmap),
            _ptr(tile_stat), _stream_handle(stream)]
    if qkv:
        _check(_lib.ssa_fwd_fp8_qkv(*head, float(v_descale), *tail), "ssa_fwd_fp8_qkv")
    else:
        _check(_lib.ssa_fwd_fp8(*head, *tail), "ssa_fwd_fp8")
    return out


def quantize_fp8(x, inv_scale: float, out=None, stream=None):
    """E4M3 codes (uint8, same shape) of fp32(x * inv_scale), nearest even, saturating."""
    import torch

    if not (isinstance(x, torch.Tensor) and x.is_cuda):
        raise ValueError("x must be a CUDA tensor")
    _require(x, "x", torch.bfloat16, x.device)
    _require(out, "out", torch.uint8, x.device, tuple(x.shape), allow_none=True)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(_lib.ssa_quantize_fp8(_ptr(x), _ptr(out), x.numel(), float(inv_scale), _stream_handle(stream)),
           "ssa_quantize_fp8")
    return out


def calibrate(q, k, v, cu_seqlens, max_seqlen: int, thresholds, softmax_scale: float = 0.0, out=None, counts=None,
              tile_stat=None, stream=None):
    """Dense attention plus, per (head, q-block) unit, the number of KV tiles
    that would be skipped at each raw lambda in ``thresholds``. Returns
    (out, counts[H, Q, N]). Passing ``tile_stat`` (float32 [H, Q, T],
    caller-allocated) selects ``ssa_calibrate_ex``, which also writes every
    tile's statistic d_j. Without ``counts`` the q-block count is read from a
    host copy of cu_seqlens (a synchronisation)."""
    import torch

    total, H, D = _shape(q)
    dev = _check_attention_args(q, k, v, cu_seqlens, out, torch.bfloat16)
    th = np.ascontiguousarray(thresholds, dtype=np.float32)
    batch = cu_seqlens.numel() - 1
    if counts is None:
        counts = torch.empty((H, num_qblocks(cu_seqlens), len(th)), dtype=torch.int32, device=dev)
    nq = _per_unit_qblocks(dev, H, total, batch, [(counts, "counts", torch.int32, (len(th),)),
                                                   (tile_stat, "tile_stat", torch.float32, (max_tiles(max_seqlen),))])
    if out is None:
        out = torch.empty_like(q)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), batch, total, int(max_seqlen), H, D, float(softmax_scale),
            th.ctypes.data, len(th), _ptr(out), _ptr(counts), nq]
    if tile_stat is not None:
        _check(_lib.ssa_calibrate_ex(*args, _ptr(tile_stat), _stream_handle(stream)), "ssa_calibrate_ex")
    else:
        _check(_lib.ssa_calibrate(*args, _stream_handle(stream)), "ssa_calibrate")
    return out, counts


def calibrate_fp8(q8, k8, v, cu_seqlens, max_seqlen: int, q_descale: float, k_descale: float, thresholds,
                  softmax_scale: float = 0.0, out=None, counts=None, v_descale=None, stream=None):
    """calibrate() on the E4M3 scores of fwd_fp8 (V bf16, or E4M3 codes with
    ``v_descale``: ssa_calibrate_fp8_qkv). Returns (out, counts[H, Q, N])."""
    import torch

    total, H, D = _shape(q8)
    qkv = v_descale is not None
    dev = _check_attention_args(q8, k8, v, cu_seqlens, out, torch.uint8, torch.uint8 if qkv else None)
    th = np.ascontiguousarray(thresholds, dtype=np.float32)
    batch = cu_seqlens.numel() - 1
    if counts is None:
        counts = torch.empty((H, num_qblocks(cu_seqlens), len(th)), dtype=torch.int32, device=dev)
    nq = _per_unit_qblocks(dev, H, total, batch, [(counts, "counts", torch.int32, (len(th),))])
    if out is None:
        out = torch.empty(v.shape, dtype=torch.bfloat16, device=v.device)
    head = [_ptr(q8), _ptr(k8), _ptr(v), _ptr(cu_seqlens), batch, total, int(max_seqlen), H, D,
            float(softmax_scale), float(q_descale), float(k_descale)]
    tail = [th.ctypes.data, len(th), _ptr(out), _ptr(counts), nq, _stream_handle(stream)]
    if qkv:
        _check(_lib.ssa_calibrate_fp8_qkv(*head, float(v_descale), *tail), "ssa_calibrate_fp8_qkv")
    else:
        _check(_lib.ssa_calibrate_fp8(*head, *tail), "ssa_calibrate_fp8")
    return out, counts


def resolve(a: float, b: float, target_sparsity: float) -> float:
    return float(_lib.ssa_resolve(a, b, target_sparsity))


def fit_logspace(sparsity, scale_factor):
    """Returns (a, b, s_min, s_max)."""
    s = np.ascontiguousarray(sparsity, dtype=np.float64)
    sf = np.ascontiguousarray(scale_factor, dtype=np.float64)
    if s.shape != sf.shape:
        raise ValueError("sparsity and scale_factor differ in length")
    out = [ctypes.c_double() for _ in range(4)]
    _check(_lib.ssa_fit_logspace(s.ctypes.data, sf.ctypes.data, len(s), *[ctypes.byref(o) for o in out]),
           "ssa_fit_logspace")
    return tuple(o.value for o in out)


def wait_timeout_check(limit_ns: int = 20_000_000, stream=None):
    """Diagnostic: run the kernels' bounded wait on a barrier nothing arrives
    on. Returns (completed, abort_flag, microseconds_waited) from the device;
    the device status then holds SSA_ERR_TIMEOUT (read it with get_error)."""
    import torch

    res = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    _check(_lib.ssa_wait_timeout_check(_ptr(res), int(limit_ns), _stream_handle(stream)), "ssa_wait_timeout_check")
    torch.cuda.synchronize()
    return tuple(int(x) for x in res.cpu().tolist())


def get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status."""
    return int(_lib.ssa_get_error(_stream_handle(stream)))


def check_device(stream=None):
    """Raise SSAError when a kernel recorded an error on this device."""
    _check(get_error(stream), "device status")


def max_tiles(max_seqlen: int) -> int:
    return (int(max_seqlen) + TILE - 1) // TILE


def bitmap_words(max_seqlen: int) -> int:
    return (max_tiles(max_seqlen) + 31) // 32


def _forward_outputs(skip_counter, decision_bitmap, tile_stat, max_seqlen):
    import torch

    return [(skip_counter, "skip_counter", torch.int32, ()),
            (decision_bitmap, "decision_bitmap", (torch.int32, torch.uint32), (bitmap_words(max_seqlen),)),
            (tile_stat, "tile_stat", torch.float32, (max_tiles(max_seqlen),))]
