"""Python binding of libbsa: two-stage block-sparse attention on B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of
``libbsa.so`` behind the C ABI of ``include/bsa.h``. PyTorch tensors serve as
device buffers and torch's current stream is passed to each call. There is no
fallback: if the library is missing or cannot load, importing this package
raises.

Functions carry the C names:

* ``bsa_block_pool(x, block_size, flags=0)``       -> pooled [B, H, nb, D] float32
  (block means, or block maxima with BSA_FLAG_MAX_POOL)
* ``bsa_block_scores_topk(q_pooled, k_pooled, topk, scores=False)`` -> idx (, S)
* ``bsa_sparse_attn_fwd(q, k, v, idx, block_size, scale=None, flags=0)`` -> o
* ``bsa_forward(q, k, v, block_size, topk_ratio, workspace=None, flags=0)`` -> o
* ``bsa_forward_host(q, k, v, block_size, topk_ratio)`` -> o, from and to
  CPU tensors (chunked copies overlapped with the compute)
* ``bsa_forward_noalloc(q, k, v, block_size, topk_ratio)`` -> o, with no
  device allocation (a fixed scratch in the library)
* ``bsa_sparse_attn_fwd_train(q, k, v, idx, block_size)`` -> (o, lse) and
  ``bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, block_size)`` -> (dq, dk, dv)
* ``bsa_adaptive_block_size(seq_len)`` -> 64, 128 or 256
* ``bsa_forward_overlap(q, k, v, block_size, topk_ratio, overlap_ratio)`` -> o
  with overlapping key windows (and ``bsa_sparse_attn_fwd_overlap``)
* ``bsa_topk_count``, ``bsa_forward_workspace_bytes``,
  ``bsa_forward_host_workspace_bytes``, ``workspace_views``, ``bsa_device_error``

q, o are [B, N, H, D]; k, v are [B, N, H_kv, D] with H a multiple of H_kv
(grouped queries; H_kv = H otherwise), contiguous, on one CUDA device
(except for bsa_forward_host). Inputs are float32, bfloat16 or
float8_e4m3fn (e4m3 gives a bfloat16 o). ``flags`` takes BSA_FLAG_CAUSAL,
BSA_FLAG_FORCE_DIAG, BSA_FLAG_MAX_POOL and BSA_GLOBAL_HEAD_PERIOD(p).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")

BSA_F32, BSA_BF16, BSA_E4M3 = 0, 1, 2
_STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_MISALIGNED",
           4: "BSA_ERR_WORKSPACE", 5: "BSA_ERR_CUDA", 6: "BSA_ERR_DEVICE"}

#: every function include/bsa.h declares
EXPORTED = ("bsa_topk_count", "bsa_forward_workspace_bytes", "bsa_block_pool",
            "bsa_block_scores_topk", "bsa_sparse_attn_fwd", "bsa_forward", "bsa_status_string",
            "bsa_last_error_detail", "bsa_device_error", "bsa_forward_noalloc",
            "bsa_block_scores_topk_ex", "bsa_sparse_attn_fwd_ex", "bsa_forward_ex",
            "bsa_forward_gqa_workspace_bytes", "bsa_block_scores_topk_gqa", "bsa_sparse_attn_fwd_gqa",
            "bsa_forward_gqa", "bsa_sparse_attn_fwd_train", "bsa_sparse_attn_bwd_workspace_bytes",
            "bsa_sparse_attn_bwd", "bsa_forward_host_workspace_bytes", "bsa_forward_host",
            "bsa_sparse_attn_fwd_train_gqa", "bsa_sparse_attn_bwd_gqa_workspace_bytes", "bsa_sparse_attn_bwd_gqa",
            "bsa_adaptive_block_size", "bsa_block_pool_ex", "bsa_overlap_window_count",
            "bsa_forward_overlap_workspace_bytes", "bsa_sparse_attn_fwd_overlap", "bsa_forward_overlap",
            "bsa_block_pool_qk")

#: variant flags of the *_ex entry points (include/bsa.h)
BSA_FLAG_CAUSAL, BSA_FLAG_FORCE_DIAG, BSA_FLAG_MAX_POOL = 1, 2, 4


def BSA_GLOBAL_HEAD_PERIOD(p: int) -> int:
    """Flag bits for global heads every p query heads (heads h with h % p == 0
    attend to every key block); p in 1..255."""
    if not 1 <= p <= 255:
        raise ValueError("the global-head period must lie in 1..255")
    return (p & 0xFF) << 8


class BsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_STATUS.get(status, status)}: {detail}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so is not built ({LIB_PATH}); run "
                          "`python -m block_sparse_attention_19_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, D, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_size_t
    F, U = ctypes.c_float, ctypes.c_uint
    sig = {
        "bsa_topk_count": ([I, D], I),
        "bsa_forward_workspace_bytes": ([I, I, I, I, I, D], Z),
        "bsa_block_pool": ([P, P, I, I, I, I, I, I, P], I),
        "bsa_block_scores_topk": ([P, P, P, P, I, I, I, I, I, P], I),
        "bsa_sparse_attn_fwd": ([P, P, P, P, P, I, I, I, I, I, I, F, I, P], I),
        "bsa_forward": ([P, P, P, P, I, I, I, I, I, D, I, P, Z, P], I),
        "bsa_status_string": ([I], ctypes.c_char_p),
        "bsa_last_error_detail": ([], ctypes.c_char_p),
        "bsa_device_error": ([ctypes.POINTER(ctypes.c_int), P], I),
        "bsa_forward_noalloc": ([P, P, P, P, I, I, I, I, I, D, I, P], I),
        "bsa_block_scores_topk_ex": ([P, P, P, P, I, I, I, I, I, U, P], I),
        "bsa_sparse_attn_fwd_ex": ([P, P, P, P, P, I, I, I, I, I, I, F, I, U, P], I),
        "bsa_forward_ex": ([P, P, P, P, I, I, I, I, I, D, I, U, P, Z, P], I),
        "bsa_forward_gqa_workspace_bytes": ([I, I, I, I, I, I, D], Z),
        "bsa_block_scores_topk_gqa": ([P, P, P, P, I, I, I, I, I, I, U, P], I),
        "bsa_sparse_attn_fwd_gqa": ([P, P, P, P, P, I, I, I, I, I, I, I, F, I, U, P], I),
        "bsa_forward_gqa": ([P, P, P, P, I, I, I, I, I, I, D, I, U, P, Z, P], I),
        "bsa_sparse_attn_fwd_train": ([P, P, P, P, P, P, I, I, I, I, I, I, F, I, U, P], I),
        "bsa_sparse_attn_bwd_workspace_bytes": ([I, I, I, I, I], Z),
        "bsa_sparse_attn_bwd": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, U, P, Z, P], I),
        "bsa_forward_host_workspace_bytes": ([I, I, I, I, I, I, D, I], Z),
        "bsa_sparse_attn_fwd_train_gqa": ([P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, U, P], I),
        "bsa_sparse_attn_bwd_gqa_workspace_bytes": ([I, I, I, I, I, I], Z),
        "bsa_sparse_attn_bwd_gqa": ([P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, F, I, U, P, Z, P], I),
        "bsa_forward_host": ([P, P, P, P, I, I, I, I, I, I, D, I, U, P, Z, P], I),
        "bsa_adaptive_block_size": ([ctypes.c_longlong], I),
        "bsa_block_pool_ex": ([P, P, I, I, I, I, I, I, U, P], I),
        "bsa_block_pool_qk": ([P, P, P, P, I, I, I, I, I, I, I, U, P], I),
        "bsa_overlap_window_count": ([I, I, D], I),
        "bsa_forward_overlap_workspace_bytes": ([I, I, I, I, I, I, D, D], Z),
        "bsa_sparse_attn_fwd_overlap": ([P, P, P, P, P, I, I, I, I, I, I, I, D, F, I, U, P], I),
        "bsa_forward_overlap": ([P, P, P, P, I, I, I, I, I, I, D, D, I, U, P, Z, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check(status: int):
    if status != 0:
        raise BsaError(status, lib.bsa_last_error_detail().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BSA_F32
    if t.dtype == torch.bfloat16:
        return BSA_BF16
    if t.dtype == torch.float8_e4m3fn:
        return BSA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype} (float32, bfloat16 or float8_e4m3fn)")


def _out_like(q: torch.Tensor) -> torch.Tensor:
    """The output tensor for inputs like q: same dtype, bfloat16 for e4m3 inputs."""
    return torch.empty(q.shape, device=q.device,
                       dtype=torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t: torch.Tensor, want, name: str):
    if tuple(t.shape) != tuple(want):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(want)}")


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """q [B, N, H, D]; k and v [B, N, H_kv, D] with H a multiple of H_kv. The
    library takes plain pointers, so a mismatch would read past a buffer: it
    is refused here, before anything reaches the device."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, N, heads, D]")
    B, N, H, D = q.shape
    Hk = k.shape[2]
    if k.shape[0] != B or k.shape[1] != N or k.shape[3] != D or Hk < 1 or H % Hk:
        raise ValueError(f"k has shape {tuple(k.shape)}; q {tuple(q.shape)} needs [B, N, H_kv, D] with H % H_kv == 0")
    _shape(v, k.shape, "v")


def _check_idx(idx: torch.Tensor, B: int, Hk: int, N: int, block_size: int):
    if idx.dim() != 4 or block_size < 1 or tuple(idx.shape[:3]) != (B, Hk, N // block_size):
        raise ValueError(f"idx has shape {tuple(idx.shape)}, expected [{B}, {Hk}, {N // max(block_size, 1)}, topk]")


def _check_out(out: torch.Tensor, q: torch.Tensor, name: str = "out"):
    _shape(out, q.shape, name)
    want = torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype
    if out.dtype != want:
        raise TypeError(f"{name} must be {want}")


def _p(t: torch.Tensor | None):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def bsa_topk_count(nb: int, topk_ratio: float) -> int:
    return lib.bsa_topk_count(int(nb), float(topk_ratio))


def bsa_forward_workspace_bytes(B: int, N: int, H: int, D: int, block_size: int, topk_ratio: float,
                                H_kv: int | None = None) -> int:
    if H_kv is None or H_kv == H:
        return lib.bsa_forward_workspace_bytes(B, N, H, D, block_size, float(topk_ratio))
    return lib.bsa_forward_gqa_workspace_bytes(B, N, H, H_kv, D, block_size, float(topk_ratio))


def bsa_overlap_window_count(N: int, block_size: int, overlap_ratio: float) -> int:
    return lib.bsa_overlap_window_count(int(N), int(block_size), float(overlap_ratio))


def bsa_forward_overlap_workspace_bytes(B: int, N: int, H: int, D: int, block_size: int, topk_ratio: float,
                                        overlap_ratio: float, H_kv: int | None = None) -> int:
    return lib.bsa_forward_overlap_workspace_bytes(B, N, H, H if H_kv is None else H_kv, D, block_size,
                                                   float(topk_ratio), float(overlap_ratio))


def bsa_forward_overlap(q, k, v, block_size: int, topk_ratio: float, overlap_ratio: float,
                        workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        flags: int = 0) -> torch.Tensor:
    """The whole path with overlapping key windows (see include/bsa.h)."""
    _check_qkv(q, k, v)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    Hk = k.shape[2]
    need = bsa_forward_overlap_workspace_bytes(B, N, H, D, block_size, topk_ratio, overlap_ratio, H_kv=Hk)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    _dev(workspace, "workspace")
    o = out if out is not None else _out_like(q)
    if out is not None:
        _check_out(out, q)
    _check(lib.bsa_forward_overlap(_p(q), _p(k), _p(v), _p(o), B, N, H, Hk, D, block_size, float(topk_ratio),
                                   float(overlap_ratio), _dtype_code(q), flags, _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(q)))
    return o


def bsa_sparse_attn_fwd_overlap(q, k, v, idx, block_size: int, overlap_ratio: float, scale: float | None = None,
                                out: torch.Tensor | None = None, flags: int = 0) -> torch.Tensor:
    """The attention over overlapping key windows: idx [B, H_kv, nb, k] of window ids."""
    _check_qkv(q, k, v)
    _check_idx(idx, q.shape[0], k.shape[2], q.shape[1], block_size)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (idx, "idx")):
        _dev(t, n)
    if idx.dtype != torch.int32:
        raise TypeError("idx must be int32")
    B, N, H, D = q.shape
    o = out if out is not None else _out_like(q)
    if out is not None:
        _check_out(out, q)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    _check(lib.bsa_sparse_attn_fwd_overlap(_p(q), _p(k), _p(v), _p(idx), _p(o), B, N, H, k.shape[2], D, block_size,
                                           idx.shape[-1], float(overlap_ratio), float(scale), _dtype_code(q), flags,
                                           _stream(q)))
    return o


def overlap_workspace_views(ws: torch.Tensor, B: int, N: int, H: int, D: int, block_size: int, topk_ratio: float,
                            overlap_ratio: float, H_kv: int | None = None):
    """The pooled q [B,H,nb,D], window means of k [B,H_kv,nb_k,D], index list
    [B,H_kv,nb,k] and scores [B,H_kv,nb,nb_k] sections of a
    bsa_forward_overlap workspace."""
    Hk = H if H_kv is None else H_kv
    nb = N // block_size
    nbk = bsa_overlap_window_count(N, block_size, overlap_ratio)
    kk = bsa_topk_count(nbk, topk_ratio)
    a256 = lambda x: (x + 255) // 256 * 256
    qpb, kpb, idxb = a256(B * H * nb * D * 4), a256(B * Hk * nbk * D * 4), a256(B * Hk * nb * kk * 4)
    base = ws.view(torch.uint8)
    qp = base[:B * H * nb * D * 4].view(torch.float32).view(B, H, nb, D)
    kp = base[qpb:qpb + B * Hk * nbk * D * 4].view(torch.float32).view(B, Hk, nbk, D)
    idx = base[qpb + kpb:qpb + kpb + B * Hk * nb * kk * 4].view(torch.int32).view(B, Hk, nb, kk)
    off = qpb + kpb + idxb
    S = base[off:off + B * Hk * nb * nbk * 4].view(torch.float32).view(B, Hk, nb, nbk)
    return qp, kp, idx, S


def bsa_adaptive_block_size(seq_len: int) -> int:
    return lib.bsa_adaptive_block_size(int(seq_len))


def bsa_block_pool(x: torch.Tensor, block_size: int, out: torch.Tensor | None = None,
                   flags: int = 0) -> torch.Tensor:
    if x.dim() != 4:
        raise ValueError("x must be [B, N, H, D]")
    B, N, H, D = x.shape
    if out is not None:
        _shape(out, (B, H, N // max(block_size, 1), D), "out")
    _dev(x, "x")
    if out is None:
        out = torch.empty((B, H, N // block_size, D), device=x.device, dtype=torch.float32)
    _check(lib.bsa_block_pool_ex(_p(x), _p(out), B, N, H, D, block_size, _dtype_code(x), flags, _stream(x)))
    return out


def bsa_block_pool_qk(q: torch.Tensor, k: torch.Tensor, block_size: int, q_out: torch.Tensor | None = None,
                      k_out: torch.Tensor | None = None, flags: int = 0):
    """Pooled q [B, H, nb, D] and pooled k [B, H_kv, nb, D] (one launch when H = H_kv)."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, N, heads, D]")
    _check_qkv(q, k, k)
    if q.dtype != k.dtype:
        raise TypeError("q and k must share one dtype")
    B, N, H, D = q.shape
    Hk = k.shape[2]
    nb = N // max(block_size, 1)
    qo = q_out if q_out is not None else torch.empty((B, H, nb, D), device=q.device, dtype=torch.float32)
    ko = k_out if k_out is not None else torch.empty((B, Hk, nb, D), device=q.device, dtype=torch.float32)
    _shape(qo, (B, H, nb, D), "q_out")
    _shape(ko, (B, Hk, nb, D), "k_out")
    for t, n in ((q, "q"), (k, "k"), (qo, "q_out"), (ko, "k_out")):
        _dev(t, n)
    _check(lib.bsa_block_pool_qk(_p(q), _p(k), _p(qo), _p(ko), B, N, H, Hk, D, block_size, _dtype_code(q), flags,
                                 _stream(q)))
    return qo, ko


def bsa_block_scores_topk(q_pooled: torch.Tensor, k_pooled: torch.Tensor, topk: int,
                          scores: bool = False, idx_out: torch.Tensor | None = None,
                          scores_out: torch.Tensor | None = None, flags: int = 0):
    """Block scores S (written to ``scores_out``, allocated if absent) and the
    top-k index list. Returns idx, or (idx, S) when ``scores`` is true.
    ``flags``: BSA_FLAG_CAUSAL / BSA_FLAG_FORCE_DIAG (bsa_block_scores_topk_ex)."""
    if q_pooled.dim() != 4 or k_pooled.dim() != 4:
        raise ValueError("pooled tensors must be [B, heads, nb, D]")
    B, H, nb, D = q_pooled.shape
    Hk = k_pooled.shape[1]  # key/value heads: fewer than H for grouped queries
    if (k_pooled.shape[0], k_pooled.shape[2], k_pooled.shape[3]) != (B, nb, D) or Hk < 1 or H % Hk:
        raise ValueError(f"k_pooled has shape {tuple(k_pooled.shape)}; q_pooled {tuple(q_pooled.shape)}")
    if idx_out is not None:
        _shape(idx_out, (B, Hk, nb, topk), "idx_out")
    if scores_out is not None:
        _shape(scores_out, (B, Hk, nb, nb), "scores_out")
    _dev(q_pooled, "q_pooled")
    _dev(k_pooled, "k_pooled")
    if q_pooled.dtype != torch.float32 or k_pooled.dtype != torch.float32:
        raise TypeError("pooled tensors must be float32")
    idx = idx_out if idx_out is not None else torch.empty((B, Hk, nb, topk), device=q_pooled.device, dtype=torch.int32)
    S = scores_out if scores_out is not None else torch.empty((B, Hk, nb, nb), device=q_pooled.device,
                                                              dtype=torch.float32)
    if Hk != H:
        _check(lib.bsa_block_scores_topk_gqa(_p(q_pooled), _p(k_pooled), _p(S), _p(idx), B, H, Hk, nb, D,
                                             topk, flags, _stream(q_pooled)))
    elif flags:
        _check(lib.bsa_block_scores_topk_ex(_p(q_pooled), _p(k_pooled), _p(S), _p(idx), B, H, nb, D, topk,
                                            flags, _stream(q_pooled)))
    else:
        _check(lib.bsa_block_scores_topk(_p(q_pooled), _p(k_pooled), _p(S), _p(idx), B, H, nb, D, topk,
                                         _stream(q_pooled)))
    return (idx, S) if scores else idx


def bsa_sparse_attn_fwd(q, k, v, idx, block_size: int, scale: float | None = None,
                        out: torch.Tensor | None = None, flags: int = 0) -> torch.Tensor:
    _check_qkv(q, k, v)
    _check_idx(idx, q.shape[0], k.shape[2], q.shape[1], block_size)
    if out is not None:
        _check_out(out, q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (idx, "idx")):
        _dev(t, n)
    if idx.dtype != torch.int32:
        raise TypeError("idx must be int32")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    Hk = k.shape[2]  # key/value heads: fewer than H for grouped queries
    topk = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = out if out is not None else _out_like(q)
    if Hk != H:
        _check(lib.bsa_sparse_attn_fwd_gqa(_p(q), _p(k), _p(v), _p(idx), _p(o), B, N, H, Hk, D, block_size,
                                           topk, float(scale), _dtype_code(q), flags, _stream(q)))
    elif flags:
        _check(lib.bsa_sparse_attn_fwd_ex(_p(q), _p(k), _p(v), _p(idx), _p(o), B, N, H, D, block_size, topk,
                                          float(scale), _dtype_code(q), flags, _stream(q)))
    else:
        _check(lib.bsa_sparse_attn_fwd(_p(q), _p(k), _p(v), _p(idx), _p(o), B, N, H, D, block_size, topk,
                                       float(scale), _dtype_code(q), _stream(q)))
    return o


def bsa_forward(q, k, v, block_size: int, topk_ratio: float, workspace: torch.Tensor | None = None,
                out: torch.Tensor | None = None, flags: int = 0) -> torch.Tensor:
    _check_qkv(q, k, v)
    if out is not None:
        _check_out(out, q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    Hk = k.shape[2]  # key/value heads: fewer than H for grouped queries
    need = bsa_forward_workspace_bytes(B, N, H, D, block_size, topk_ratio, H_kv=Hk)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    o = out if out is not None else _out_like(q)
    nbytes = workspace.numel() * workspace.element_size()
    if Hk != H:
        _check(lib.bsa_forward_gqa(_p(q), _p(k), _p(v), _p(o), B, N, H, Hk, D, block_size, float(topk_ratio),
                                   _dtype_code(q), flags, _p(workspace), nbytes, _stream(q)))
    elif flags:
        _check(lib.bsa_forward_ex(_p(q), _p(k), _p(v), _p(o), B, N, H, D, block_size, float(topk_ratio),
                                  _dtype_code(q), flags, _p(workspace), nbytes, _stream(q)))
    else:
        _check(lib.bsa_forward(_p(q), _p(k), _p(v), _p(o), B, N, H, D, block_size, float(topk_ratio),
                               _dtype_code(q), _p(workspace), nbytes, _stream(q)))
    return o


def bsa_forward_host_workspace_bytes(B: int, N: int, H: int, D: int, block_size: int, topk_ratio: float,
                                     dtype: torch.dtype, H_kv: int | None = None) -> int:
    """Device workspace bytes of bsa_forward_host (its two chunk slots)."""
    code = _dtype_code(torch.empty(0, dtype=dtype))
    return int(lib.bsa_forward_host_workspace_bytes(B, N, H, H if H_kv is None else H_kv, D, block_size,
                                                    float(topk_ratio), code))


def bsa_forward_host(q, k, v, block_size: int, topk_ratio: float, out: torch.Tensor | None = None,
                     flags: int = 0, workspace: torch.Tensor | None = None, device=None,
                     synchronize: bool = True) -> torch.Tensor:
    """The whole forward from host tensors: q [B, N, H, D], k and v [B, N, H_kv, D]
    on the CPU (pinned memory lets the copies overlap the compute), o returned
    (or written to `out`) on the CPU. The library copies head-group chunks to
    `device` (default: the current CUDA device) on its own streams, computes
    them on the current stream there and copies the results back. With
    synchronize=False the call returns once the work is enqueued; the output
    is complete when the current stream of `device` is."""
    _check_qkv(q, k, v)
    if out is not None:
        _check_out(out, q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CPU tensor")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    B, N, H, D = q.shape
    Hk = k.shape[2]
    need = bsa_forward_host_workspace_bytes(B, N, H, D, block_size, topk_ratio, q.dtype, H_kv=Hk)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=dev, dtype=torch.uint8)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype,
                          pin_memory=True)
    elif out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous CPU tensor")
    with torch.cuda.device(dev):
        st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        _check(lib.bsa_forward_host(_p(q), _p(k), _p(v), _p(out), B, N, H, Hk, D, block_size, float(topk_ratio),
                                    _dtype_code(q), flags, _p(workspace), workspace.numel(), st))
        if synchronize:
            torch.cuda.current_stream(dev).synchronize()
    return out


def bsa_sparse_attn_fwd_train(q, k, v, idx, block_size: int, scale: float | None = None, flags: int = 0,
                              out: torch.Tensor | None = None, lse: torch.Tensor | None = None):
    """The attention forward that also returns lse [B,H,N] (ln of each row's
    softmax denominator), for bsa_sparse_attn_bwd. Returns (o, lse). k and v
    may have fewer heads than q (grouped queries; idx per key/value head)."""
    _check_qkv(q, k, v)
    _check_idx(idx, q.shape[0], k.shape[2], q.shape[1], block_size)
    if out is not None:
        _check_out(out, q)
    if lse is not None:
        _shape(lse, (q.shape[0], q.shape[2], q.shape[1]), "lse")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (idx, "idx")):
        _dev(t, n)
    B, N, H, D = q.shape
    Hk = k.shape[2]
    topk = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = out if out is not None else _out_like(q)
    lse = lse if lse is not None else torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    _check(lib.bsa_sparse_attn_fwd_train_gqa(_p(q), _p(k), _p(v), _p(idx), _p(o), _p(lse), B, N, H, Hk, D,
                                             block_size, topk, float(scale), _dtype_code(q), flags, _stream(q)))
    return o, lse


def bsa_sparse_attn_bwd(q, k, v, o, do, idx, lse, block_size: int, scale: float | None = None, flags: int = 0,
                        workspace: torch.Tensor | None = None):
    """Gradients (dq, dk, dv) of the attention over the kept blocks with the
    index lists held fixed; o and lse from bsa_sparse_attn_fwd_train. With
    grouped queries (k, v with fewer heads than q) dk and dv are per
    key/value head, summed over the group's query heads."""
    _check_qkv(q, k, v)
    _check_idx(idx, q.shape[0], k.shape[2], q.shape[1], block_size)
    _check_out(o, q, "o")
    _shape(do, q.shape, "do")
    _shape(lse, (q.shape[0], q.shape[2], q.shape[1]), "lse")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do"), (idx, "idx"), (lse, "lse")):
        _dev(t, n)
    B, N, H, D = q.shape
    Hk = k.shape[2]
    topk = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    need = lib.bsa_sparse_attn_bwd_gqa_workspace_bytes(B, N, H, Hk, D, block_size)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=q.device, dtype=torch.uint8)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    _check(lib.bsa_sparse_attn_bwd_gqa(_p(q), _p(k), _p(v), _p(o), _p(do), _p(idx), _p(lse), _p(dq), _p(dk),
                                       _p(dv), B, N, H, Hk, D, block_size, topk, float(scale), _dtype_code(q),
                                       flags, _p(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(q)))
    return dq, dk, dv


def bsa_forward_noalloc(q, k, v, block_size: int, topk_ratio: float, out: torch.Tensor | None = None) -> torch.Tensor:
    """bsa_forward with its intermediates in the library's fixed device scratch
    (for callers that cannot allocate device memory; see include/bsa.h for the
    size limit and the sharing rules)."""
    _check_qkv(q, k, v)
    _shape(k, q.shape, "k")  # one key/value head per query head
    if out is not None:
        _check_out(out, q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n)
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    o = out if out is not None else _out_like(q)
    _check(lib.bsa_forward_noalloc(_p(q), _p(k), _p(v), _p(o), B, N, H, D, block_size, float(topk_ratio),
                                   _dtype_code(q), _stream(q)))
    return o


def bsa_device_error(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device error word."""
    code = ctypes.c_int(0)
    stream = torch.cuda.current_stream(device).cuda_stream
    _check(lib.bsa_device_error(ctypes.byref(code), ctypes.c_void_p(stream)))
    return code.value


def workspace_views(ws: torch.Tensor, B: int, N: int, H: int, D: int, block_size: int, topk_ratio: float,
                    with_scores: bool = False, H_kv: int | None = None):
    """The pooled q [B,H,nb,D], pooled k [B,H_kv,nb,D], index-list [B,H_kv,nb,k]
    (and block-score [B,H_kv,nb,nb]) sections of a bsa_forward(_gqa)
    workspace (the layout of include/bsa.h: 256-byte aligned sections in that
    order)."""
    Hk = H if H_kv is None else H_kv
    nb = N // block_size
    kk = bsa_topk_count(nb, topk_ratio)
    a256 = lambda x: (x + 255) // 256 * 256
    qpb, kpb, idxb = a256(B * H * nb * D * 4), a256(B * Hk * nb * D * 4), a256(B * Hk * nb * kk * 4)
    base = ws.view(torch.uint8)
    qp = base[:B * H * nb * D * 4].view(torch.float32).view(B, H, nb, D)
    kp = base[qpb:qpb + B * Hk * nb * D * 4].view(torch.float32).view(B, Hk, nb, D)
    idx = base[qpb + kpb:qpb + kpb + B * Hk * nb * kk * 4].view(torch.int32).view(B, Hk, nb, kk)
    if not with_scores:
        return qp, kp, idx
    off = qpb + kpb + idxb
    S = base[off:off + B * Hk * nb * nb * 4].view(torch.float32).view(B, Hk, nb, nb)
    return qp, kp, idx, S
