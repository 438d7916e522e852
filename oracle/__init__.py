"""Float64 CPU oracle for two-stage block-sparse attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package; the product path (``block_sparse_attention_19_b200``) never does, and
this package imports nothing from it.

The arithmetic lives in ``bsa_oracle.c`` (plain C, float64, OpenMP over
independent rows only); this module builds it with gcc and marshals numpy
arrays through ctypes.  Each function follows the definition on the pages:

* "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
  "SparseFormer 注意力实现": mean-pool q/k over blocks, score blocks,
  keep int(topk_ratio * nb) blocks with top-k, attend over the kept blocks
  with scale 1/sqrt(D).
* "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析", §2.1 and §2.2:
  Softmax(Mask(QK^T/sqrt(d_k)))V with a block mask from a coarse block score.

Every function here is pinned by ``tests/test_oracle.py`` against closed forms,
library routines (numpy matmul / lexsort, torch SDPA in float64), brute force
and invariants; nothing in this package is "parity unpinned".

Inputs may be float32, float64, bfloat16 or FP8 E4M3; bfloat16 is passed as
its raw 16-bit patterns in a ``numpy.uint16`` array and E4M3 as raw bytes in a
``numpy.uint8`` array.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64, E4M3 = 0, 1, 2, 3
_lib = None


def build(force: bool = False) -> str:
    """Compile ``bsa_oracle.c`` into ``liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i, d = ctypes.c_int, ctypes.c_double
        lib.oracle_topk_count.argtypes = [i, d]
        lib.oracle_topk_count.restype = i
        lib.oracle_block_pool.argtypes = [P, i, i, i, i, i, i, P]
        lib.oracle_block_pool_max.argtypes = [P, i, i, i, i, i, i, P]
        lib.oracle_adaptive_block_size.argtypes = [ctypes.c_longlong]
        lib.oracle_adaptive_block_size.restype = i
        lib.oracle_block_scores.argtypes = [P, P, i, i, i, i, P, i, P]
        lib.oracle_topk_row.argtypes = [P, i, i, P]
        lib.oracle_topk.argtypes = [P, ctypes.c_long, i, i, P]
        lib.oracle_sparse_attn.argtypes = [P, P, P, i, i, i, i, i, i, P, i, P, i, d, P]
        lib.oracle_topk_ex.argtypes = [P, ctypes.c_long, i, i, P, i, P]
        lib.oracle_sparse_attn_ex.argtypes = [P, P, P, i, i, i, i, i, i, P, i, P, i, d, i, P]
        lib.oracle_sparse_attn_gqa.argtypes = [P, P, P, i, i, i, i, i, i, i, P, i, P, i, d, i, P]
        lib.oracle_sparse_attn_bwd.argtypes = [P, P, P, P, i, i, i, i, i, i, P, i, P, i, d, i, P, P, P]
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = d
        lib.oracle_num_threads.restype = i
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _as_input(x: np.ndarray):
    """Return (contiguous array, dtype code) for a q/k/v tensor."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.uint8:
        return x, E4M3
    raise TypeError("oracle inputs must be float32, float64, bf16 bits (uint16) or e4m3 bytes (uint8), "
                    f"got {x.dtype}")


def e4m3_to_double(code: int) -> float:
    """Value of an FP8 E4M3 byte (sign, 4-bit exponent with bias 7, 3-bit
    mantissa, subnormals at exponent 0, NaN at S.1111.111; no infinities)."""
    return _load().oracle_e4m3_to_double(int(code))


def num_threads() -> int:
    return _load().oracle_num_threads()


def topk_count(nb: int, topk_ratio: float) -> int:
    """k = int(topk_ratio * nb) exactly as Python evaluates it ([SF] step 2)."""
    return _load().oracle_topk_count(int(nb), float(topk_ratio))


def block_pool(x: np.ndarray, block_size: int, pool: str = "mean") -> np.ndarray:
    """[B,N,H,D] -> block means [B,H,nb,D] in float64 ([SF] step 1), or with
    ``pool="max"`` the element-wise block maxima ([MSA] §2.2, "block-internal
    extreme value")."""
    x, code = _as_input(x)
    B, N, H, D = x.shape
    if N % block_size:
        raise ValueError("N must be a multiple of block_size")
    if pool not in ("mean", "max"):
        raise ValueError("pool must be 'mean' or 'max'")
    nb = N // block_size
    out = np.empty((B, H, nb, D), np.float64)
    fn = _load().oracle_block_pool if pool == "mean" else _load().oracle_block_pool_max
    fn(_ptr(x), code, B, N, H, D, block_size, _ptr(out))
    return out


def adaptive_block_size(seq_len: int) -> int:
    """Block size for an input length ([MSA] §4.2): 64 below 500,000 tokens,
    128 below 1,000,000, else 256; -1 for a length below 1."""
    return _load().oracle_adaptive_block_size(int(seq_len))


def _rows(rows, B: int, H: int, nb: int):
    """(nrows, pointer, array) for a query-block list: ``rows`` broadcast to
    [B, H, nrows] (so [1, 1, nrows] picks the same blocks in every batch
    entry and head), or (nb, None, None) for all blocks. The C routines read
    B * H * nrows entries, so anything else is refused here."""
    if rows is None:
        return nb, None, None
    r = np.asarray(rows)
    if r.ndim != 3:
        raise ValueError(f"rows must be [B, H, nrows], got shape {r.shape}")
    r = np.ascontiguousarray(np.broadcast_to(r, (B, H, r.shape[-1])), np.int32)
    if r.size and (r.min() < 0 or r.max() >= nb):
        raise ValueError(f"rows must lie in [0, {nb})")
    return r.shape[-1], _ptr(r), r


def block_scores(qp: np.ndarray, kp: np.ndarray, rows: np.ndarray | None = None) -> np.ndarray:
    """Block scores S[b,h,r,j] = qp[b,h,rows[b,h,r]] . kp[b,h,j] ([SF] step 1).

    ``rows`` is an int array [B,H,nrows] of query-block ids (None = all)."""
    qp = np.ascontiguousarray(qp, np.float64)
    kp = np.ascontiguousarray(kp, np.float64)
    B, H, nb, D = qp.shape
    nrows, rp, rows = _rows(rows, B, H, nb)
    out = np.empty((B, H, nrows, nb), np.float64)
    _load().oracle_block_scores(_ptr(qp), _ptr(kp), B, H, nb, D, rp, nrows, _ptr(out))
    return out


CAUSAL, FORCE_DIAG = 1, 2


def topk(scores: np.ndarray, k: int, causal: bool = False, force_diag: bool = False,
         qblocks: np.ndarray | None = None) -> np.ndarray:
    """Top-k block ids of every score row, ties to the lower id, ascending ([SF] step 2).

    With ``causal`` the row of query block i ranks only blocks j <= i and keeps
    min(k, i+1) of them (with ``force_diag`` block i always, plus the best
    j < i), padding the row with -1.  ``qblocks`` gives the query block of each
    row (shape of ``scores`` without its last axis); None means the rows are all
    nb query blocks in order."""
    s = np.ascontiguousarray(scores, np.float64)
    nb = s.shape[-1]
    if not (1 <= k <= nb):
        raise ValueError("need 1 <= k <= nb")
    rows = int(np.prod(s.shape[:-1]))
    out = np.empty(s.shape[:-1] + (k,), np.int32)
    if not causal:
        _load().oracle_topk(_ptr(s), rows, nb, k, _ptr(out))
        return out
    flags = CAUSAL | (FORCE_DIAG if force_diag else 0)
    qb = None if qblocks is None else np.ascontiguousarray(np.broadcast_to(qblocks, s.shape[:-1]), np.int32)
    _load().oracle_topk_ex(_ptr(s), rows, nb, k, None if qb is None else _ptr(qb), flags, _ptr(out))
    return out


def sparse_attn(q, k, v, idx, block_size: int, scale: float | None = None, rows=None,
                causal: bool = False) -> np.ndarray:
    """Exact softmax attention over the selected key blocks ([SF] step 3, [MSA] §2.1).

    ``idx`` is int [B,H,nrows,k] (the selected key blocks of each listed query
    block; entries below 0 select nothing); ``rows`` is int [B,H,nrows] (None =
    all nb query blocks in order).  With ``causal`` query token n ignores key
    tokens t > n.  Returns float64 [B,H,nrows,block_size,D]."""
    q, code = _as_input(q)
    k_, code_k = _as_input(k)
    v, code_v = _as_input(v)
    if not (code == code_k == code_v):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    nb = N // block_size
    idx = np.ascontiguousarray(idx, np.int32)
    kk = idx.shape[-1]
    nrows, rp, rows = _rows(rows, B, H, nb)
    if idx.shape != (B, H, nrows, kk):
        raise ValueError(f"idx shape {idx.shape} != {(B, H, nrows, kk)}")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, H, nrows, block_size, D), np.float64)
    if causal or (idx < 0).any():
        _load().oracle_sparse_attn_ex(_ptr(q), _ptr(k_), _ptr(v), code, B, N, H, D, block_size,
                                      _ptr(idx), kk, rp, nrows, float(scale), CAUSAL if causal else 0,
                                      _ptr(out))
    else:
        _load().oracle_sparse_attn(_ptr(q), _ptr(k_), _ptr(v), code, B, N, H, D, block_size,
                                   _ptr(idx), kk, rp, nrows, float(scale), _ptr(out))
    return out


def forward(q, k, v, block_size: int, topk_ratio: float, rows=None, scale=None,
            causal: bool = False, force_diag: bool = False, pool: str = "mean") -> dict:
    """The whole path of the [SF] listing on the oracle: pool, score, select, attend.

    ``rows`` (int [B,H,nrows]) restricts the scored / attended query blocks to
    a sample; pooling of k always covers every block since selection needs all
    of them. ``pool`` is "mean" (the listing) or "max" (block maxima).  Returns a dict with qp, kp, scores, idx, o, k and timings."""
    t0 = time.perf_counter()
    qn, _ = _as_input(q)
    B, N, H, D = qn.shape
    nb = N // block_size
    kk = topk_count(nb, topk_ratio)
    qp = block_pool(q, block_size, pool)
    kp = block_pool(k, block_size, pool)
    S = block_scores(qp, kp, rows)
    idx = topk(S, kk, causal=causal, force_diag=force_diag, qblocks=rows)
    o = sparse_attn(q, k, v, idx, block_size, scale=scale, rows=rows, causal=causal)
    return {"qp": qp, "kp": kp, "scores": S, "idx": idx, "o": o, "k": kk,
            "seconds": time.perf_counter() - t0}


def sparse_attn_bwd(q, k, v, do, idx, block_size: int, scale: float | None = None,
                    causal: bool = False, rows=None):
    """Gradients (dq, dk, dv) of the attention over the kept blocks with the
    index lists held fixed (the top-k indices carry no gradient): for each query
    token, dS_t = p_t (dO . v_t - dO . o), dq = scale sum_t dS_t k_t,
    dk_t += scale dS_t q, dv_t += p_t dO. ``idx`` [B,H,nb,k] for all query blocks
    (entries below 0 select nothing); ``do`` has q's dtype. ``rows`` (int
    [B,H,nrows]) sums only those query blocks' contributions (a timing
    sample). Returns float64 [B,N,H,D] arrays."""
    q, code = _as_input(q)
    k_, code_k = _as_input(k)
    v, code_v = _as_input(v)
    do, code_o = _as_input(do)
    if not (code == code_k == code_v == code_o):
        raise TypeError("q, k, v, do must share one dtype")
    B, N, H, D = q.shape
    nb = N // block_size
    idx = np.ascontiguousarray(idx, np.int32)
    kk = idx.shape[-1]
    if idx.shape != (B, H, nb, kk):
        raise ValueError(f"idx shape {idx.shape} != {(B, H, nb, kk)}")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    dq, dk, dv = (np.empty((B, N, H, D), np.float64) for _ in range(3))
    nrows, rp, rows = _rows(rows, B, H, nb)
    _load().oracle_sparse_attn_bwd(_ptr(q), _ptr(k_), _ptr(v), _ptr(do), code, B, N, H, D, block_size,
                                   _ptr(idx), kk, rp, nrows, float(scale), CAUSAL if causal else 0,
                                   _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


# ---------------------------------------------------------------- grouped-query variant
# Readings ("从M2.7到M3" §3.1: the attention block is GQA-based): q has H heads,
# k and v have Hkv = H / G; query head h reads key/value head h // G; each
# key/value head has one selection, scored with the group's pooled query (the
# mean over its G heads of their block means).

def group_pool(qp: np.ndarray, Hkv: int) -> np.ndarray:
    """Pooled queries [B,H,nb,D] -> the group means [B,Hkv,nb,D] (heads h with h // G == g)."""
    B, H, nb, D = qp.shape
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    return np.asarray(qp, np.float64).reshape(B, Hkv, H // Hkv, nb, D).mean(axis=2)


def sparse_attn_gqa(q, k, v, idx, block_size: int, scale: float | None = None, rows=None,
                    causal: bool = False) -> np.ndarray:
    """sparse_attn with Hkv key/value heads: q [B,N,H,D], k and v [B,N,Hkv,D];
    ``idx`` [B,H,nrows,k] and ``rows`` [B,H,nrows] are per query head.
    Returns float64 [B,H,nrows,block_size,D]."""
    q, code = _as_input(q)
    k_, code_k = _as_input(k)
    v, code_v = _as_input(v)
    if not (code == code_k == code_v):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, D = q.shape
    Hkv = k_.shape[2]
    if H % Hkv or k_.shape != (B, N, Hkv, D) or v.shape != k_.shape:
        raise ValueError("need k, v of shape [B,N,Hkv,D] with H a multiple of Hkv")
    nb = N // block_size
    idx = np.ascontiguousarray(idx, np.int32)
    kk = idx.shape[-1]
    nrows, rp, rows = _rows(rows, B, H, nb)
    if idx.shape != (B, H, nrows, kk):
        raise ValueError(f"idx shape {idx.shape} != {(B, H, nrows, kk)}")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, H, nrows, block_size, D), np.float64)
    _load().oracle_sparse_attn_gqa(_ptr(q), _ptr(k_), _ptr(v), code, B, N, H, Hkv, D, block_size,
                                   _ptr(idx), kk, rp, nrows, float(scale), CAUSAL if causal else 0,
                                   _ptr(out))
    return out


def forward_gqa(q, k, v, block_size: int, topk_ratio: float, rows=None, scale=None,
                causal: bool = False, force_diag: bool = False, pool: str = "mean") -> dict:
    """The whole path with grouped queries. ``rows`` (int [B,Hkv,nrows]) picks
    query blocks per key/value head; every query head of the group is attended
    for those blocks. Returns qp (per head), qg (group means), kp, scores and
    idx (per key/value head), idx_q / rows_q (expanded to query heads) and o
    [B,H,nrows,bs,D]."""
    qn, _ = _as_input(q)
    kn, _ = _as_input(k)
    B, N, H, D = qn.shape
    Hkv = kn.shape[2]
    G = H // Hkv
    nb = N // block_size
    kk = topk_count(nb, topk_ratio)
    if rows is not None:
        _, _, rows = _rows(rows, B, Hkv, nb)
    qp = block_pool(q, block_size, pool)
    qg = group_pool(qp, Hkv)
    kp = block_pool(k, block_size, pool)
    S = block_scores(qg, kp, rows)
    idx = topk(S, kk, causal=causal, force_diag=force_diag, qblocks=rows)
    idx_q = np.repeat(idx, G, axis=1)
    rows_q = None if rows is None else np.repeat(np.asarray(rows, np.int32), G, axis=1)
    o = sparse_attn_gqa(q, k, v, idx_q, block_size, scale=scale, rows=rows_q, causal=causal)
    return {"qp": qp, "qg": qg, "kp": kp, "scores": S, "idx": idx, "idx_q": idx_q, "rows_q": rows_q,
            "o": o, "k": kk}


# ---------------------------------------------------------------- global heads
# Reading ("从M2.7到M3" §5.3: add global attention heads, e.g. one global head in
# every four): query head h is global when h % period == 0 (the first head of
# every run of `period` heads); a global head attends to every key block (with
# the causal flag: every block j <= i, token-masked as usual), the other heads
# to their selected blocks.

def global_head_rows(idx_q: np.ndarray, nb: int, period: int, causal: bool = False, rows=None) -> np.ndarray:
    """Per-query-head index rows with global heads: ``idx_q`` [B,H,nrows,k]
    (the selection of each query head's rows) widened to nb entries; rows of
    global heads list every key block (causal: blocks 0..i, then -1), the
    others their k blocks followed by -1. ``rows`` [B,H,nrows] gives the query
    block of each row (None: all nb blocks in order)."""
    B, H, nrows, k = idx_q.shape
    out = np.full((B, H, nrows, nb), -1, np.int32)
    out[..., :k] = idx_q
    qb = np.broadcast_to(np.arange(nrows), (B, H, nrows)) if rows is None else np.broadcast_to(rows, (B, H, nrows))
    for h in range(0, H, period):
        for b in range(B):
            for r in range(nrows):
                n = qb[b, h, r] + 1 if causal else nb
                out[b, h, r, :] = -1
                out[b, h, r, :n] = np.arange(n)
    return out


def forward_global(q, k, v, block_size: int, topk_ratio: float, period: int, causal: bool = False,
                   force_diag: bool = False, pool: str = "mean", rows=None) -> dict:
    """forward_gqa with global heads every ``period`` query heads. Returns the
    forward_gqa dict with idx_q replaced by the widened per-query-head rows
    and o recomputed over them."""
    r = forward_gqa(q, k, v, block_size, topk_ratio, rows=rows, causal=causal, force_diag=force_diag, pool=pool)
    qn, _ = _as_input(q)
    nb = qn.shape[1] // block_size
    idx_w = global_head_rows(r["idx_q"], nb, period, causal, r["rows_q"])
    r["idx_q"] = idx_w
    r["o"] = sparse_attn_gqa(q, k, v, idx_w, block_size, rows=r["rows_q"], causal=causal)
    return r


# ---------------------------------------------------------------- overlapping key blocks
# Reading ("从M2.7到M3" §5.3: against losses at block boundaries, overlapping
# blocks with overlap_ratio = 0.25): key blocks become windows of block_size
# tokens that overlap their neighbours by ov = int(overlap_ratio * block_size)
# tokens, i.e. start every s = block_size - ov tokens; the last window is
# moved back to end at token N, so nb_k = ceil((N - block_size) / s) + 1
# windows cover the sequence. Query blocks stay disjoint. Each window is
# scored by its mean key, k = int(topk_ratio * nb_k) windows are kept per
# query block, and each query row attends to the union of the kept windows'
# tokens (a token two kept windows share counts once).

def window_starts(N: int, block_size: int, ov: int) -> np.ndarray:
    """First token of every key window."""
    if not 0 <= ov < block_size or N < block_size:
        raise ValueError("need 0 <= ov < block_size <= N")
    s = block_size - ov
    nbk = -(-(N - block_size) // s) + 1
    return np.minimum(np.arange(nbk) * s, N - block_size)


def window_pool(x, block_size: int, ov: int) -> np.ndarray:
    """Mean of every key window: [B,N,H,D] -> [B,H,nb_k,D] float64."""
    xn, code = _as_input(x)
    xd = _to_f64(xn, code)
    B, N, H, D = xd.shape
    w = window_starts(N, block_size, ov)
    out = np.empty((B, H, len(w), D))
    for j, t0 in enumerate(w):
        out[:, :, j] = xd[:, t0:t0 + block_size].sum(axis=1) / block_size
    return out


def _to_f64(x: np.ndarray, code: int) -> np.ndarray:
    """Exact float64 values of an oracle input array."""
    if code == BF16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if code == E4M3:
        lut = np.array([e4m3_to_double(c) for c in range(256)])
        return lut[x]
    return x.astype(np.float64)


def attend_token_sets(q, k, v, tokens, block_size: int, scale: float | None = None) -> np.ndarray:
    """Softmax attention of every query row of block i over an explicit token
    set: tokens[b][g][i] is the sorted array of key tokens of (b, key/value
    head g, query block i). q [B,N,H,D], k and v [B,N,Hkv,D]; query head h
    reads key/value head h // (H / Hkv). Returns float64 [B,H,nb,bs,D]."""
    qn, cq = _as_input(q)
    kn, ck = _as_input(k)
    vn, cv = _as_input(v)
    qd, kd, vd = _to_f64(qn, cq), _to_f64(kn, ck), _to_f64(vn, cv)
    B, N, H, D = qd.shape
    Hkv = kd.shape[2]
    G = H // Hkv
    nb = N // block_size
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, H, nb, block_size, D))
    for b in range(B):
        for h in range(H):
            g = h // G
            for i in range(nb):
                t = np.asarray(tokens[b][g][i])
                logits = qd[b, i * block_size:(i + 1) * block_size, h] @ kd[b, t, g].T * scale
                w = np.exp(logits - logits.max(axis=1, keepdims=True))
                out[b, h, i] = (w @ vd[b, t, g]) / w.sum(axis=1, keepdims=True)
    return out


def window_token_sets(idx: np.ndarray, N: int, block_size: int, ov: int):
    """The union of the tokens of each row's kept windows: idx [B,Hkv,nb,k]
    (window ids, entries below 0 select nothing) -> nested lists of sorted
    token arrays [b][g][i]."""
    w = window_starts(N, block_size, ov)
    B, Hkv, nb, _ = idx.shape
    return [[[np.unique(np.concatenate([np.arange(w[j], w[j] + block_size) for j in idx[b, g, i] if j >= 0]))
              for i in range(nb)] for g in range(Hkv)] for b in range(B)]


def forward_overlap(q, k, v, block_size: int, topk_ratio: float, overlap_ratio: float, pool: str = "mean") -> dict:
    """The whole path with overlapping key windows (see above); grouped
    queries as in forward_gqa. Returns qp, qg, kp (window means), scores
    [B,Hkv,nb,nb_k], idx [B,Hkv,nb,k], o [B,H,nb,bs,D], ov and nb_k."""
    if pool != "mean":
        raise ValueError("overlapping windows are mean-pooled")
    qn, _ = _as_input(q)
    kn, _ = _as_input(k)
    B, N, H, D = qn.shape
    Hkv = kn.shape[2]
    ov = int(overlap_ratio * block_size)
    qp = block_pool(q, block_size)
    qg = group_pool(qp, Hkv)
    kp = window_pool(k, block_size, ov)
    nbk = kp.shape[2]
    kk = topk_count(nbk, topk_ratio)
    S = np.matmul(qg, kp.transpose(0, 1, 3, 2))  # [B, Hkv, nb, nb_k]
    idx = topk(S, kk)
    o = attend_token_sets(q, k, v, window_token_sets(idx, N, block_size, ov), block_size)
    return {"qp": qp, "qg": qg, "kp": kp, "scores": S, "idx": idx, "o": o, "ov": ov, "nbk": nbk, "k": kk}


def o_to_bnhd(o: np.ndarray) -> np.ndarray:
    """Reorder an all-rows oracle output [B,H,nb,bs,D] to [B,N,H,D]."""
    B, H, nb, bs, D = o.shape
    return o.reshape(B, H, nb * bs, D).transpose(0, 2, 1, 3).copy()
