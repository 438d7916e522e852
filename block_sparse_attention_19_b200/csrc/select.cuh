// select.cuh -- step 2: top-k block selection from the block scores.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 2: torch.topk(block_scores, k) over the key
// blocks. Readings fixed here: ties go to the lower key-block index; each
// output row lists its k blocks in ascending order (a canonical order, so
// results compare exactly).
//
// One warp per score row, scores as order-preserving 32-bit keys. The k-th
// largest key is bracketed by bisection (on the score value, then on the
// key) until at most 64 keys remain in the bracket, which are sorted exactly
// (about 8 counting passes on typical rows instead of 32). For nb <= 1024
// the keys sit in registers (block_topk_kernel); longer rows are converted
// once into shared memory and counted from there (block_topk_wide_kernel;
// rows too long to stage fall back to a bitwise search read from L2). One
// ordered ballot pass then emits every key above the k-th largest plus the
// lowest-index keys equal to it.
#pragma once

#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Order-preserving map float -> uint32 (larger float <=> larger key). -0 is
// mapped as +0: the two compare equal, so they must tie (and go to the lower
// index) like any other equal scores.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  u = u == 0x80000000u ? 0u : u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// Number of the warp's keys >= t (one redux.sync instead of a shuffle tree).
template <int KPL>
__device__ __forceinline__ int warp_count_ge(const uint32_t (&key)[KPL], uint32_t t) {
  unsigned c = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) c += key[i] >= t;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, c));
}

// Bitonic sort of 64 keys held two per lane (element i = lane in a, lane + 32
// in b) into descending order across the warp.
__device__ __forceinline__ void warp_sort64_desc(uint32_t& a, uint32_t& b, int lane) {
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {
        // partners i and i + 32 sit in the same lane; size is 64: one descending block
        const uint32_t hi = max(a, b), lo = min(a, b);
        a = hi;
        b = lo;
      } else {
#pragma unroll
        for (int slot = 0; slot < 2; ++slot) {
          uint32_t& x = slot == 0 ? a : b;
          const int i = lane + 32 * slot;
          const uint32_t y = __shfl_xor_sync(0xffffffffu, x, stride);
          const bool lower = (i & stride) == 0;
          const bool desc = (i & size) == 0;
          x = (lower == desc) ? max(x, y) : min(x, y);
        }
      }
    }
  }
}

// Key of a score for the register path: float_key with the -0 fix done by
// an add, and clamped to >= 1 (this merges the two lowest NaN patterns only)
// so that the padding key 0 never enters a bracket, a count or the output.
__device__ __forceinline__ uint32_t score_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 + 0 = +0
  const uint32_t flip = static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u;
  return max(u ^ flip, 1u);
}

// One warp selects the k largest of a row of nb <= 32 * KPL scores held as
// keys in registers, lane-major: lane l holds keys j = l * KPL + t, so
// ascending j is lane order and each lane loads a contiguous run (float4
// loads when `vec`: the row starts 16-byte aligned and nb % 4 == 0). The
// k-th largest key is bracketed by bisection (up to 12 steps on the score
// value, then on the key, which needs at most 32 steps) until the bracket
// [lo, hi) holds at most 64 keys, which are then sorted exactly; a bracket
// that cannot be split holds equal keys only. `cand` is 64 words of shared
// memory private to the warp.
template <int KPL>
__device__ __forceinline__ void select_row_bracket(const float* srow, int nb, int nvalid, int k,
                                                   int32_t* out, int lane, uint32_t* cand, bool vec) {
  uint32_t key[KPL];
  const int j0 = lane * KPL;
  if (KPL % 4 == 0 && vec) {
#pragma unroll
    for (int v = 0; v < KPL / 4; ++v) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      const int j = j0 + 4 * v;
      if (j < nb) f = __ldg(reinterpret_cast<const float4*>(srow + j0) + v);  // nb % 4 == 0
      key[4 * v] = j < nvalid ? score_key(f.x) : 0u;
      key[4 * v + 1] = j + 1 < nvalid ? score_key(f.y) : 0u;
      key[4 * v + 2] = j + 2 < nvalid ? score_key(f.z) : 0u;
      key[4 * v + 3] = j + 3 < nvalid ? score_key(f.w) : 0u;
    }
  } else {
#pragma unroll
    for (int t = 0; t < KPL; ++t) key[t] = j0 + t < nvalid ? score_key(__ldg(srow + j0 + t)) : 0u;
  }
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    kmin = min(kmin, key[t] == 0u ? 0xFFFFFFFFu : key[t]);  // padding is not a key
    kmax = max(kmax, key[t]);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // invariant: count(key >= lo) = clo >= k > chi = count(key >= hi); hi may be 2^32
  uint32_t lo = kmin;
  uint64_t hi = static_cast<uint64_t>(kmax) + 1;
  int clo = nvalid, chi = 0;
#pragma unroll 1
  for (int it = 0; it < 64 && clo - chi > 64 && hi - lo > 1; ++it) {
    const float flo = key_float(lo), fhi = key_float(static_cast<uint32_t>(hi - 1));
    const float fm = 0.5f * flo + 0.5f * fhi;
    uint32_t p = float_key(fm);
    // value steps first (fast on smooth score distributions), then key
    // midpoints, which end in at most 32 steps whatever the distribution
    if (it >= 12 || !(isfinite(fm) && p > lo && static_cast<uint64_t>(p) < hi))
      p = lo + static_cast<uint32_t>((hi - lo) >> 1);
    const int c = warp_count_ge(key, p);
    if (c >= k) {
      lo = p;
      clo = c;
    } else {
      hi = p;
      chi = c;
    }
  }
  // T = the k-th largest key, gt = #keys > T, eq = #keys == T
  uint32_t T;
  int gt, eq;
  if (hi - lo == 1) {
    T = lo;  // the bracket holds copies of one key
    gt = chi;
    eq = clo - chi;
  } else if (clo - chi <= 64) {
    // gather the bracket's keys (in any order) and sort them
    const uint32_t top = static_cast<uint32_t>(hi - 1);
    unsigned mine = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) mine += key[t] >= lo && key[t] <= top;
    unsigned incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = static_cast<int>(__shfl_sync(0xffffffffu, incl, 31));
    int off = static_cast<int>(incl - mine);
#pragma unroll
    for (int t = 0; t < KPL; ++t)
      if (key[t] >= lo && key[t] <= top && off < 64) cand[off++] = key[t];
    __syncwarp();
    uint32_t a = lane < total ? cand[lane] : 0u, b = lane + 32 < total ? cand[lane + 32] : 0u;
    __syncwarp();
    warp_sort64_desc(a, b, lane);
    const int r = k - chi - 1;  // 0 <= r < clo - chi <= 64
    const uint32_t va = __shfl_sync(0xffffffffu, a, r & 31), vb = __shfl_sync(0xffffffffu, b, r & 31);
    T = r < 32 ? va : vb;
    // every key == T lies in the bracket; keys above it are the chi keys >= hi
    gt = chi + __popc(__ballot_sync(0xffffffffu, a > T)) + __popc(__ballot_sync(0xffffffffu, b > T));
    eq = __popc(__ballot_sync(0xffffffffu, a == T)) + __popc(__ballot_sync(0xffffffffu, b == T));
  } else {
    // not narrowed in time (pathological rows): exact bitwise search
    T = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = T | (1u << bit);
      if (warp_count_ge(key, c) >= k) T = c;
    }
    gt = T == 0xFFFFFFFFu ? 0 : warp_count_ge(key, T + 1);
    eq = warp_count_ge(key, T) - gt;
  }
  const int need_eq = k - gt;  // >= 1 by the choice of T
  // this lane's picks as a bit mask over t (padding keys are 0 < T)
  uint32_t sel = 0;
  if (eq == need_eq) {
    // no tie straddles the cut: the selection is every key >= T
#pragma unroll
    for (int t = 0; t < KPL; ++t) sel |= (key[t] >= T ? 1u : 0u) << t;
  } else {
    // keys equal to T are taken in ascending j (lane order, then t) until k
    uint32_t eqm = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      sel |= (key[t] > T ? 1u : 0u) << t;
      eqm |= (key[t] == T ? 1u : 0u) << t;
    }
    const int neq = __popc(eqm);
    int incl = neq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int take = need_eq - (incl - neq);  // equal keys this lane still takes
    for (; take > 0 && eqm; --take) {
      sel |= eqm & (0u - eqm);  // lowest remaining equal key
      eqm &= eqm - 1u;
    }
  }
  const int nsel = __popc(sel);
  int incl = nsel;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  for (int pos = incl - nsel; sel && pos < k; ++pos) {
    out[pos] = j0 + __ffs(sel) - 1;
    sel &= sel - 1u;
  }
}

// Same selection with the keys re-read from shared memory (any nb).
__device__ __forceinline__ void select_row_smem(const float* srow, int nb, int k, int32_t* out,
                                                int lane) {
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < nb; j += 32) cnt += float_key(srow[j]) >= cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= k) T = cand;
  }
  int gt = 0;
  for (int j = lane; j < nb; j += 32) gt += float_key(srow[j]) > T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  const int need_eq = k - gt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < nb ? float_key(srow[j]) : 0u;
    const bool eq = (j < nb) && key == T;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_ballot & lt_mask);
    const bool sel = (j < nb) && (key > T || (eq && eq_rank < need_eq));
    const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sel_ballot & lt_mask);
    if (sel && pos < k) out[pos] = j;
    written += __popc(sel_ballot);
    eq_seen += __popc(eq_ballot);
  }
}

// Row length a warp stages in shared memory for nb > 1024: whole 128-key
// chunks (the tail is padding key 0).
__host__ __device__ constexpr int staged_row_keys(int nb) { return (nb + 127) & ~127; }

// The selection of select_row_bracket for a row too long for registers:
// keys (score_key, padding 0) staged once in shared memory, nbp of them
// (a multiple of 128). Counting passes read four keys per lane per
// 16-byte load; the bracket is narrowed on the score value, then on the key,
// to at most 64 keys, which are gathered and sorted; the emission is one
// ordered ballot pass. `cand` is 64 words of shared memory private to the warp.
__device__ __forceinline__ void select_row_staged(const uint32_t* keys, int nbp, int nvalid, int k,
                                                  int32_t* out, int lane, uint32_t* cand) {
  const uint4* kv = reinterpret_cast<const uint4*>(keys);
  const int nv4 = nbp / 4;
  auto count_ge = [&](uint32_t t) {
    unsigned c = 0;
    for (int q = lane; q < nv4; q += 32) {
      const uint4 u = kv[q];
      c += (u.x >= t) + (u.y >= t) + (u.z >= t) + (u.w >= t);
    }
    return static_cast<int>(__reduce_add_sync(0xffffffffu, c));
  };
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int q = lane; q < nv4; q += 32) {
    const uint4 u = kv[q];
    const uint32_t e[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      kmin = min(kmin, e[t] == 0u ? 0xFFFFFFFFu : e[t]);  // padding is not a key
      kmax = max(kmax, e[t]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // invariant: count(key >= lo) = clo >= k > chi = count(key >= hi); hi may be 2^32
  uint32_t lo = kmin;
  uint64_t hi = static_cast<uint64_t>(kmax) + 1;
  int clo = nvalid, chi = 0;
#pragma unroll 1
  for (int it = 0; it < 64 && clo - chi > 64 && hi - lo > 1; ++it) {
    const float flo = key_float(lo), fhi = key_float(static_cast<uint32_t>(hi - 1));
    const float fm = 0.5f * flo + 0.5f * fhi;
    uint32_t p = float_key(fm);
    if (it >= 12 || !(isfinite(fm) && p > lo && static_cast<uint64_t>(p) < hi))
      p = lo + static_cast<uint32_t>((hi - lo) >> 1);
    const int c = count_ge(p);
    if (c >= k) {
      lo = p;
      clo = c;
    } else {
      hi = p;
      chi = c;
    }
  }
  uint32_t T;
  int gt;
  if (hi - lo == 1) {
    T = lo;
    gt = chi;
  } else if (clo - chi <= 64) {
    // gather the bracket's keys and sort them
    const uint32_t top = static_cast<uint32_t>(hi - 1);
    const uint32_t lt_mask = (1u << lane) - 1u;
    int base = 0;
    for (int j0 = 0; j0 < nbp; j0 += 32) {
      const uint32_t key = keys[j0 + lane];
      const bool in = key >= lo && key <= top;
      const uint32_t b = __ballot_sync(0xffffffffu, in);
      const int pos = base + __popc(b & lt_mask);
      if (in && pos < 64) cand[pos] = key;
      base += __popc(b);
    }
    __syncwarp();
    const int total = base;
    uint32_t a = lane < total ? cand[lane] : 0u, b = lane + 32 < total ? cand[lane + 32] : 0u;
    __syncwarp();
    warp_sort64_desc(a, b, lane);
    const int r = k - chi - 1;  // 0 <= r < clo - chi <= 64
    const uint32_t va = __shfl_sync(0xffffffffu, a, r & 31), vb = __shfl_sync(0xffffffffu, b, r & 31);
    T = r < 32 ? va : vb;
    gt = chi + __popc(__ballot_sync(0xffffffffu, a > T)) + __popc(__ballot_sync(0xffffffffu, b > T));
  } else {
    // not narrowed in time (pathological rows): exact bitwise search
    T = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = T | (1u << bit);
      if (count_ge(c) >= k) T = c;
    }
    gt = T == 0xFFFFFFFFu ? 0 : count_ge(T + 1);
  }
  // keys above T, then the lowest-index keys equal to T, in ascending index
  const int need_eq = k - gt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
  for (int j0 = 0; j0 < nbp && written < k; j0 += 32) {
    const uint32_t key = keys[j0 + lane];
    const bool eq = key == T;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_ballot & lt_mask);
    const bool sel = key > T || (eq && eq_rank < need_eq);
    const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
    const int pos = written + __popc(sel_ballot & lt_mask);
    if (sel && pos < k) out[pos] = j0 + lane;
    written += __popc(sel_ballot);
    eq_seen += __popc(eq_ballot);
  }
}

// Row setup shared by the two top-k kernels: the output row, and with the
// causal flag the candidates [0, ncand) and the count ksel ranked among them
// (row r is query block i = r % nb: only key blocks j <= i are ranked and
// min(k, i + 1) are kept; with kFlagForceDiag block i always, plus the best
// j < i; the row is padded with -1). Returns false when nothing is ranked.
__device__ __forceinline__ bool topk_row_setup(long r, int nb, int k, unsigned flags, int32_t* out, int lane,
                                               int& ncand, int& ksel) {
  ncand = nb;
  ksel = k;
  if (flags & kFlagCausal) {
    const int i = static_cast<int>(r % nb);
    const bool force = (flags & kFlagForceDiag) != 0;
    const int n = min(k, i + 1);
    ncand = force ? i : i + 1;
    ksel = force ? n - 1 : n;
    if (force && lane == 0) out[ksel] = i;  // above every ranked id: the list stays ascending
    for (int t = n + lane; t < k; t += 32) out[t] = -1;
    if (ksel == 0) return false;
  }
  return true;
}

// grid.x = ceil(rows / kSelWarps); one warp per row of S ([rows, nb]), nb <= 1024:
// keys in registers.
__global__ void __launch_bounds__(kSelThreads, 4)
    block_topk_kernel(const float* __restrict__ S, int32_t* __restrict__ idx, long rows, int nb,
                      int k, unsigned flags) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ uint32_t cand[kSelWarps][64];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long r = static_cast<long>(blockIdx.x) * kSelWarps + warp;
  if (r >= rows) return;
  const float* srow = S + r * nb;
  int32_t* out = idx + r * static_cast<long>(k);
  const bool vec = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0;
  int ncand, ksel;
  if (!topk_row_setup(r, nb, k, flags, out, lane, ncand, ksel)) return;
  if (nb <= 32)
    select_row_bracket<1>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
  else if (nb <= 64)
    select_row_bracket<2>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
  else if (nb <= 128)
    select_row_bracket<4>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
  else if (nb <= 256)
    select_row_bracket<8>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
  else if (nb <= 512)
    select_row_bracket<16>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
  else
    select_row_bracket<32>(srow, nb, ncand, ksel, out, lane, cand[warp], vec);
}

// The same for nb > 1024. Dynamic shared memory: kSelWarps *
// staged_row_keys(nb) keys when stage_rows (the keys of each warp's row,
// converted once), else none (rows too long to stage are searched bit by bit
// from L2).
__global__ void __launch_bounds__(kSelThreads, 1)
    block_topk_wide_kernel(const float* __restrict__ S, int32_t* __restrict__ idx, long rows, int nb,
                           int k, int stage_rows, unsigned flags) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) uint32_t sel_keys[];
  __shared__ uint32_t cand[kSelWarps][64];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long r = static_cast<long>(blockIdx.x) * kSelWarps + warp;
  if (r >= rows) return;
  const float* srow = S + r * nb;
  int32_t* out = idx + r * static_cast<long>(k);
  const bool vec = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0;
  int ncand, ksel;
  if (!topk_row_setup(r, nb, k, flags, out, lane, ncand, ksel)) return;
  if (stage_rows) {
    const int nbp = staged_row_keys(nb);
    uint32_t* keys = sel_keys + static_cast<long>(warp) * nbp;
    if (vec) {
      // 16-byte loads (nb % 4 == 0), several in flight per lane
#pragma unroll 4
      for (int j = 4 * lane; j < nbp; j += 128) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < nb) f = __ldg(reinterpret_cast<const float4*>(srow + j));
        uint4 u;
        u.x = j < ncand ? score_key(f.x) : 0u;
        u.y = j + 1 < ncand ? score_key(f.y) : 0u;
        u.z = j + 2 < ncand ? score_key(f.z) : 0u;
        u.w = j + 3 < ncand ? score_key(f.w) : 0u;
        *reinterpret_cast<uint4*>(keys + j) = u;
      }
    } else {
      for (int j = lane; j < nbp; j += 32) keys[j] = j < ncand ? score_key(__ldg(srow + j)) : 0u;
    }
    __syncwarp();
    select_row_staged(keys, nbp, ncand, ksel, out, lane, cand[warp]);
  } else {
    select_row_smem(srow, ncand, ksel, out, lane);  // rows too long to stage: read them from L2
  }
}

}  // namespace bsa
