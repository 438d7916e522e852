// select.cuh -- step 2: top-k block selection from the block scores.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 2: torch.topk(block_scores, k) over the key
// blocks. Readings fixed here: ties go to the lower key-block index; each
// output row lists its k blocks in ascending order (a canonical order, so
// results compare exactly).
//
// One warp per score row, scores as order-preserving 32-bit keys. For
// nb <= 1024 the keys sit in registers and the k-th largest key is
// bracketed by bisection (on the score value, then on the key) until at most
// 64 keys remain in the bracket, which are sorted exactly (about 8 counting
// passes on typical rows instead of 32); longer rows use a bitwise binary search over the keys
// staged in shared memory. One ordered ballot pass then emits every key above
// the k-th largest plus the lowest-index keys equal to it.
#pragma once

#include <stdint.h>

namespace bsa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

// Order-preserving map float -> uint32 (larger float <=> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Per-lane key capacity of the register path of phase B (nb <= 32 * KPL).
template <int KPL>
__device__ __forceinline__ void select_row_regs(const float* srow, int nb, int k, int32_t* out,
                                                int lane) {
  uint32_t key[KPL];
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const int j = t * 32 + lane;
    key[t] = j < nb ? float_key(srow[j]) : 0u;  // padding key 0 is never counted (cand >= 1)
  }
  // T = largest key value with #{key >= T} >= k: the k-th largest key.
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) cnt += key[t] >= cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= k) T = cand;
  }
  int gt = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) gt += key[t] > T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  const int need_eq = k - gt;  // >= 1 by the choice of T

  // ordered emission: ascending j, lanes cover 32 consecutive j per step
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const int j = t * 32 + lane;
    const bool eq = (j < nb) && key[t] == T;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_ballot & lt_mask);
    const bool sel = (j < nb) && (key[t] > T || (eq && eq_rank < need_eq));
    const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(sel_ballot & lt_mask)] = j;
    written += __popc(sel_ballot);
    eq_seen += __popc(eq_ballot);
  }
}

__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

template <int KPL>
__device__ __forceinline__ int warp_count_ge(const uint32_t (&key)[KPL], uint32_t t) {
  int c = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) c += key[i] >= t;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  return c;
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

// Same result as select_row_regs with far fewer passes on typical rows: the
// k-th largest key is bracketed by bisection (up to 12 steps on the score
// value, then on the key, which needs at most 32 steps) until the bracket
// [lo, hi) holds at most 64 keys, which are then sorted exactly; a
// bracket that cannot be split holds equal keys only. `cand` is 64 words of
// shared memory private to the warp.
template <int KPL>
__device__ __forceinline__ void select_row_bracket(const float* srow, int nb, int k, int32_t* out,
                                                   int lane, uint32_t* cand) {
  uint32_t key[KPL];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const int j = t * 32 + lane;
    key[t] = j < nb ? float_key(srow[j]) : 0u;  // padding 0 never reaches a bracket above 0
    if (j < nb) {
      kmin = min(kmin, key[t]);
      kmax = max(kmax, key[t]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  // invariant: count(key >= lo) = clo >= k > chi = count(key >= hi); hi may be 2^32
  uint32_t lo = kmin;
  uint64_t hi = static_cast<uint64_t>(kmax) + 1;
  int clo = nb, chi = 0;
  if (kmin == 0u) clo = warp_count_ge(key, 0u) - (KPL * 32 - nb);  // real keys of value 0
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
  uint32_t T;
  if (hi - lo == 1) {
    T = lo;  // the bracket holds copies of one key
  } else if (clo - chi <= 64) {
    // gather the bracket's keys and take the (k - chi)-th largest exactly
    int base = 0;
    const uint32_t lt_mask0 = (1u << lane) - 1u;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      const bool in = key[t] >= lo && static_cast<uint64_t>(key[t]) < hi && t * 32 + lane < nb;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (in) cand[base + __popc(bal & lt_mask0)] = key[t];
      base += __popc(bal);
    }
    __syncwarp();
    uint32_t a = lane < base ? cand[lane] : 0u, b = lane + 32 < base ? cand[lane + 32] : 0u;
    __syncwarp();
    warp_sort64_desc(a, b, lane);
    const int r = k - chi - 1;
    const uint32_t va = __shfl_sync(0xffffffffu, a, r & 31), vb = __shfl_sync(0xffffffffu, b, r & 31);
    T = r < 32 ? va : vb;
  } else {
    // not narrowed in time (pathological rows): exact bitwise search
    T = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = T | (1u << bit);
      if (warp_count_ge(key, c) >= k) T = c;
    }
  }
  const int gt = T == 0xFFFFFFFFu ? 0 : warp_count_ge(key, T + 1);
  const int need_eq = k - gt;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const int j = t * 32 + lane;
    const bool eq = (j < nb) && key[t] == T;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_ballot & lt_mask);
    const bool sel = (j < nb) && (key[t] > T || (eq && eq_rank < need_eq));
    const uint32_t sel_ballot = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(sel_ballot & lt_mask)] = j;
    written += __popc(sel_ballot);
    eq_seen += __popc(eq_ballot);
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
    if (sel) out[written + __popc(sel_ballot & lt_mask)] = j;
    written += __popc(sel_ballot);
    eq_seen += __popc(eq_ballot);
  }
}

// grid.x = ceil(rows / kSelWarps); one warp per row of S ([rows, nb]).
// Dynamic shared memory: kSelWarps * nb floats when nb > 1024 and stage_rows, else none.
__global__ void __launch_bounds__(kSelThreads)
    block_topk_kernel(const float* __restrict__ S, int32_t* __restrict__ idx, long rows, int nb,
                      int k, int stage_rows) {
  extern __shared__ __align__(16) float sel_rows[];
  __shared__ uint32_t cand[kSelWarps][64];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long r = static_cast<long>(blockIdx.x) * kSelWarps + warp;
  if (r >= rows) return;
  const float* srow = S + r * nb;
  int32_t* out = idx + r * static_cast<long>(k);
  if (nb <= 32)
    select_row_bracket<1>(srow, nb, k, out, lane, cand[warp]);
  else if (nb <= 64)
    select_row_bracket<2>(srow, nb, k, out, lane, cand[warp]);
  else if (nb <= 128)
    select_row_bracket<4>(srow, nb, k, out, lane, cand[warp]);
  else if (nb <= 256)
    select_row_bracket<8>(srow, nb, k, out, lane, cand[warp]);
  else if (nb <= 512)
    select_row_bracket<16>(srow, nb, k, out, lane, cand[warp]);
  else if (nb <= 1024)
    select_row_bracket<32>(srow, nb, k, out, lane, cand[warp]);
  else if (stage_rows) {
    // the row is re-read once per key bit: stage it in shared memory
    float* row = sel_rows + static_cast<long>(warp) * nb;
    if ((nb & 3) == 0) {
      for (int j = lane * 4; j < nb; j += 128)
        *reinterpret_cast<float4*>(row + j) = __ldg(reinterpret_cast<const float4*>(srow + j));
    } else {
      for (int j = lane; j < nb; j += 32) row[j] = __ldg(srow + j);
    }
    __syncwarp();
    select_row_smem(row, nb, k, out, lane);
  } else {
    select_row_smem(srow, nb, k, out, lane);  // rows too long to stage: read them from L2
  }
}

}  // namespace bsa
