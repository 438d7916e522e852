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
// (about 8 counting passes on typical rows instead of 32). For nb <= 4096
// the keys sit in registers (block_topk_kernel up to 1024,
// block_topk_reg_wide_kernel beyond); longer rows are converted once into
// shared memory and counted from there (block_topk_wide_kernel; rows too long
// to stage fall back to a bitwise search read from L2). One
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

// Reductions over the NW warps that share one row (a whole CTA when NW > 1,
// whose threads all call every member in the same order). Each warp reduces
// its lanes with redux/shuffles; with NW > 1 the warp results meet in shared
// memory behind one __syncthreads, in two buffers used alternately (a buffer
// is rewritten only after the barrier of the next reduction, which every
// thread reaches after reading it).
template <int NW>
struct RowGroup {
  uint32_t* buf;  // 2 x NW x 4 words of shared memory (NW > 1)
  int warp, lane, par;
  __device__ __forceinline__ RowGroup(uint32_t* b, int w, int l) : buf(b), warp(w), lane(l), par(0) {}
  // four values at once: op 0 = add, 1 = min, 2 = max (u32), 3 = float add
  __device__ __forceinline__ void reduce4(uint32_t (&v)[4], const int (&op)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (op[i] == 0) v[i] = __reduce_add_sync(0xffffffffu, v[i]);
      else if (op[i] == 1) v[i] = __reduce_min_sync(0xffffffffu, v[i]);
      else if (op[i] == 2) v[i] = __reduce_max_sync(0xffffffffu, v[i]);
      else {
        float f = __uint_as_float(v[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
        v[i] = __float_as_uint(f);
      }
    }
    if constexpr (NW > 1) {
      uint32_t* b = buf + par * NW * 4;
      if (lane == 0)
#pragma unroll
        for (int i = 0; i < 4; ++i) b[warp * 4 + i] = v[i];
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t r = b[i];
        for (int w = 1; w < NW; ++w) {
          const uint32_t x = b[w * 4 + i];
          if (op[i] == 0) r += x;
          else if (op[i] == 1) r = min(r, x);
          else if (op[i] == 2) r = max(r, x);
          else r = __float_as_uint(__uint_as_float(r) + __uint_as_float(x));
        }
        v[i] = r;
      }
      par ^= 1;
    }
  }
  __device__ __forceinline__ int sum(unsigned x) {
    uint32_t v[4] = {x, 0u, 0u, 0u};
    const int op[4] = {0, 0, 0, 0};
    reduce4(v, op);
    return static_cast<int>(v[0]);
  }
  // exclusive prefix of x over the group's threads in (warp, lane) order,
  // and the total
  __device__ __forceinline__ int prefix(int x, int& total) {
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int before = incl - x;
    const int wtot = __shfl_sync(0xffffffffu, incl, 31);
    total = wtot;
    if constexpr (NW > 1) {
      uint32_t* b = buf + par * NW * 4;
      if (lane == 0) b[warp * 4] = static_cast<uint32_t>(wtot);
      __syncthreads();
      total = 0;
      for (int w = 0; w < NW; ++w) {
        const int t = static_cast<int>(b[w * 4]);
        if (w < warp) before += t;
        total += t;
      }
      par ^= 1;
    }
    return before;
  }
};

// Number of the group's keys >= t.
template <int KPL, int NW>
__device__ __forceinline__ int group_count_ge(const uint32_t (&key)[KPL], uint32_t t, RowGroup<NW>& grp) {
  unsigned c = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) c += key[i] >= t;
  return grp.sum(c);
}

// Pivot for a target count t inside the bracket: the score value where the
// row is expected to hold t keys at or above it, from a Gaussian model of the
// whole row (first pass: mean mu, deviation sd over n scores) or from a
// linear count between the bracket ends (later passes: count clo at value
// flo, chi at fhi). Returns 0 (no pivot) when the estimate is not strictly
// inside the bracket (lo, hi).
__device__ __forceinline__ uint32_t interp_pivot(int t, bool gaussian, float mu, float sd, float n, float flo,
                                                 float fhi, int clo, int chi, uint32_t lo, uint64_t hi) {
  float x;
  if (gaussian) {
    // count(>= x) = n (1 - Phi((x - mu) / sd))  =>  x = mu + sd sqrt(2) erfinv(1 - 2 t / n)
    const float q = fminf(fmaxf(1.0f - 2.0f * static_cast<float>(t) / n, -0.999999f), 0.999999f);
    x = mu + sd * 1.41421356f * erfinvf(q);
  } else {
    x = flo + (fhi - flo) * (static_cast<float>(clo - t) / static_cast<float>(clo - chi));
  }
  if (!isfinite(x)) return 0u;
  const uint32_t p = float_key(x);
  return (p > lo && static_cast<uint64_t>(p) < hi) ? p : 0u;
}

// NW warps (one CTA when NW > 1) select the k largest of a row of
// nb <= 32 * NW * KPL scores held as keys in registers, thread-major: thread
// g = 32 * warp + lane holds keys j = g * KPL + t, so ascending j is thread
// order and each thread loads a contiguous run (float4 loads when `vec`: the
// row starts 16-byte aligned and nb % 4 == 0). The k-th largest key is
// bracketed first (groups of several warps) with two pivots per counting
// pass, placed where about k + 24 and k - 24 keys are expected at or above
// them (a Gaussian model of the row for the first pass, a linear count
// between the bracket ends after it; up to 4 such passes), then by bisection (up to 12 steps on the score
// value, then on the key, which needs at most 32 steps), until the bracket
// [lo, hi) holds at most 64 keys, which are then sorted exactly; a bracket
// that cannot be split holds equal keys only. `cand` is 64 words of shared
// memory private to the group. (A single warp skips the pivot passes.)
template <int KPL, int NW>
__device__ __forceinline__ void select_row_group(const float* srow, int nb, int nvalid, int k, int32_t* out,
                                                 int warp, int lane, uint32_t* cand, bool vec, RowGroup<NW>& grp) {
  constexpr int W = (KPL + 31) / 32;  // 32-key words of a thread's selection masks
  uint32_t key[KPL];
  float sx = 0.f, sxx = 0.f;  // sum and sum of squares of the thread's valid scores (NW > 1)
  const int j0 = (warp * 32 + lane) * KPL;
  if (KPL % 4 == 0 && vec) {
#pragma unroll
    for (int v = 0; v < KPL / 4; ++v) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      const int j = j0 + 4 * v;
      if (j < nb) f = __ldg(reinterpret_cast<const float4*>(srow + j0) + v);  // nb % 4 == 0
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool valid = j + e < nvalid;
        key[4 * v + e] = valid ? score_key(fv[e]) : 0u;
        if constexpr (NW > 1) {
          const float x = valid ? fv[e] : 0.f;
          sx += x;
          sxx = fmaf(x, x, sxx);
        }
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      const bool valid = j0 + t < nvalid;
      const float x = valid ? __ldg(srow + j0 + t) : 0.f;
      key[t] = valid ? score_key(x) : 0u;
      if constexpr (NW > 1) {
        sx += x;
        sxx = fmaf(x, x, sxx);
      }
    }
  }
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    kmin = min(kmin, key[t] == 0u ? 0xFFFFFFFFu : key[t]);  // padding is not a key
    kmax = max(kmax, key[t]);
  }
  if constexpr (NW > 1) {
    uint32_t v[4] = {kmin, kmax, __float_as_uint(sx), __float_as_uint(sxx)};
    const int op[4] = {1, 2, 3, 3};
    grp.reduce4(v, op);
    kmin = v[0];
    kmax = v[1];
    sx = __uint_as_float(v[2]);
    sxx = __uint_as_float(v[3]);
  } else {
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
  }
  // invariant: count(key >= lo) = clo >= k > chi = count(key >= hi); hi may be 2^32
  uint32_t lo = kmin;
  uint64_t hi = static_cast<uint64_t>(kmax) + 1;
  int clo = nvalid, chi = 0;
  // The pivot passes save counting passes, which matter most when every pass
  // costs a group barrier: measured faster than bisection alone for groups of
  // 4 warps on 4096-key rows, slower for one warp on rows of <= 1024 keys
  // (the model's fixed cost is then not paid back).
  if constexpr (NW > 1) {
    const float n = static_cast<float>(nvalid), mu = sx / n;
    const float sd = sqrtf(fmaxf(sxx / n - mu * mu, 0.f));
#pragma unroll 1
    for (int it = 0; it < 4 && clo - chi > 64 && hi - lo > 1; ++it) {
      const float flo = key_float(lo), fhi = key_float(static_cast<uint32_t>(hi - 1));
      const bool gauss = it == 0 && sd > 0.f;
      // pivot 1 should keep >= k keys above it, pivot 2 fewer than k
      const uint32_t p1 = interp_pivot(min(clo, k + 24), gauss, mu, sd, n, flo, fhi, clo, chi, lo, hi);
      uint32_t p2 = interp_pivot(max(chi, k - 24), gauss, mu, sd, n, flo, fhi, clo, chi, lo, hi);
      if (p1 == 0u && p2 == 0u) break;  // no estimate inside the bracket: bisect
      if (p2 != 0u && p2 <= p1) p2 = 0u;
      unsigned c1 = 0, c2 = 0;
#pragma unroll
      for (int t = 0; t < KPL; ++t) {
        c1 += key[t] >= p1;  // p1 == 0 counts every key (and padding): not used
        c2 += key[t] >= p2;
      }
      uint32_t v[4] = {c1, c2, 0u, 0u};
      const int op[4] = {0, 0, 0, 0};
      grp.reduce4(v, op);
      const int n1 = static_cast<int>(v[0]), n2 = static_cast<int>(v[1]);
      // counts fall as the pivot rises, so the two updates never conflict
      if (p1 != 0u) {
        if (n1 >= k) { lo = p1; clo = n1; } else { hi = p1; chi = n1; }
      }
      if (p2 != 0u && static_cast<uint64_t>(p2) < hi && p2 > lo) {
        if (n2 >= k) { lo = p2; clo = n2; } else { hi = p2; chi = n2; }
      }
    }
  }
#pragma unroll 1
  for (int it = 0; it < 64 && clo - chi > 64 && hi - lo > 1; ++it) {
    const float flo = key_float(lo), fhi = key_float(static_cast<uint32_t>(hi - 1));
    const float fm = 0.5f * flo + 0.5f * fhi;
    uint32_t p = float_key(fm);
    // value steps first (fast on smooth score distributions), then key
    // midpoints, which end in at most 32 steps whatever the distribution
    if (it >= 12 || !(isfinite(fm) && p > lo && static_cast<uint64_t>(p) < hi))
      p = lo + static_cast<uint32_t>((hi - lo) >> 1);
    const int c = group_count_ge(key, p, grp);
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
    // gather the bracket's keys (in any order) and sort them (every warp of
    // the group sorts the same 64 keys)
    const uint32_t top = static_cast<uint32_t>(hi - 1);
    unsigned mine = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) mine += key[t] >= lo && key[t] <= top;
    int total;
    int off = grp.prefix(static_cast<int>(mine), total);
#pragma unroll
    for (int t = 0; t < KPL; ++t)
      if (key[t] >= lo && key[t] <= top && off < 64) cand[off++] = key[t];
    if constexpr (NW > 1) __syncthreads(); else __syncwarp();
    uint32_t a = lane < total ? cand[lane] : 0u, b = lane + 32 < total ? cand[lane + 32] : 0u;
    if constexpr (NW > 1) __syncthreads(); else __syncwarp();
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
      if (group_count_ge(key, c, grp) >= k) T = c;
    }
    gt = T == 0xFFFFFFFFu ? 0 : group_count_ge(key, T + 1, grp);
    eq = group_count_ge(key, T, grp) - gt;
  }
  const int need_eq = k - gt;  // >= 1 by the choice of T
  // this thread's picks as bit masks over t, word t / 32 (padding keys are 0 < T)
  uint32_t sel[W];
#pragma unroll
  for (int w = 0; w < W; ++w) sel[w] = 0u;
  if (eq == need_eq) {
    // no tie straddles the cut: the selection is every key >= T
#pragma unroll
    for (int t = 0; t < KPL; ++t) sel[t / 32] |= (key[t] >= T ? 1u : 0u) << (t % 32);
  } else {
    // keys equal to T are taken in ascending j (thread order, then t) until k
    uint32_t eqm[W];
#pragma unroll
    for (int w = 0; w < W; ++w) eqm[w] = 0u;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      sel[t / 32] |= (key[t] > T ? 1u : 0u) << (t % 32);
      eqm[t / 32] |= (key[t] == T ? 1u : 0u) << (t % 32);
    }
    int neq = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) neq += __popc(eqm[w]);
    int all_eq;
    int take = need_eq - grp.prefix(neq, all_eq);  // equal keys this thread still takes
#pragma unroll
    for (int w = 0; w < W; ++w)
      for (; take > 0 && eqm[w]; --take) {
        sel[w] |= eqm[w] & (0u - eqm[w]);  // lowest remaining equal key
        eqm[w] &= eqm[w] - 1u;
      }
  }
  int nsel = 0;
#pragma unroll
  for (int w = 0; w < W; ++w) nsel += __popc(sel[w]);
  int all_sel;
  int pos = grp.prefix(nsel, all_sel);
#pragma unroll
  for (int w = 0; w < W; ++w)
    for (uint32_t m = sel[w]; m && pos < k; ++pos) {
      out[pos] = j0 + 32 * w + __ffs(m) - 1;
      m &= m - 1u;
    }
}

// One warp per row (keys in registers).
template <int KPL>
__device__ __forceinline__ void select_row_bracket(const float* srow, int nb, int nvalid, int k,
                                                   int32_t* out, int lane, uint32_t* cand, bool vec) {
  RowGroup<1> grp(nullptr, 0, lane);
  select_row_group<KPL, 1>(srow, nb, nvalid, k, out, 0, lane, cand, vec, grp);
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
// Only the lanes of one warp write (`writer`); every caller gets the counts.
__device__ __forceinline__ bool topk_row_setup(long r, int nb, int k, unsigned flags, int32_t* out, int lane,
                                               int& ncand, int& ksel, bool writer = true) {
  ncand = nb;
  ksel = k;
  if (flags & kFlagCausal) {
    const int i = static_cast<int>(r % nb);
    const bool force = (flags & kFlagForceDiag) != 0;
    const int n = min(k, i + 1);
    ncand = force ? i : i + 1;
    ksel = force ? n - 1 : n;
    if (writer) {
      if (force && lane == 0) out[ksel] = i;  // above every ranked id: the list stays ascending
      for (int t = n + lane; t < k; t += 32) out[t] = -1;
    }
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

// One CTA of 4 warps per row for 1024 < nb <= 4096: the keys stay in
// registers (16 or 32 per thread), the four warps reduce through shared
// memory, and many small CTAs per SM keep enough rows in flight.
constexpr int kSelGroupThreads = 128;
constexpr int kSelGroupWarps = kSelGroupThreads / 32;

__global__ void __launch_bounds__(kSelGroupThreads, 8)
    block_topk_group_kernel(const float* __restrict__ S, int32_t* __restrict__ idx, long rows, int nb, int k,
                            unsigned flags) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ uint32_t cand[64];
  __shared__ uint32_t red[2 * kSelGroupWarps * 4];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long r = blockIdx.x;
  if (r >= rows) return;  // whole CTA: the barriers below stay uniform
  const float* srow = S + r * nb;
  int32_t* out = idx + r * static_cast<long>(k);
  const bool vec = (nb & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0;
  int ncand, ksel;
  // warp 0 writes the causal padding of the row
  const bool ranked = topk_row_setup(r, nb, k, flags, out, lane, ncand, ksel, warp == 0);
  if (!ranked) return;  // uniform over the CTA: it depends on the row only
  RowGroup<kSelGroupWarps> grp(red, warp, lane);
  if (nb <= 2048)
    select_row_group<16, kSelGroupWarps>(srow, nb, ncand, ksel, out, warp, lane, cand, vec, grp);
  else
    select_row_group<32, kSelGroupWarps>(srow, nb, ncand, ksel, out, warp, lane, cand, vec, grp);
}

// The same for nb > 4096. Dynamic shared memory: kSelWarps *
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
