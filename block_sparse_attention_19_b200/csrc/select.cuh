// select.cuh -- steps 1b + 2: block scores and top-k block selection.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现": block_scores = einsum of the pooled q and k per
// (b, h) (an nb x nb matrix), then torch.topk(block_scores, k) over the key
// blocks. Readings fixed here: float32 dot products with no 1/sqrt(D) factor;
// ties go to the lower key-block index; each output row lists its k blocks in
// ascending order (a canonical order, so results are exactly comparable).
//
// One CTA owns R consecutive query blocks of one (b, h). Phase A computes the
// R score rows S[r, 0..nb) in float32 FFMA (each thread owns two key-block
// columns at a time; pooled q rows are broadcast from shared memory, pooled k
// rows stream from L2) and keeps them in shared memory. Phase B selects per
// row with one warp: the k-th largest score is found exactly by a bitwise
// binary search over order-preserving 32-bit keys, then one ordered pass
// emits every key above it plus the lowest-index keys equal to it.
#pragma once

#include <stdint.h>

namespace bsa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelSmemScoreBytes = 128 * 1024;  // R * nb * 4 bytes at most

// Order-preserving map float -> uint32 (larger float <=> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Rows per CTA for a given nb (power of two, R * nb * 4 <= kSelSmemScoreBytes).
inline int select_rows_per_cta(int nb) {
  int r = 32;
  while (r > 1 && static_cast<long>(r) * nb * 4 > kSelSmemScoreBytes) r >>= 1;
  return r;
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

// grid.x = B * H * ceil(nb / R). Dynamic shared memory: R * D floats (pooled q
// rows) + R * nb floats (score rows).
template <int R>
__global__ void __launch_bounds__(kSelThreads, 1)
    block_scores_topk_kernel(const float* __restrict__ qp, const float* __restrict__ kp,
                             float* __restrict__ scores_out, int32_t* __restrict__ idx, int H,
                             int nb, int D, int k) {
  extern __shared__ __align__(16) float sel_smem[];
  float* qs = sel_smem;         // [R][D]
  float* ss = sel_smem + R * D;  // [R][nb]

  const int tiles = (nb + R - 1) / R;
  const int tile = blockIdx.x % tiles;
  const long bh = blockIdx.x / tiles;
  const int i0 = tile * R;
  const int rows = min(R, nb - i0);
  const float* qbase = qp + (bh * nb + i0) * D;
  const float* kbase = kp + bh * nb * D;
  const int tid = threadIdx.x;

  for (int e = tid; e < R * D; e += kSelThreads) qs[e] = (e < rows * D) ? qbase[e] : 0.f;
  __syncthreads();

  // ---- phase A: S[r][j] = sum_d qs[r][d] * kp[j][d], two columns per thread
  for (int j0 = 2 * tid; j0 < nb; j0 += 2 * kSelThreads) {
    const bool two = j0 + 1 < nb;
    const float4* k0 = reinterpret_cast<const float4*>(kbase + static_cast<long>(j0) * D);
    const float4* k1 = reinterpret_cast<const float4*>(kbase + static_cast<long>(two ? j0 + 1 : j0) * D);
    float a0[R], a1[R];
#pragma unroll
    for (int r = 0; r < R; ++r) a0[r] = a1[r] = 0.f;
#pragma unroll 2
    for (int d4 = 0; d4 < D / 4; ++d4) {
      const float4 x = __ldg(k0 + d4);
      const float4 y = __ldg(k1 + d4);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 q = reinterpret_cast<const float4*>(qs + r * D)[d4];
        a0[r] = fmaf(q.x, x.x, a0[r]);
        a0[r] = fmaf(q.y, x.y, a0[r]);
        a0[r] = fmaf(q.z, x.z, a0[r]);
        a0[r] = fmaf(q.w, x.w, a0[r]);
        a1[r] = fmaf(q.x, y.x, a1[r]);
        a1[r] = fmaf(q.y, y.y, a1[r]);
        a1[r] = fmaf(q.z, y.z, a1[r]);
        a1[r] = fmaf(q.w, y.w, a1[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      ss[r * nb + j0] = a0[r];
      if (two) ss[r * nb + j0 + 1] = a1[r];
    }
    if (scores_out != nullptr) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r < rows) {
          float* srow = scores_out + (bh * nb + i0 + r) * static_cast<long>(nb);
          srow[j0] = a0[r];
          if (two) srow[j0 + 1] = a1[r];
        }
      }
    }
  }
  __syncthreads();

  // ---- phase B: one warp per row
  const int warp = tid / 32, lane = tid % 32;
  for (int r = warp; r < rows; r += kSelWarps) {
    const float* srow = ss + r * nb;
    int32_t* out = idx + (bh * nb + i0 + r) * static_cast<long>(k);
    if (nb <= 32)
      select_row_regs<1>(srow, nb, k, out, lane);
    else if (nb <= 64)
      select_row_regs<2>(srow, nb, k, out, lane);
    else if (nb <= 128)
      select_row_regs<4>(srow, nb, k, out, lane);
    else if (nb <= 256)
      select_row_regs<8>(srow, nb, k, out, lane);
    else if (nb <= 512)
      select_row_regs<16>(srow, nb, k, out, lane);
    else if (nb <= 1024)
      select_row_regs<32>(srow, nb, k, out, lane);
    else
      select_row_smem(srow, nb, k, out, lane);
  }
}

}  // namespace bsa
