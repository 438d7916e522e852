// attn_simt.cuh -- step 3 for float32 inputs: exact softmax attention over the
// selected key blocks, in float32 on CUDA cores.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 3 (sparse_attn_cuda with scale 1/sqrt(D));
// page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §2.1 (softmax of the
// masked, scaled QK^T times V).
//
// float32 inputs are held to an absolute error of 1e-4, which TF32 tensor
// cores cannot meet, so this path uses FFMA. One CTA (4 warps) owns 16 query
// rows of one (b, h, query block); it streams the selected key blocks through
// shared memory in tiles of 64 keys and keeps a flash-style running max, sum
// and output per row (each warp owns 4 rows; lane l owns output columns
// l, l+32, ...). Logits for a tile are computed one key per lane.
// An index row ends at its first -1 entry; with kFlagCausal key token t is
// left out for query token n when t > n.
#pragma once

#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kSimtThreads = 128;
constexpr int kSimtRows = 16;  // query rows per CTA
constexpr int kSimtKeys = 64;  // keys per shared-memory tile

template <int D>
struct SimtSmem {
  float q[kSimtRows][D];
  float k[kSimtKeys][D + 1];  // +1: conflict-free per-lane row reads
  float v[kSimtKeys][D];
  float p[4][kSimtKeys];      // per-warp probabilities of the current row
};

// grid.x = B * H * nb * (bs / kSimtRows). gperiod > 0: query heads h with
// h % gperiod == 0 are global heads (every key block, 0..i when causal).
// ws < bs: index entries name key windows starting at min(e * ws, N - bs)
// (nkb of them), and keys the previous kept window holds are masked.
template <int D>
__global__ void __launch_bounds__(kSimtThreads)
    sparse_attn_simt_kernel(const float* __restrict__ q, const float* __restrict__ kmat,
                            const float* __restrict__ v, const int32_t* __restrict__ idx,
                            float* __restrict__ o, int N, int H, int Hkv, int bs, int k, float scale,
                            unsigned flags, int gperiod, int ws, int nkb) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char simt_raw[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(simt_raw);
  constexpr int DL = D / 32;  // output columns per lane

  const int nb = N / bs;
  const int chunks = bs / kSimtRows;
  long u = blockIdx.x;
  const int chunk = static_cast<int>(u % chunks);
  u /= chunks;
  const int i = static_cast<int>(u % nb);
  u /= nb;
  const int h = static_cast<int>(u % H);
  const long b = u / H;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const long row_stride = static_cast<long>(H) * D;  // q and o rows
  const long kv_stride = static_cast<long>(Hkv) * D;  // k and v rows
  const int g = h / (H / Hkv);                        // key/value head of query head h
  const float* qb = q + (b * N) * row_stride + static_cast<long>(h) * D;
  const float* kb = kmat + (b * N) * kv_stride + static_cast<long>(g) * D;
  const float* vb = v + (b * N) * kv_stride + static_cast<long>(g) * D;
  const int n0 = i * bs + chunk * kSimtRows;

  for (int e = tid; e < kSimtRows * D; e += kSimtThreads) {
    const int r = e / D, d = e % D;
    sm.q[r][d] = qb[static_cast<long>(n0 + r) * row_stride + d];
  }

  float m[4], l[4], acc[4][DL];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < DL; ++c) acc[rr][c] = 0.f;
  }

  const int32_t* sel = idx + ((b * Hkv + g) * static_cast<long>(nb) + i) * k;
  const int tiles_per_block = bs / kSimtKeys;
  const bool causal = (flags & kFlagCausal) != 0;
  // a global head (h % gperiod == 0) attends to every block, 0..i when causal
  const bool dense = gperiod > 0 && h % gperiod == 0;
  const int nsel = dense ? (causal ? i + 1 : nb) : k;
  int prev_end = 0;  // overlapping windows: first token past the previous kept window
  for (int s = 0; s < nsel; ++s) {
    int blk = dense ? s : sel[s];
    if (blk < 0) {
      if (s > 0) break;  // the row's valid entries end here (a row of only -1 reads block 0)
      blk = 0;
    }
    const int lim_blk = dense ? nb : nkb;
    blk = blk >= lim_blk ? lim_blk - 1 : blk;
    const int w0 = dense ? blk * bs : min(blk * ws, N - bs);  // first token of the window
    // keys of this window before `dup_end` were in the previous kept window
    const int dup_end = (!dense && s > 0 && ws < bs) ? prev_end : 0;
    prev_end = w0 + bs;
    for (int tt = 0; tt < tiles_per_block; ++tt) {
      const int t0 = w0 + tt * kSimtKeys;
      __syncthreads();  // previous tile fully consumed
      for (int e = tid; e < kSimtKeys * D; e += kSimtThreads) {
        const int r = e / D, d = e % D;
        sm.k[r][d] = kb[static_cast<long>(t0 + r) * kv_stride + d];
        sm.v[r][d] = vb[static_cast<long>(t0 + r) * kv_stride + d];
      }
      __syncthreads();
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = warp * 4 + rr;
        // logits of keys lane and lane + 32
        float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
          const float qd = sm.q[r][d];
          s0 = fmaf(qd, sm.k[lane][d], s0);
          s1 = fmaf(qd, sm.k[lane + 32][d], s1);
        }
        s0 *= scale;
        s1 *= scale;
        if (causal) {
          if (t0 + lane > n0 + r) s0 = -INFINITY;
          if (t0 + lane + 32 > n0 + r) s1 = -INFINITY;
        }
        if (t0 + lane < dup_end) s0 = -INFINITY;
        if (t0 + lane + 32 < dup_end) s1 = -INFINITY;
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m[rr], mx);
        // reference point of the exponentials: finite even while every key so
        // far is masked (then alpha and p are 0, as are l and acc)
        const float m_ref = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = expf(m[rr] - m_ref);  // 0 on the first tile (m = -inf)
        const float p0 = expf(s0 - m_ref), p1 = expf(s1 - m_ref);
        float ps = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l[rr] = l[rr] * alpha + ps;
        m[rr] = m_new;
        sm.p[warp][lane] = p0;
        sm.p[warp][lane + 32] = p1;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < DL; ++c) acc[rr][c] *= alpha;
#pragma unroll 8
        for (int t = 0; t < kSimtKeys; ++t) {
          const float pt = sm.p[warp][t];
#pragma unroll
          for (int c = 0; c < DL; ++c) acc[rr][c] = fmaf(pt, sm.v[t][lane + 32 * c], acc[rr][c]);
        }
        __syncwarp();
      }
    }
  }

  float* ob = o + (b * N) * row_stride + static_cast<long>(h) * D;
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    const float inv = 1.0f / l[rr];
#pragma unroll
    for (int c = 0; c < DL; ++c) ob[static_cast<long>(n0 + r) * row_stride + lane + 32 * c] = acc[rr][c] * inv;
  }
}

}  // namespace bsa
