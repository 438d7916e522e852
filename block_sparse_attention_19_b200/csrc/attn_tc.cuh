// attn_tc.cuh -- step 3 for bfloat16 inputs on the sm_100a tensor cores.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 3: sparse_attn_cuda(q, k, v, topk_indices,
// block_size, scale=1/sqrt(D)); page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现
// 全解析" §2.2: full attention inside the chosen blocks. For every query row,
// o = softmax(scale * q K_sel^T) V_sel over the tokens of the selected blocks.
//
// Design (one CTA per (b, h, query block, 128-row part of the block)):
//   * The selected key blocks are walked as "key tiles" of up to 128 rows:
//     block_size 128 -> one block per tile; 256 -> two tiles per block;
//     64 -> two blocks per tile (the last tile has 64 rows when k is odd).
//   * Warp 0 (one lane) is the TMA producer: it loads the query tile once and
//     gathers each key tile's K and V rows by block index into a 2-stage
//     shared-memory ring (128-byte swizzled boxes of 64 rows x 64 columns).
//   * Warp 1 (one lane) issues tcgen05.mma: S_t = Q K_t^T into one of two TMEM
//     score buffers, then O += P_t V_t into a TMEM output accumulator; S_{t+1}
//     is issued before PV_t so the tensor core works while softmax runs.
//   * Warps 2-5 (128 threads, one query row each) run the online softmax:
//     read their S row from TMEM, keep a running max in the log2 domain that
//     is only moved when it grows by more than 8 (so O is rarely rescaled),
//     write P = exp2(S * scale * log2 e - max) as bf16 into shared memory in
//     the MMA operand layout, and finally normalise O by the running sum and
//     store the output row.
//   * Every mbarrier wait is bounded; a timeout sets the device error word and
//     an abort flag, all roles leave their loops, in-flight copies and MMAs
//     are drained (bounded) and TMEM is freed.
// Accumulation is float32 throughout (TMEM); P is rounded to bf16 for the
// second MMA.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kTcThreads = 192;  // 6 warps: producer, MMA, 4 x softmax
constexpr int kKeyTile = 128;    // key rows per tile
constexpr int kStages = 2;       // K/V pipeline depth

template <int D, int BM>
struct TcLayout {
  static constexpr int kChunks = D / 64;  // 128-byte column chunks across D
  static constexpr uint32_t kQBytes = BM * D * 2;
  static constexpr uint32_t kKVBytes = kKeyTile * D * 2;  // one stage of K (or V)
  static constexpr uint32_t kPBytes = BM * kKeyTile * 2;  // one P buffer
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + kQBytes;
  static constexpr uint32_t kVOff = kKOff + kStages * kKVBytes;
  static constexpr uint32_t kPOff = kVOff + kStages * kKVBytes;
  static constexpr uint32_t kBarOff = kPOff + 2 * kPBytes;
  static constexpr uint32_t kBytes = kBarOff + 256;
  static constexpr uint32_t kSmemAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t kTmemCols = 512;             // S0 | S1 | O
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kColO + D <= kTmemCols, "TMEM budget");
};

struct TcBarriers {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t mma_drained;
  uint32_t tmem_base;
  int abort;
};

// Rows of key tile t: (first token row of each 64-row half, halves used).
__device__ __forceinline__ int tile_keys(int t, int bs, int k) {
  return (bs == 64 && 2 * t + 1 >= k) ? 64 : 128;
}

__device__ __forceinline__ int clamp_block(int blk, int nb) {
  return blk < 0 ? 0 : (blk >= nb ? nb - 1 : blk);
}

__device__ __forceinline__ int half_row0(const int32_t* sel, int t, int half, int bs, int nb) {
  if (bs == 64) return clamp_block(__ldg(sel + 2 * t + half), nb) * 64;
  if (bs == 128) return clamp_block(__ldg(sel + t), nb) * 128 + half * 64;
  return clamp_block(__ldg(sel + t / 2), nb) * 256 + (t % 2) * 128 + half * 64;  // bs == 256
}

// grid.x = B * H * nb * parts, parts = max(1, bs / BM).
template <int D, int BM>
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, int N,
                          int H, int bs, int k, float scale_log2) {
  using L = TcLayout<D, BM>;
  extern __shared__ unsigned char tc_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  TcBarriers& bar = *reinterpret_cast<TcBarriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;

  const int nb = N / bs;
  const int parts = bs > BM ? bs / BM : 1;
  long u = blockIdx.x;
  const int part = static_cast<int>(u % parts);
  u /= parts;
  const int i = static_cast<int>(u % nb);
  u /= nb;
  const int h = static_cast<int>(u % H);
  const int b = static_cast<int>(u / H);
  const int32_t* sel = idx + ((static_cast<long>(b) * H + h) * nb + i) * k;
  const int T = bs == 64 ? (k + 1) / 2 : (bs == 128 ? k : 2 * k);  // key tiles

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.p_full[s], 4);
      mbar_init(&bar.pv_done[s], 1);
    }
    mbar_init(&bar.mma_drained, 1);
    bar.abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      const uint64_t keep = policy_evict_last();    // gathered K/V: reused across query blocks
      const uint64_t stream = policy_evict_first();  // query tile: read once
      int issued_k[kStages] = {0, 0}, issued_v[kStages] = {0, 0};
      bool ok = true;
      mbar_arrive_expect_tx(&bar.q_full, L::kQBytes);
      const int qrow0 = i * bs + part * BM;
      for (int hh = 0; hh < BM / 64; ++hh)
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(smem + L::kQOff + c * (BM * 128) + hh * 64 * 128, &tm_q, &bar.q_full, c * 64,
                      h, qrow0 + hh * 64, b, stream);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % kStages, use = t / kStages;
        const int halves = tile_keys(t, bs, k) / 64;
        const uint32_t bytes = halves * 64 * D * 2;
        int row0[2];
        for (int hf = 0; hf < halves; ++hf) row0[hf] = half_row0(sel, t, hf, bs, nb);
        if (t >= kStages) ok = mbar_wait(&bar.k_empty[s], (use - 1) & 1, abort_flag, 101);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar.k_full[s], bytes);
        for (int hf = 0; hf < halves; ++hf)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + L::kKOff + s * L::kKVBytes + c * (kKeyTile * 128) + hf * 64 * 128,
                        &tm_k, &bar.k_full[s], c * 64, h, row0[hf], b, keep);
        issued_k[s] = use + 1;
        if (t >= kStages) ok = mbar_wait(&bar.v_empty[s], (use - 1) & 1, abort_flag, 102);
        if (!ok) break;
        mbar_arrive_expect_tx(&bar.v_full[s], bytes);
        for (int hf = 0; hf < halves; ++hf)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + L::kVOff + s * L::kKVBytes + c * (kKeyTile * 128) + hf * 64 * 128,
                        &tm_v, &bar.v_full[s], c * 64, h, row0[hf], b, keep);
        issued_v[s] = use + 1;
      }
      // drain: every copy this thread issued has landed before TMEM/smem teardown
      mbar_wait_teardown(&bar.q_full, 0);
      for (int s = 0; s < kStages; ++s) {
        if (issued_k[s]) mbar_wait_teardown(&bar.k_full[s], (issued_k[s] - 1) & 1);
        if (issued_v[s]) mbar_wait_teardown(&bar.v_full[s], (issued_v[s] - 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kSBO = 1024;  // 8 rows x 128 bytes
      const uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);  // P K-major, V MN-major
      bool ok = mbar_wait(&bar.q_full, 0, abort_flag, 201);
      for (int t = 0; t <= T && ok; ++t) {
        if (t < T) {  // ---- S_t = Q K_t^T
          const int s = t % kStages, use = t / kStages;
          const int nk = tile_keys(t, bs, k);
          ok = mbar_wait(&bar.k_full[s], use & 1, abort_flag, 202);
          if (ok && t >= 2) ok = mbar_wait(&bar.p_full[t % 2], ((t - 2) / 2) & 1, abort_flag, 203);
          if (!ok) break;
          tc_fence_after();
          const uint32_t idesc_s = idesc_bf16_f32(BM, nk, 0, 0);
          const uint32_t d_tmem = tmem + ((t % 2) ? L::kColS1 : L::kColS0);
          const uint32_t kbase = sbase + L::kKOff + s * L::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t coff = (kk % 4) * 32;  // 16 bf16 = 32 bytes along K
            const uint64_t ad = smem_desc_sw128(sbase + L::kQOff + (kk / 4) * (BM * 128) + coff, 16, kSBO);
            const uint64_t bd = smem_desc_sw128(kbase + (kk / 4) * (kKeyTile * 128) + coff, 16, kSBO);
            mma_bf16_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar.s_full[t % 2]);
          mma_commit(&bar.k_empty[s]);
        }
        if (t >= 1) {  // ---- O += P_j V_j, j = t - 1
          const int j = t - 1;
          const int s = j % kStages, use = j / kStages;
          const int nk = tile_keys(j, bs, k);
          ok = mbar_wait(&bar.p_full[j % 2], (j / 2) & 1, abort_flag, 204);
          if (ok) ok = mbar_wait(&bar.v_full[s], use & 1, abort_flag, 205);
          if (!ok) break;
          tc_fence_after();
          const uint32_t pbase = sbase + L::kPOff + (j % 2) * L::kPBytes;
          const uint32_t vbase = sbase + L::kVOff + s * L::kKVBytes;
          for (int kk = 0; kk < nk / 16; ++kk) {
            const uint64_t ad =
                smem_desc_sw128(pbase + (kk / 4) * (BM * 128) + (kk % 4) * 32, 16, kSBO);
            // V tile is MN-major: next 16 key rows are 16 * 128 bytes further;
            // the leading offset steps between 64-column chunks of D.
            const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, kKeyTile * 128, kSBO);
            mma_bf16_ss(tmem + L::kColO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar.pv_done[j % 2]);
          mma_commit(&bar.v_empty[s]);
        }
      }
      // every MMA this thread issued has completed before teardown
      mma_commit(&bar.mma_drained);
      mbar_wait_teardown(&bar.mma_drained, 0);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax / epilogue
    const int quad = warp % 4;  // TMEM lane quadrant this warp may access
    const bool active = BM == 128 || lane < 16;
    const int row = BM == 128 ? quad * 32 + lane : quad * 16 + lane;  // row in the query tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int nk = tile_keys(j, bs, k);
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.s_full[j % 2], (j / 2) & 1, abort_flag, 301));
      if (!ok) break;
      tc_fence_after();
      // S row of this thread: sv[c][e] = column 32 c + e (chunks 2, 3 only when nk == 128)
      uint32_t sv[4][32];
      {
        const uint32_t scol = lane_base + ((j % 2) ? L::kColS1 : L::kColS0);
        tmem_ld32(scol, sv[0]);
        tmem_ld32(scol + 32, sv[1]);
        if (nk == 128) {
          tmem_ld32(scol + 64, sv[2]);
          tmem_ld32(scol + 96, sv[3]);
        }
        tmem_wait_ld();
      }
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fmaxf(__uint_as_float(sv[0][e]), __uint_as_float(sv[1][e])));
      if (nk == 128) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          mx = fmaxf(mx, fmaxf(__uint_as_float(sv[2][e]), __uint_as_float(sv[3][e])));
      }
      mx *= scale_log2;
      float m_new = m_run;
      if (j == 0 || mx > m_run + 8.0f) m_new = mx;
      const bool rescale = active && j > 0 && m_new != m_run;
      // P buffer j%2 was last read by PV_{j-2}
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.pv_done[j % 2], ((j - 2) / 2) & 1, abort_flag, 302));
        if (!ok) break;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar.pv_done[(j - 1) % 2], ((j - 1) / 2) & 1, abort_flag, 303));
        if (!ok) break;
        tc_fence_after();
        const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
        l_run *= alpha;
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const uint32_t ocol = lane_base + L::kColO + c * 32;
          tmem_ld32(ocol, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(ocol, r);
        }
        tmem_wait_st();
      }
      m_run = m_new;
      // P = exp2(S * scale_log2 - m) as bf16, K-major 128-byte-swizzled rows
      float psum = 0.f;
      const uint32_t prow = sbase + L::kPOff + (j % 2) * L::kPBytes + row * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (c == 1 && nk == 64) break;
#pragma unroll
        for (int u8 = 0; u8 < 8; ++u8) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = c * 64 + u8 * 8 + e;
            p[e] = fast_exp2(fmaf(__uint_as_float(sv[col / 32][col % 32]), scale_log2, -m_run));
            psum += p[e];
          }
          if (active)
            st_shared_v4(prow + c * (BM * 128) + ((u8 ^ (row & 7)) * 16), pack_bf16x2(p[0], p[1]),
                         pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
        }
      }
      l_run += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[j % 2]);
    }
    // ---- epilogue: O / l -> bf16 -> global
    if (ok && T > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.pv_done[(T - 1) % 2], ((T - 1) / 2) & 1, abort_flag, 304));
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const long n = static_cast<long>(i) * bs + part * BM + row;
      __nv_bfloat16* orow = o + ((static_cast<long>(b) * N + n) * H + h) * D;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(lane_base + L::kColO + c * 32, r);
        tmem_wait_ld();
        if (active) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv, __uint_as_float(r[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv, __uint_as_float(r[e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + e) = w;
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace bsa
