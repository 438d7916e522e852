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
//   * Warp 0 feeds shared memory with TMA: lane 0 loads the query tile and
//     gathers each key tile's K rows by block index, lane 1 gathers the V
//     rows, each into its own ring of stages (128-byte swizzled 64x64 boxes).
//   * Warp 1 (one lane) issues tcgen05.mma in the order S_0, S_1, PV_0, S_2,
//     PV_1, ...: S_t = Q K_t^T into one of two TMEM score buffers, and
//     O += P_j V_j with P read from TMEM and O accumulated in TMEM.
//   * Warps 2-9 (256 threads) run the online softmax. Two warps share a TMEM
//     lane quadrant (32 query rows): one takes key columns 0-63 of each tile,
//     the other 64-127. Per tile a thread reads its half row of S from TMEM,
//     publishes its partial row max to its partner, and -- unless its own
//     half already exceeds the running max by more than 8 -- computes
//     P = exp2(S * scale * log2 e - m) with the running max while the
//     partner's value arrives; only when the combined max grows by more than
//     8 (rare) is P recomputed and O in TMEM rescaled. A quarter of the
//     exponentials run as a polynomial on the FMA pipe to relieve the MUFU
//     unit. P is stored to TMEM as packed bf16 once the previous P.V product
//     has finished with it. At the end the partners add their row sums and
//     each normalises and stores half of the O row.
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

constexpr int kSoftmaxWarps = 8;
constexpr int kTcThreads = 64 + 32 * kSoftmaxWarps;  // TMA, MMA, 8 x softmax
constexpr int kKeyTile = 128;                        // key rows per tile
constexpr int kMaxStages = 6;

template <int D, int BM>
struct TcLayout {
  static constexpr int kStages = D == 128 ? 3 : 6;  // K (and V) ring depth
  static constexpr int kChunks = D / 64;           // 128-byte column chunks across D
  static constexpr uint32_t kQBytes = BM * D * 2;
  static constexpr uint32_t kKVBytes = kKeyTile * D * 2;  // one stage of K (or V)
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + kQBytes;
  static constexpr uint32_t kVOff = kKOff + kStages * kKVBytes;
  static constexpr uint32_t kRedOff = kVOff + kStages * kKVBytes;  // [2 parity][2 half][128] floats
  static constexpr uint32_t kBarOff = kRedOff + 2 * 2 * 128 * 4;
  static constexpr uint32_t kBytes = kBarOff + 512;
  static constexpr uint32_t kTmemCols = 512;  // S0 | S1 | O | P
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;
  static_assert(kStages <= kMaxStages, "stage count");
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(kColO + D <= kColP && kColP + 64 <= kTmemCols, "TMEM budget");
};

struct TcBarriers {
  uint64_t q_full;
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[2];
  uint64_t p_full;   // phase j: all softmax warps stored P_j (and finished any O rescale)
  uint64_t pv_done;  // phase j: O += P_j V_j completed
  uint64_t pair[4];  // per lane quadrant: both partner warps published their partial row data
  uint64_t mma_drained;
  uint32_t tmem_base;
  int abort;
  int kvalid;  // valid entries of the index row (at least 1)
};
static_assert(sizeof(TcBarriers) <= 512, "barrier area");

// Keys in key tile t (128, or 64 for the last tile of an odd k at block_size 64).
__device__ __forceinline__ int tile_keys(int t, int bs, int k) {
  return (bs == 64 && 2 * t + 1 >= k) ? 64 : 128;
}

__device__ __forceinline__ int clamp_block(int blk, int nb) {
  return blk < 0 ? 0 : (blk >= nb ? nb - 1 : blk);
}

// First token row of 64-row half `half` of key tile t.
__device__ __forceinline__ int half_row0(const int32_t* sel, int t, int half, int bs, int nb) {
  if (bs == 64) return clamp_block(__ldg(sel + 2 * t + half), nb) * 64;
  if (bs == 128) return clamp_block(__ldg(sel + t), nb) * 128 + half * 64;
  return clamp_block(__ldg(sel + t / 2), nb) * 256 + (t % 2) * 128 + half * 64;  // bs == 256
}

// P = exp2(s * scale_log2 - m) for this thread's 64 scores, packed as bf16
// pairs (low half = even key), and their float32 sum.
__device__ __forceinline__ void softmax_exps(const uint32_t (&sv)[2][32], float scale_log2, float m,
                                             uint32_t (&pk)[32], float& psum) {
  float ps[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) ps[e] = 0.f;
#pragma unroll
  for (int e = 0; e < 64; e += 2) {
    const float x0 = fmaf(__uint_as_float(sv[e / 32][e % 32]), scale_log2, -m);
    const float x1 = fmaf(__uint_as_float(sv[e / 32][e % 32 + 1]), scale_log2, -m);
    float p0, p1;
    if ((e / 2) % 4 == 3) {  // one pair in four on the FMA pipe
      p0 = exp2_poly(x0);
      p1 = exp2_poly(x1);
    } else {
      p0 = fast_exp2(x0);
      p1 = fast_exp2(x1);
    }
    ps[(e / 2) % 8] += p0 + p1;
    pk[e / 2] = pack_bf16x2(p0, p1);
  }
  psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
}

// grid.x = B * H * nb * parts, parts = max(1, bs / BM).
template <int D, int BM>
__global__ void __launch_bounds__(kTcThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, int N,
                          int H, int Hkv, int bs, int k, float scale_log2, unsigned flags) {
  using L = TcLayout<D, BM>;
  constexpr int KS = L::kStages;
  extern __shared__ __align__(1024) unsigned char tc_raw[];
  // The swizzled operand tiles need 1024-byte alignment; the layout uses the
  // whole shared-memory budget, so there is no slack to realign: refuse to
  // run (before touching any barrier or TMEM) if the base is not aligned.
  if ((smem_u32(tc_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(401);
    return;
  }
  unsigned char* smem = tc_raw;
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
  const int g = h / (H / Hkv);  // key/value head (and selection) of query head h
  const int32_t* sel = idx + ((static_cast<long>(b) * Hkv + g) * nb + i) * k;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    mbar_init(&bar.s_full[0], 1);
    mbar_init(&bar.s_full[1], 1);
    mbar_init(&bar.p_full, kSoftmaxWarps);
    mbar_init(&bar.pv_done, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bar.pair[q], 64);
    mbar_init(&bar.mma_drained, 1);
    bar.abort = 0;
    // a row lists its blocks, then pads with -1; a row of only -1 reads block 0
    bar.kvalid = max(index_row_valid(sel, k), 1);
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
  const int kv = bar.kvalid;
  const int T = bs == 64 ? (kv + 1) / 2 : (bs == 128 ? kv : 2 * kv);  // key tiles

  if (warp == 0) {
    // ============================================================ TMA producers
    // lane 0: query tile and K ring; lane 1: V ring
    if (lane < 2) {
      const uint64_t keep = policy_evict_last();  // gathered K/V: reused across query blocks
      const bool is_k = lane == 0;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint64_t* full = is_k ? bar.k_full : bar.v_full;
      uint64_t* empty = is_k ? bar.k_empty : bar.v_empty;
      const uint32_t ring = is_k ? L::kKOff : L::kVOff;
      int issued[kMaxStages];
      for (int s = 0; s < KS; ++s) issued[s] = 0;
      bool ok = true;
      if (is_k) {
        const uint64_t stream = policy_evict_first();  // query tile: read once
        mbar_arrive_expect_tx(&bar.q_full, L::kQBytes);
        const int qrow0 = i * bs + part * BM;
        for (int hh = 0; hh < BM / 64; ++hh)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + L::kQOff + c * (BM * 128) + hh * 64 * 128, &tm_q, &bar.q_full,
                        c * 64, h, qrow0 + hh * 64, b, stream);
      }
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % KS, use = t / KS;
        const int halves = tile_keys(t, bs, kv) / 64;
        int row0[2];
        for (int hf = 0; hf < halves; ++hf) row0[hf] = half_row0(sel, t, hf, bs, nb);
        if (t >= KS) ok = mbar_wait(&empty[s], (use - 1) & 1, abort_flag, is_k ? 101 : 102);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[s], halves * 64 * D * 2);
        for (int hf = 0; hf < halves; ++hf)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + ring + s * L::kKVBytes + c * (kKeyTile * 128) + hf * 64 * 128, map,
                        &full[s], c * 64, g, row0[hf], b, keep);
        issued[s] = use + 1;
      }
      // drain: every copy this thread issued has landed before teardown
      if (is_k) mbar_wait_teardown(&bar.q_full, 0);
      for (int s = 0; s < KS; ++s)
        if (issued[s]) mbar_wait_teardown(&full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    // S_t reuses the TMEM score buffer of S_{t-2}, whose softmax finished
    // before PV_{t-2} (issued earlier in this order) was issued.
    if (lane == 0) {
      constexpr uint32_t kSBO = 1024;  // 8 rows x 128 bytes
      const uint32_t idesc_pv = idesc_bf16_f32(BM, D, 0, 1);  // P from TMEM, V MN-major
      bool ok = mbar_wait(&bar.q_full, 0, abort_flag, 201);
      for (int t = 0; t <= T && ok; ++t) {
        if (t < T) {  // ---- S_t = Q K_t^T
          const int s = t % KS, use = t / KS;
          const int nk = tile_keys(t, bs, kv);
          ok = mbar_wait(&bar.k_full[s], use & 1, abort_flag, 202);
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
          const int s = j % KS, use = j / KS;
          const int nk = tile_keys(j, bs, kv);
          ok = mbar_wait(&bar.p_full, j & 1, abort_flag, 204);
          if (ok) ok = mbar_wait(&bar.v_full[s], use & 1, abort_flag, 205);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vbase = sbase + L::kVOff + s * L::kKVBytes;
          for (int kk = 0; kk < nk / 16; ++kk) {
            // V tile is MN-major: next 16 key rows are 16 * 128 bytes further;
            // the leading offset steps between 64-column chunks of D.
            const uint64_t bd = smem_desc_sw128(vbase + kk * 16 * 128, kKeyTile * 128, kSBO);
            mma_bf16_ts(tmem + L::kColO, tmem + L::kColP + kk * 8, bd, idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar.pv_done);
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
    const int sw = warp - 2;    // 0..7
    const int quad = warp % 4;  // TMEM lane quadrant this warp may access
    const int half = sw / 4;    // key columns [64 half, 64 half + 64) of each tile
    const bool active = BM == 128 || lane < 16;
    const int row = BM == 128 ? quad * 32 + lane : quad * 16 + lane;  // row in the query tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    // partial-row exchange slots [parity][half][quad * 32 + lane]: indexed by
    // thread, not by row, because the idle lanes of an M = 64 tile would alias
    // rows of the next quadrant
    float* red = reinterpret_cast<float*>(smem + L::kRedOff);
    const int slot = quad * 32 + lane;
    uint64_t* pair = &bar.pair[quad];
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const bool has = half == 0 || tile_keys(j, bs, kv) == 128;  // this half holds keys
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.s_full[j % 2], (j / 2) & 1, abort_flag, 301));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][32];  // this thread's 64 scores of the tile
      float mx = -INFINITY;
      if (has) {
        const uint32_t scol = lane_base + ((j % 2) ? L::kColS1 : L::kColS0) + half * 64;
        tmem_ld32(scol, sv[0]);
        tmem_ld32(scol + 32, sv[1]);
        tmem_wait_ld();
        if (flags & kFlagCausal) {
          // key c of this half is token kbase + c; keys after the thread's
          // query token (c > lim) are left out (only the diagonal block)
          const int kbase = half_row0(sel, j, half, bs, nb);
          const int lim = i * bs + part * BM + row - kbase;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (e > lim) sv[0][e] = __float_as_uint(-INFINITY);
            if (e + 32 > lim) sv[1][e] = __float_as_uint(-INFINITY);
          }
        }
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = fmaxf(__uint_as_float(sv[0][e]), __uint_as_float(sv[1][e]));
#pragma unroll
        for (int e = 8; e < 32; ++e)
          m8[e % 8] = fmaxf(m8[e % 8], fmaxf(__uint_as_float(sv[0][e]), __uint_as_float(sv[1][e])));
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      // publish the partial row max; meanwhile exponentiate with the running
      // max unless this half alone already moves it
      red[((j & 1) * 2 + half) * 128 + slot] = mx;
      mbar_arrive(pair);
      uint32_t pk[32];
      float psum = 0.f;
      bool have = false;
      if (has && j > 0 && mx * scale_log2 <= m_run + 8.0f) {
        softmax_exps(sv, scale_log2, m_run, pk, psum);
        have = true;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(pair, j & 1, abort_flag, 305));
      if (!ok) break;
      const float mt = fmaxf(mx, red[((j & 1) * 2 + (half ^ 1)) * 128 + slot]) * scale_log2;
      const float m_new = (j == 0 || mt > m_run + 8.0f) ? mt : m_run;
      if (has && (!have || m_new != m_run)) softmax_exps(sv, scale_log2, m_new, pk, psum);
      const bool rescale = active && j > 0 && m_new != m_run;
      // PV_{j-1} done: the TMEM P columns are free and O holds every earlier tile
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.pv_done, (j - 1) & 1, abort_flag, 302));
        if (!ok) break;
      }
      tc_fence_after();
      if (has) tmem_st32(lane_base + L::kColP + half * 32, pk);  // keys 64 half .. 64 half + 63
      if (__any_sync(0xffffffffu, rescale)) {
        const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
        l_run *= alpha;
        // rare path: keep its register footprint small
        uint32_t r[16];
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          const uint32_t ocol = lane_base + L::kColO + half * (D / 2) + c * 16;
          tmem_ld16(ocol, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(ocol, r);
        }
      }
      tmem_wait_st();
      m_run = m_new;
      l_run += psum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full);
    }
    // ---- epilogue: O / (l_half0 + l_half1) -> bf16 -> global, half the columns each
    if (ok && T > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.pv_done, (T - 1) & 1, abort_flag, 304));
    if (ok) {
      red[((T & 1) * 2 + half) * 128 + slot] = l_run;
      mbar_arrive(pair);
      ok = __all_sync(0xffffffffu, mbar_wait(pair, T & 1, abort_flag, 306));
    }
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / (l_run + red[((T & 1) * 2 + (half ^ 1)) * 128 + slot]);
      const long n = static_cast<long>(i) * bs + part * BM + row;
      __nv_bfloat16* orow = o + ((static_cast<long>(b) * N + n) * H + h) * D + half * (D / 2);
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tmem_ld32(lane_base + L::kColO + half * (D / 2) + c * 32, r);
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
