// bwd.cuh -- backward pass of the attention over the kept blocks.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现": step 2 keeps key blocks with torch.topk, whose
// indices carry no gradient, so the gradients are those of step 3 (the
// attention over the kept blocks, "从M2.7到M3" §2.1 Softmax(Mask(QK^T/sqrt(d_k)))V)
// with the index lists held fixed. Per query token n and kept key token t:
//   p = exp(scale q.k - lse_n), D_n = dO_n . o_n, dP = dO_n . v_t,
//   dS = p (dP - D_n), dq_n = scale sum_t dS k_t,
//   dk_t = scale sum_n dS q_n, dv_t = sum_n p dO_n.
// The forward leaves lse (ln of each row's softmax denominator).
//
// Kernels:
//  * bwd_mask_kernel: the transpose of the selection as a bit matrix
//    [B, H, nb, ceil(nb / 32)] (bit i of row j: query block i kept key
//    block j); deterministic (atomicOr of bits).
//  * bwd_rowdot_kernel: D_n = dO_n . o_n in float32.
//  * bwd_dq_kernel: one CTA per 128-row query tile walks its kept key tiles:
//    S = Q K^T and dP = dO V^T (tcgen05, TMEM), then dS (bf16, over S in
//    TMEM) and dQ += dS K; dQ accumulates in TMEM.
//  * bwd_dkdv_kernel: one CTA per 128-key tile walks the query tiles that
//    kept its block (the bit row): S^T = K Q^T and dP^T = V dO^T, then P^T
//    and dS^T (bf16 over S^T and dP^T) and dV += P^T dO, dK += dS^T Q; all
//    four products and both accumulators live in TMEM (512 columns).
// Each CTA has a TMA producer warp, an MMA warp (one issuing thread) and four
// compute warps (one row per thread); every wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kBwdThreads = 192;  // producer warp, MMA warp, 4 compute warps

// ---------------------------------------------------------------- transpose
// grid.x = ceil(B * H * nb * k / 256)
__global__ void bwd_mask_kernel(const int32_t* __restrict__ idx, uint32_t* __restrict__ mask,
                                long entries, int nb, int k, int words) {
  const long e = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= entries) return;
  const int j = __ldg(idx + e);
  if (j < 0 || j >= nb) return;
  const long row = e / k;                   // (b, h, i)
  const int i = static_cast<int>(row % nb);
  const long bh = row / nb;
  atomicOr(mask + (bh * nb + j) * words + i / 32, 1u << (i % 32));
}

// ---------------------------------------------------------------- D_n
// One warp per row: D_n = sum_d dO[n, d] * o[n, d] (bf16 inputs, float32 sum),
// written to dsum [B, H, N]. grid.x = ceil(B * N * H / 8), 256 threads.
__global__ void bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                                  float* __restrict__ dsum, long rows, int N, int H, int D) {
  const long r = static_cast<long>(blockIdx.x) * 8 + threadIdx.x / 32;  // (b, n, h) row of [B, N, H, D]
  const int lane = threadIdx.x % 32;
  if (r >= rows) return;
  float acc = 0.f;
  for (int d = lane * 2; d < D; d += 64) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(o + r * D + d);
    const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162*>(dO + r * D + d);
    acc = fmaf(__low2float(a), __low2float(g), acc);
    acc = fmaf(__high2float(a), __high2float(g), acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int h = static_cast<int>(r % H);
    const long bn = r / H;
    const int n = static_cast<int>(bn % N);
    const long b = bn / N;
    dsum[(b * H + h) * N + n] = acc;
  }
}

// ---------------------------------------------------------------- shared pieces
template <int D>
struct BwdLayout {
  static constexpr uint32_t kTile = 128 * D * 2;  // a 128-row bf16 tile
  static constexpr int kChunks = D / 64;          // 128-byte column chunks
  static constexpr int kXStages = 3, kYStages = 2;
  static constexpr uint32_t kOffA = 0;                           // dq: Q, dO     dkdv: K, V
  static constexpr uint32_t kOffX = 2 * kTile;                   // dq: K ring    dkdv: Q ring
  static constexpr uint32_t kOffY = kOffX + kXStages * kTile;    // dq: V ring    dkdv: dO ring
  static constexpr uint32_t kBarOff = kOffY + kYStages * kTile;
  static constexpr uint32_t kStatOff = kBarOff + 256;  // dkdv: float [2 tiles][lse2, D][128 queries]
  static constexpr uint32_t kBytes = kStatOff + 2 * 2 * 128 * 4;
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Ring X holds the operand each tile reads twice, first by the score-like
// product issued a tile ahead and last by the accumulating product (dq: K;
// dkdv: Q), so it is three deep; ring Y (dq: V; dkdv: dO) is two deep.
struct BwdBarriers {
  uint64_t a_full;          // the two resident tiles
  uint64_t x_full[3], x_empty[3];
  uint64_t y_full[2], y_empty[2];
  uint64_t prod_full;       // phase t: both score-like products of tile t done
  uint64_t s_loaded;        // phase t: the compute warps hold tile t's S (dkdv: S^T)
  uint64_t p_loaded;        // dq, phase t: the compute warps hold tile t's dP
  uint64_t soft_full;       // phase t: tile t's bf16 operands stored
  uint64_t half_full;       // dkdv, phase t: the operands of tile t's first 64 queries stored
  uint64_t stats_ready[2];  // dkdv, tile t's query statistics in shared memory (slot t % 2)
  uint64_t acc_free;        // dq, phase t: dQ += dS(t) K(t) done, the dS columns are free
  uint64_t done;            // the last accumulating products done
  uint64_t drained;
  uint32_t tmem_base;
  int abort;
  int tiles;   // key tiles (dq) or query tiles (dkdv) this CTA walks
  int blocks;  // dkdv: query blocks that kept this key block (per query head of the group)
  int half[2];  // block_size 64: valid key blocks (dq) or keeping query blocks (dkdv) of each stacked block
};
static_assert(sizeof(BwdBarriers) <= 256, "barrier area");

// First token row of 64-row half hf of tile t of a row of kept blocks:
// block sel[t / tpb], 128-row part t % tpb.
__device__ __forceinline__ int bwd_tile_row(const int32_t* sel, int t, int hf, int bs, int nb) {
  const int tpb = bs / 128;
  int blk = __ldg(sel + t / tpb);
  blk = blk < 0 ? 0 : (blk >= nb ? nb - 1 : blk);
  return blk * bs + (t % tpb) * 128 + hf * 64;
}

// Loads one 128-row tile (two 64-row boxes per 128-byte chunk) at token row
// `row` of head h, batch b into `dst`, completing on `bar`.
template <int D>
__device__ __forceinline__ void bwd_load_tile(unsigned char* dst, const CUtensorMap* map, uint64_t* bar,
                                              int h, int row, int b, uint64_t policy) {
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int c = 0; c < BwdLayout<D>::kChunks; ++c)
      tma_load_4d(dst + c * (128 * 128) + hf * 64 * 128, map, bar, c * 64, h, row + hf * 64, b, policy);
}

// The same tile from two 64-row pieces at token rows row0 (rows 0-63) and
// row1 (rows 64-127): block_size 64 stacks two blocks in one tile.
template <int D>
__device__ __forceinline__ void bwd_load_tile2(unsigned char* dst, const CUtensorMap* map, uint64_t* bar,
                                               int h, int row0, int row1, int b, uint64_t policy) {
#pragma unroll
  for (int hf = 0; hf < 2; ++hf)
#pragma unroll
    for (int c = 0; c < BwdLayout<D>::kChunks; ++c)
      tma_load_4d(dst + c * (128 * 128) + hf * 64 * 128, map, bar, c * 64, h, hf == 0 ? row0 : row1, b, policy);
}

// Key block of entry t of an index row (-1 padding reads block 0).
__device__ __forceinline__ int bwd_entry_block(const int32_t* sel, int t, int nb) {
  const int blk = __ldg(sel + t);
  return blk < 0 ? 0 : (blk >= nb ? nb - 1 : blk);
}

// 32 bf16 pairs of a row chunk to 16 packed words.
__device__ __forceinline__ void bwd_pack16(const float (&v)[32], uint32_t (&w)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
}

// ---------------------------------------------------------------- dQ
// grid.x = B * H * nb * (bs / 128): one CTA per 128-row query tile, which
// walks the key tiles of its query block's kept blocks.
// kStack (block_size 64): grid.x = B * H * ceil(nb / 2); the 128-row tile
// stacks query blocks 2u (rows 0-63) and 2u + 1 (rows 64-127, absent when
// 2u + 1 = nb), and key tile t stacks the t-th kept block of each (keys
// 0-63, 64-127), as in the forward. Rows see only their own block's 64 key
// columns (and none once their list has ended), so dS is zero on the other
// quadrants and dQ += dS K sums each row's own keys only.
// TMEM: S [0, 128), dP [128, 256), dQ [256, 256 + D), dS (bf16) [384, 448).
// dS has columns of its own, so the products of tile t+1 need only wait
// until the compute warps have read tile t's S and dP into registers: dP(t+1)
// runs while tile t's dS is being computed, S(t+1) right after its last S
// load, and dQ += dS(t) K(t) after them.
template <int D, bool kCausal, bool kStack = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const int32_t* __restrict__ idx, const float* __restrict__ lse,
                  const float* __restrict__ dsum, __nv_bfloat16* __restrict__ dq, int N, int H, int Hkv,
                  int bs, int k, float scale, float scale_log2) {
  using L = BwdLayout<D>;
  extern __shared__ __align__(1024) unsigned char bwd_raw[];
  if ((smem_u32(bwd_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(701);
    return;
  }
  unsigned char* smem = bwd_raw;
  BwdBarriers& bar = *reinterpret_cast<BwdBarriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;
  constexpr uint32_t kColS = 0, kColP = 128, kColQ = 256, kColDS = 384;
  constexpr int XS = L::kXStages, YS = L::kYStages;

  const int nb = N / bs, tpb = kStack ? 1 : bs / 128;
  long u = blockIdx.x;
  int part = 0, i;
  if (kStack) {
    const int per = (nb + 1) / 2;
    i = 2 * static_cast<int>(u % per);  // blocks i and i + 1
    u /= per;
  } else {
    part = static_cast<int>(u % tpb);
    u /= tpb;
    i = static_cast<int>(u % nb);
    u /= nb;
  }
  const int h = static_cast<int>(u % H);
  const int b = static_cast<int>(u / H);
  const long bh = static_cast<long>(b) * H + h;
  const int g = h / (H / Hkv);  // the key/value head (and selection) of query head h
  const int qrow0 = kStack ? i * 64 : i * bs + part * 128;
  const bool second = kStack && i + 1 < nb;  // the stacked second block exists
  const int32_t* sel = idx + ((static_cast<long>(b) * Hkv + g) * nb + i) * k;
  const int32_t* sel1 = second ? sel + k : sel;  // kStack: the index row of block i + 1
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bar.a_full, 1);
    for (int s = 0; s < XS; ++s) {
      mbar_init(&bar.x_full[s], 1);
      mbar_init(&bar.x_empty[s], 1);
    }
    for (int s = 0; s < YS; ++s) {
      mbar_init(&bar.y_full[s], 1);
      mbar_init(&bar.y_empty[s], 1);
    }
    mbar_init(&bar.prod_full, 1);
    mbar_init(&bar.s_loaded, 4);
    mbar_init(&bar.p_loaded, 4);
    mbar_init(&bar.soft_full, 4);
    mbar_init(&bar.acc_free, 1);
    mbar_init(&bar.done, 1);
    mbar_init(&bar.drained, 1);
    bar.abort = 0;
    if (kStack) {
      bar.half[0] = max(index_row_valid(sel, k), 1);
      bar.half[1] = second ? max(index_row_valid(sel1, k), 1) : 0;
      bar.tiles = max(bar.half[0], bar.half[1]);
    } else {
      bar.tiles = max(index_row_valid(sel, k), 1) * tpb;  // a row of only -1 reads block 0
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int T = bar.tiles;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    // ============================================================ TMA producers
    // lane 0: Q and dO, then the K ring; lane 1: the V ring
    if (lane < 2) {
      const bool is_x = lane == 0;
      const int S = is_x ? XS : YS;
      uint64_t* full = is_x ? bar.x_full : bar.y_full;
      uint64_t* empty = is_x ? bar.x_empty : bar.y_empty;
      const uint32_t ring = is_x ? L::kOffX : L::kOffY;
      const CUtensorMap* map = is_x ? &tm_k : &tm_v;
      const uint64_t keep = policy_evict_last();
      if (is_x) {
        const uint64_t stream = policy_evict_first();
        mbar_arrive_expect_tx(&bar.a_full, 2 * L::kTile);
        bwd_load_tile<D>(smem + L::kOffA, &tm_q, &bar.a_full, h, qrow0, b, stream);
        bwd_load_tile<D>(smem + L::kOffA + L::kTile, &tm_do, &bar.a_full, h, qrow0, b, stream);
      }
      int issued[XS] = {};
      bool ok = true;
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % S, use = t / S;
        if (t >= S) ok = mbar_wait(&empty[s], (use - 1) & 1, abort_flag, is_x ? 711 : 712);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[s], L::kTile);
        if (kStack)  // entries past a list's end read block 0 (their columns are masked)
          bwd_load_tile2<D>(smem + ring + s * L::kTile, map, &full[s], g, bwd_entry_block(sel, t, nb) * 64,
                            bwd_entry_block(sel1, t, nb) * 64, b, keep);
        else
          bwd_load_tile<D>(smem + ring + s * L::kTile, map, &full[s], g, bwd_tile_row(sel, t, 0, bs, nb), b, keep);
        issued[s] = use + 1;
      }
      if (is_x) mbar_wait_teardown(&bar.a_full, 0);
      for (int s = 0; s < S; ++s)
        if (issued[s]) mbar_wait_teardown(&full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_q = idesc_bf16_f32(128, D, 0, 1);  // dS from TMEM, K used MN-major
      const uint64_t dqd = smem_desc_sw128(sbase + L::kOffA, 16, 1024);
      const uint64_t ddo = smem_desc_sw128(sbase + L::kOffA + L::kTile, 16, 1024);
      const uint64_t dx = smem_desc_sw128(sbase + L::kOffX, 16, 1024);              // K, K-major
      const uint64_t dx_mn = smem_desc_sw128(sbase + L::kOffX, 128 * 128, 1024);    // K, MN-major
      const uint64_t dy = smem_desc_sw128(sbase + L::kOffY, 16, 1024);              // V, K-major
      constexpr uint64_t kStep = L::kTile >> 4;
      bool ok = mbar_wait(&bar.a_full, 0, abort_flag, 721);
      // dP(t) = dO V(t)^T; frees its V ring entry when done
      auto issue_dp = [&](int t) {
        ok = ok && mbar_wait(&bar.y_full[t % YS], (t / YS) & 1, abort_flag, 723);
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
          mma_bf16_ss(tmem + kColP, ddo + off, dy + (t % YS) * kStep + off, id_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.y_empty[t % YS]);
      };
      // S(t) = Q K(t)^T
      auto issue_s = [&](int t) {
        ok = ok && mbar_wait(&bar.x_full[t % XS], (t / XS) & 1, abort_flag, 724);
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
          mma_bf16_ss(tmem + kColS, dqd + off, dx + (t % XS) * kStep + off, id_s, kk > 0 ? 1u : 0u);
        }
      };
      if (T > 0) {
        issue_dp(0);
        issue_s(0);
        if (ok) mma_commit(&bar.prod_full);
      }
      for (int t = 0; t < T && ok; ++t) {
        if (t + 1 < T) {
          // tile t+1's products overwrite S and dP once the compute warps hold them
          ok = mbar_wait(&bar.p_loaded, t & 1, abort_flag, 725);
          issue_dp(t + 1);
          ok = ok && mbar_wait(&bar.s_loaded, t & 1, abort_flag, 726);
          issue_s(t + 1);
          if (!ok) break;
          mma_commit(&bar.prod_full);
        }
        // dQ += dS(t) K(t)
        ok = mbar_wait(&bar.soft_full, t & 1, abort_flag, 722);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + kColQ, tmem + kColDS + kk * 8, dx_mn + (t % XS) * kStep + ((kk * 16 * 128) >> 4), id_q,
                      (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar.x_empty[t % XS]);
        mma_commit(&bar.acc_free);
      }
      if (ok) mma_commit(&bar.done);
      mma_commit(&bar.drained);
      mbar_wait_teardown(&bar.drained, 0);
    }
    __syncwarp();
  } else {
    // ============================================================ dS, then the dQ epilogue
    const int quad = warp % 4;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const long n = qrow0 + row;
    // kStack: rows 64 hq.. belong to stacked block hq; an absent block's rows are skipped
    const int hq = kStack ? row / 64 : 0;
    const bool live = !kStack || hq == 0 || second;
    const float lse2 = live ? __ldg(lse + bh * N + n) * 1.4426950408889634f : 0.f;  // log2 units
    const float dn = live ? __ldg(dsum + bh * N + n) : 0.f;
    const int vt = kStack ? (live ? bar.half[hq] : 0) : T;  // tiles holding keys of this row
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.prod_full, t & 1, abort_flag, 731));
      if (!ok) break;
      tc_fence_after();
      // the row's key columns of this tile are [clo, lim]: keys c with
      // kbase + c > n are masked (causal); kStack: only the row's own block's
      // 64 columns, none past the end of its list
      int clo = 0, lim = 1 << 30;
      if (kStack) {
        clo = 64 * hq;
        lim = t < vt ? clo + 63 : -1;
        if (kCausal && t < vt)
          lim = min(lim, static_cast<int>(n - bwd_entry_block(hq == 0 ? sel : sel1, t, nb) * 64) + clo);
      } else if (kCausal) {
        lim = static_cast<int>(n - bwd_tile_row(sel, t, 0, bs, nb));
      }
      // the whole dP row, then the tensor core may overwrite it
      uint32_t p0[32], p1[32], p2[32], p3[32];
      tmem_ld32(lane_base + kColP, p0);
      tmem_ld32(lane_base + kColP + 32, p1);
      tmem_ld32(lane_base + kColP + 64, p2);
      tmem_ld32(lane_base + kColP + 96, p3);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_loaded);
      // S in 32-column pieces; dS packed to bf16 as it is made
      uint32_t w0[16], w1[16], w2[16], w3[16];
      auto piece = [&](int c, const uint32_t (&pv)[32], uint32_t (&w)[16]) {
        uint32_t sv[32];
        tmem_ld32(lane_base + kColS + c * 32, sv);
        tmem_wait_ld();
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.s_loaded);
        }
        float ds[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = c * 32 + e;
          const float p =
              (col > lim || col < clo) ? 0.f : fast_exp2(fmaf(__uint_as_float(sv[e]), scale_log2, -lse2));
          ds[e] = p * (__uint_as_float(pv[e]) - dn);
        }
        bwd_pack16(ds, w);
      };
      piece(0, p0, w0);
      piece(1, p1, w1);
      piece(2, p2, w2);
      piece(3, p3, w3);
      // the dS columns are free once dQ(t-1) has read them
      if (t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar.acc_free, (t - 1) & 1, abort_flag, 733));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st16(lane_base + kColDS, w0);
      tmem_st16(lane_base + kColDS + 16, w1);
      tmem_st16(lane_base + kColDS + 32, w2);
      tmem_st16(lane_base + kColDS + 48, w3);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.soft_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.done, 0, abort_flag, 732));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* out = dq + ((static_cast<long>(b) * N + (live ? n : 0)) * H + h) * D;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(lane_base + kColQ + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w4;
          w4.x = pack_bf16x2(__uint_as_float(r[e]) * scale, __uint_as_float(r[e + 1]) * scale);
          w4.y = pack_bf16x2(__uint_as_float(r[e + 2]) * scale, __uint_as_float(r[e + 3]) * scale);
          w4.z = pack_bf16x2(__uint_as_float(r[e + 4]) * scale, __uint_as_float(r[e + 5]) * scale);
          w4.w = pack_bf16x2(__uint_as_float(r[e + 6]) * scale, __uint_as_float(r[e + 7]) * scale);
          if (live) *reinterpret_cast<uint4*>(out + c * 32 + e) = w4;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
// Query block of the u-th query tile of a bit row (tpb tiles per block):
// walks the set bits in ascending order. `w` and `cur` carry the position.
__device__ __forceinline__ int bwd_next_block(const uint32_t* row, int words, int& w, uint32_t& cur) {
  while (cur == 0 && w + 1 < words) cur = __ldg(row + ++w);
  const int i = w * 32 + __ffs(cur) - 1;
  cur &= cur - 1;
  return i;
}

// grid.x = B * Hkv * nb * (bs / 128): one CTA per 128-key tile of key/value
// head g, which walks, for each of the G = H / Hkv query heads of its group in
// turn, the query tiles of the query blocks that kept its block (bit row of
// `mask`, one per key/value head: the group shares its selection).
// TMEM: S^T [0, 128), dP^T [128, 256), dV [256, 256 + D), dK [256 + D, 256 + 2D).
// The compute warps read the whole S^T row first, so S^T(t+1) is computed
// while tile t's P^T and dS^T are made; those go over dP^T, 32-query piece
// c at columns 128 + 32c: P^T in its first 16 columns, dS^T in the last 16
// (each piece is read before it is overwritten).
// kStack (block_size 64): grid.x = B * Hkv * ceil(nb / 2); the 128-key tile
// stacks key blocks 2u (keys 0-63) and 2u + 1 (keys 64-127, absent when
// 2u + 1 = nb), and query tile t stacks the t-th query block that kept each
// (queries 0-63, 64-127), so S^T is used on its diagonal quadrants only:
// a key row sees only its own block's 64 query columns, none once its bit
// row is exhausted, and P^T and dS^T are zero elsewhere.
template <int D, bool kCausal, bool kStack = false>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const uint32_t* __restrict__ mask, const float* __restrict__ lse,
                    const float* __restrict__ dsum, __nv_bfloat16* __restrict__ dk,
                    __nv_bfloat16* __restrict__ dv, int N, int H, int Hkv, int bs, float scale,
                    float scale_log2) {
  using L = BwdLayout<D>;
  static_assert(256 + 2 * D <= 512, "TMEM columns");
  extern __shared__ __align__(1024) unsigned char bwd_raw[];
  if ((smem_u32(bwd_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(702);
    return;
  }
  unsigned char* smem = bwd_raw;
  BwdBarriers& bar = *reinterpret_cast<BwdBarriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;
  constexpr uint32_t kColS = 0, kColP = 128, kColV = 256, kColK = 256 + D;
  constexpr int XS = L::kXStages, YS = L::kYStages;

  const int nb = N / bs, tpb = kStack ? 1 : bs / 128, words = (nb + 31) / 32;
  long u = blockIdx.x;
  int part = 0, j;
  if (kStack) {
    const int per = (nb + 1) / 2;
    j = 2 * static_cast<int>(u % per);  // key blocks j and j + 1
    u /= per;
  } else {
    part = static_cast<int>(u % tpb);
    u /= tpb;
    j = static_cast<int>(u % nb);
    u /= nb;
  }
  const int g = static_cast<int>(u % Hkv);
  const int b = static_cast<int>(u / Hkv);
  const int G = H / Hkv;
  const int krow0 = kStack ? j * 64 : j * bs + part * 128;  // first key token of this tile
  const bool second = kStack && j + 1 < nb;                  // the stacked second key block exists
  const uint32_t* mrow = mask + ((static_cast<long>(b) * Hkv + g) * nb + j) * words;
  const uint32_t* mrow1 = second ? mrow + words : mrow;      // kStack: the bit row of key block j + 1
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bar.a_full, 1);
    for (int s = 0; s < XS; ++s) {
      mbar_init(&bar.x_full[s], 1);
      mbar_init(&bar.x_empty[s], 1);
    }
    for (int s = 0; s < YS; ++s) {
      mbar_init(&bar.y_full[s], 1);
      mbar_init(&bar.y_empty[s], 1);
    }
    mbar_init(&bar.prod_full, 1);
    mbar_init(&bar.s_loaded, 4);
    mbar_init(&bar.soft_full, 4);
    mbar_init(&bar.half_full, 4);
    for (int s = 0; s < 2; ++s) mbar_init(&bar.stats_ready[s], 4);
    mbar_init(&bar.done, 1);
    mbar_init(&bar.drained, 1);
    bar.abort = 0;
    int blocks = 0;
    for (int w = 0; w < words; ++w) blocks += __popc(__ldg(mrow + w));
    if (kStack) {
      int blocks1 = 0;
      if (second)
        for (int w = 0; w < words; ++w) blocks1 += __popc(__ldg(mrow1 + w));
      bar.half[0] = blocks;
      bar.half[1] = blocks1;
      blocks = max(blocks, blocks1);  // query tiles per query head
    }
    bar.blocks = blocks;
    bar.tiles = G * blocks * tpb;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int U = bar.tiles, UB = bar.blocks * tpb;  // tiles in all, tiles per query head
  const int H0 = kStack ? bar.half[0] : 0, H1 = kStack ? bar.half[1] : 0;
  const uint32_t sbase = smem_u32(smem);
  // Tile t is query tile t % UB of query head g * G + t / UB; the bit row is
  // walked again for each query head.
  auto walk = [&](int t, int& w, uint32_t& cur, int& qb, int& hq) {
    const int tt = t % UB;
    if (tt == 0) {
      w = 0;
      cur = __ldg(mrow);
      hq = g * G + t / UB;
    }
    if (tt % tpb == 0) qb = bwd_next_block(mrow, words, w, cur);
    return qb * bs + (tt % tpb) * 128;  // first query token of the tile
  };
  // kStack: both bit rows walked side by side; a row already exhausted keeps
  // query block 0 (its columns are masked). Returns the tile's query blocks
  // of the two halves (qb0 for keys 0-63, qb1 for keys 64-127).
  auto walk2 = [&](int t, int (&w2)[2], uint32_t (&cur2)[2], int (&qb2)[2], int& hq) {
    const int tt = t % UB;
    if (tt == 0) {
      w2[0] = w2[1] = 0;
      cur2[0] = __ldg(mrow);
      cur2[1] = __ldg(mrow1);
      hq = g * G + t / UB;
    }
    qb2[0] = tt < H0 ? bwd_next_block(mrow, words, w2[0], cur2[0]) : 0;
    qb2[1] = tt < H1 ? bwd_next_block(mrow1, words, w2[1], cur2[1]) : 0;
  };

  if (warp == 0) {
    // ============================================================ TMA producers
    // lane 0: K and V, then the Q ring; lane 1: the dO ring
    if (lane < 2 && U > 0) {
      const bool is_x = lane == 0;
      const int S = is_x ? XS : YS;
      uint64_t* full = is_x ? bar.x_full : bar.y_full;
      uint64_t* empty = is_x ? bar.x_empty : bar.y_empty;
      const uint32_t ring = is_x ? L::kOffX : L::kOffY;
      const CUtensorMap* map = is_x ? &tm_q : &tm_do;
      const uint64_t keep = policy_evict_last();
      if (is_x) {
        const uint64_t stream = policy_evict_first();
        mbar_arrive_expect_tx(&bar.a_full, 2 * L::kTile);
        bwd_load_tile<D>(smem + L::kOffA, &tm_k, &bar.a_full, g, krow0, b, stream);
        bwd_load_tile<D>(smem + L::kOffA + L::kTile, &tm_v, &bar.a_full, g, krow0, b, stream);
      }
      int issued[XS] = {};
      bool ok = true;
      int w = 0, qb = 0, hq = 0, w2[2] = {0, 0}, qb2[2] = {0, 0};
      uint32_t cur = 0, cur2[2] = {0u, 0u};
      for (int t = 0; t < U && ok; ++t) {
        const int s = t % S, use = t / S;
        int row = 0;
        if (kStack) walk2(t, w2, cur2, qb2, hq);
        else row = walk(t, w, cur, qb, hq);
        if (t >= S) ok = mbar_wait(&empty[s], (use - 1) & 1, abort_flag, is_x ? 741 : 742);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[s], L::kTile);
        if (kStack)
          bwd_load_tile2<D>(smem + ring + s * L::kTile, map, &full[s], hq, qb2[0] * 64, qb2[1] * 64, b, keep);
        else
          bwd_load_tile<D>(smem + ring + s * L::kTile, map, &full[s], hq, row, b, keep);
        issued[s] = use + 1;
      }
      if (is_x) mbar_wait_teardown(&bar.a_full, 0);
      for (int s = 0; s < S; ++s)
        if (issued[s]) mbar_wait_teardown(&full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0 && U > 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_a = idesc_bf16_f32(128, D, 0, 1);  // P^T / dS^T from TMEM, dO / Q MN-major
      const uint64_t dkd = smem_desc_sw128(sbase + L::kOffA, 16, 1024);
      const uint64_t dvd = smem_desc_sw128(sbase + L::kOffA + L::kTile, 16, 1024);
      const uint64_t dx = smem_desc_sw128(sbase + L::kOffX, 16, 1024);              // Q, K-major
      const uint64_t dx_mn = smem_desc_sw128(sbase + L::kOffX, 128 * 128, 1024);    // Q, MN-major
      const uint64_t dy = smem_desc_sw128(sbase + L::kOffY, 16, 1024);              // dO, K-major
      const uint64_t dy_mn = smem_desc_sw128(sbase + L::kOffY, 128 * 128, 1024);    // dO, MN-major
      constexpr uint64_t kStep = L::kTile >> 4;
      bool ok = mbar_wait(&bar.a_full, 0, abort_flag, 751);
      // S^T(t) = K Q(t)^T
      auto issue_s = [&](int t) {
        ok = ok && mbar_wait(&bar.x_full[t % XS], (t / XS) & 1, abort_flag, 753);
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
          mma_bf16_ss(tmem + kColS, dkd + off, dx + (t % XS) * kStep + off, id_s, kk > 0 ? 1u : 0u);
        }
      };
      // dP^T(t) = V dO(t)^T
      auto issue_dp = [&](int t) {
        ok = ok && mbar_wait(&bar.y_full[t % YS], (t / YS) & 1, abort_flag, 754);
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4;
          mma_bf16_ss(tmem + kColP, dvd + off, dy + (t % YS) * kStep + off, id_s, kk > 0 ? 1u : 0u);
        }
      };
      issue_s(0);
      issue_dp(0);
      if (ok) mma_commit(&bar.prod_full);
      for (int t = 0; t < U && ok; ++t) {
        // S^T(t+1) once the compute warps hold S^T(t)
        if (t + 1 < U) {
          ok = mbar_wait(&bar.s_loaded, t & 1, abort_flag, 755);
          issue_s(t + 1);
          if (!ok) break;
        }
        // dV += P^T(t) dO(t), dK += dS^T(t) Q(t), queries 0-63 as soon as
        // their operands are stored, then 64-127; the 16 queries of
        // instruction kk sit in piece kk / 2, at its column 8 (kk % 2)
        const uint64_t dq_mn = dx_mn + (t % XS) * kStep, ddo_mn = dy_mn + (t % YS) * kStep;
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          ok = mbar_wait(hq == 0 ? &bar.half_full : &bar.soft_full, t & 1, abort_flag, hq == 0 ? 756 : 752);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * hq; kk < 4 * hq + 4; ++kk)
            mma_bf16_ts(tmem + kColV, tmem + kColP + 32 * (kk / 2) + 8 * (kk % 2), ddo_mn + ((kk * 16 * 128) >> 4),
                        id_a, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 4 * hq; kk < 4 * hq + 4; ++kk)
            mma_bf16_ts(tmem + kColK, tmem + kColP + 32 * (kk / 2) + 8 * (kk % 2) + 16,
                        dq_mn + ((kk * 16 * 128) >> 4), id_a, (t > 0 || kk > 0) ? 1u : 0u);
        }
        if (!ok) break;
        mma_commit(&bar.x_empty[t % XS]);
        mma_commit(&bar.y_empty[t % YS]);
        // dP^T(t+1) overwrites the columns the products above read (in order)
        if (t + 1 < U) {
          issue_dp(t + 1);
          if (!ok) break;
          mma_commit(&bar.prod_full);
        }
      }
      if (ok) mma_commit(&bar.done);
      mma_commit(&bar.drained);
      mbar_wait_teardown(&bar.drained, 0);
    }
    __syncwarp();
  } else {
    // ============================================================ P^T, dS^T, then the epilogue
    const int quad = warp % 4;
    const int kr = quad * 32 + lane;  // key row of the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const long key = krow0 + kr;
    // kStack: key rows 64 hk.. belong to stacked key block hk; an absent
    // block's rows are not written
    const int hk = kStack ? kr / 64 : 0;
    const bool live = !kStack || hk == 0 || second;
    bool ok = true;
    int w = 0, qb = 0, hq = 0, w2[2] = {0, 0}, qb2[2] = {0, 0};
    uint32_t cur = 0, cur2[2] = {0u, 0u};
    float* stats = reinterpret_cast<float*>(smem + L::kStatOff);
    for (int t = 0; t < U; ++t) {
      // query token of the thread's column kr (stats), and of column 0 of the tile
      int qrow0 = 0, qtok;
      if (kStack) {
        walk2(t, w2, cur2, qb2, hq);
        qtok = qb2[kr / 64] * 64 + kr % 64;
      } else {
        qrow0 = walk(t, w, cur, qb, hq);
        qtok = qrow0 + kr;
      }
      const long bh = static_cast<long>(b) * H + hq;
      // the tile's per-query ln-sum (as log2) and D, one query per thread,
      // into slot t % 2. The slot's previous tile, t - 2, is done: this warp
      // has seen tile t - 1's products complete, which the MMA thread issues
      // only after every compute warp has stored tile t - 2's operands.
      float* st_lse = stats + (t & 1) * 256;
      float* st_dn = st_lse + 128;
      st_lse[kr] = __ldg(lse + bh * N + qtok) * 1.4426950408889634f;
      st_dn[kr] = __ldg(dsum + bh * N + qtok);
      // kStack: the row's query columns [clo, chi] (its own block's, none once
      // its bit row is exhausted) and the first query token of its block
      const int tt = t % (UB > 0 ? UB : 1);
      const int clo = kStack ? 64 * hk : 0;
      const int chi = kStack ? ((live && tt < (hk == 0 ? H0 : H1)) ? clo + 63 : -1) : 127;
      const int qbase = kStack ? qb2[hk] * 64 - clo : qrow0;  // query token of column c: qbase + c
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.stats_ready[t & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.prod_full, t & 1, abort_flag, 761));
      if (!ok) break;
      tc_fence_after();
      // the whole S^T row, then the tensor core may overwrite it
      uint32_t s0[32], s1[32], s2[32], s3[32];
      tmem_ld32(lane_base + kColS, s0);
      tmem_ld32(lane_base + kColS + 32, s1);
      tmem_ld32(lane_base + kColS + 64, s2);
      tmem_ld32(lane_base + kColS + 96, s3);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.s_loaded);
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.stats_ready[t & 1], (t >> 1) & 1, abort_flag, 763));
      if (!ok) break;
      auto piece = [&](int c, const uint32_t (&sv)[32]) {
        uint32_t pv[32];
        tmem_ld32(lane_base + kColP + c * 32, pv);
        tmem_wait_ld();
        // this piece's 32 query columns (the same for every lane: broadcast reads)
        float lq[32], dq_[32];
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 a = *reinterpret_cast<const float4*>(st_lse + c * 32 + e);
          const float4 d = *reinterpret_cast<const float4*>(st_dn + c * 32 + e);
          lq[e] = a.x, lq[e + 1] = a.y, lq[e + 2] = a.z, lq[e + 3] = a.w;
          dq_[e] = d.x, dq_[e + 1] = d.y, dq_[e + 2] = d.z, dq_[e + 3] = d.w;
        }
        float pt[32], dst[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float lse2 = lq[e];
          const float dn = dq_[e];
          const int col = c * 32 + e;
          const bool masked = col < clo || col > chi || (kCausal && key > qbase + col);
          const float p = masked ? 0.f : fast_exp2(fmaf(__uint_as_float(sv[e]), scale_log2, -lse2));
          pt[e] = p;
          dst[e] = p * (__uint_as_float(pv[e]) - dn);
        }
        uint32_t wp[16], wd[16];
        bwd_pack16(pt, wp);
        bwd_pack16(dst, wd);
        tmem_st16(lane_base + kColP + c * 32, wp);       // over dP^T columns this piece has read
        tmem_st16(lane_base + kColP + c * 32 + 16, wd);
      };
      piece(0, s0);
      piece(1, s1);
      // queries 0-63 are ready for the accumulating products
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.half_full);
      piece(2, s2);
      piece(3, s3);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.soft_full);
    }
    if (ok && U > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar.done, 0, abort_flag, 762));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* ov = dv + ((static_cast<long>(b) * N + key) * Hkv + g) * D;
      __nv_bfloat16* ok_ = dk + ((static_cast<long>(b) * N + key) * Hkv + g) * D;
      uint32_t r[32];
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? kColV : kColK;
        const float f = which == 0 ? 1.0f : scale;
        __nv_bfloat16* out = which == 0 ? ov : ok_;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          if (U > 0) {
            tmem_ld32(lane_base + col + c * 32, r);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;  // no query block kept this key block
          }
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w4;
            w4.x = pack_bf16x2(__uint_as_float(r[e]) * f, __uint_as_float(r[e + 1]) * f);
            w4.y = pack_bf16x2(__uint_as_float(r[e + 2]) * f, __uint_as_float(r[e + 3]) * f);
            w4.z = pack_bf16x2(__uint_as_float(r[e + 4]) * f, __uint_as_float(r[e + 5]) * f);
            w4.w = pack_bf16x2(__uint_as_float(r[e + 6]) * f, __uint_as_float(r[e + 7]) * f);
            if (live) *reinterpret_cast<uint4*>(out + c * 32 + e) = w4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bsa
