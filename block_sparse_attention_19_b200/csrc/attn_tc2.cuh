// attn_tc2.cuh -- step 3 for bfloat16 or e4m3 inputs on the tensor cores:
// two 128-row query tiles per CTA so that the tensor core works on one tile
// while the softmax runs on the other.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 3 (sparse_attn_cuda, scale 1/sqrt(D)); page
// "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §2.2 (full attention inside
// the chosen blocks): o = softmax(scale * q K_sel^T) V_sel per query row.
//
// Work unit (one CTA): two "streams" A and B of 128 query rows each.
//   * block_size 256: the two halves of one query block. They share the key
//     list, so every gathered K/V tile feeds both streams.
//   * block_size 128 with an even number of query heads per key/value head:
//     one query block of two heads of a group, which share the key list.
//   * block_size 128 otherwise: two consecutive query blocks of one head,
//     each with its own key list; K/V tiles of the two streams alternate in
//     the rings. With an odd number of blocks the last CTA runs stream A only.
//   * block_size 64 (kStack): each stream stacks two consecutive query blocks
//     (see the kernel's comment).
// Roles:
//   * warp 0 (one lane): TMA loads of both query tiles and the K ring; warp 2
//     (one lane): the V ring. Rings are filled in the order the MMA consumes
//     them.
//   * warp 1, lane 0: tcgen05.mma issue in the order S_A(0), S_B(0), then per
//     key tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1). The softmax warps
//     release K ring entries (they see each S complete); the issuing thread
//     commits only the S the softmax waits for and the V entry it just read.
//     S_X lives in TMEM columns of stream X; P_X (bf16, or e4m3) is written
//     over the first 64 (32) of them (block_size 64 with e4m3: 16, each block
//     in its own lanes) and read from TMEM as the A operand of PV_X; O_X
//     accumulates in TMEM. With the causal mask and one query block per
//     stream (bf16), the first half of PV_X(j) starts once the first half of
//     P_X(j) is stored. Because tcgen05.mma ops of one thread run
//     in order, S_X(j+1) cannot overwrite P_X(j) before PV_X(j) has read it,
//     and the completion of S_X(j+1) implies that PV_X(j) is done (so O_X is
//     stable).
//   * warps 4-7 (stream A) and 8-11 (stream B): one query row per thread.
//     Per tile a thread loads its whole S row from TMEM into registers (the
//     softmax warp groups take registers from warp group 0 with setmaxnreg),
//     takes the row max; the running max (log2 domain) moves only when the
//     tile max exceeds it by more than 8, in which case O_X is rescaled in
//     TMEM; then P = exp2(S * scale * log2 e - m) with two-wide float32
//     instructions (one key pair in four via a polynomial on the FMA pipe),
//     stored packed over the first columns of S.
//   * warp 3 idle.
// Every wait is bounded; on a timeout the device error word and an abort flag
// are set, roles leave their loops, copies and MMAs are drained, TMEM is freed.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kTc2Threads = 384;  // 12 warps
constexpr int kTc2MaxStages = 12;
// Register split: warp group 0 (producers, MMA issuer) gives registers to
// the two softmax warp groups, which hold a whole 128-column S row. The sum
// must fit in the launch allocation (kTc2Threads x the kernel's register
// count), which the host verifies: kTc2LaunchRegs is what the split needs.
constexpr uint32_t kTc2RegsLow = 80, kTc2RegsHigh = 208;
constexpr uint32_t kTc2LaunchRegs = (128 * kTc2RegsLow + 256 * kTc2RegsHigh + kTc2Threads - 1) / kTc2Threads;

// F8: FP8 E4M3 inputs (one byte per element) instead of bfloat16.
template <int D, bool F8 = false>
struct Tc2Layout {
  static constexpr int kElem = F8 ? 1 : 2;                  // bytes per element
  static constexpr uint32_t kTileBytes = 128 * D * kElem;  // a 128-row Q, K or V tile
  static constexpr int kKStages = F8 ? (D == 64 ? 12 : 6) : (D == 128 ? 3 : 6);
  static constexpr int kVStages = F8 ? (D == 64 ? 12 : 6) : (D == 128 ? 2 : 6);
  // A tile is stored as column chunks of kRowBytes per row in the swizzled
  // layout the MMA reads: 128-byte rows (128-byte swizzle), or 64-byte rows
  // (64-byte swizzle) when a whole row is 64 bytes (e4m3 with D = 64).
  static constexpr uint32_t kRowBytes = D * kElem < 128 ? D * kElem : 128;
  static constexpr int kChunks = D * kElem / kRowBytes;     // column chunks of a row
  static constexpr int kChunkElems = kRowBytes / kElem;     // elements per chunk (TMA box width)
  static constexpr uint32_t kChunkBytes = 128 * kRowBytes;  // one chunk of a 128-row tile
  static constexpr uint32_t kHalfBytes = 64 * kRowBytes;    // 64 rows of a chunk (one TMA box)
  static constexpr uint32_t kSBO = 8 * kRowBytes;           // 8-row swizzle atom
  static constexpr uint32_t kLayout = kRowBytes == 128 ? 2u : 4u;  // descriptor layout field
  static constexpr int kStepsPerRow = kRowBytes / 32;       // 32-byte MMA K steps per chunk row
  static constexpr uint32_t kQOff = 0;  // Q_A, Q_B
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + kKStages * kTileBytes;
  static constexpr uint32_t kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr uint32_t kBytes = kBarOff + 512;
  static constexpr uint32_t kTmemCols = 512;  // S_A | S_B | O_A | O_B
  __device__ static constexpr uint32_t col_s(int x) { return 128u * x; }
  __device__ static constexpr uint32_t col_o(int x) { return 256u + 128u * x; }
  static_assert(kBytes <= 232448, "shared memory budget");
  static_assert(kKStages <= kTc2MaxStages && kVStages <= kTc2MaxStages, "stage count");
};

struct Tc2Barriers {
  uint64_t q_full;
  uint64_t k_full[kTc2MaxStages], k_empty[kTc2MaxStages];
  uint64_t v_full[kTc2MaxStages], v_empty[kTc2MaxStages];
  uint64_t s_full[2];   // phase j: S_X(j) computed
  uint64_t p_full[2];   // phase j: P_X(j) stored (and O_X rescaled if needed)
  uint64_t p_half[2];   // phase j: keys 0-63 of P_X(j) stored (causal bf16 tiles of one block)
  uint64_t pv_last[2];  // phase 0: the last PV_X completed
  uint64_t mma_drained;
  uint32_t tmem_base;
  int abort;
  int tiles[2];  // key tiles of stream A and B (valid index entries, x2 for block_size 256)
  int valid[4];  // block_size 64: valid index entries of the four query blocks
};
static_assert(sizeof(Tc2Barriers) <= 512, "barrier area");

// Key block of entry t of an index row; a global head has no index row
// (sel == nullptr) and walks every block in order.
__device__ __forceinline__ int sel_block(const int32_t* sel, int t, int nb) {
  return sel ? clamp_block(__ldg(sel + t), nb) : t;
}

// Key windows: entry t of an index row names key window e, whose first token
// is min(e * ws, N - bs) (ws = bs: the disjoint blocks; ws < bs: windows that
// overlap by bs - ws tokens, the last one ending at token N). A global head
// (sel == nullptr) walks the disjoint blocks. nkb: windows per head.
// kVar = false compiles the plain method only (an index row of disjoint
// blocks for every head), so its kernels carry none of this.
struct KeyWin {
  int bs, N, ws, nkb;
};
template <bool kVar>
__device__ __forceinline__ int win_start(const int32_t* sel, int t, const KeyWin& kw) {
  if constexpr (!kVar) return clamp_block(__ldg(sel + t), kw.nkb) * kw.bs;
  if (!sel) return t * kw.bs;
  return min(clamp_block(__ldg(sel + t), kw.nkb) * kw.ws, kw.N - kw.bs);
}
// Leading tokens of entry t's window that entry t - 1's window already holds
// (entries ascend, so only the previous window can reach into this one).
__device__ __forceinline__ int win_dup(const int32_t* sel, int t, const KeyWin& kw) {
  if (!sel || t == 0 || kw.ws >= kw.bs || __ldg(sel + t) < 0) return 0;
  return max(0, win_start<true>(sel, t - 1, kw) + kw.bs - win_start<true>(sel, t, kw));
}

// Valid entries of an index row; for a global head (sel == nullptr) every
// block, or with the causal mask the blocks 0..i of query block i.
template <bool kCausal>
__device__ __forceinline__ int sel_valid(const int32_t* sel, int k, int i, int nb) {
  return sel ? index_row_valid(sel, k) : (kCausal ? i + 1 : nb);  // sel == nullptr only with kVar
}

// Token row where 64-row half `hf` of stream `x`'s key tile t starts.
template <bool kVar>
__device__ __forceinline__ int tc2_key_row(const int32_t* sel_a, const int32_t* sel_b, int x,
                                           int t, int hf, const KeyWin& kw) {
  if (kw.bs == 128) return win_start<kVar>(x == 0 ? sel_a : sel_b, t, kw) + hf * 64;
  return win_start<kVar>(sel_a, t / 2, kw) + (t % 2) * 128 + hf * 64;  // bs == 256
}

// Columns c < lo of 32 scores of a row become -inf (keys another kept window
// already contributed).
__device__ __forceinline__ void tc2_mask_before(uint32_t (&r)[32], int c0, int lo) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (c0 + e < lo) r[e] = __float_as_uint(-INFINITY);
}

// Causal mask on 32 scores of a row: column c0 + e becomes -inf when it is
// above lim.
__device__ __forceinline__ void tc2_mask_after(uint32_t (&r)[32], int c0, int lim) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (c0 + e > lim) r[e] = __float_as_uint(-INFINITY);
}

// The max of 64 scores.
__device__ __forceinline__ float tc2_max64(const uint32_t (&s0)[32], const uint32_t (&s1)[32]) {
  float m4[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) m4[e] = fmaxf(__uint_as_float(s0[2 * e]), __uint_as_float(s0[2 * e + 1]));
#pragma unroll
  for (int pr = 4; pr < 32; ++pr) {
    const float a = __uint_as_float(pr < 16 ? s0[(2 * pr) & 31] : s1[(2 * pr) & 31]);
    const float c = __uint_as_float(pr < 16 ? s0[(2 * pr + 1) & 31] : s1[(2 * pr + 1) & 31]);
    m4[pr % 4] = fmax3(m4[pr % 4], a, c);
  }
  return fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
}

// O_X *= alpha for the thread's row (alpha is 1 on rows whose max stayed).
template <int D>
__device__ __forceinline__ void tc2_rescale_o(uint32_t ocol, float alpha) {
  uint32_t r[16];
#pragma unroll 1
  for (int c = 0; c < D / 16; ++c) {
    tmem_ld16(ocol + c * 16, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
    tmem_st16(ocol + c * 16, r);
  }
}

// P = exp2(S * scale_log2 - m) for 32 scores of a row, packed as the P.V
// product reads it from TMEM: bf16 two per column (16 columns) or e4m3 four
// per column (8), the lowest key in the lowest bits; one key pair in four via
// the polynomial exp2. ps: four partial sums of the float32 P, accumulated.
template <bool kF8>
__device__ __forceinline__ void tc2_make_p32(const uint32_t (&sv)[32], float m, float scale_log2,
                                             uint32_t (&pk)[kF8 ? 8 : 16], uint64_t (&ps)[4]) {
  const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-m, -m);
#pragma unroll
  for (int pr = 0; pr < 16; ++pr) {
    const uint64_t x2 = f2_fma(f2(__uint_as_float(sv[2 * pr]), __uint_as_float(sv[2 * pr + 1])), sc2, nm2);
    uint64_t p2;
    if (pr % 4 == 1) {
      p2 = exp2_poly2(x2);
    } else {
      float x0, x1;
      f2_split(x2, x0, x1);
      p2 = f2(fast_exp2(x0), fast_exp2(x1));
    }
    ps[pr % 4] = f2_add(ps[pr % 4], p2);
    float p0, p1;
    f2_split(p2, p0, p1);
    if constexpr (kF8) {
      const uint32_t h16 = pack_e4m3x2(p0, p1);
      if (pr % 2 == 0)
        pk[pr / 2] = h16;
      else
        pk[pr / 2] |= h16 << 16;
    } else {
      pk[pr] = pack_bf16x2(p0, p1);
    }
  }
}

// grid.x = B * H * ceil(nb / 2) for block_size 128, B * H * nb for 256.
// kStack (block_size 64): grid.x = B * H * ceil(nb / 4); stream x stacks
// query blocks 4u + 2x (rows 0-63) and 4u + 2x + 1 (rows 64-127), and its
// key tile t stacks the t-th kept block of each (keys 0-63, 64-127). The
// 128 x 128 score tile is then block diagonal: rows 0-63 keep keys 0-63,
// rows 64-127 keys 64-127; the other quadrants are computed and discarded,
// and P is zero there, so one M = 128 product serves both blocks (the same
// tensor time as two M = 64 products, with every TMEM lane and softmax
// thread in use). With e4m3 inputs P.V is issued per block instead, with the
// output-lane mask: each block's P (its 64 keys, 16 columns) times its half
// of the V tile into its own lanes of O, so no zero half is stored and a
// block whose list has ended issues no P.V.
// kCausal: key tokens after the query token are masked (kFlagCausal).
// lse (optional, [B, H, N] float32): ln sum_t exp(scale q_n . k_t) per row.
// gperiod > 0: query heads h with h % gperiod == 0 are global heads, which
// read no index row and attend to every key block (blocks 0..i when causal);
// query heads are then never paired in a CTA.
// ws < bs: the index rows name overlapping key windows (see KeyWin; nkb
// windows per head); a key that the row's previous kept window already
// holds is masked, so each token of the union counts once (not causal).
// Both need kVar; the plain method's instances (kVar = false) ignore
// gperiod, ws and nkb.
template <int D, bool kCausal, bool kF8 = false, bool kStack = false, bool kVar = false>
__global__ void __launch_bounds__(kTc2Threads, 1)
    sparse_attn_tc2_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, int N,
                           int H, int Hkv, int bs, int k, float scale_log2, float* __restrict__ lse,
                           int gperiod, int ws, int nkb) {
  using L = Tc2Layout<D, kF8>;
  // MMA steps: K = 32 bytes of the row per instruction (16 bf16 or 32 e4m3)
  constexpr int kStepsS = D * L::kElem / 32;
  constexpr int kKeysPerStep = 32 / L::kElem;
  constexpr int kStepsPV = 128 / kKeysPerStep;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(1024) unsigned char tc2_raw[];
  // swizzled tiles need 1024-byte alignment and the layout has no slack
  if ((smem_u32(tc2_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(402);
    return;
  }
  unsigned char* smem = tc2_raw;
  Tc2Barriers& bar = *reinterpret_cast<Tc2Barriers*>(smem + L::kBarOff);
  volatile int* abort_flag = &bar.abort;

  const int nb = N / bs;
  const KeyWin kw{bs, N, kVar ? ws : bs, kVar ? nkb : nb};
  // What the two query tiles (streams) of a CTA are:
  //  - block_size 256: the two 128-row halves of one query block of one head;
  //  - block_size 128, an even number G of query heads per key/value head:
  //    one query block of two heads of the same group;
  //  - otherwise: two consecutive query blocks of one head.
  // In the first two the streams read the same key tiles (one selection),
  // so each K and V tile is loaded once for both.
  const int G = H / Hkv;
  const bool head_pairs = !kStack && bs == 128 && (G % 2) == 0 && (!kVar || gperiod == 0);
  const bool shared_kv = !kStack && (bs == 256 || head_pairs);
  long u = blockIdx.x;
  int iA, b, qh[2];
  if (kStack) {
    const int per_bh = (nb + 3) / 4;
    iA = 4 * static_cast<int>(u % per_bh);
    u /= per_bh;
    qh[0] = qh[1] = static_cast<int>(u % H);
    b = static_cast<int>(u / H);
  } else if (head_pairs) {
    iA = static_cast<int>(u % nb);
    u /= nb;
    const int hp = static_cast<int>(u % (H / 2));
    b = static_cast<int>(u / (H / 2));
    qh[0] = 2 * hp;
    qh[1] = 2 * hp + 1;
  } else {
    const int per_bh = bs == 256 ? nb : (nb + 1) / 2;
    const int unit = static_cast<int>(u % per_bh);
    u /= per_bh;
    qh[0] = qh[1] = static_cast<int>(u % H);
    b = static_cast<int>(u / H);
    iA = bs == 256 ? unit : 2 * unit;
  }
  const int g = qh[0] / G;  // the key/value head (and selection) of both streams
  const int nstreams = kStack ? (iA + 2 < nb ? 2 : 1) : ((!shared_kv && iA + 1 >= nb) ? 1 : 2);
  // stream x covers query rows [row0[x], row0[x] + 128) of query head qh[x]
  const int row0[2] = {iA * bs, kStack ? (iA + 2) * 64
                                       : (bs == 256 ? iA * bs + 128 : (head_pairs ? iA * bs : (iA + 1) * bs))};
  const long bg = static_cast<long>(b) * Hkv + g;
  // both streams belong to one query head whenever global heads exist
  const bool dense = kVar && gperiod > 0 && qh[0] % gperiod == 0;
  const int iB = iA + 1 < nb ? iA + 1 : iA;
  const int32_t* sel_a = dense ? nullptr : idx + (bg * nb + iA) * k;
  const int32_t* sel_b = shared_kv ? sel_a : (dense ? nullptr : idx + (bg * nb + iB) * k);
  // kStack: index rows of query blocks iA + q (an absent second block of a
  // stream takes its first block's row, whose rows are then not written)
  const int32_t* sel4[4];
  int blk4[4];
  if (kStack)
    for (int q = 0; q < 4; ++q) {
      blk4[q] = iA + q < nb ? iA + q : min(iA + (q & 2), nb - 1);
      sel4[q] = dense ? nullptr : idx + (bg * nb + blk4[q]) * k;
    }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    // a K entry is released by the softmax warp group(s) that saw its S
    // complete; a V entry by an MMA commit right after its last P.V product
    for (int s = 0; s < KS; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], shared_kv ? 2 : 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.p_full[x], 4);
      mbar_init(&bar.p_half[x], 4);
      mbar_init(&bar.pv_last[x], 1);
    }
    mbar_init(&bar.mma_drained, 1);
    bar.abort = 0;
    // key tiles per stream: the valid entries of its index row (at least one,
    // so that a row of only -1 still reads block 0 instead of nothing)
    if (kStack) {
      // a stream walks as many tiles as the longer of its two rows
      for (int q = 0; q < 4; ++q)
        bar.valid[q] = iA + q < nb ? max(sel_valid<kCausal>(sel4[q], k, blk4[q], nb), 1) : 0;
      bar.tiles[0] = max(bar.valid[0], bar.valid[1]);
      bar.tiles[1] = max(bar.valid[2], bar.valid[3]);
    } else {
      const int ta = max(sel_valid<kCausal>(sel_a, k, iA, nb), 1);
      const int tb = nstreams == 2 && !shared_kv ? max(sel_valid<kCausal>(sel_b, k, iB, nb), 1) : 0;
      const int tpb = bs == 256 ? 2 : 1;  // key tiles per block
      bar.tiles[0] = tpb * ta;
      bar.tiles[1] = shared_kv ? tpb * ta : tb;
    }
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
  const int TA = bar.tiles[0], TB = bar.tiles[1];
  // Ring order of the K and V loads: one per (stream, tile), alternating A, B
  // while both streams have tiles, then the longer stream alone; one per tile
  // when the streams share their key tiles.
  const int Tmin = min(TA, TB);
  const int nloads = shared_kv ? TA : TA + TB;
  auto load_index = [&](int x, int t) {
    return shared_kv ? t : (t < Tmin ? 2 * t + x : 2 * Tmin + (t - Tmin));
  };
  // register split: each role adjusts its own allowance on entry (warp
  // group 0: producers, MMA issuer and the idle warp 3 give registers away)
  if (warp == 0 || warp == 2) {
    regs_decrease<kTc2RegsLow>();
    // ============================================================ TMA producers
    // warp 0: query tiles and the K ring; warp 2: the V ring. Separate warps,
    // so that one producer suspended in a wait never holds up the other.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int S = is_k ? KS : VS;
      const uint64_t keep = policy_evict_last();  // gathered K/V: reused across query blocks
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint64_t* full = is_k ? bar.k_full : bar.v_full;
      uint64_t* empty = is_k ? bar.k_empty : bar.v_empty;
      const uint32_t ring = is_k ? L::kKOff : L::kVOff;
      int issued[kTc2MaxStages];
      for (int s = 0; s < S; ++s) issued[s] = 0;
      bool ok = true;
      if (is_k) {
        const uint64_t stream = policy_evict_first();  // query tiles: read once
        mbar_arrive_expect_tx(&bar.q_full, nstreams * L::kTileBytes);
        for (int x = 0; x < nstreams; ++x)
          for (int hh = 0; hh < 2; ++hh)
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_4d(smem + L::kQOff + x * L::kTileBytes + c * L::kChunkBytes + hh * L::kHalfBytes,
                          &tm_q, &bar.q_full, c * L::kChunkElems, qh[x], row0[x] + hh * 64, b, stream);
      }
      for (int n = 0; n < nloads && ok; ++n) {
        const int s = n % S, use = n / S;
        // inverse of load_index
        const int x = shared_kv ? 0 : (n < 2 * Tmin ? (n & 1) : (TA > TB ? 0 : 1));
        const int t = shared_kv ? n : (n < 2 * Tmin ? (n >> 1) : Tmin + (n - 2 * Tmin));
        int r[2];
        for (int hf = 0; hf < 2; ++hf)
          r[hf] = kStack ? win_start<kVar>(sel4[2 * x + hf], t, kw)  // -1 entries load block 0, unused
                         : tc2_key_row<kVar>(sel_a, sel_b, x, t, hf, kw);
        if (n >= S) ok = mbar_wait(&empty[s], (use - 1) & 1, abort_flag, is_k ? 111 : 112);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[s], L::kTileBytes);
        for (int hf = 0; hf < 2; ++hf)
          for (int c = 0; c < L::kChunks; ++c)
            tma_load_4d(smem + ring + s * L::kTileBytes + c * L::kChunkBytes + hf * L::kHalfBytes, map,
                        &full[s], c * L::kChunkElems, g, r[hf], b, keep);
        issued[s] = use + 1;
      }
      if (is_k) mbar_wait_teardown(&bar.q_full, 0);
      for (int s = 0; s < S; ++s)
        if (issued[s]) mbar_wait_teardown(&full[s], (issued[s] - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    regs_decrease<kTc2RegsLow>();
    // ============================================================ MMA issuer
    // One thread feeds the tensor core, and a tcgen05.mma issue returns only
    // when the previous instruction starts, so any work between instructions
    // is idle tensor time: the loop body is straight-line, waits take a
    // one-instruction fast path, descriptors move by plain adds, and the only
    // commit per group is the one the softmax needs (ring entries are released
    // by the softmax warps, which see each S complete).
    if (lane == 0) {
      const uint32_t idesc_s = kF8 ? idesc_e4m3_f32(128, 128, 0, 0) : idesc_bf16_f32(128, 128, 0, 0);
      // P from TMEM, V MN-major
      const uint32_t idesc_pv = kF8 ? idesc_e4m3_f32(128, D, 0, 1) : idesc_bf16_f32(128, D, 0, 1);
      const uint64_t dq0 = smem_desc_swz(sbase + L::kQOff, 16, L::kSBO, L::kLayout);
      const uint64_t dk0 = smem_desc_swz(sbase + L::kKOff, 16, L::kSBO, L::kLayout);
      // V MN-major: the leading offset steps between column chunks of D
      const uint64_t dv0 = smem_desc_swz(sbase + L::kVOff, L::kChunkBytes, L::kSBO, L::kLayout);
      constexpr uint64_t kTileStep = L::kTileBytes >> 4;
      // ring index of stream x's tile t (K and V rings are filled in the same order)
      bool ok = mbar_wait(&bar.q_full, 0, abort_flag, 211);
      // kStack with e4m3: valid index entries of the four query blocks (0: absent)
      int vq[4] = {0, 0, 0, 0};
      if constexpr (kStack && kF8)
        for (int q = 0; q < 4; ++q) vq[q] = bar.valid[q];
      // The rings are consumed in load order: kn and vn are the next K and
      // V loads (a load serves both streams, stream B last, when they share
      // their key tiles).
      int kn = 0, vn = 0;
      // S_X(0)
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (!ok || x >= nstreams) break;
        const int n = kn;
        if (!shared_kv || x == 1) ++kn;
        ok = mbar_wait_fast(&bar.k_full[n % KS], (n / KS) & 1, abort_flag, 212);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dq = dq0 + x * kTileStep, dk = dk0 + (n % KS) * kTileStep;
#pragma unroll
        for (int kk = 0; kk < kStepsS; ++kk) {
          const uint64_t off =
              ((kk / L::kStepsPerRow) * L::kChunkBytes + (kk % L::kStepsPerRow) * 32) >> 4;
          if (kF8)
            mma_f8_ss(tmem + L::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
          else
            mma_bf16_ss(tmem + L::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar.s_full[x]);
      }
      const int Tmax = max(TA, TB);
      for (int j = 0; j < Tmax && ok; ++j) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int Tx = x == 0 ? TA : TB;
          if (j >= Tx) continue;  // this stream is done (or absent)
          const bool more = j + 1 < Tx;
          // PV_X(j) needs P_X(j) and V(x, j); S_X(j+1) needs K(x, j+1)
          const int nv = vn, nk = kn;
          const bool last_user = !shared_kv || x == 1;
          vn += last_user;
          if (more) kn += last_user;
          // causal bf16 tiles of one query block: the first half of PV_X(j)
          // starts once keys 0-63 of P_X(j) are stored (A/B: causal c4 20.9 ->
          // 20.2 ms; without the mask, where both streams stay busy to the
          // end, it measured 1% slower)
          constexpr bool kHalfP = !kStack && !kF8 && kCausal;
          ok = mbar_wait_fast(kHalfP ? &bar.p_half[x] : &bar.p_full[x], j & 1, abort_flag, 213) &&
               mbar_wait_fast(&bar.v_full[nv % VS], (nv / VS) & 1, abort_flag, 214) &&
               (!more || mbar_wait_fast(&bar.k_full[nk % KS], (nk / KS) & 1, abort_flag, 215));
          if (!ok) break;
          tc_fence_after();
          const uint64_t dv = dv0 + (nv % VS) * kTileStep;
          const uint32_t a_tmem = tmem + L::col_s(x);
          if constexpr (kStack && kF8) {
            // e4m3: block hf of the stream multiplies its own P (the first
            // columns of S) by its half of the V tile, into its own lanes of
            // O, and issues nothing once its list has ended. (With bf16 one
            // P.V over the whole tile, with the other block's half of P zero,
            // measured faster.)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              if (j >= vq[2 * x + hf]) continue;
#pragma unroll
              for (int kk = 0; kk < kStepsPV / 2; ++kk) {
                const uint64_t bv = dv + ((((kStepsPV / 2) * hf + kk) * kKeysPerStep * L::kRowBytes) >> 4);
                mma_f8_ts_half(tmem + L::col_o(x), a_tmem + kk * 8, bv, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u,
                               hf == 0);
              }
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kStepsPV; ++kk) {
              if (kHalfP && kk == kStepsPV / 2) {
                ok = mbar_wait_fast(&bar.p_full[x], j & 1, abort_flag, 216);
                if (!ok) break;
                tc_fence_after();
              }
              // kKeysPerStep keys: 8 TMEM columns of P, kKeysPerStep rows of V
              const uint64_t bv = dv + ((kk * kKeysPerStep * L::kRowBytes) >> 4);
              if (kF8)
                mma_f8_ts(tmem + L::col_o(x), a_tmem + kk * 8, bv, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
              else
                mma_bf16_ts(tmem + L::col_o(x), a_tmem + kk * 8, bv, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          // the V ring is shallow, so its entry is freed as soon as the product is done
          if (last_user) mma_commit(&bar.v_empty[nv % VS]);
          if (more) {
            const uint64_t dq = dq0 + x * kTileStep, dk = dk0 + (nk % KS) * kTileStep;
#pragma unroll
            for (int kk = 0; kk < kStepsS; ++kk) {
              const uint64_t off =
              ((kk / L::kStepsPerRow) * L::kChunkBytes + (kk % L::kStepsPerRow) * 32) >> 4;
              if (kF8)
                mma_f8_ss(tmem + L::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
              else
                mma_bf16_ss(tmem + L::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar.s_full[x]);
          } else {
            mma_commit(&bar.pv_last[x]);
          }
        }
      }
      mma_commit(&bar.mma_drained);
      mbar_wait_teardown(&bar.mma_drained, 0);
    }
    __syncwarp();
  } else if (warp == 3) {
    regs_decrease<kTc2RegsLow>();
  } else if ((warp - 4) / 4 < nstreams) {
    regs_increase<kTc2RegsHigh>();
    // ============================================================ softmax / epilogue
    const int x = (warp - 4) / 4;
    const int quad = warp % 4;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t scol = lane_base + L::col_s(x);
    const uint32_t ocol = lane_base + L::col_o(x);
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    const int Tx = x == 0 ? TA : TB;
    // kStack: valid tiles of the thread's query block; rows of an absent block are not written
    const int vt = kStack ? bar.valid[2 * x + quad / 2] : Tx;
    const bool live = !kStack || iA + 2 * x + quad / 2 < nb;
    for (int j = 0; j < Tx; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar.s_full[x], j & 1, abort_flag, 311));
      if (!ok) break;
      tc_fence_after();
      if (quad == 0 && lane == 0) {
        // S_X(j) is complete: the K tile it read can be refilled
        mbar_arrive(&bar.k_empty[load_index(x, j) % KS]);
      }
      if constexpr (kStack) {
        // rows 64 hf.. of the stream belong to query block iA + 2x + hf, whose
        // keys are columns 64 hf.. of the tile
        const int hf = quad / 2;
        if (j >= vt) {
          // this block's list has ended (or the block is absent): with bf16
          // the tile's P.V reads its lanes, so its P is zero; with e4m3 its
          // half of P.V is not issued
          if constexpr (!kF8) {
            uint32_t z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0;
            tmem_st32(scol, z);
            tmem_st32(scol + 32, z);
          }
        } else {
          uint32_t s0[32], s1[32];
          tmem_ld32(scol + 64 * hf, s0);
          tmem_ld32(scol + 64 * hf + 32, s1);
          tmem_wait_ld();
          if (kCausal) {
            // keys c > lim of the block follow the thread's query token
            const int lim = row0[x] + row - win_start<kVar>(sel4[2 * x + hf], j, kw);
            if (lim < 63) {
              tc2_mask_after(s0, 0, lim);
              tc2_mask_after(s1, 32, lim);
            }
          }
          if constexpr (kVar) {
            // overlapping windows: keys the previous kept window holds
            const int dup = win_dup(sel4[2 * x + hf], j, kw);
            if (dup > 0) {
              tc2_mask_before(s0, 0, dup);
              tc2_mask_before(s1, 32, dup);
            }
          }
          const float mt = tc2_max64(s0, s1) * scale_log2;
          const float m_new = (j == 0 || mt > m_run + 8.0f) ? mt : m_run;
          const bool rescale = j > 0 && m_new != m_run;
          if (__any_sync(0xffffffffu, rescale)) {
            const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
            l_run *= alpha;
            tc2_rescale_o<D>(ocol, alpha);
          }
          m_run = m_new;
          uint64_t ps[4] = {0, 0, 0, 0};
          uint32_t pk0[kF8 ? 8 : 16], pk1[kF8 ? 8 : 16];
          tc2_make_p32<kF8>(s0, m_new, scale_log2, pk0, ps);
          tc2_make_p32<kF8>(s1, m_new, scale_log2, pk1, ps);
          if constexpr (kF8) {
            // the block's 64 keys over the first columns of S, which its
            // half of P.V reads in its own lanes
            tmem_st8(scol, pk0);
            tmem_st8(scol + 8, pk1);
          } else {
            // P of the block's keys; zeros where the tile holds the other block's
            uint32_t z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0;
            tmem_st16(scol + 32 * hf, pk0);
            tmem_st16(scol + 32 * hf + 16, pk1);
            tmem_st32(scol + 32 * (1 - hf), z);
          }
          float a0, a1;
          f2_split(f2_add(f2_add(ps[0], ps[1]), f2_add(ps[2], ps[3])), a0, a1);
          l_run += a0 + a1;
        }
        tmem_wait_st();
      } else {
        // first key token of this tile; with the causal flag a tile that
        // reaches past the tile's first query token masks key c for row r when
        // kbase + c > qbase + r (only the diagonal block does)
        const int kbase = kCausal ? tc2_key_row<kVar>(sel_a, sel_b, x, j, 0, kw) : 0;
        const bool mask_tile = kCausal && kbase + 127 > row0[x];
        // The whole S row in registers: four TMEM loads, one wait.
        uint32_t sa[32], sb[32], sc[32], sd[32];
        tmem_ld32(scol, sa);
        tmem_ld32(scol + 32, sb);
        tmem_ld32(scol + 64, sc);
        tmem_ld32(scol + 96, sd);
        tmem_wait_ld();
        if (mask_tile) {
          // keys c > lim of this tile lie after the thread's query token
          const int lim = row0[x] + row - kbase;
          tc2_mask_after(sa, 0, lim);
          tc2_mask_after(sb, 32, lim);
          tc2_mask_after(sc, 64, lim);
          tc2_mask_after(sd, 96, lim);
        }
        if constexpr (kVar) {
          // overlapping windows: keys of this tile the previous kept window
          // holds (block_size 256: the window's second tile starts at key 128)
          const int lo = win_dup(x == 0 ? sel_a : sel_b, bs == 256 ? j / 2 : j, kw) - (bs == 256 ? (j % 2) * 128 : 0);
          if (lo > 0) {
            tc2_mask_before(sa, 0, lo);
            tc2_mask_before(sb, 32, lo);
            tc2_mask_before(sc, 64, lo);
            tc2_mask_before(sd, 96, lo);
          }
        }
#define BSA_S(i) __uint_as_float((i) < 32 ? sa[(i) & 31] : (i) < 64 ? sb[(i) & 31] : (i) < 96 ? sc[(i) & 31] : sd[(i) & 31])
        float m4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) m4[e] = fmaxf(BSA_S(2 * e), BSA_S(2 * e + 1));
#pragma unroll
        for (int pr = 4; pr < 64; ++pr) m4[pr % 4] = fmax3(m4[pr % 4], BSA_S(2 * pr), BSA_S(2 * pr + 1));
        const float mt = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]) * scale_log2;
        // the running max moves only when the tile max exceeds it by more than 8
        const float m_new = (j == 0 || mt > m_run + 8.0f) ? mt : m_run;
        const bool rescale = j > 0 && m_new != m_run;
        if (__any_sync(0xffffffffu, rescale)) {
          // S_X(j) is complete, so PV_X(j-1) has finished accumulating into O_X
          const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.0f;
          l_run *= alpha;
          uint32_t r[16];
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            tmem_ld16(ocol + c * 16, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16(ocol + c * 16, r);
          }
        }
        m_run = m_new;
        // P = exp2(S * scale_log2 - m) for key pairs with two-wide float32
        // instructions; one pair in four takes the polynomial exp2 on the FMA
        // pipe (the split measured fastest: the softmax is bound by issue slots
        // more than by MUFU). P is stored over the first columns of S: packed
        // bf16, two per column (64 columns), or e4m3, four per column (32).
        uint32_t pa[32], pb[kF8 ? 1 : 32];
        uint64_t ps[4] = {0, 0, 0, 0};
        {
          const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-m_new, -m_new);
#pragma unroll
          for (int pr = 0; pr < 64; ++pr) {
            const uint64_t x2 = f2_fma(f2(BSA_S(2 * pr), BSA_S(2 * pr + 1)), sc2, nm2);
            uint64_t p2;
            if (pr % 4 == 1) {
              p2 = exp2_poly2(x2);
            } else {
              float x0, x1;
              f2_split(x2, x0, x1);
              p2 = f2(fast_exp2(x0), fast_exp2(x1));
            }
            ps[pr % 4] = f2_add(ps[pr % 4], p2);
            float p0, p1;
            f2_split(p2, p0, p1);
            if (kF8) {
              // four e4m3 per 32-bit column, the lowest byte the lowest key
              const uint32_t h16 = pack_e4m3x2(p0, p1);
              if (pr % 2 == 0)
                pa[pr / 2] = h16;
              else
                pa[pr / 2] |= h16 << 16;
            } else if (pr < 32) {
              pa[pr] = pack_bf16x2(p0, p1);
              if (kCausal && pr == 31) {
                // keys 0-63 stored: the first half of PV_X(j) may start
                tmem_st32(scol, pa);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar.p_half[x]);
              }
            } else {
              pb[pr - 32] = pack_bf16x2(p0, p1);
            }
          }
        }
#undef BSA_S
        if constexpr (kF8) {
          tmem_st32(scol, pa);
        } else {
          if constexpr (!kCausal) tmem_st32(scol, pa);  // (causal: stored above)
          tmem_st32(scol + 32, pb);
        }
        tmem_wait_st();
        {
          float a0, a1;
          f2_split(f2_add(f2_add(ps[0], ps[1]), f2_add(ps[2], ps[3])), a0, a1);
          l_run += a0 + a1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.p_full[x]);
    }
    // ---- epilogue: O_X / l -> bf16 -> global
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar.pv_last[x], 0, abort_flag, 314));
    if (ok && live) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const long n = row0[x] + row;
      // natural log of the row's softmax denominator (m_run is in log2 units)
      if (lse) lse[(static_cast<long>(b) * H + qh[x]) * N + n] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      __nv_bfloat16* orow = o + ((static_cast<long>(b) * N + n) * H + qh[x]) * D;
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(ocol + c * 32, r);
        tmem_wait_ld();
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

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace bsa
