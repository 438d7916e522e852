// scores_tc.cuh -- step 1b: block scores on the tensor cores in split TF32.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 1: block_scores = einsum of the pooled q and
// k, per (b, h): S[i, j] = qbar_i . kbar_j (an nb x nb matrix per head);
// page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §3.3: block scoring as a
// matrix product.
//
// Float32 accuracy from TF32 tensor cores: each operand is split exactly as
// x = hi + lo with hi = x with its 13 low mantissa bits cleared (what a TF32
// product reads) and lo = x - hi (exact in float32, |lo| < 2^-10 |x|); the
// product is taken as hi.hi + hi.lo + lo.hi, dropping lo.lo and the TF32
// truncation of each lo (each below 2^-20 of the product), accumulated in
// float32 in TMEM. The error per score stays inside float32 FFMA's own
// worst-case bound of D * 2^-24 * sum_d |qbar_d kbar_d| (measured: about half
// of it, 2^-18 of sum_d |qbar_d kbar_d| at D = 128).
//
// Persistent, warp-specialised kernel, one CTA per SM, tiles of 128 rows x
// ntile (128 or 256) columns of S taken round-robin:
//  * warps 0-7, two groups of four: group g loads the float32 rows of every
//    other 32-column chunk of the pooled operands straight into registers
//    (coalesced), splits them and writes hi and lo to shared-memory stage g in
//    the 128-byte-swizzled K-major layout. With two groups each has two chunk
//    times to cover the L2 latency of its loads.
//  * warp 12: one thread issues 3 x 4 tcgen05.mma (kind::tf32, K = 8 each)
//    per chunk into one of two TMEM accumulators (2 x 256 columns), so a
//    tile's epilogue overlaps the next tile's products.
//  * warps 8-11: the epilogue. Each warp reads its 32 TMEM lanes (rows) 32
//    columns at a time, writes them to a swizzled staging box and stores the
//    box with a TMA tensor store, which clips rows and columns beyond nb.
//    When the row pitch nb * 4 bytes is not a multiple of 16 (nb % 4 != 0) a
//    tensor map cannot describe S and the warp stores rows directly instead.
// Shared memory traffic, not the tensor pipe, sets the pace: per chunk of a
// 128 x 256 tile the products read 144 KB and the split writes 96 KB.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kScM = 128, kScChunk = 32;  // tile rows, d per chunk
constexpr int kScSplitWarps = 8, kScEpiWarp0 = 8, kScMmaWarp = 12;
constexpr int kScThreads = 13 * 32;
constexpr uint32_t kScAHalf = kScM * kScChunk * 4;          // 16 KB: A hi (or lo) of one chunk
constexpr uint32_t kScBHalf = 256 * kScChunk * 4;           // 32 KB
constexpr uint32_t kScStage = 2 * kScAHalf + 2 * kScBHalf;  // 96 KB
constexpr uint32_t kScStagingOff = 2 * kScStage;            // 192 KB
constexpr uint32_t kScBox = 32 * 128;                       // 32 rows x 32 floats
constexpr uint32_t kScBarOff = kScStagingOff + 4 * 2 * kScBox;  // 224 KB
constexpr uint32_t kScSmem = kScBarOff + 128 + 1024;            // + barriers + alignment
constexpr uint32_t kScTmemCols = 512;                           // two 256-column accumulators

// Instruction descriptor: kind::tf32, f32 accumulate, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 3-D tiled TMA store of one shared-memory box (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// At most one bulk group of this thread still reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Every bulk group of this thread complete.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

struct ScTile {
  long bh;
  int i0, j0;
};

__device__ __forceinline__ ScTile sc_tile(long t, int nbq, int nbk, int ntile) {
  const int mt = (nbq + kScM - 1) / kScM, nt = (nbk + ntile - 1) / ntile;
  ScTile r;
  r.j0 = static_cast<int>(t % nt) * ntile;
  t /= nt;
  r.i0 = static_cast<int>(t % mt) * kScM;
  r.bh = t / mt;
  return r;
}

// grid.x = min(tiles, SMs); S = qbar kbar^T as [B*H, nbq, nbk] float32 (nbq
// query blocks, nbk key blocks or windows; nbq = nbk but for overlapping key
// windows). tm_s describes S as {nbk, nbq, B*H} with 32 x 32 boxes (used when
// tma_store).
// kGroup: grouped queries (H = G * Hkv query heads): the A operand of score
// matrix (b, g) is the mean of the pooled rows of query heads g*G .. g*G+G-1
// (summed in float32, then scaled by 1/G).
template <int NT, bool kGroup>
__global__ void __launch_bounds__(kScThreads, 1)
    block_scores_tc_kernel(const float* __restrict__ qp, const float* __restrict__ kp,
                           float* __restrict__ S, const __grid_constant__ CUtensorMap tm_s, int nbq,
                           int nbk, int D, long ntiles, int tma_store, int H, int Hkv) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int ntile = NT;
  extern __shared__ unsigned char sc_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(sc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScBarOff);  // [2] stage split, count 128
  uint64_t* freed = full + 2;                                      // [2] stage read by the MMAs
  uint64_t* acc_full = full + 4;                                   // [2] accumulator complete
  uint64_t* acc_empty = full + 6;                                  // [2] accumulator drained, count 128
  uint64_t* drained = full + 8;                                    // all MMAs of the CTA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + 10);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int nch = D / kScChunk;
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&freed[s], 1);
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 128);
    }
    mbar_init(drained, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kScMmaWarp) {
    tmem_alloc(tmem_slot, kScTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kScSplitWarps) {
    // ============================================================ load + split
    const int grp = warp / 4, gt = tid % 128;
    constexpr int per = 8 + NT / 16;             // float4 per thread per chunk: 8 of A, 8 or 16 of B
    const int rsub = gt >> 3, q4 = gt & 7;       // row within a 16-row slab, float4 within the 128 B row
    const uint32_t swz = static_cast<uint32_t>(q4 ^ (rsub & 7)) * 16u;  // 128-byte swizzle
    unsigned char* st = smem + grp * kScStage;
    bool ok = true;
    long i = 0;
    for (long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      const ScTile tl = sc_tile(tile, nbq, nbk, ntile);
      // this thread's rows: i0 + rsub + 16 u of qbar, j0 + rsub + 16 u of kbar
      // tl.bh = b * Hkv + g: the query rows of (b, g) start at head g * G of batch b
      const int G = kGroup ? H / Hkv : 1;
      const long qhead = kGroup ? (tl.bh / Hkv) * H + (tl.bh % Hkv) * G : tl.bh;
      const float4* pa = reinterpret_cast<const float4*>(
                             qp + (qhead * nbq + tl.i0 + rsub) * static_cast<long>(D)) + q4;
      const long hstep = static_cast<long>(nbq) * D / 4;  // float4 per query head
      const float4* pb = reinterpret_cast<const float4*>(
                             kp + (tl.bh * nbk + tl.j0 + rsub) * static_cast<long>(D)) + q4;
      const int ra = nbq - tl.i0 - rsub, rb = nbk - tl.j0 - rsub;  // rows left below this thread's first
      const int step = 4 * D;                                   // float4 per 16 rows
      for (int c = 0; c < nch; ++c) {
        const long gi = i * nch + c;  // chunk number within this CTA; stage and group = gi % 2
        if ((gi & 1) != grp) continue;
        float4 v[per];
#pragma unroll
        for (int u = 0; u < per; ++u) {
          const bool is_a = u < 8;
          const int uu = is_a ? u : u - 8;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (16 * uu < (is_a ? ra : rb))
            v[u] = __ldg((is_a ? pa : pb) + uu * step + c * (kScChunk / 4));
          if (kGroup && is_a && 16 * uu < ra) {
            for (int gg = 1; gg < G; ++gg) {
              const float4 w = __ldg(pa + gg * hstep + uu * step + c * (kScChunk / 4));
              v[u].x += w.x;
              v[u].y += w.y;
              v[u].z += w.z;
              v[u].w += w.w;
            }
            const float inv = 1.0f / static_cast<float>(G);
            v[u].x *= inv;
            v[u].y *= inv;
            v[u].z *= inv;
            v[u].w *= inv;
          }
        }
        const long use = gi >> 1;
        if (use > 0) ok = mbar_wait(&freed[grp], static_cast<uint32_t>((use - 1) & 1), abort_flag, 601);
        if (!ok) break;
        const uint32_t m = 0xFFFFE000u;
#pragma unroll
        for (int u = 0; u < per; ++u) {
          const bool is_a = u < 8;
          const int r = rsub + (is_a ? u : u - 8) * 16;
          unsigned char* hi = st + (is_a ? 0u : 2 * kScAHalf);
          unsigned char* lo = hi + (is_a ? kScAHalf : kScBHalf);
          const uint32_t off = static_cast<uint32_t>(r) * 128u + swz;
          float4 h, l;
          h.x = __uint_as_float(__float_as_uint(v[u].x) & m);
          h.y = __uint_as_float(__float_as_uint(v[u].y) & m);
          h.z = __uint_as_float(__float_as_uint(v[u].z) & m);
          h.w = __uint_as_float(__float_as_uint(v[u].w) & m);
          l.x = v[u].x - h.x;
          l.y = v[u].y - h.y;
          l.z = v[u].z - h.z;
          l.w = v[u].w - h.w;
          *reinterpret_cast<float4*>(hi + off) = h;
          *reinterpret_cast<float4*>(lo + off) = l;
        }
        fence_proxy_async_smem();
        mbar_arrive(&full[grp]);
      }
    }
  } else if (warp == kScMmaWarp) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32_f32(kScM, ntile);
      // stage 0 descriptors; the start-address field holds addr >> 4, so
      // stage 1 is a plain add of kScStage >> 4 (addresses stay below 256 KB)
      const uint32_t base = smem_u32(smem);
      const uint64_t dah = smem_desc_sw128(base, 16, 1024);
      const uint64_t dal = smem_desc_sw128(base + kScAHalf, 16, 1024);
      const uint64_t dbh = smem_desc_sw128(base + 2 * kScAHalf, 16, 1024);
      const uint64_t dbl = smem_desc_sw128(base + 2 * kScAHalf + kScBHalf, 16, 1024);
      bool ok = true;
      long i = 0;
      for (long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
        const int buf = static_cast<int>(i & 1);
        if (i >= 2) ok = mbar_wait_fast(&acc_empty[buf], static_cast<uint32_t>(((i >> 1) - 1) & 1), abort_flag, 602);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf) * 256u;
        for (int c = 0; c < nch && ok; ++c) {
          const long gi = i * nch + c;
          const int s = static_cast<int>(gi & 1);
          ok = mbar_wait_fast(&full[s], static_cast<uint32_t>((gi >> 1) & 1), abort_flag, 603);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>(s) * (kScStage >> 4);
#pragma unroll
          for (int kk = 0; kk < kScChunk / 8; ++kk) {
            const uint64_t o = so + ((kk * 32) >> 4);  // 8 floats = 32 bytes along K
            mma_tf32_ss(d, dah + o, dbh + o, idesc, (c > 0 || kk > 0) ? 1u : 0u);
            mma_tf32_ss(d, dah + o, dbl + o, idesc, 1u);
            mma_tf32_ss(d, dal + o, dbh + o, idesc, 1u);
          }
          mma_commit(&freed[s]);
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
      mma_commit(drained);
      mbar_wait_teardown(drained, 0);
    }
    __syncwarp();
  } else {
    // ============================================================ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 = tile rows
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    unsigned char* staging = smem + kScStagingOff + quarter * 2 * kScBox;
    uint32_t nstore = 0;
    bool ok = true;
    long i = 0;
    for (long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      const ScTile tl = sc_tile(tile, nbq, nbk, ntile);
      const int buf = static_cast<int>(i & 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], static_cast<uint32_t>((i >> 1) & 1), abort_flag, 604));
      if (!ok) break;
      tc_fence_after();
      const int row0 = tl.i0 + quarter * 32;
      if (row0 < nbq) {
        for (int cc = 0; cc < ntile / 32; ++cc) {
          const int col0 = tl.j0 + cc * 32;
          if (col0 >= nbk) break;
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + static_cast<uint32_t>(buf * 256 + cc * 32), r);
          tmem_wait_ld();
          if (tma_store) {
            unsigned char* box = staging + (nstore & 1u) * kScBox;
            if (lane == 0) bulk_wait_read_1();  // the store that last read this box is done with it
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                  make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tm_s, box, col0, row0, static_cast<int>(tl.bh));
              bulk_commit_group();
            }
            ++nstore;
          } else {
            const int row = row0 + lane;
            if (row < nbq) {
              float* dst = S + (tl.bh * nbq + row) * static_cast<long>(nbk) + col0;
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (col0 + e < nbk) dst[e] = __uint_as_float(r[e]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kScMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kScTmemCols);
  }
}

}  // namespace bsa
