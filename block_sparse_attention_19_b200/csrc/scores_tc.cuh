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
// product reads) and lo = x - hi (exact in float32); the product is taken as
// hi.hi + hi.lo + lo.hi, dropping lo.lo (relative size 2^-22) and the TF32
// truncation of lo (2^-11 of lo), accumulated in float32 in TMEM. The error
// per score is below about 2^-20 * sum_d |qbar_d kbar_d|, far inside float32
// FFMA's own worst-case bound of D * 2^-24 * sum_d |qbar_d kbar_d| for D >= 64.
//
// One CTA (4 warps) computes a 128 x 256 tile of S for one (b, h). The pooled
// rows are read as float32 in 32-column chunks, split by the threads and
// written to shared memory in the 128-byte-swizzled K-major layout; one
// thread issues 3 x 4 tcgen05.mma (kind::tf32, K = 8 each) per chunk while
// the threads already load the next chunk; the accumulator is read back from
// TMEM one row per thread and written to S through a swizzled shared-memory
// transpose so that whole rows are stored coalesced. Rows or columns beyond nb
// are zero operands and are not written.
#pragma once

#include <stdint.h>

#include "bsa_ptx.cuh"

namespace bsa {

constexpr int kScThreads = 128;
constexpr int kScM = 128, kScN = 256, kScChunk = 32;  // tile rows, tile columns, d per chunk
constexpr uint32_t kScAHalf = kScM * kScChunk * 4;     // 16 KB: A hi (or lo) of one chunk
constexpr uint32_t kScBHalf = kScN * kScChunk * 4;     // 32 KB
constexpr uint32_t kScSmem = 2 * kScAHalf + 2 * kScBHalf + 1024 + 64;  // + alignment + barrier

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

// Splits the float4 at src into hi / lo halves and writes them at byte
// offset `off` of the hi and lo buffers.
__device__ __forceinline__ void split_store(float4 v, unsigned char* hi, unsigned char* lo,
                                            uint32_t off) {
  const uint32_t m = 0xFFFFE000u;
  float4 h, l;
  h.x = __uint_as_float(__float_as_uint(v.x) & m);
  h.y = __uint_as_float(__float_as_uint(v.y) & m);
  h.z = __uint_as_float(__float_as_uint(v.z) & m);
  h.w = __uint_as_float(__float_as_uint(v.w) & m);
  l.x = v.x - h.x;
  l.y = v.y - h.y;
  l.z = v.z - h.z;
  l.w = v.w - h.w;
  *reinterpret_cast<float4*>(hi + off) = h;
  *reinterpret_cast<float4*>(lo + off) = l;
}

// grid.x = B * H * ceil(nb / 128) * ceil(nb / 256)
__global__ void __launch_bounds__(kScThreads, 1)
    block_scores_tc_kernel(const float* __restrict__ qp, const float* __restrict__ kp,
                           float* __restrict__ S, int nb, int D) {
  extern __shared__ unsigned char sc_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(sc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* a_hi = smem;
  unsigned char* a_lo = a_hi + kScAHalf;
  unsigned char* b_hi = a_lo + kScAHalf;
  unsigned char* b_lo = b_hi + kScBHalf;
  uint64_t* done = reinterpret_cast<uint64_t*>(b_lo + kScBHalf);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(done + 2);

  const int mt = (nb + kScM - 1) / kScM, ntl = (nb + kScN - 1) / kScN;
  long u = blockIdx.x;
  const int tn = static_cast<int>(u % ntl);
  u /= ntl;
  const int tm = static_cast<int>(u % mt);
  const long bh = u / mt;
  const int i0 = tm * kScM, j0 = tn * kScN;
  const float* qbase = qp + bh * nb * static_cast<long>(D);
  const float* kbase = kp + bh * nb * static_cast<long>(D);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  if (tid == 0) {
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kScN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_tf32_f32(kScM, kScN);
  const uint64_t dah = smem_desc_sw128(smem_u32(a_hi), 16, 1024);
  const uint64_t dal = smem_desc_sw128(smem_u32(a_lo), 16, 1024);
  const uint64_t dbh = smem_desc_sw128(smem_u32(b_hi), 16, 1024);
  const uint64_t dbl = smem_desc_sw128(smem_u32(b_lo), 16, 1024);
  bool ok = true;

  const int nchunks = D / kScChunk;
  // Each thread moves 24 float4 per chunk (8 of A, 16 of B). All of a
  // chunk's loads are issued before any is used, and the next chunk's loads
  // are issued while the tensor core works on the current one.
  constexpr int kPer = (kScM + kScN) * (kScChunk / 4) / kScThreads;  // 24
  float4 v[kPer];
  auto load_chunk = [&](int c) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kScThreads;
      const bool is_a = e < kScM * (kScChunk / 4);
      const int ee = is_a ? e : e - kScM * (kScChunk / 4);
      const int r = ee / (kScChunk / 4), q4 = ee % (kScChunk / 4);
      const int grow = (is_a ? i0 : j0) + r;
      v[u] = grow < nb ? __ldg(reinterpret_cast<const float4*>((is_a ? qbase : kbase) +
                                                               static_cast<long>(grow) * D + c * kScChunk) + q4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_chunk(0);
  for (int c = 0; c < nchunks; ++c) {
    if (c > 0) {
      // the previous chunk's products must have read shared memory; the
      // outcome is agreed by the whole CTA, which has barriers below
      ok = __syncthreads_and(mbar_wait(done, (c - 1) & 1, abort_flag, 501));
      if (!ok) break;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kScThreads;
      const bool is_a = e < kScM * (kScChunk / 4);
      const int ee = is_a ? e : e - kScM * (kScChunk / 4);
      const int r = ee / (kScChunk / 4), q4 = ee % (kScChunk / 4);
      const uint32_t off = r * 128 + ((q4 ^ (r & 7)) * 16);  // 128-byte swizzle
      if (is_a)
        split_store(v[u], a_hi, a_lo, off);
      else
        split_store(v[u], b_hi, b_lo, off);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kScChunk / 8; ++kk) {
        const uint64_t o = (kk * 32) >> 4;  // 8 floats = 32 bytes along K
        const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
        mma_tf32_ss(tmem, dah + o, dbh + o, idesc, acc);
        mma_tf32_ss(tmem, dah + o, dbl + o, idesc, 1u);
        mma_tf32_ss(tmem, dal + o, dbh + o, idesc, 1u);
      }
      mma_commit(done);
    }
    __syncwarp();
    if (c + 1 < nchunks) load_chunk(c + 1);
  }
  {
    const bool w = ok ? mbar_wait(done, (nchunks - 1) & 1, abort_flag, 502) : false;
    ok = __syncthreads_and(w);
  }
  if (ok) {
    // Epilogue through shared memory (the operand buffers are free now): each
    // thread writes its row's 128 accumulators of one half of the tile with a
    // 16-byte XOR swizzle, then each warp writes whole rows out coalesced.
    tc_fence_after();
    float* stage = reinterpret_cast<float*>(smem);  // [128 rows][128 floats], 64 KB
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      __syncthreads();  // previous half copied out
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(lane_base + half * 128 + cc * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int chunk = cc * 8 + q;  // 16-byte chunk of the 512-byte row
          *reinterpret_cast<float4*>(stage + row * 128 + ((chunk ^ (row & 31)) * 4)) =
              make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                          __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        }
      }
      __syncthreads();
      const int col0 = j0 + half * 128;
      for (int rr = warp; rr < kScM; rr += kScThreads / 32) {
        if (i0 + rr >= nb) break;
        float* dst = S + (bh * nb + i0 + rr) * static_cast<long>(nb) + col0;
        const float4 w = *reinterpret_cast<const float4*>(stage + rr * 128 + ((lane ^ (rr & 31)) * 4));
        const int col = col0 + lane * 4;
        if ((nb & 3) == 0 && col + 4 <= nb) {
          *reinterpret_cast<float4*>(dst + lane * 4) = w;
        } else {
          const float e4[4] = {w.x, w.y, w.z, w.w};
          for (int e = 0; e < 4; ++e)
            if (col + e < nb) dst[lane * 4 + e] = e4[e];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kScN);
  }
}

}  // namespace bsa
