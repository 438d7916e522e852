// pool.cuh -- step 1a: block mean-pooling of q and k.
//
// Page "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
// "SparseFormer 注意力实现", step 1: the mean over each block of block_size
// tokens, per batch entry and head, of q and of k. Output layout here is
// head-major [B, H, nb, D] float32 so that each (b, h) score matrix reads
// contiguous rows. With kMax the pooled vector is the element-wise maximum
// over the block's rows instead (page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析"
// §2.2: block-based methods score blocks by their block-internal extreme
// value); the maximum of stored values is exact.
//
// HBM-bound: every element of q and k is read exactly once with 16-byte
// vector loads; the block's rows for all heads are contiguous in memory
// (bs * H * D elements), so a work item is (tensor, b, block i, column group)
// and its warps stream whole 512-byte row segments. Sums are float32.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace bsa {

constexpr int kPoolThreads = 256;
// Rows of a block are split over this many row groups whatever the row width
// (the host launches kPoolRowGroups * cw threads), so every block mean is
// summed in the same order for any number of heads: the host-buffer path
// pools one head group at a time and must match the whole tensor.
constexpr int kPoolRowGroups = 4;

struct PoolTask {
  const void* x;  // [B, N, H, D]
  float* xp;      // [B, H, nb, D]
};

// Accumulation of one element: a sum (mean pooling) or a maximum.
template <bool kMax>
__device__ __forceinline__ void pool_acc(float& a, float x) {
  if constexpr (kMax) a = fmaxf(a, x);
  else a += x;
}

template <typename T>
struct Vec16;  // 16 bytes of T, converted to floats and accumulated
template <>
struct Vec16<float> {
  static constexpr int kN = 4;
  template <bool kMax>
  __device__ __forceinline__ static void add(float* acc, const uint4& u) {
    pool_acc<kMax>(acc[0], __uint_as_float(u.x));
    pool_acc<kMax>(acc[1], __uint_as_float(u.y));
    pool_acc<kMax>(acc[2], __uint_as_float(u.z));
    pool_acc<kMax>(acc[3], __uint_as_float(u.w));
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kN = 8;
  template <bool kMax>
  __device__ __forceinline__ static void add(float* acc, const uint4& u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      pool_acc<kMax>(acc[2 * t], __uint_as_float(w[t] << 16));
      pool_acc<kMax>(acc[2 * t + 1], __uint_as_float(w[t] & 0xFFFF0000u));
    }
  }
};

template <>
struct Vec16<__nv_fp8_e4m3> {
  static constexpr int kN = 16;
  template <bool kMax>
  __device__ __forceinline__ static void add(float* acc, const uint4& u) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      __nv_fp8x4_e4m3 x;
      x.__x = w[t];
      const float4 f = static_cast<float4>(x);  // exact: byte 0 -> .x
      pool_acc<kMax>(acc[4 * t], f.x);
      pool_acc<kMax>(acc[4 * t + 1], f.y);
      pool_acc<kMax>(acc[4 * t + 2], f.z);
      pool_acc<kMax>(acc[4 * t + 3], f.w);
    }
  }
};

// Columns (16-byte units) one work item covers: the largest divisor of the
// row width up to kPoolThreads / kPoolRowGroups = 64.
inline int pool_column_group(int C) {
  int cw = C < kPoolThreads / kPoolRowGroups ? C : kPoolThreads / kPoolRowGroups;
  while (C % cw) --cw;
  return cw;
}

// grid.x = ntasks * B * nb * (C / cw), blockDim.x = kPoolRowGroups * cw. Each
// CTA reduces bs rows of one group of cw 16-byte columns of one block; row r
// goes to row group r % kPoolRowGroups, and the groups' partial sums are
// added in group order. kWin: item i is the key window of rows
// min(i * stride, N - bs) .. + bs - 1 (stride < bs: overlapping windows, the
// last one ending at row N), one of nwin; otherwise block i of the N / bs
// disjoint blocks (stride and nwin unused: measured 8% faster on c4 than the
// general form, which keeps the plain method on its own instance).
template <typename T, bool kMax = false, bool kWin = false>
__global__ void __launch_bounds__(kPoolThreads)
    block_pool_kernel(PoolTask t0, PoolTask t1, int B, int N, int H, int D, int bs, int cw, int stride,
                      int nwin) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int V = Vec16<T>::kN;
  const int nb = kWin ? nwin : N / bs;
  const int C = H * D / V;  // 16-byte columns per row
  const int ngroups = C / cw;
  const int G = blockDim.x / cw;  // kPoolRowGroups (read at run time: the compiled loop is faster)

  long item = blockIdx.x;
  const int cg = static_cast<int>(item % ngroups);
  item /= ngroups;
  const int i = static_cast<int>(item % nb);
  item /= nb;
  const int b = static_cast<int>(item % B);
  const int which = static_cast<int>(item / B);
  const PoolTask task = which == 0 ? t0 : t1;

  const int tid = threadIdx.x;
  const int col = tid % cw;
  const int rg = tid / cw;
  const int c = cg * cw + col;  // 16-byte column within the row

  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = kMax ? -INFINITY : 0.f;

  if (rg < G) {
    const size_t row0 = kWin ? static_cast<size_t>(min(i * stride, N - bs)) : static_cast<size_t>(i) * bs;
    const uint4* base = reinterpret_cast<const uint4*>(task.x) + (static_cast<size_t>(b) * N + row0) * C + c;
    int r = rg;
    // 4 independent loads in flight per thread
    for (; r + 3 * G < bs; r += 4 * G) {
      uint4 u0 = __ldg(base + static_cast<size_t>(r) * C);
      uint4 u1 = __ldg(base + static_cast<size_t>(r + G) * C);
      uint4 u2 = __ldg(base + static_cast<size_t>(r + 2 * G) * C);
      uint4 u3 = __ldg(base + static_cast<size_t>(r + 3 * G) * C);
      Vec16<T>::template add<kMax>(acc, u0);
      Vec16<T>::template add<kMax>(acc, u1);
      Vec16<T>::template add<kMax>(acc, u2);
      Vec16<T>::template add<kMax>(acc, u3);
    }
    for (; r < bs; r += G) Vec16<T>::template add<kMax>(acc, __ldg(base + static_cast<size_t>(r) * C));
  }

  // combine the row groups
  __shared__ float part[kPoolThreads * V];
  if (rg < G) {
#pragma unroll
    for (int e = 0; e < V; ++e) part[(rg * cw + col) * V + e] = acc[e];
  }
  __syncthreads();
  if (rg == 0) {
    for (int g = 1; g < G; ++g)
#pragma unroll
      for (int e = 0; e < V; ++e) pool_acc<kMax>(acc[e], part[(g * cw + col) * V + e]);
    const float inv = kMax ? 1.0f : 1.0f / static_cast<float>(bs);  // bs is a power of two: exact
    const int h = (c * V) / D;
    const int d0 = (c * V) % D;
    float* out = task.xp + ((static_cast<size_t>(b) * H + h) * nb + i) * D + d0;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(out + e) =
          make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
  }
}

}  // namespace bsa
