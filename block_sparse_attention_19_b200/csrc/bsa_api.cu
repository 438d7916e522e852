// bsa_api.cu -- the C ABI declared in include/bsa.h: argument checks,
// workspace layout, tensor-map encoding and kernel launches. The whole library
// is this one translation unit (it includes the kernel headers), so the
// device-side error word has a single definition.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "attn_simt.cuh"
#include "attn_tc2.cuh"
#include "bwd.cuh"
#include "bsa.h"
#include "bsa_ptx.cuh"
#include "pool.cuh"
#include "scores_tc.cuh"
#include "select.cuh"

namespace {

thread_local char g_detail[512] = "";

bsa_status fail(bsa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return s;
}

bsa_status ok() {
  g_detail[0] = '\0';
  return BSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------------ shapes

bsa_status check_dims(int B, int N, int H, int D, int block_size) {
  if (B < 1 || N < 1 || H < 1 || D < 1 || block_size < 1)
    return fail(BSA_ERR_INVALID_ARG, "sizes must be positive (B=%d N=%d H=%d D=%d block_size=%d)",
                B, N, H, D, block_size);
  if (N % block_size != 0)
    return fail(BSA_ERR_INVALID_ARG, "N=%d is not a multiple of block_size=%d", N, block_size);
  if (D != 64 && D != 128) return fail(BSA_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", D);
  if (block_size != 64 && block_size != 128 && block_size != 256)
    return fail(BSA_ERR_UNSUPPORTED, "block_size=%d (supported: 64, 128, 256)", block_size);
  if (static_cast<long long>(B) * H > (1ll << 24) || static_cast<long long>(N) > (1ll << 30))
    return fail(BSA_ERR_UNSUPPORTED, "B*H or N too large for the launch grid");
  return BSA_OK;
}

static_assert(BSA_FLAG_CAUSAL == bsa::kFlagCausal && BSA_FLAG_FORCE_DIAG == bsa::kFlagForceDiag,
              "flag values of the header and the kernels");

// The global-head period carried in bits 8-15 of the flags (0: none).
int global_period(unsigned flags) { return static_cast<int>((flags >> 8) & 0xFFu); }

bsa_status check_flags(unsigned flags) {
  if (flags & ~(BSA_FLAG_CAUSAL | BSA_FLAG_FORCE_DIAG | BSA_FLAG_MAX_POOL | BSA_GLOBAL_HEAD_PERIOD(255)))
    return fail(BSA_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if ((flags & BSA_FLAG_FORCE_DIAG) && !(flags & BSA_FLAG_CAUSAL))
    return fail(BSA_ERR_INVALID_ARG, "BSA_FLAG_FORCE_DIAG needs BSA_FLAG_CAUSAL");
  return BSA_OK;
}

bsa_status check_heads(int H, int Hkv) {
  if (Hkv < 1 || H % Hkv != 0)
    return fail(BSA_ERR_INVALID_ARG, "H=%d must be a positive multiple of H_kv=%d", H, Hkv);
  return BSA_OK;
}

bsa_status check_dtype(bsa_dtype dt) {
  if (dt != BSA_F32 && dt != BSA_BF16 && dt != BSA_E4M3)
    return fail(BSA_ERR_UNSUPPORTED, "dtype %d", static_cast<int>(dt));
  return BSA_OK;
}

// ------------------------------------------------------------------ device

// The kernels are built for sm_100a only.
bsa_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BSA_ERR_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  static int cached_ok[64] = {0};  // 0 unknown, 1 ok, -1 unsupported
  if (dev < 64 && cached_ok[dev] == 1) return BSA_OK;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) {
    if (dev < 64) cached_ok[dev] = -1;
    return fail(BSA_ERR_DEVICE, "device %d is sm_%d%d; libbsa is built for sm_100a", dev, major, minor);
  }
  if (dev < 64) cached_ok[dev] = 1;
  return BSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B, N, H, D] bf16 (or e4m3 with e4m3 = true) tensor as a 4-D TMA map
// {D, H, N, B}; box = 128 bytes of a row (64 bf16 or 128 e4m3 columns) x 1
// head x 64 rows x 1 batch, 128-byte swizzle (the UMMA K-/MN-major layout);
// a row of only 64 bytes (e4m3, D = 64) is one 64-byte box with the 64-byte
// swizzle.
bsa_status make_bnhd_map(CUtensorMap* map, const void* base, int B, int N, int H, int D,
                         bool e4m3 = false) {
  auto encode = tensor_map_encoder();
  if (!encode) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t es = e4m3 ? 1 : 2;
  const cuuint32_t row_bytes = static_cast<cuuint64_t>(D) * es < 128 ? static_cast<cuuint32_t>(D * es) : 128u;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * es, static_cast<cuuint64_t>(H) * D * es,
                           static_cast<cuuint64_t>(N) * H * D * es};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(row_bytes / es), 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return BSA_OK;
}

// ------------------------------------------------------------------ launches

// Launches `kernel` with programmatic stream serialization: it may be
// scheduled while the previous kernel of the stream finishes (the forward
// path's kernels wait for their predecessor on entry, pdl_wait).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// One pooling launch for element type T: the block maxima with max pooling,
// the key windows when `win` (mean only), else the block means.
template <typename T>
cudaError_t launch_pool_t(bool maxp, bool win, unsigned g, unsigned threads, cudaStream_t st, bsa::PoolTask t0,
                          bsa::PoolTask t1, int B, int N, int H, int D, int bs, int cw, int stride, int nwin) {
  if (win)
    return launch_pdl(bsa::block_pool_kernel<T, false, true>, g, threads, 0, st, t0, t1, B, N, H, D, bs, cw, stride,
                      nwin);
  if (maxp)
    return launch_pdl(bsa::block_pool_kernel<T, true>, g, threads, 0, st, t0, t1, B, N, H, D, bs, cw, stride, nwin);
  return launch_pdl(bsa::block_pool_kernel<T>, g, threads, 0, st, t0, t1, B, N, H, D, bs, cw, stride, nwin);
}

// stride > 0 pools overlapping key windows (stride rows apart, nwin of
// them); 0 means the disjoint blocks.
bsa_status launch_pool(const void* x0, float* p0, const void* x1, float* p1, int ntasks, int B,
                       int N, int H, int D, int bs, bsa_dtype dt, unsigned flags, cudaStream_t st,
                       int stride = 0, int nwin = 0) {
  const int V = dt == BSA_F32 ? 4 : (dt == BSA_E4M3 ? 16 : 8);  // elements per 16 bytes
  const int C = H * D / V;
  const int cw = bsa::pool_column_group(C);
  const bool win = stride > 0;
  const long grid = static_cast<long>(ntasks) * B * (win ? nwin : N / bs) * (C / cw);
  if (grid > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "pool grid too large");
  bsa::PoolTask t0{x0, p0}, t1{x1 ? x1 : x0, p1 ? p1 : p0};
  const unsigned g = static_cast<unsigned>(grid);
  const unsigned threads = static_cast<unsigned>(bsa::kPoolRowGroups * cw);
  const bool maxp = (flags & BSA_FLAG_MAX_POOL) != 0;
  cudaError_t e;
  if (dt == BSA_F32)
    e = launch_pool_t<float>(maxp, win, g, threads, st, t0, t1, B, N, H, D, bs, cw, stride, nwin);
  else if (dt == BSA_E4M3)
    e = launch_pool_t<__nv_fp8_e4m3>(maxp, win, g, threads, st, t0, t1, B, N, H, D, bs, cw, stride, nwin);
  else
    e = launch_pool_t<__nv_bfloat16>(maxp, win, g, threads, st, t0, t1, B, N, H, D, bs, cw, stride, nwin);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "block_pool_kernel launch");
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

// Block scores S = qbar kbar^T per (b, h) on the tensor cores (split TF32),
// written to S [B, H, nb, nb] by TMA tensor stores when a row of S is a
// multiple of 16 bytes; then the top-k selection reads S back.
// H query heads, Hkv key/value heads (score matrices); H > Hkv averages each
// group's pooled queries.
bsa_status launch_scores(const float* qp, const float* kp, float* S, int B, int H, int Hkv, int nb,
                         int D, cudaStream_t st, int nbk = 0) {
  if (nbk <= 0) nbk = nb;  // key windows per head (nb but for overlapping windows)
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    for (auto fn : {bsa::block_scores_tc_kernel<128, false>, bsa::block_scores_tc_kernel<256, false>,
                    bsa::block_scores_tc_kernel<128, true>, bsa::block_scores_tc_kernel<256, true>}) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bsa::kScSmem);
      if (e != cudaSuccess) return cuda_fail(e, "scores smem attribute");
    }
    attr_set[dev] = true;
  }
  // 128-wide score tiles up to nb = 256 (256-wide ones would leave most SMs
  // idle there), 256-wide beyond; the choice depends on nb alone, so that a
  // subset of the heads is scored exactly like the whole tensor
  const int ntile = nbk <= 256 ? 128 : 256;
  const long ntiles = static_cast<long>(B) * Hkv * ((nb + bsa::kScM - 1) / bsa::kScM) *
                      ((nbk + ntile - 1) / ntile);
  const int tma_store = (nbk % 4 == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0) ? 1 : 0;
  CUtensorMap tm_s;
  std::memset(&tm_s, 0, sizeof(tm_s));
  if (tma_store) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(nbk), static_cast<cuuint64_t>(nb),
                          static_cast<cuuint64_t>(B) * Hkv};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(nbk) * 4,
                             static_cast<cuuint64_t>(nb) * nbk * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&tm_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, S, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "score tensor map failed (%d)", static_cast<int>(r));
  }
  const long grid = ntiles < sm_count() ? ntiles : sm_count();
  const unsigned gr = static_cast<unsigned>(grid);
  const bool grouped = H != Hkv;
  auto kern = ntile == 128 ? (grouped ? bsa::block_scores_tc_kernel<128, true> : bsa::block_scores_tc_kernel<128, false>)
                            : (grouped ? bsa::block_scores_tc_kernel<256, true> : bsa::block_scores_tc_kernel<256, false>);
  cudaError_t e = launch_pdl(kern, gr, bsa::kScThreads, bsa::kScSmem, st, qp, kp, S, tm_s, nb, nbk, D, ntiles,
                             tma_store, H, Hkv);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "block_scores_tc_kernel launch");
}

// rows = B * H * nbq rows of nb scores each (nbq = nb but for overlapping
// key windows, which are not causal).
bsa_status launch_topk(const float* S, int32_t* idx, int B, int H, int nb, int k, unsigned flags,
                       cudaStream_t st, int nbq = 0) {
  const long rows = static_cast<long>(B) * H * (nbq > 0 ? nbq : nb);
  const long grid = (rows + bsa::kSelWarps - 1) / bsa::kSelWarps;
  if (grid > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "top-k grid too large");
  cudaError_t e;
  if (nb <= 1024) {
    e = launch_pdl(bsa::block_topk_kernel, static_cast<unsigned>(grid), bsa::kSelThreads, 0, st, S, idx, rows, nb,
                   k, flags);
  } else if (nb <= 4096) {
    if (rows > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "top-k grid too large");
    e = launch_pdl(bsa::block_topk_group_kernel, static_cast<unsigned>(rows), bsa::kSelGroupThreads, 0, st, S,
                   idx, rows, nb, k, flags);
  } else {
    // long rows: each warp stages its row's keys in shared memory when they fit
    const size_t stage_bytes = static_cast<size_t>(bsa::kSelWarps) * bsa::staged_row_keys(nb) * sizeof(uint32_t);
    const bool stage = stage_bytes <= 200 * 1024;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
      e = cudaFuncSetAttribute(bsa::block_topk_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      if (e != cudaSuccess) return cuda_fail(e, "top-k smem attribute");
      attr_set[dev] = true;
    }
    e = launch_pdl(bsa::block_topk_wide_kernel, static_cast<unsigned>(grid), bsa::kSelThreads,
                   stage ? stage_bytes : 0, st, S, idx, rows, nb, k, stage ? 1 : 0, flags);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "top-k kernel launch");
}

bsa_status launch_select(const float* qp, const float* kp, float* S, int32_t* idx, int B, int H,
                         int Hkv, int nb, int D, int k, unsigned flags, cudaStream_t st, int nbk = 0) {
  bsa_status s;
  if (nbk <= 0) nbk = nb;
  if ((s = launch_scores(qp, kp, S, B, H, Hkv, nb, D, st, nbk)) != BSA_OK) return s;
  return launch_topk(S, idx, B, Hkv, nbk, k, flags, st, nb);
}

template <int D>
bsa_status launch_attn_simt(const float* q, const float* k, const float* v, const int32_t* idx,
                            float* o, int B, int N, int H, int Hkv, int bs, int kk, float scale,
                            unsigned flags, cudaStream_t st, int ws, int nkb) {
  const size_t smem = sizeof(bsa::SimtSmem<D>);
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bsa::sparse_attn_simt_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "simt smem attribute");
    attr_set[dev] = true;
  }
  const long grid = static_cast<long>(B) * H * (N / bs) * (bs / bsa::kSimtRows);
  if (grid > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "attention grid too large");
  cudaError_t e = launch_pdl(bsa::sparse_attn_simt_kernel<D>, static_cast<unsigned>(grid), bsa::kSimtThreads, smem,
                             st, q, k, v, idx, o, N, H, Hkv, bs, kk, scale, flags, global_period(flags), ws, nkb);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "sparse_attn_simt_kernel launch");
}

template <int D, bool kCausal, bool kF8, bool kStack, bool kVar>
bsa_status launch_attn_tc2_as(const void* q, const void* k, const void* v, const int32_t* idx, void* o,
                              int B, int N, int H, int Hkv, int bs, int kk, float scale,
                              float* lse, int gperiod, int ws, int nkb, cudaStream_t st) {
  using L = bsa::Tc2Layout<D, kF8>;
  CUtensorMap mq, mk, mv;
  bsa_status s;
  if ((s = make_bnhd_map(&mq, q, B, N, H, D, kF8)) != BSA_OK) return s;
  if ((s = make_bnhd_map(&mk, k, B, N, Hkv, D, kF8)) != BSA_OK) return s;
  if ((s = make_bnhd_map(&mv, v, B, N, Hkv, D, kF8)) != BSA_OK) return s;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bsa::sparse_attn_tc2_kernel<D, kCausal, kF8, kStack, kVar>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return cuda_fail(e, "tc2 smem attribute");
    // The kernel moves registers between warp groups (setmaxnreg); an increase
    // that the launch allocation cannot cover would wait forever, so refuse
    // to launch unless the compiled register count covers the split.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, bsa::sparse_attn_tc2_kernel<D, kCausal, kF8, kStack, kVar>);
    if (e != cudaSuccess) return cuda_fail(e, "tc2 attributes");
    if (fa.numRegs < static_cast<int>(bsa::kTc2LaunchRegs))
      return fail(BSA_ERR_UNSUPPORTED, "attention kernel built with %d registers/thread, its register split needs %u",
                  fa.numRegs, bsa::kTc2LaunchRegs);
    attr_set[dev] = true;
  }
  const int nb = N / bs;
  // the kernel's CTA layouts: halves of a 256-block; two query heads of a
  // group on one block (an even group size); two blocks of one head
  // block_size 64: two streams of two stacked query blocks each
  const bool head_pairs = bs == 128 && ((H / Hkv) % 2) == 0 && gperiod == 0;
  const long grid = kStack       ? static_cast<long>(B) * H * ((nb + 3) / 4)
                    : head_pairs ? static_cast<long>(B) * (H / 2) * nb
                                 : static_cast<long>(B) * H * (bs == 256 ? nb : (nb + 1) / 2);
  if (grid > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "attention grid too large");
  const float scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e = launch_pdl(bsa::sparse_attn_tc2_kernel<D, kCausal, kF8, kStack, kVar>, static_cast<unsigned>(grid),
                             bsa::kTc2Threads, L::kBytes, st, mq, mk, mv, idx, static_cast<__nv_bfloat16*>(o), N, H,
                             Hkv, bs, kk, scale_log2, lse, gperiod, ws, nkb);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "sparse_attn_tc2_kernel launch");
}

template <int D, bool kF8 = false, bool kStack = false>
bsa_status launch_attn_tc2(const void* q, const void* k, const void* v, const int32_t* idx, void* o,
                           int B, int N, int H, int Hkv, int bs, int kk, float scale, unsigned flags,
                           float* lse, cudaStream_t st, int ws, int nkb) {
  const int gp = global_period(flags);
  // global heads and overlapping windows run their own instances, so the
  // plain method's kernels carry none of their code
  const bool var = gp > 0 || ws < bs;
#define BSA_TC2_ARGS q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, lse, gp, ws, nkb, st
  if (flags & BSA_FLAG_CAUSAL)
    return var ? launch_attn_tc2_as<D, true, kF8, kStack, true>(BSA_TC2_ARGS)
               : launch_attn_tc2_as<D, true, kF8, kStack, false>(BSA_TC2_ARGS);
  return var ? launch_attn_tc2_as<D, false, kF8, kStack, true>(BSA_TC2_ARGS)
             : launch_attn_tc2_as<D, false, kF8, kStack, false>(BSA_TC2_ARGS);
#undef BSA_TC2_ARGS
}

// ws < bs: index entries name overlapping key windows ws tokens apart (nkb
// of them); 0 means the disjoint blocks.
bsa_status launch_attn(const void* q, const void* k, const void* v, const int32_t* idx, void* o,
                       int B, int N, int H, int Hkv, int D, int bs, int kk, float scale, bsa_dtype dt,
                       unsigned flags, cudaStream_t st, float* lse = nullptr, int ws = 0, int nkb = 0) {
  if (ws <= 0) {
    ws = bs;
    nkb = N / bs;
  }
  if (dt == BSA_F32) {
    const float *fq = static_cast<const float*>(q), *fk = static_cast<const float*>(k),
                *fv = static_cast<const float*>(v);
    float* fo = static_cast<float*>(o);
    return D == 64 ? launch_attn_simt<64>(fq, fk, fv, idx, fo, B, N, H, Hkv, bs, kk, scale, flags, st, ws, nkb)
                   : launch_attn_simt<128>(fq, fk, fv, idx, fo, B, N, H, Hkv, bs, kk, scale, flags, st, ws, nkb);
  }
  if (dt == BSA_E4M3) {
    if (D == 64)
      return bs == 64 ? launch_attn_tc2<64, true, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb)
                      : launch_attn_tc2<64, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb);
    return bs == 64 ? launch_attn_tc2<128, true, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb)
                    : launch_attn_tc2<128, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb);
  }
  if (bs == 64)
    return D == 64 ? launch_attn_tc2<64, false, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb)
                   : launch_attn_tc2<128, false, true>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb);
  return D == 64 ? launch_attn_tc2<64>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb)
                 : launch_attn_tc2<128>(q, k, v, idx, o, B, N, H, Hkv, bs, kk, scale, flags, lse, st, ws, nkb);
}

// Backward: transpose of the selection (bit matrix), D_n, dQ, dK/dV.
struct BwdWorkspace {
  uint32_t* mask;  // [B, Hkv, nb, ceil(nb / 32)]
  float* dsum;     // [B, H, N]
  size_t bytes;
};

BwdWorkspace bwd_workspace_layout(void* base, int B, int N, int H, int Hkv, int bs) {
  const size_t nb = static_cast<size_t>(N / bs), words = (nb + 31) / 32;
  const size_t mb = align256(static_cast<size_t>(B) * Hkv * nb * words * sizeof(uint32_t));
  const size_t db = align256(static_cast<size_t>(B) * H * N * sizeof(float));
  unsigned char* p = static_cast<unsigned char*>(base);
  BwdWorkspace w;
  w.mask = reinterpret_cast<uint32_t*>(p);
  w.dsum = reinterpret_cast<float*>(p + mb);
  w.bytes = mb + db;
  return w;
}

template <int D, bool kCausal, bool kStack>
bsa_status launch_bwd_as(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const int32_t* idx, const float* lse, const BwdWorkspace& w, void* dq, void* dk,
                         void* dv, int B, int N, int H, int Hkv, int bs, int kk, float scale, cudaStream_t st) {
  using L = bsa::BwdLayout<D>;
  CUtensorMap mq, mk, mv, mdo;
  bsa_status s;
  if ((s = make_bnhd_map(&mq, q, B, N, H, D)) != BSA_OK) return s;
  if ((s = make_bnhd_map(&mk, k, B, N, Hkv, D)) != BSA_OK) return s;
  if ((s = make_bnhd_map(&mv, v, B, N, Hkv, D)) != BSA_OK) return s;
  if ((s = make_bnhd_map(&mdo, dO, B, N, H, D)) != BSA_OK) return s;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bsa::bwd_dq_kernel<D, kCausal, kStack>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bsa::bwd_dkdv_kernel<D, kCausal, kStack>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::kBytes);
    if (e != cudaSuccess) return cuda_fail(e, "backward smem attribute");
    attr_set[dev] = true;
  }
  const int nb = N / bs, words = (nb + 31) / 32;
  // 1. the transpose of the selection, as bits
  cudaError_t e = cudaMemsetAsync(w.mask, 0, static_cast<size_t>(B) * Hkv * nb * words * sizeof(uint32_t), st);
  if (e != cudaSuccess) return cuda_fail(e, "backward mask clear");
  const long entries = static_cast<long>(B) * Hkv * nb * kk;
  bsa::bwd_mask_kernel<<<static_cast<unsigned>((entries + 255) / 256), 256, 0, st>>>(idx, w.mask, entries, nb,
                                                                                     kk, words);
  // 2. D_n = dO_n . o_n
  const long rows = static_cast<long>(B) * N * H;
  bsa::bwd_rowdot_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), w.dsum, rows, N, H, D);
  // 3. dQ per query tile, 4. dK and dV per key tile of each key/value head
  // (block_size 64: one tile per pair of blocks, stacked)
  const long tiles_per_bh = kStack ? (nb + 1) / 2 : static_cast<long>(nb) * (bs / 128);
  const long qtiles = static_cast<long>(B) * H * tiles_per_bh;
  const long ktiles = static_cast<long>(B) * Hkv * tiles_per_bh;
  if (qtiles > 0x7fffffffL) return fail(BSA_ERR_UNSUPPORTED, "backward grid too large");
  const float scale_log2 = scale * 1.4426950408889634f;
  bsa::bwd_dq_kernel<D, kCausal, kStack><<<static_cast<unsigned>(qtiles), bsa::kBwdThreads, L::kBytes, st>>>(
      mq, mk, mv, mdo, idx, lse, w.dsum, static_cast<__nv_bfloat16*>(dq), N, H, Hkv, bs, kk, scale, scale_log2);
  bsa::bwd_dkdv_kernel<D, kCausal, kStack><<<static_cast<unsigned>(ktiles), bsa::kBwdThreads, L::kBytes, st>>>(
      mq, mk, mv, mdo, w.mask, lse, w.dsum, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), N,
      H, Hkv, bs, scale, scale_log2);
  e = cudaGetLastError();
  return e == cudaSuccess ? BSA_OK : cuda_fail(e, "backward launches");
}

bsa_status launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                      const int32_t* idx, const float* lse, const BwdWorkspace& w, void* dq, void* dk, void* dv,
                      int B, int N, int H, int Hkv, int D, int bs, int kk, float scale, unsigned flags,
                      cudaStream_t st) {
  const bool causal = (flags & BSA_FLAG_CAUSAL) != 0;
#define BSA_BWD_ARGS q, k, v, o, dO, idx, lse, w, dq, dk, dv, B, N, H, Hkv, bs, kk, scale, st
  if (bs == 64) {
    if (D == 64)
      return causal ? launch_bwd_as<64, true, true>(BSA_BWD_ARGS) : launch_bwd_as<64, false, true>(BSA_BWD_ARGS);
    return causal ? launch_bwd_as<128, true, true>(BSA_BWD_ARGS) : launch_bwd_as<128, false, true>(BSA_BWD_ARGS);
  }
  if (D == 64)
    return causal ? launch_bwd_as<64, true, false>(BSA_BWD_ARGS) : launch_bwd_as<64, false, false>(BSA_BWD_ARGS);
  return causal ? launch_bwd_as<128, true, false>(BSA_BWD_ARGS) : launch_bwd_as<128, false, false>(BSA_BWD_ARGS);
#undef BSA_BWD_ARGS
}

struct Workspace {
  float* qp;
  float* kp;
  int32_t* idx;
  float* scores;
  size_t bytes;
};

// q_pooled [B,H,nb,D] | k_pooled [B,Hkv,nb,D] | idx [B,Hkv,nb,k] | scores
// [B,Hkv,nb,nb], each section 256-byte aligned
Workspace workspace_layout(void* base, int B, int N, int H, int Hkv, int D, int bs, int k) {
  const size_t nb = static_cast<size_t>(N / bs);
  const size_t qpb = align256(static_cast<size_t>(B) * H * nb * D * sizeof(float));
  const size_t kpb = align256(static_cast<size_t>(B) * Hkv * nb * D * sizeof(float));
  const size_t idxb = align256(static_cast<size_t>(B) * Hkv * nb * k * sizeof(int32_t));
  const size_t scb = align256(static_cast<size_t>(B) * Hkv * nb * nb * sizeof(float));
  unsigned char* p = static_cast<unsigned char*>(base);
  Workspace w;
  w.qp = reinterpret_cast<float*>(p);
  w.kp = reinterpret_cast<float*>(p + qpb);
  w.idx = reinterpret_cast<int32_t*>(p + qpb + kpb);
  w.scores = reinterpret_cast<float*>(p + qpb + kpb + idxb);
  w.bytes = qpb + kpb + idxb + scb;
  return w;
}

}  // namespace

// ---- overlapping key windows: window plan, workspace layout, flag checks

namespace {

// ov = int(overlap_ratio * block_size) tokens of overlap (Python int() of the
// double product), windows ws = block_size - ov apart, nbk of them; false if
// the ratio is outside [0, 1) or N < block_size.
bool overlap_plan(int N, int bs, double overlap_ratio, int& ws, int& nbk) {
  if (!std::isfinite(overlap_ratio) || overlap_ratio < 0.0 || overlap_ratio >= 1.0 || N < bs || bs < 1) return false;
  const int ov = static_cast<int>(overlap_ratio * static_cast<double>(bs));
  if (ov < 0 || ov >= bs) return false;
  ws = bs - ov;
  nbk = (N - bs + ws - 1) / ws + 1;
  return true;
}

// q_pooled [B,H,nb,D] | k window means [B,Hkv,nbk,D] | idx [B,Hkv,nb,k] |
// scores [B,Hkv,nb,nbk], each section 256-byte aligned
Workspace overlap_workspace_layout(void* base, int B, int N, int H, int Hkv, int D, int bs, int nbk, int k) {
  const size_t nb = static_cast<size_t>(N / bs);
  const size_t qpb = align256(static_cast<size_t>(B) * H * nb * D * sizeof(float));
  const size_t kpb = align256(static_cast<size_t>(B) * Hkv * nbk * D * sizeof(float));
  const size_t idxb = align256(static_cast<size_t>(B) * Hkv * nb * k * sizeof(int32_t));
  const size_t scb = align256(static_cast<size_t>(B) * Hkv * nb * nbk * sizeof(float));
  unsigned char* p = static_cast<unsigned char*>(base);
  Workspace w;
  w.qp = reinterpret_cast<float*>(p);
  w.kp = reinterpret_cast<float*>(p + qpb);
  w.idx = reinterpret_cast<int32_t*>(p + qpb + kpb);
  w.scores = reinterpret_cast<float*>(p + qpb + kpb + idxb);
  w.bytes = qpb + kpb + idxb + scb;
  return w;
}

bsa_status check_overlap_flags(unsigned flags) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if (flags & (BSA_FLAG_CAUSAL | BSA_FLAG_FORCE_DIAG))
    return fail(BSA_ERR_UNSUPPORTED, "overlapping key windows are not causal");
  if (flags & BSA_FLAG_MAX_POOL) return fail(BSA_ERR_UNSUPPORTED, "overlapping key windows are mean-pooled");
  return BSA_OK;
}

}  // namespace

// ==================================================================== C ABI

extern "C" {

int bsa_topk_count(int nb, double topk_ratio) {
  if (nb < 1 || !std::isfinite(topk_ratio) || topk_ratio < 0.0) return -1;
  const double prod = topk_ratio * static_cast<double>(nb);
  if (prod >= 2147483647.0) return -1;
  return static_cast<int>(prod);  // truncation == Python int() for prod >= 0
}

size_t bsa_forward_gqa_workspace_bytes(int B, int N, int H, int Hkv, int D, int block_size,
                                       double topk_ratio) {
  if (check_dims(B, N, H, D, block_size) != BSA_OK || check_heads(H, Hkv) != BSA_OK) return 0;
  const int k = bsa_topk_count(N / block_size, topk_ratio);
  if (k < 1 || k > N / block_size) return 0;
  return workspace_layout(nullptr, B, N, H, Hkv, D, block_size, k).bytes;
}

size_t bsa_forward_workspace_bytes(int B, int N, int H, int D, int block_size, double topk_ratio) {
  return bsa_forward_gqa_workspace_bytes(B, N, H, H, D, block_size, topk_ratio);
}

const char* bsa_status_string(bsa_status s) {
  switch (s) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported size or type";
    case BSA_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case BSA_ERR_WORKSPACE: return "workspace missing or too small";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_DEVICE: return "no usable sm_100 device";
  }
  return "unknown status";
}

const char* bsa_last_error_detail(void) { return g_detail; }

int bsa_adaptive_block_size(long long seq_len) {
  if (seq_len < 1) return -1;
  if (seq_len < 500000) return 64;
  if (seq_len < 1000000) return 128;
  return 256;
}

bsa_status bsa_block_pool_ex(const void* x, float* x_pooled, int B, int N, int H, int D, int block_size,
                             bsa_dtype dt, unsigned flags, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  if (!x || !x_pooled) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(x_pooled)) return fail(BSA_ERR_MISALIGNED, "x or x_pooled");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_pool(x, x_pooled, nullptr, nullptr, 1, B, N, H, D, block_size, dt, flags,
                       static_cast<cudaStream_t>(stream))) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_block_pool(const void* x, float* x_pooled, int B, int N, int H, int D,
                          int block_size, bsa_dtype dt, void* stream) {
  return bsa_block_pool_ex(x, x_pooled, B, N, H, D, block_size, dt, 0u, stream);
}

bsa_status bsa_block_pool_qk(const void* q, const void* k, float* q_pooled, float* k_pooled, int B, int N, int H,
                             int H_kv, int D, int block_size, bsa_dtype dt, unsigned flags, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, H_kv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  if (!q || !k || !q_pooled || !k_pooled) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pooled) || !aligned16(k_pooled))
    return fail(BSA_ERR_MISALIGNED, "q, k, q_pooled or k_pooled");
  if ((s = check_device()) != BSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (H == H_kv)  // one launch for both tensors, as bsa_forward pools them
    return (s = launch_pool(q, q_pooled, k, k_pooled, 2, B, N, H, D, block_size, dt, flags, st)) != BSA_OK ? s : ok();
  if ((s = launch_pool(q, q_pooled, nullptr, nullptr, 1, B, N, H, D, block_size, dt, flags, st)) != BSA_OK) return s;
  if ((s = launch_pool(k, k_pooled, nullptr, nullptr, 1, B, N, H_kv, D, block_size, dt, flags, st)) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_block_scores_topk_gqa(const float* q_pooled, const float* k_pooled, float* scores,
                                     int32_t* idx, int B, int H, int Hkv, int nb, int D, int k,
                                     unsigned flags, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if (B < 1 || H < 1 || nb < 1) return fail(BSA_ERR_INVALID_ARG, "sizes must be positive");
  if ((s = check_heads(H, Hkv)) != BSA_OK) return s;
  if (D != 64 && D != 128) return fail(BSA_ERR_UNSUPPORTED, "D=%d (supported: 64, 128)", D);
  if (nb > 32768) return fail(BSA_ERR_UNSUPPORTED, "nb=%d > 32768", nb);
  if (k < 1 || k > nb) return fail(BSA_ERR_INVALID_ARG, "k=%d outside [1, nb=%d]", k, nb);
  if (!q_pooled || !k_pooled || !idx || !scores) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q_pooled) || !aligned16(k_pooled) || !aligned16(idx) || !aligned16(scores))
    return fail(BSA_ERR_MISALIGNED, "q_pooled, k_pooled, idx or scores");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_select(q_pooled, k_pooled, scores, idx, B, H, Hkv, nb, D, k, flags,
                         static_cast<cudaStream_t>(stream))) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_block_scores_topk_ex(const float* q_pooled, const float* k_pooled, float* scores,
                                    int32_t* idx, int B, int H, int nb, int D, int k, unsigned flags,
                                    void* stream) {
  return bsa_block_scores_topk_gqa(q_pooled, k_pooled, scores, idx, B, H, H, nb, D, k, flags, stream);
}

bsa_status bsa_block_scores_topk(const float* q_pooled, const float* k_pooled, float* scores,
                                 int32_t* idx, int B, int H, int nb, int D, int k, void* stream) {
  return bsa_block_scores_topk_ex(q_pooled, k_pooled, scores, idx, B, H, nb, D, k, 0u, stream);
}

bsa_status bsa_sparse_attn_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* idx,
                                   void* o, int B, int N, int H, int Hkv, int D, int block_size, int kk,
                                   float scale, bsa_dtype dt, unsigned flags, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, Hkv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  const int nb = N / block_size;
  if (kk < 1 || kk > nb) return fail(BSA_ERR_INVALID_ARG, "k=%d outside [1, nb=%d]", kk, nb);
  if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(BSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (!q || !k || !v || !idx || !o) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o))
    return fail(BSA_ERR_MISALIGNED, "q, k, v, idx or o");
  if (o == q || o == k || o == v) return fail(BSA_ERR_INVALID_ARG, "o aliases an input");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_attn(q, k, v, idx, o, B, N, H, Hkv, D, block_size, kk, scale, dt, flags,
                       static_cast<cudaStream_t>(stream))) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_sparse_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* idx,
                                  void* o, int B, int N, int H, int D, int block_size, int kk,
                                  float scale, bsa_dtype dt, unsigned flags, void* stream) {
  return bsa_sparse_attn_fwd_gqa(q, k, v, idx, o, B, N, H, H, D, block_size, kk, scale, dt, flags, stream);
}

bsa_status bsa_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                               void* o, int B, int N, int H, int D, int block_size, int kk,
                               float scale, bsa_dtype dt, void* stream) {
  return bsa_sparse_attn_fwd_ex(q, k, v, idx, o, B, N, H, D, block_size, kk, scale, dt, 0u, stream);
}

bsa_status bsa_forward_gqa(const void* q, const void* k, const void* v, void* o, int B, int N,
                           int H, int Hkv, int D, int block_size, double topk_ratio, bsa_dtype dt,
                           unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, Hkv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  const int nb = N / block_size;
  if (nb > 32768) return fail(BSA_ERR_UNSUPPORTED, "nb=%d > 32768", nb);
  if (!std::isfinite(topk_ratio) || topk_ratio < 0.0 || topk_ratio > 1.0)
    return fail(BSA_ERR_INVALID_ARG, "topk_ratio=%g outside [0, 1]", topk_ratio);
  const int kk = bsa_topk_count(nb, topk_ratio);
  if (kk < 1) return fail(BSA_ERR_INVALID_ARG, "k = int(%g * %d) = %d < 1", topk_ratio, nb, kk);
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_MISALIGNED, "q, k, v or o");
  if (o == q || o == k || o == v) return fail(BSA_ERR_INVALID_ARG, "o aliases an input");
  const Workspace w = workspace_layout(workspace, B, N, H, Hkv, D, block_size, kk);
  if (!workspace || workspace_bytes < w.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", w.bytes, workspace ? workspace_bytes : 0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(BSA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if ((s = check_device()) != BSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  if (H == Hkv) {
    if ((s = launch_pool(q, w.qp, k, w.kp, 2, B, N, H, D, block_size, dt, flags, st)) != BSA_OK) return s;
  } else {
    if ((s = launch_pool(q, w.qp, nullptr, nullptr, 1, B, N, H, D, block_size, dt, flags, st)) != BSA_OK) return s;
    if ((s = launch_pool(k, w.kp, nullptr, nullptr, 1, B, N, Hkv, D, block_size, dt, flags, st)) != BSA_OK) return s;
  }
  if ((s = launch_select(w.qp, w.kp, w.scores, w.idx, B, H, Hkv, nb, D, kk, flags, st)) != BSA_OK) return s;
  if ((s = launch_attn(q, k, v, w.idx, o, B, N, H, Hkv, D, block_size, kk, scale, dt, flags, st)) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_forward_ex(const void* q, const void* k, const void* v, void* o, int B, int N,
                          int H, int D, int block_size, double topk_ratio, bsa_dtype dt,
                          unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  return bsa_forward_gqa(q, k, v, o, B, N, H, H, D, block_size, topk_ratio, dt, flags, workspace,
                         workspace_bytes, stream);
}

bsa_status bsa_forward(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                       int D, int block_size, double topk_ratio, bsa_dtype dt, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return bsa_forward_ex(q, k, v, o, B, N, H, D, block_size, topk_ratio, dt, 0u, workspace,
                        workspace_bytes, stream);
}

// ---- overlapping key windows

extern "C" int bsa_overlap_window_count(int N, int block_size, double overlap_ratio) {
  int ws = 0, nbk = 0;
  if (N < 1 || block_size < 1 || N % block_size != 0 || !overlap_plan(N, block_size, overlap_ratio, ws, nbk)) return -1;
  return nbk;
}

extern "C" size_t bsa_forward_overlap_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size,
                                                      double topk_ratio, double overlap_ratio) {
  if (check_dims(B, N, H, D, block_size) != BSA_OK || check_heads(H, H_kv) != BSA_OK) return 0;
  int ws = 0, nbk = 0;
  if (!overlap_plan(N, block_size, overlap_ratio, ws, nbk) || nbk > 32768) return 0;
  const int kk = bsa_topk_count(nbk, topk_ratio);
  if (kk < 1 || kk > nbk) return 0;
  return overlap_workspace_layout(nullptr, B, N, H, H_kv, D, block_size, nbk, kk).bytes;
}

extern "C" bsa_status bsa_sparse_attn_fwd_overlap(const void* q, const void* k, const void* v, const int32_t* idx,
                                                  void* o, int B, int N, int H, int H_kv, int D, int block_size,
                                                  int topk, double overlap_ratio, float scale, bsa_dtype dt,
                                                  unsigned flags, void* stream) {
  bsa_status s;
  if ((s = check_overlap_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, H_kv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  int ws = 0, nbk = 0;
  if (!overlap_plan(N, block_size, overlap_ratio, ws, nbk))
    return fail(BSA_ERR_INVALID_ARG, "overlap_ratio=%g outside [0, 1)", overlap_ratio);
  if (topk < 1 || topk > nbk) return fail(BSA_ERR_INVALID_ARG, "k=%d outside [1, nb_k=%d]", topk, nbk);
  if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(BSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (!q || !k || !v || !idx || !o) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o))
    return fail(BSA_ERR_MISALIGNED, "q, k, v, idx or o");
  if (o == q || o == k || o == v) return fail(BSA_ERR_INVALID_ARG, "o aliases an input");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_attn(q, k, v, idx, o, B, N, H, H_kv, D, block_size, topk, scale, dt, flags,
                       static_cast<cudaStream_t>(stream), nullptr, ws, nbk)) != BSA_OK)
    return s;
  return ok();
}

extern "C" bsa_status bsa_forward_overlap(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                                          int H_kv, int D, int block_size, double topk_ratio, double overlap_ratio,
                                          bsa_dtype dt, unsigned flags, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  bsa_status s;
  if ((s = check_overlap_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, H_kv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  int ws = 0, nbk = 0;
  if (!overlap_plan(N, block_size, overlap_ratio, ws, nbk))
    return fail(BSA_ERR_INVALID_ARG, "overlap_ratio=%g outside [0, 1)", overlap_ratio);
  if (nbk > 32768) return fail(BSA_ERR_UNSUPPORTED, "nb_k=%d > 32768", nbk);
  if (!std::isfinite(topk_ratio) || topk_ratio < 0.0 || topk_ratio > 1.0)
    return fail(BSA_ERR_INVALID_ARG, "topk_ratio=%g outside [0, 1]", topk_ratio);
  const int kk = bsa_topk_count(nbk, topk_ratio);
  if (kk < 1) return fail(BSA_ERR_INVALID_ARG, "k = int(%g * %d) = %d < 1", topk_ratio, nbk, kk);
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(BSA_ERR_MISALIGNED, "q, k, v or o");
  if (o == q || o == k || o == v) return fail(BSA_ERR_INVALID_ARG, "o aliases an input");
  const Workspace w = overlap_workspace_layout(workspace, B, N, H, H_kv, D, block_size, nbk, kk);
  if (!workspace || workspace_bytes < w.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", w.bytes, workspace ? workspace_bytes : 0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(BSA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if ((s = check_device()) != BSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nb = N / block_size;
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  if ((s = launch_pool(q, w.qp, nullptr, nullptr, 1, B, N, H, D, block_size, dt, flags, st)) != BSA_OK) return s;
  if ((s = launch_pool(k, w.kp, nullptr, nullptr, 1, B, N, H_kv, D, block_size, dt, flags, st, ws, nbk)) != BSA_OK)
    return s;
  if ((s = launch_select(w.qp, w.kp, w.scores, w.idx, B, H, H_kv, nb, D, kk, flags, st, nbk)) != BSA_OK) return s;
  if ((s = launch_attn(q, k, v, w.idx, o, B, N, H, H_kv, D, block_size, kk, scale, dt, flags, st, nullptr, ws, nbk)) !=
      BSA_OK)
    return s;
  return ok();
}

// ---- training: the forward with the row log-sum-exp, and the backward

// The shapes the training entry points cover: bf16, D in {64, 128},
// block_size 64, 128 or 256, H a multiple of H_kv.
bsa_status check_train(int B, int N, int H, int Hkv, int D, int block_size, int kk, bsa_dtype dt, unsigned flags) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, Hkv)) != BSA_OK) return s;
  if (dt != BSA_BF16) return fail(BSA_ERR_UNSUPPORTED, "training entry points take bf16");
  if (global_period(flags) != 0) return fail(BSA_ERR_UNSUPPORTED, "training entry points have no global heads");
  const int nb = N / block_size;
  if (kk < 1 || kk > nb) return fail(BSA_ERR_INVALID_ARG, "k=%d outside [1, nb=%d]", kk, nb);
  return BSA_OK;
}

bsa_status bsa_sparse_attn_fwd_train_gqa(const void* q, const void* k, const void* v, const int32_t* idx,
                                         void* o, float* lse, int B, int N, int H, int H_kv, int D,
                                         int block_size, int kk, float scale, bsa_dtype dt, unsigned flags,
                                         void* stream) {
  bsa_status s;
  if ((s = check_train(B, N, H, H_kv, D, block_size, kk, dt, flags)) != BSA_OK) return s;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(BSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (!q || !k || !v || !idx || !o || !lse) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) || !aligned16(lse))
    return fail(BSA_ERR_MISALIGNED, "q, k, v, idx, o or lse");
  if (o == q || o == k || o == v) return fail(BSA_ERR_INVALID_ARG, "o aliases an input");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_attn(q, k, v, idx, o, B, N, H, H_kv, D, block_size, kk, scale, dt, flags,
                       static_cast<cudaStream_t>(stream), lse)) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_sparse_attn_fwd_train(const void* q, const void* k, const void* v, const int32_t* idx,
                                     void* o, float* lse, int B, int N, int H, int D, int block_size,
                                     int kk, float scale, bsa_dtype dt, unsigned flags, void* stream) {
  return bsa_sparse_attn_fwd_train_gqa(q, k, v, idx, o, lse, B, N, H, H, D, block_size, kk, scale, dt, flags,
                                       stream);
}

size_t bsa_sparse_attn_bwd_gqa_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size) {
  if (check_dims(B, N, H, D, block_size) != BSA_OK || check_heads(H, H_kv) != BSA_OK) return 0;
  return bwd_workspace_layout(nullptr, B, N, H, H_kv, block_size).bytes;
}

size_t bsa_sparse_attn_bwd_workspace_bytes(int B, int N, int H, int D, int block_size) {
  return bsa_sparse_attn_bwd_gqa_workspace_bytes(B, N, H, H, D, block_size);
}

bsa_status bsa_sparse_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                   const int32_t* idx, const float* lse, void* dq, void* dk, void* dv, int B,
                                   int N, int H, int H_kv, int D, int block_size, int kk, float scale,
                                   bsa_dtype dt, unsigned flags, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  bsa_status s;
  if ((s = check_train(B, N, H, H_kv, D, block_size, kk, dt, flags)) != BSA_OK) return s;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(BSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (!q || !k || !v || !o || !dO || !idx || !lse || !dq || !dk || !dv)
    return fail(BSA_ERR_INVALID_ARG, "null pointer");
  const void* ptrs[] = {q, k, v, o, dO, idx, lse, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(BSA_ERR_MISALIGNED, "a tensor is not 16-byte aligned");
  const void* outs[] = {dq, dk, dv};
  const void* ins[] = {q, k, v, o, dO};
  for (const void* a : outs)
    for (const void* b : ins)
      if (a == b) return fail(BSA_ERR_INVALID_ARG, "a gradient aliases an input");
  const BwdWorkspace w = bwd_workspace_layout(workspace, B, N, H, H_kv, block_size);
  if (!workspace || workspace_bytes < w.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", w.bytes, workspace ? workspace_bytes : 0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(BSA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if ((s = check_device()) != BSA_OK) return s;
  if ((s = launch_bwd(q, k, v, o, dO, idx, lse, w, dq, dk, dv, B, N, H, H_kv, D, block_size, kk, scale, flags,
                      static_cast<cudaStream_t>(stream))) != BSA_OK)
    return s;
  return ok();
}

bsa_status bsa_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                               const int32_t* idx, const float* lse, void* dq, void* dk, void* dv, int B,
                               int N, int H, int D, int block_size, int kk, float scale, bsa_dtype dt,
                               unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  return bsa_sparse_attn_bwd_gqa(q, k, v, o, dO, idx, lse, dq, dk, dv, B, N, H, H, D, block_size, kk, scale, dt,
                                 flags, workspace, workspace_bytes, stream);
}

bsa_status bsa_device_error(int* code_out, void* stream) {
  if (!code_out) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  bsa_status s;
  if ((s = check_device()) != BSA_OK) return s;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int code = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&code, bsa::g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  e = cudaMemcpyToSymbol(bsa::g_device_error, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
  *code_out = code;
  return ok();
}

}  // extern "C"

// ==================================================================== forward without allocation
//
// bsa_forward needs a workspace (pooled q, pooled k, the index list and the
// block-score matrix) that the caller allocates. Some callers cannot allocate device memory at all: a
// plugin running inside a host application that owns the whole device-memory
// budget, or a latency-critical loop where a cudaMalloc (and the implicit
// device synchronisation it may bring) is not allowed. bsa_forward_noalloc
// serves them from a fixed scratch array that is part of the library image.
//
// The array below lives in device memory of every GPU that loads this
// library, from module load until process exit. Host code must not use its
// name as a device address (on the host it is only a stand-in symbol): the
// device address is looked up once per device with cudaGetSymbolAddress.

static __device__ __align__(256) unsigned char g_noalloc_scratch[BSA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};
unsigned long long g_noalloc_ctx[64] = {};  // id of the context the address belongs to

// Unique id of the current context (cuCtxGetId: ids are never reused within
// a process), 0 when it cannot be read.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device. The lookup
// (with that device current) runs on the first call on each device and again
// whenever the device's context has changed since (a cudaDeviceReset destroys
// the context and the next one loads the module anew, possibly elsewhere);
// when the context id cannot be read, it runs on every call.
bsa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(BSA_ERR_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(BSA_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  // 0 when no context is current yet: the lookup below then creates it
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context_id();  // the context the address belongs to
  }
  *out = g_noalloc_ptr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" bsa_status bsa_forward_noalloc(const void* q, const void* k, const void* v, void* o,
                                          int B, int N, int H, int D, int block_size,
                                          double topk_ratio, bsa_dtype dt, void* stream) {
  bsa_status s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if (!std::isfinite(topk_ratio) || topk_ratio < 0.0 || topk_ratio > 1.0)
    return fail(BSA_ERR_INVALID_ARG, "topk_ratio=%g outside [0, 1]", topk_ratio);
  const size_t need = bsa_forward_workspace_bytes(B, N, H, D, block_size, topk_ratio);
  if (need == 0) return fail(BSA_ERR_INVALID_ARG, "k = int(topk_ratio * nb) < 1");
  if (need > static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES))
    return fail(BSA_ERR_WORKSPACE,
                "these sizes need %zu bytes of scratch; the built-in scratch holds %zu bytes "
                "(use bsa_forward with a caller-provided workspace)",
                need, static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES));
  if ((s = check_device()) != BSA_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != BSA_OK) return s;
  // Nothing in the scratch has to start at zero: every byte the forward's
  // kernels read was written earlier in the same call.
  return bsa_forward(q, k, v, o, B, N, H, D, block_size, topk_ratio, dt, scratch,
                     static_cast<size_t>(BSA_NOALLOC_SCRATCH_BYTES), stream);
}

// ---- the whole path from host buffers, copies overlapped with the compute

namespace {

size_t elem_bytes(bsa_dtype dt) { return dt == BSA_F32 ? 4 : (dt == BSA_BF16 ? 2 : 1); }
size_t out_elem_bytes(bsa_dtype dt) { return dt == BSA_F32 ? 4 : 2; }  // e4m3 inputs give bf16 o

// The job is cut into chunks of (one batch entry, gc consecutive key/value
// heads with their G query heads each): independent problems, each held on
// the device as compact [1, N, heads, D] tensors. Two chunk slots let the
// copies of one chunk run while the other computes.
constexpr size_t kHostChunkBytes = size_t(64) << 20;  // aim: at least this much input+output per chunk

struct HostPlan {
  int gc = 0, chunks = 0, slots = 0;
  size_t q = 0, kv = 0, o = 0, ws = 0, slot = 0, bytes = 0;
};

HostPlan host_plan(int B, int N, int H, int Hkv, int D, int bs, double ratio, bsa_dtype dt) {
  HostPlan p;
  const int G = H / Hkv;
  const size_t es = elem_bytes(dt), oes = out_elem_bytes(dt);
  const size_t per_g = static_cast<size_t>(N) * D * (G * es + 2 * es + G * oes);
  p.gc = Hkv;
  for (int gc = 1; gc <= Hkv; ++gc)
    if (Hkv % gc == 0 && static_cast<size_t>(gc) * per_g >= kHostChunkBytes) {
      p.gc = gc;
      break;
    }
  p.chunks = B * (Hkv / p.gc);
  p.slots = p.chunks > 1 ? 2 : 1;
  p.q = align256(static_cast<size_t>(N) * G * p.gc * D * es);
  p.kv = align256(static_cast<size_t>(N) * p.gc * D * es);
  p.o = align256(static_cast<size_t>(N) * G * p.gc * D * oes);
  p.ws = align256(bsa_forward_gqa_workspace_bytes(1, N, G * p.gc, p.gc, D, bs, ratio));
  p.slot = p.q + 2 * p.kv + p.o + p.ws;
  p.bytes = p.ws == 0 ? 0 : p.slots * p.slot;
  return p;
}

// Per device: the copy-in and copy-out streams and the events that order the
// chunk slots (guarded by g_host_mu while a call enqueues its work).
struct HostStreams {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, end = nullptr, in[2] = {}, comp[2] = {}, out[2] = {};
};
HostStreams g_host[64];
std::mutex g_host_mu;

bsa_status host_streams(int dev, HostStreams** out) {
  HostStreams& h = g_host[dev];
  if (!h.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&h.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h.d2h, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&h.start, &h.end, &h.in[0], &h.in[1], &h.comp[0], &h.comp[1], &h.out[0], &h.out[1]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "host-path streams and events");
    h.ready = true;
  }
  *out = &h;
  return BSA_OK;
}

// The N token rows of a head group as one 2-D copy: `width` bytes per token,
// rows `spitch` bytes apart in the source and `dpitch` in the destination.
cudaError_t copy_heads(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width, int N,
                       cudaMemcpyKind kind, cudaStream_t st) {
  return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, static_cast<size_t>(N), kind, st);
}

}  // namespace

extern "C" size_t bsa_forward_host_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size,
                                                   double topk_ratio, bsa_dtype dt) {
  if (check_dtype(dt) != BSA_OK) return 0;
  if (check_dims(B, N, H, D, block_size) != BSA_OK || check_heads(H, H_kv) != BSA_OK) return 0;
  return host_plan(B, N, H, H_kv, D, block_size, topk_ratio, dt).bytes;
}

extern "C" bsa_status bsa_forward_host(const void* q, const void* k, const void* v, void* o, int B, int N,
                                       int H, int H_kv, int D, int block_size, double topk_ratio, bsa_dtype dt,
                                       unsigned flags, void* workspace, size_t workspace_bytes, void* stream) {
  bsa_status s;
  if ((s = check_flags(flags)) != BSA_OK) return s;
  if ((s = check_dims(B, N, H, D, block_size)) != BSA_OK) return s;
  if ((s = check_heads(H, H_kv)) != BSA_OK) return s;
  if ((s = check_dtype(dt)) != BSA_OK) return s;
  if (!q || !k || !v || !o) return fail(BSA_ERR_INVALID_ARG, "null pointer");
  const HostPlan p = host_plan(B, N, H, H_kv, D, block_size, topk_ratio, dt);
  if (p.bytes == 0) return fail(BSA_ERR_INVALID_ARG, "k = int(topk_ratio * nb) < 1 or topk_ratio outside [0, 1]");
  if (!workspace || workspace_bytes < p.bytes)
    return fail(BSA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", p.bytes, workspace ? workspace_bytes : 0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(BSA_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  if ((s = check_device()) != BSA_OK) return s;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(BSA_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostStreams* hs = nullptr;
  if ((s = host_streams(dev, &hs)) != BSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = H / H_kv, groups = H_kv / p.gc;
  const size_t es = elem_bytes(dt), oes = out_elem_bytes(dt);
  // host rows: one token of all heads; chunk rows: one token of the chunk's heads
  const size_t q_row = static_cast<size_t>(H) * D * es, kv_row = static_cast<size_t>(H_kv) * D * es;
  const size_t o_row = static_cast<size_t>(H) * D * oes;
  const size_t cq_row = static_cast<size_t>(G) * p.gc * D * es, ckv_row = static_cast<size_t>(p.gc) * D * es;
  const size_t co_row = static_cast<size_t>(G) * p.gc * D * oes;
  // the internal streams start after the work already on `stream`
  if ((e = cudaEventRecord(hs->start, st)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = cudaStreamWaitEvent(hs->h2d, hs->start, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  if ((e = cudaStreamWaitEvent(hs->d2h, hs->start, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  for (int c = 0; c < p.chunks; ++c) {
    const int sl = c % p.slots, b = c / groups, g0 = (c % groups) * p.gc;
    unsigned char* base = static_cast<unsigned char*>(workspace) + sl * p.slot;
    unsigned char *dq = base, *dk = base + p.q, *dv = dk + p.kv, *dout = dv + p.kv, *dws = dout + p.o;
    const size_t tok = static_cast<size_t>(b) * N;  // first token row of batch entry b
    const unsigned char* hq = static_cast<const unsigned char*>(q) + tok * q_row + static_cast<size_t>(g0) * G * D * es;
    const unsigned char* hk = static_cast<const unsigned char*>(k) + tok * kv_row + static_cast<size_t>(g0) * D * es;
    const unsigned char* hv = static_cast<const unsigned char*>(v) + tok * kv_row + static_cast<size_t>(g0) * D * es;
    unsigned char* ho = static_cast<unsigned char*>(o) + tok * o_row + static_cast<size_t>(g0) * G * D * oes;
    // copy in once the slot's previous chunk has been computed
    if (c >= p.slots && (e = cudaStreamWaitEvent(hs->h2d, hs->comp[sl], 0)) != cudaSuccess)
      return cuda_fail(e, "stream wait");
    if ((e = copy_heads(dq, cq_row, hq, q_row, cq_row, N, cudaMemcpyHostToDevice, hs->h2d)) != cudaSuccess ||
        (e = copy_heads(dk, ckv_row, hk, kv_row, ckv_row, N, cudaMemcpyHostToDevice, hs->h2d)) != cudaSuccess ||
        (e = copy_heads(dv, ckv_row, hv, kv_row, ckv_row, N, cudaMemcpyHostToDevice, hs->h2d)) != cudaSuccess)
      return cuda_fail(e, "host to device copy");
    if ((e = cudaEventRecord(hs->in[sl], hs->h2d)) != cudaSuccess) return cuda_fail(e, "event record");
    // compute once the inputs are in and the slot's previous output is out
    if ((e = cudaStreamWaitEvent(st, hs->in[sl], 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
    if (c >= p.slots && (e = cudaStreamWaitEvent(st, hs->out[sl], 0)) != cudaSuccess)
      return cuda_fail(e, "stream wait");
    if ((s = bsa_forward_gqa(dq, dk, dv, dout, 1, N, G * p.gc, p.gc, D, block_size, topk_ratio, dt, flags, dws,
                             p.ws, st)) != BSA_OK)
      return s;
    if ((e = cudaEventRecord(hs->comp[sl], st)) != cudaSuccess) return cuda_fail(e, "event record");
    // copy out
    if ((e = cudaStreamWaitEvent(hs->d2h, hs->comp[sl], 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
    if ((e = copy_heads(ho, o_row, dout, co_row, co_row, N, cudaMemcpyDeviceToHost, hs->d2h)) != cudaSuccess)
      return cuda_fail(e, "device to host copy");
    if ((e = cudaEventRecord(hs->out[sl], hs->d2h)) != cudaSuccess) return cuda_fail(e, "event record");
  }
  // `stream` continues after the last output copy
  if ((e = cudaEventRecord(hs->end, hs->d2h)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = cudaStreamWaitEvent(st, hs->end, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
  return ok();
}
