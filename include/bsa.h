/*
 * bsa.h -- C ABI of libbsa: two-stage block-sparse attention on NVIDIA B200
 * (sm_100a).
 *
 * The method (page "2026 新一代卷积与 Transformer 网络架构", qqiyuan.cn,
 * section "SparseFormer 注意力实现"; page "从M2.7到M3：多模态模型稀疏注意力架构
 * 设计与实现全解析", cloud.baidu.com, §2.1-§2.2):
 *   1. mean-pool q and k over blocks of block_size tokens and score every query
 *      block against every key block: S[b,h,i,j] = qbar[b,h,i,:] . kbar[b,h,j,:];
 *   2. keep, per (b, h, query block i), the k = floor(topk_ratio * nb) key
 *      blocks with the largest scores (ties go to the lower block index);
 *   3. for every query row n of block i, o[n] = softmax(scale * q[n] K_sel^T) V_sel
 *      with K_sel / V_sel the k * block_size rows of the kept blocks and
 *      scale = 1/sqrt(D) by default. Attention is non-causal.
 *
 * Conventions for every entry point:
 *   - Tensors are dense and row-major. q, k, v, o are [B, N, H, D] (the head
 *     axis inside the token axis, as the "SparseFormer 注意力实现" section takes them); pooled
 *     tensors are [B, H, nb, D] float32; index lists are [B, H, nb, k] int32,
 *     each row strictly ascending by key-block id.
 *   - All pointers are DEVICE pointers unless stated otherwise. The caller owns
 *     every buffer; the library allocates nothing on any call and keeps no
 *     pointer after a call returns.
 *   - Every device pointer must be 16-byte aligned (BSA_ERR_MISALIGNED).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Work is enqueued asynchronously; a call returns once its kernels
 *     are launched. Faults inside a kernel surface at the caller's next
 *     synchronisation; bsa_device_error() reports bounded-wait timeouts.
 *   - Argument errors are detected on the host before anything is launched and
 *     leave all buffers untouched. bsa_last_error_detail() then describes the
 *     error (thread-local, valid until the next call on the same thread).
 *   - Supported sizes: D in {64, 128}; block_size in {64, 128, 256};
 *     N a multiple of block_size; 1 <= k <= nb; B, H >= 1. Offsets are
 *     64-bit, so tensor sizes are bounded only by device memory.
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, N % block_size != 0, k out of range */
  BSA_ERR_UNSUPPORTED = 2, /* D / block_size / dtype / size outside what the kernels implement */
  BSA_ERR_MISALIGNED = 3,  /* a device pointer not 16-byte aligned */
  BSA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than bsa_forward_workspace_bytes() */
  BSA_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  BSA_ERR_DEVICE = 6       /* no usable sm_100 device for this call */
} bsa_status;

typedef enum {
  BSA_F32 = 0, /* float32 q/k/v/o; attention in float32 on CUDA cores */
  BSA_BF16 = 1, /* bfloat16 q/k/v/o; attention on tcgen05 tensor cores, float32 accumulate */
  /* FP8 E4M3 q/k/v with bfloat16 o (page "2026 新一代卷积与 Transformer 网络架构",
   * section "基准测试": SparseFormer run in FP8; its closing advice: use FP8
   * tensor cores). The stored e4m3 values are the inputs (a caller with
   * scaled FP8 folds the q and k scales into `scale` and multiplies o by the
   * v scale). Both products run as tcgen05 kind::f8f6f4 with float32
   * accumulation; the softmax weights P are rounded to e4m3 (round to
   * nearest, saturating) for the P.V product, the row sums use float32 P.
   * D = 64 and 128. */
  BSA_E4M3 = 2
} bsa_dtype;

/* Number of kept key blocks: floor(topk_ratio * nb) evaluated in IEEE double,
 * which equals the Python int() of that product that page "2026 新一代卷积与
 * Transformer 网络架构" (section "SparseFormer 注意力实现", step 2) uses. Returns -1 if nb < 1 or topk_ratio is negative or not finite.
 * Pure host function. */
int bsa_topk_count(int nb, double topk_ratio);

/* Bytes of device workspace bsa_forward() needs for these sizes: pooled q,
 * pooled k, the index list and the [B, H, nb, nb] float32 block-score matrix,
 * in that order, each section 256-byte aligned. Returns 0 when the arguments
 * are invalid. Pure host function. */
size_t bsa_forward_workspace_bytes(int B, int N, int H, int D, int block_size, double topk_ratio);

/* Step 1a (page "2026 新一代卷积与 Transformer 网络架构", section "SparseFormer
 * 注意力实现", step 1: the mean of each block of block_size consecutive tokens,
 * per batch entry and head):
 *   x_pooled[b, h, i, d] = (1/block_size) * sum_{t<block_size} x[b, i*block_size + t, h, d]
 * x: [B, N, H, D] of dtype dt (read only). x_pooled: [B, H, nb, D] float32
 * (written). Sums are accumulated in float32. */
bsa_status bsa_block_pool(const void* x, float* x_pooled, int B, int N, int H, int D,
                          int block_size, bsa_dtype dt, void* stream);

/* Step 1a for q and k together: q_pooled [B, H, nb, D] and k_pooled
 * [B, H_kv, nb, D] as bsa_block_pool_ex writes them (H a multiple of H_kv;
 * flags as for bsa_block_pool_ex). One kernel launch when H = H_kv (the
 * pooling bsa_forward runs), two otherwise. */
bsa_status bsa_block_pool_qk(const void* q, const void* k, float* q_pooled, float* k_pooled, int B, int N, int H,
                             int H_kv, int D, int block_size, bsa_dtype dt, unsigned flags, void* stream);

/* Steps 1b + 2 (same page and section, steps 1 and 2: the dot product of every
 * pooled query block with every pooled key block of the same (b, h), then the
 * topk largest of each row):
 *   S[b, h, i, j] = sum_d q_pooled[b, h, i, d] * k_pooled[b, h, j, d]
 *   idx[b, h, i, :] = the topk key blocks j with the largest S[b, h, i, j],
 *                     ties to the lower j, written in ascending j.
 * q_pooled, k_pooled: [B, H, nb, D] float32 (read). scores: [B, H, nb, nb]
 * float32 (written with S; the selection then reads it back). idx:
 * [B, H, nb, topk] int32 (written). S is computed on the tensor cores with
 * float32 accuracy (each operand split into two TF32 parts, three products
 * accumulated in float32); there is no 1/sqrt(D) factor (it would not change
 * the ranking). Two kernel launches. */
bsa_status bsa_block_scores_topk(const float* q_pooled, const float* k_pooled, float* scores,
                                 int32_t* idx, int B, int H, int nb, int D, int topk, void* stream);

/* Step 3 (same page and section, step 3: softmax attention of each query row
 * over the tokens of its block's kept key blocks, with a given scale): for
 * every (b, h, query block i) and every row n of that block,
 *   o[b, n, h, :] = sum_t softmax_t(scale * q[b,n,h,:] . k[b,t,h,:]) v[b,t,h,:]
 * over the tokens t of the key blocks idx[b, h, i, 0..topk).
 * q, k, v: [B, N, H, D] of dtype dt (read). idx: [B, H, nb, topk] int32 with
 * entries in [0, nb) and each row strictly ascending (read; a negative entry
 * ends its row, as in bsa_sparse_attn_fwd_ex, and entries >= nb are clamped
 * by the kernel). o: [B, N, H, D] of dtype dt (written);
 * o must not alias q, k or v. scale: softmax scale (> 0, finite). */
bsa_status bsa_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                               void* o, int B, int N, int H, int D, int block_size, int topk,
                               float scale, bsa_dtype dt, void* stream);

/* The whole path: bsa_block_pool on q and k, bsa_block_scores_topk (scores in
 * the workspace), bsa_sparse_attn_fwd with scale = 1/sqrt(D); four kernel
 * launches on `stream`, no host synchronisation. k = bsa_topk_count(N / block_size,
 * topk_ratio) must be >= 1. workspace: device buffer of at least
 * bsa_forward_workspace_bytes(...) bytes, 256-byte aligned, owned by the caller
 * and not used concurrently by another call. */
bsa_status bsa_forward(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                       int D, int block_size, double topk_ratio, bsa_dtype dt, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Block size for an input length (page "从M2.7到M3：多模态模型稀疏注意力架构设计与
 * 实现全解析" §4.2, dynamic block selection): 64 below 500,000 tokens, 128
 * below 1,000,000, else 256. Returns -1 for seq_len < 1. Pure host function. */
int bsa_adaptive_block_size(long long seq_len);

/* ---- Variants (flags of the _ex entry points) -------------------------
 * The base entry points above are the _ex ones with flags = 0.
 *
 * BSA_FLAG_CAUSAL: the causal variant. Page "从M2.7到M3：多模态模型稀疏注意力
 *   架构设计与实现全解析" §2.1 writes the attention as
 *   Softmax(Mask(QK^T/sqrt(d_k)))V; with a causal mask the readings are:
 *   - selection: query block i ranks only key blocks j <= i and keeps
 *     n_i = min(topk, i + 1) of them; its index row lists them ascending and
 *     pads the remaining topk - n_i entries with -1;
 *   - attention: query token n never sees key token t > n (so, of the kept
 *     blocks, only the diagonal block i is masked token by token).
 * BSA_FLAG_FORCE_DIAG (with BSA_FLAG_CAUSAL): block i is always kept and the
 *   other n_i - 1 are the highest-scoring blocks j < i.
 * Other bits (beyond those defined below) are reserved and rejected
 * (BSA_ERR_INVALID_ARG). */
#define BSA_FLAG_CAUSAL 1u
#define BSA_FLAG_FORCE_DIAG 2u
/* BSA_FLAG_MAX_POOL: blocks are pooled by their element-wise maximum over
 *   the block's rows instead of the mean, for q and k alike (page "从M2.7到M3：
 *   多模态模型稀疏注意力架构设计与实现全解析" §2.2, comparison table: block-based
 *   methods such as MSA/MoBA score a block by its block-internal extreme
 *   value). Read by the pooling step (bsa_block_pool_ex and the whole-path
 *   entry points); the score, selection and attention steps are unchanged
 *   and ignore it. Composes with the causal flags. */
#define BSA_FLAG_MAX_POOL 4u
/* BSA_GLOBAL_HEAD_PERIOD(p), p in 1..255 (bits 8-15 of the flags): global
 *   attention heads (page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §5.3:
 *   one global head in every four, against losses at block boundaries).
 *   Reading: query head h is global when h % p == 0 and attends to every key
 *   block (with BSA_FLAG_CAUSAL: every block j <= i, token-masked as usual),
 *   reading no index row; the other heads attend over their selection.
 *   Read by the attention step (and the whole-path entry points, which still
 *   select blocks for every head); the training entry points refuse it
 *   (BSA_ERR_UNSUPPORTED). p = 1 makes every head dense. */
#define BSA_GLOBAL_HEAD_PERIOD(p) ((((unsigned)(p)) & 0xFFu) << 8)

/* bsa_block_pool with variant flags: BSA_FLAG_MAX_POOL pools by the
 * element-wise block maximum (x_pooled[b, h, i, d] = max_t x[b, i*block_size
 * + t, h, d], exact); the causal flags do not change pooling. */
bsa_status bsa_block_pool_ex(const void* x, float* x_pooled, int B, int N, int H, int D, int block_size,
                             bsa_dtype dt, unsigned flags, void* stream);

/* bsa_block_scores_topk with variant flags (see above). With
 * BSA_FLAG_CAUSAL, scores is still written in full (all nb x nb entries). */
bsa_status bsa_block_scores_topk_ex(const float* q_pooled, const float* k_pooled, float* scores,
                                    int32_t* idx, int B, int H, int nb, int D, int topk,
                                    unsigned flags, void* stream);

/* bsa_sparse_attn_fwd with variant flags. idx rows may end in -1 entries
 * (rows as bsa_block_scores_topk_ex writes them): a row's valid entries are
 * its leading entries >= 0, which must be strictly ascending, and a row needs
 * at least one (a row of only -1 reads block 0). With BSA_FLAG_CAUSAL, key
 * token t is left out of the softmax of query token n when t > n; the caller
 * is responsible for keeping blocks j <= i (the kernel masks tokens, it does
 * not check the list). */
bsa_status bsa_sparse_attn_fwd_ex(const void* q, const void* k, const void* v, const int32_t* idx,
                                  void* o, int B, int N, int H, int D, int block_size, int topk,
                                  float scale, bsa_dtype dt, unsigned flags, void* stream);

/* bsa_forward with variant flags; same workspace. */
bsa_status bsa_forward_ex(const void* q, const void* k, const void* v, void* o, int B, int N,
                          int H, int D, int block_size, double topk_ratio, bsa_dtype dt,
                          unsigned flags, void* workspace, size_t workspace_bytes, void* stream);

/* ---- Grouped-query attention ------------------------------------------
 * Page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §3.1: the MSA attention
 * block is GQA-based. Readings: q (and o) have H heads, k and v have H_kv
 * heads, H = G * H_kv; query head h reads key/value head h / G. Each
 * key/value head has one block selection per query block, scored with the
 * group's pooled query: the mean over its G query heads of their block means
 * (equal, by linearity, to the mean of the G heads' block scores); every
 * query head of the group then attends over that selection. H_kv = H is the
 * plain method (the _ex entry points are these with H_kv = H). Flags as for
 * the _ex entry points. Error codes as for the plain entry points, plus
 * BSA_ERR_INVALID_ARG when H is not a positive multiple of H_kv. */

/* Workspace bytes of bsa_forward_gqa: pooled q [B, H, nb, D], pooled k
 * [B, H_kv, nb, D], the index list [B, H_kv, nb, topk] and the block scores
 * [B, H_kv, nb, nb] (float32). 0 if the arguments are invalid. */
size_t bsa_forward_gqa_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size,
                                       double topk_ratio);

/* q_pooled: [B, H, nb, D] float32 (the per-head block means, as
 * bsa_block_pool writes them). k_pooled: [B, H_kv, nb, D]. scores:
 * [B, H_kv, nb, nb] float32 (written: S[b, g] = qbar_g kbar_g^T with qbar_g
 * the group mean, summed in float32 and scaled by 1/G). idx:
 * [B, H_kv, nb, topk] int32 (written). */
bsa_status bsa_block_scores_topk_gqa(const float* q_pooled, const float* k_pooled, float* scores,
                                     int32_t* idx, int B, int H, int H_kv, int nb, int D, int topk,
                                     unsigned flags, void* stream);

/* q, o: [B, N, H, D]; k, v: [B, N, H_kv, D]; idx: [B, H_kv, nb, topk] (the
 * selection of each key/value head, rows as bsa_sparse_attn_fwd_ex reads
 * them). With an even G and block_size 128, two query heads of a group are
 * computed together and share every gathered key/value tile. */
bsa_status bsa_sparse_attn_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* idx,
                                   void* o, int B, int N, int H, int H_kv, int D, int block_size,
                                   int topk, float scale, bsa_dtype dt, unsigned flags, void* stream);

/* The whole path with grouped queries: pooling of q (H heads) and k (H_kv),
 * scores and selection per key/value head, attention per query head; four
 * or five kernel launches on `stream`. */
bsa_status bsa_forward_gqa(const void* q, const void* k, const void* v, void* o, int B, int N,
                           int H, int H_kv, int D, int block_size, double topk_ratio, bsa_dtype dt,
                           unsigned flags, void* workspace, size_t workspace_bytes, void* stream);

/* ---- Overlapping key windows ------------------------------------------
 * Page "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析" §5.3: overlapping blocks
 * (overlap_ratio = 0.25) against losses at block boundaries. Readings: key
 * blocks become windows of block_size tokens that overlap by
 * ov = int(overlap_ratio * block_size) tokens, i.e. window e starts at token
 * min(e * (block_size - ov), N - block_size) (the last window ends at token
 * N); there are nb_k = ceil((N - block_size) / (block_size - ov)) + 1 of
 * them. Query blocks stay the disjoint blocks of block_size tokens. Each
 * window is scored by its mean key, k = int(topk_ratio * nb_k) windows are
 * kept per query block (ties to the lower window, ascending), and each query
 * row attends to the union of the kept windows' tokens (a token two kept
 * windows share counts once). overlap_ratio in [0, 1); 0 is the plain
 * method. Not causal (BSA_FLAG_CAUSAL and BSA_FLAG_MAX_POOL return
 * BSA_ERR_UNSUPPORTED); global heads (BSA_GLOBAL_HEAD_PERIOD) attend to
 * every token as usual. H a multiple of H_kv as in the _gqa entry points. */

/* nb_k for these sizes, or -1 if N % block_size != 0 or overlap_ratio is
 * outside [0, 1). Pure host function. */
int bsa_overlap_window_count(int N, int block_size, double overlap_ratio);

/* Workspace bytes of bsa_forward_overlap: pooled q [B, H, nb, D], window
 * means of k [B, H_kv, nb_k, D], the index list [B, H_kv, nb, k] and the
 * scores [B, H_kv, nb, nb_k] (float32), each section 256-byte aligned; 0 if
 * the arguments are invalid. */
size_t bsa_forward_overlap_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size,
                                           double topk_ratio, double overlap_ratio);

/* The attention step over overlapping key windows: idx [B, H_kv, nb, topk]
 * holds window ids in [0, nb_k) (ascending; a negative entry ends its row),
 * the rest as bsa_sparse_attn_fwd_gqa. */
bsa_status bsa_sparse_attn_fwd_overlap(const void* q, const void* k, const void* v, const int32_t* idx,
                                       void* o, int B, int N, int H, int H_kv, int D, int block_size,
                                       int topk, double overlap_ratio, float scale, bsa_dtype dt,
                                       unsigned flags, void* stream);

/* The whole path with overlapping key windows: pooling of q (blocks) and of
 * k (windows), scores [nb x nb_k] and selection per key/value head, the
 * attention; five kernel launches on `stream`. */
bsa_status bsa_forward_overlap(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                               int H_kv, int D, int block_size, double topk_ratio, double overlap_ratio,
                               bsa_dtype dt, unsigned flags, void* workspace, size_t workspace_bytes,
                               void* stream);

/* ---- The whole path from host memory ----------------------------------
 * bsa_forward_gqa on HOST buffers: q [B, N, H, D], k and v [B, N, H_kv, D]
 * and o [B, N, H, D] live in host memory (page-locked memory lets the copies
 * run asynchronously). The (batch entry, key/value head) problems are
 * independent, so the job is cut into chunks of one batch entry and a group
 * of consecutive key/value heads (with their query heads), sized to at least
 * 64 MB of inputs and output where the head count allows. Each chunk is
 * copied into a compact device slot on an internal copy-in stream, computed
 * on `stream` exactly as bsa_forward_gqa computes it (the same kernels, so
 * the same results bit for bit), and copied out on an internal copy-out
 * stream; two slots let the copies of one chunk overlap the compute of the
 * other. Work already on `stream` is finished before the first copy, and
 * `stream` resumes after the last output copy: synchronize `stream` before
 * reading o. The host buffers must stay valid until then.
 * workspace: device memory of bsa_forward_host_workspace_bytes() bytes,
 * 256-byte aligned (the chunk slots: q, k, v, o copies and a forward
 * workspace each). Calls on one device are serialized while they enqueue
 * (the internal streams are per device). Errors as for bsa_forward_gqa;
 * argument errors return before anything is enqueued, but a CUDA error
 * returned after the first chunk may leave earlier copies and kernels
 * running on the internal streams, so synchronize the device before reusing
 * the buffers after such an error. */
size_t bsa_forward_host_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size,
                                        double topk_ratio, bsa_dtype dt);

bsa_status bsa_forward_host(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                            int H_kv, int D, int block_size, double topk_ratio, bsa_dtype dt, unsigned flags,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ---- Training: forward with the row log-sum-exp, and the backward -------
 * Step 2 of the "SparseFormer 注意力实现" section keeps blocks by a top-k, whose indices
 * carry no gradient, so the backward is the gradient of step 3 (the
 * attention over the kept blocks) with the index lists held fixed. Per query
 * token n and kept key token t (p = softmax weight, o = output):
 *   D_n = dO_n . o_n,  dS = p (dO_n . v_t - D_n),
 *   dq_n = scale sum_t dS k_t,  dk_t = scale sum_n dS q_n,  dv_t = sum_n p dO_n.
 * Covered shapes: dt = BSA_BF16, D = 64 or 128, block_size 64, 128 or 256
 * (others: BSA_ERR_UNSUPPORTED; block_size 64 stacks two blocks per 128-row
 * tile as the forward does); H a multiple of H_kv in the _gqa forms, where query
 * head h reads key/value head h / (H / H_kv) and that head's selection (idx
 * [B, H_kv, nb, topk], as bsa_sparse_attn_fwd_gqa reads it), and dk, dv sum
 * over the group's query heads. Flags: as for the _ex entry points
 * (BSA_FLAG_CAUSAL masks as in the forward). */

/* bsa_sparse_attn_fwd_ex that also writes lse [B, H, N] float32 (written):
 * ln sum_t exp(scale q_n . k_t) over the row's kept (unmasked) key tokens. */
bsa_status bsa_sparse_attn_fwd_train(const void* q, const void* k, const void* v, const int32_t* idx,
                                     void* o, float* lse, int B, int N, int H, int D, int block_size,
                                     int topk, float scale, bsa_dtype dt, unsigned flags, void* stream);

/* The same with grouped queries: q, o, lse per query head ([B, N, H, D],
 * [B, H, N]); k, v [B, N, H_kv, D]; idx [B, H_kv, nb, topk]. */
bsa_status bsa_sparse_attn_fwd_train_gqa(const void* q, const void* k, const void* v, const int32_t* idx,
                                         void* o, float* lse, int B, int N, int H, int H_kv, int D,
                                         int block_size, int topk, float scale, bsa_dtype dt, unsigned flags,
                                         void* stream);

/* Workspace bytes of bsa_sparse_attn_bwd: the transpose of the selection as
 * a bit matrix [B, H, nb, ceil(nb / 32)] and D [B, H, N] float32. */
size_t bsa_sparse_attn_bwd_workspace_bytes(int B, int N, int H, int D, int block_size);

/* Workspace bytes of bsa_sparse_attn_bwd_gqa: the bit matrix per key/value
 * head [B, H_kv, nb, ceil(nb / 32)] and D [B, H, N] float32. */
size_t bsa_sparse_attn_bwd_gqa_workspace_bytes(int B, int N, int H, int H_kv, int D, int block_size);

/* Gradients dq, dk, dv ([B, N, H, D] bf16, written) of the attention of
 * bsa_sparse_attn_fwd_train, given q, k, v, its output o and lse, the output
 * gradient dO ([B, N, H, D] bf16) and the same idx, scale and flags. Four
 * kernel launches (and one memset) on `stream`: the transpose of idx, D, dQ
 * (one CTA per 128-row query tile over its kept key tiles) and dK/dV (one
 * CTA per 128-key tile over the query tiles that kept its block; a key block
 * no query block kept gets zero gradients). The gradients must not alias the
 * inputs. Deterministic: every sum has a fixed order. */
bsa_status bsa_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                               const int32_t* idx, const float* lse, void* dq, void* dk, void* dv, int B,
                               int N, int H, int D, int block_size, int topk, float scale, bsa_dtype dt,
                               unsigned flags, void* workspace, size_t workspace_bytes, void* stream);

/* The same with grouped queries: dq [B, N, H, D]; dk, dv [B, N, H_kv, D],
 * each the sum over the G = H / H_kv query heads of its group (one CTA per
 * 128-key tile of a key/value head walks the kept query tiles of all G heads
 * in turn, so the sum keeps a fixed order). */
bsa_status bsa_sparse_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                   const int32_t* idx, const float* lse, void* dq, void* dk, void* dv, int B,
                                   int N, int H, int H_kv, int D, int block_size, int topk, float scale,
                                   bsa_dtype dt, unsigned flags, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* Size of the fixed device scratch that bsa_forward_noalloc uses: 64 MiB. */
#define BSA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* bsa_forward without a caller workspace, for callers that cannot allocate
 * device memory (for example a plugin inside a host application that owns the
 * whole device-memory budget, or a loop where cudaMalloc and its implicit
 * synchronisation are not allowed). The pages have no counterpart of this
 * entry point; it only changes where the intermediates live.
 *
 * Arguments and results are those of bsa_forward minus the workspace. The
 * whole bsa_forward workspace -- pooled q, pooled k, the index list and the
 * [B, H, nb, nb] float32 block-score matrix, which is most of it (B*H*nb^2*4
 * bytes: 64 MiB is reached at B*H*nb^2 = 2^24, e.g. 16 heads at nb = 1024) --
 * goes to a fixed 256-byte aligned array of BSA_NOALLOC_SCRATCH_BYTES in the
 * library's device image: every GPU that loads libbsa holds it until the
 * process exits. Sizes whose workspace (bsa_forward_workspace_bytes) exceeds
 * it return BSA_ERR_WORKSPACE before anything is launched. The call
 * allocates nothing (no cudaMalloc/cudaFree).
 * The first call on each device (and the first call after the device's
 * context was destroyed, e.g. by cudaDeviceReset, which reloads the module
 * and may move the array) looks up the array's device address
 * (cudaGetSymbolAddress, with that device current), so make that first call
 * before any stream capture. All calls on a device share the one array and
 * it keeps the last call's contents (nothing in it needs to start at zero):
 * calls that may overlap on the GPU (different streams, or concurrent host
 * threads) race on it and must be serialised by the caller. */
bsa_status bsa_forward_noalloc(const void* q, const void* k, const void* v, void* o, int B, int N,
                               int H, int D, int block_size, double topk_ratio, bsa_dtype dt,
                               void* stream);

/* Static description of a status code. */
const char* bsa_status_string(bsa_status s);

/* Detail of the last error returned on this thread ("" if none). */
const char* bsa_last_error_detail(void);

/* Reads and clears the device-side error word of the current device: 0 when no
 * kernel gave up on a bounded wait since the last call, otherwise the code of
 * the first wait that timed out. Synchronises `stream` first. */
bsa_status bsa_device_error(int* code_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
