/*
 * bsa_oracle.c -- float64 CPU oracle for two-stage block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference definition that the
 * CUDA library is checked against.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it; no product code path calls it.
 * It shares no code, header or constant with the CUDA library.
 *
 * Sources (web pages; cited by title and section):
 *   [SF]  "2026 新一代卷积与 Transformer 网络架构" (qqiyuan.cn), section
 *         "SparseFormer 注意力实现": block_sparse_attention(q, k, v,
 *         block_size=64, topk_ratio=0.3) with q/k/v of shape [B, N, H, D];
 *         step 1 mean-pools q and k over blocks and forms block scores,
 *         step 2 keeps int(topk_ratio * num_blocks) key blocks per query
 *         block with torch.topk, step 3 runs attention over the kept blocks
 *         with scale = 1/sqrt(D).
 *   [MSA] "从M2.7到M3：多模态模型稀疏注意力架构设计与实现全解析"
 *         (cloud.baidu.com), §2.1 (Attention = Softmax(Mask(QK^T/sqrt(d_k)))V)
 *         and §2.2 (coarse block scoring, then full attention inside the
 *         chosen blocks).
 *
 * Readings where the pages are silent or garbled (each one is listed in the
 * design notes as well):
 *   - The [SF] einsum 'bhid,bhjd->bhij' is applied to the pooled tensors
 *     after moving the head axis next to the batch axis, so the scores are
 *     per (b, h) and of size nb x nb, as the comment on step 1 states.
 *   - The block score carries no 1/sqrt(D) factor (the [SF] code has none);
 *     a positive factor would not change the ranking anyway.
 *   - Pooled means are kept in float64 (no rounding to the input type).
 *   - Ties in the top-k go to the lower key-block index; each selected list
 *     is emitted in ascending block order.
 *   - Attention is non-causal.
 *
 * Every function works in float64.  Inputs may be float32, bfloat16 (raw
 * 16-bit patterns), FP8 E4M3 (raw bytes) or float64; each element is
 * converted exactly to double.
 * Parallelism (OpenMP) is only over independent output rows; the arithmetic
 * inside a row follows the definition in plain order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F64 2
#define ORACLE_E4M3 3

/* FP8 E4M3 (the "fn" variant: no infinities): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 holds subnormals (m / 8 * 2^-6); the
 * pattern with every exponent and mantissa bit set is NaN. */
double oracle_e4m3_to_double(uint8_t x) {
  int sign = x >> 7, e = (x >> 3) & 15, m = x & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Exact conversion of one stored element to double. */
static double elem(const void* base, int dtype, size_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
  if (dtype == ORACLE_F64) return ((const double*)base)[i];
  if (dtype == ORACLE_E4M3) return oracle_e4m3_to_double(((const uint8_t*)base)[i]);
  /* bfloat16: the high 16 bits of an IEEE float32. */
  uint32_t bits = ((uint32_t)((const uint16_t*)base)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Offset of element (b, n, h, d) of a contiguous [B, N, H, D] tensor. */
static size_t at_bnhd(int N, int H, int D, int b, int n, int h, int d) {
  return (((size_t)b * N + n) * H + h) * D + d;
}

/* [SF] step 2: k = int(topk_ratio * num_blocks), Python int() of a double. */
int oracle_topk_count(int nb, double topk_ratio) {
  double prod = topk_ratio * (double)nb;
  if (!(prod >= 0.0)) return -1;
  return (int)prod; /* truncation toward zero == Python int() for prod >= 0 */
}

/* [SF] step 1 (q.view(B, nb, bs, H, D).mean(2)):
 * xp[b, h, i, d] = (1/bs) * sum_{t < bs} x[b, i*bs + t, h, d].
 * Output layout [B, H, nb, D]. */
void oracle_block_pool(const void* x, int dtype, int B, int N, int H, int D, int bs,
                       double* xp) {
  int nb = N / bs;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i)
        for (int d = 0; d < D; ++d) {
          double s = 0.0;
          for (int t = 0; t < bs; ++t) s += elem(x, dtype, at_bnhd(N, H, D, b, i * bs + t, h, d));
          xp[(((size_t)b * H + h) * nb + i) * D + d] = s / (double)bs;
        }
}

/* Max-pooled variant ([MSA] §2.2, the comparison table: block-based methods
 * such as MSA/MoBA score blocks by their "block-internal extreme value").
 * Reading: the pooled vector of a block is its element-wise maximum over
 * the block's block_size rows, for q and k alike, in place of the mean:
 * xp[b, h, i, d] = max_{t < bs} x[b, i*bs + t, h, d]. Output [B, H, nb, D]. */
void oracle_block_pool_max(const void* x, int dtype, int B, int N, int H, int D, int bs, double* xp) {
  int nb = N / bs;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i)
        for (int d = 0; d < D; ++d) {
          double m = elem(x, dtype, at_bnhd(N, H, D, b, i * bs, h, d));
          for (int t = 1; t < bs; ++t) {
            double e = elem(x, dtype, at_bnhd(N, H, D, b, i * bs + t, h, d));
            if (e > m) m = e;
          }
          xp[(((size_t)b * H + h) * nb + i) * D + d] = m;
        }
}

/* [MSA] §4.2 (performance tuning, dynamic block selection): the block size
 * chosen from the input length: 64 below 500,000 tokens, 128 below
 * 1,000,000, else 256. Returns -1 for a length below 1. */
int oracle_adaptive_block_size(long long seq_len) {
  if (seq_len < 1) return -1;
  if (seq_len < 500000) return 64;
  if (seq_len < 1000000) return 128;
  return 256;
}

/* [SF] step 1 (einsum of pooled q and pooled k, per (b, h)):
 * S[b, h, r, j] = sum_d qp[b, h, rows[b,h,r], d] * kp[b, h, j, d]
 * for the nrows query blocks listed per (b, h) in rows[B, H, nrows]
 * (rows == NULL means all nb query blocks, nrows == nb). */
void oracle_block_scores(const double* qp, const double* kp, int B, int H, int nb, int D,
                         const int* rows, int nrows, double* S) {
#pragma omp parallel for collapse(3) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int r = 0; r < nrows; ++r) {
        size_t bh = (size_t)b * H + h;
        int i = rows ? rows[bh * nrows + r] : r;
        const double* qi = qp + (bh * nb + i) * D;
        for (int j = 0; j < nb; ++j) {
          const double* kj = kp + (bh * nb + j) * D;
          double s = 0.0;
          for (int d = 0; d < D; ++d) s += qi[d] * kj[d];
          S[(bh * nrows + r) * nb + j] = s;
        }
      }
}

/* Ordering for the top-k: larger score first, equal scores by lower index. */
typedef struct {
  double s;
  int j;
} scored_block;

static int by_score_then_index(const void* a, const void* b) {
  const scored_block* x = (const scored_block*)a;
  const scored_block* y = (const scored_block*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

static int ascending_int(const void* a, const void* b) {
  int x = *(const int*)a, y = *(const int*)b;
  return (x > y) - (x < y);
}

/* [SF] step 2 for one row: the k key blocks with the largest scores (ties to
 * the lower block index), written to idx[0..k) in ascending block order. */
void oracle_topk_row(const double* s_row, int nb, int k, int* idx) {
  scored_block* order = (scored_block*)malloc((size_t)nb * sizeof(scored_block));
  for (int j = 0; j < nb; ++j) {
    order[j].s = s_row[j];
    order[j].j = j;
  }
  qsort(order, (size_t)nb, sizeof(scored_block), by_score_then_index);
  for (int t = 0; t < k; ++t) idx[t] = order[t].j;
  qsort(idx, (size_t)k, sizeof(int), ascending_int);
  free(order);
}

/* [SF] step 2 over many rows: S is [nrows_total, nb], idx is [nrows_total, k]. */
void oracle_topk(const double* S, long nrows_total, int nb, int k, int* idx) {
#pragma omp parallel for schedule(static)
  for (long r = 0; r < nrows_total; ++r) oracle_topk_row(S + r * nb, nb, k, idx + r * k);
}

void oracle_sparse_attn_gqa(const void* q, const void* kmat, const void* v, int dtype, int B, int N,
                            int H, int Hkv, int D, int bs, const int* idx, int k, const int* rows,
                            int nrows, double scale, int flags, double* o);

/* [SF] step 3 / [MSA] §2.1-§2.2: for every query row n of query block i,
 *   l_t = scale * sum_d q[b,n,h,d] * k[b,t,h,d]   for t in the selected blocks,
 *   o[n] = sum_t exp(l_t - max l) v[b,t,h,:] / sum_t exp(l_t - max l).
 * The selected blocks of (b, h, rows[b,h,r]) are idx[b, h, r, 0..k).
 * Output o is [B, H, nrows, bs, D] (float64). rows == NULL means all nb.
 * The arithmetic is written out once, in oracle_sparse_attn_gqa below (with
 * one key/value head per query head it is exactly this definition). */
void oracle_sparse_attn(const void* q, const void* kmat, const void* v, int dtype, int B, int N,
                        int H, int D, int bs, const int* idx, int k, const int* rows, int nrows,
                        double scale, double* o) {
  oracle_sparse_attn_gqa(q, kmat, v, dtype, B, N, H, H, D, bs, idx, k, rows, nrows, scale, 0, o);
}

/* Number of OpenMP threads the oracle runs with (reported by the CPU baseline). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------
 * Causal variant (readings, listed in the design notes as well):
 *   - query block i may select only key blocks j <= i, so it keeps
 *     n_i = min(k, i + 1) blocks;
 *   - with force_diag, block i itself is always kept and the other n_i - 1
 *     are the highest-scoring blocks j < i;
 *   - a selected list holds its n_i ids in ascending order, followed by
 *     k - n_i entries of -1;
 *   - inside the selected blocks, query token n sees key token t only if
 *     t <= n ([MSA] §2.1: Softmax(Mask(QK^T/sqrt(d_k)))V, with the causal
 *     mask), so only the diagonal block is masked token by token.
 * ------------------------------------------------------------------------ */
#define ORACLE_CAUSAL 1
#define ORACLE_FORCE_DIAG 2

/* Causal top-k for query block i of one row of scores. */
void oracle_topk_row_causal(const double* s_row, int nb, int i, int k, int force_diag, int* idx) {
  int n = k < i + 1 ? k : i + 1;
  int ncand = force_diag ? i : i + 1; /* candidates ranked by score */
  int nrank = force_diag ? n - 1 : n; /* how many of them are kept */
  scored_block* order = (scored_block*)malloc((size_t)(ncand > 0 ? ncand : 1) * sizeof(scored_block));
  for (int j = 0; j < ncand; ++j) {
    order[j].s = s_row[j];
    order[j].j = j;
  }
  qsort(order, (size_t)ncand, sizeof(scored_block), by_score_then_index);
  for (int t = 0; t < nrank; ++t) idx[t] = order[t].j;
  if (force_diag) idx[nrank] = i;
  qsort(idx, (size_t)n, sizeof(int), ascending_int);
  for (int t = n; t < k; ++t) idx[t] = -1;
  free(order);
  (void)nb;
}

/* Top-k over many rows with flags (bit 0: causal, bit 1: force the diagonal
 * block). qblock[r] is the query block of row r (NULL: r % nb). */
void oracle_topk_ex(const double* S, long nrows_total, int nb, int k, const int* qblock, int flags,
                    int* idx) {
#pragma omp parallel for schedule(static)
  for (long r = 0; r < nrows_total; ++r) {
    if (flags & ORACLE_CAUSAL) {
      int i = qblock ? qblock[r] : (int)(r % nb);
      oracle_topk_row_causal(S + r * nb, nb, i, k, (flags & ORACLE_FORCE_DIAG) != 0, idx + r * k);
    } else {
      oracle_topk_row(S + r * nb, nb, k, idx + r * k);
    }
  }
}

/* oracle_sparse_attn with flags: entries of idx below 0 select nothing, and
 * with ORACLE_CAUSAL key token t is left out of the softmax of query token n
 * when t > n. (Written out in oracle_sparse_attn_gqa, with Hkv = H.) */
void oracle_sparse_attn_ex(const void* q, const void* kmat, const void* v, int dtype, int B, int N,
                           int H, int D, int bs, const int* idx, int k, const int* rows, int nrows,
                           double scale, int flags, double* o) {
  oracle_sparse_attn_gqa(q, kmat, v, dtype, B, N, H, H, D, bs, idx, k, rows, nrows, scale, flags, o);
}

/* ------------------------------------------------------------------------
 * Grouped-query variant ([MSA] §3.1: the attention block is GQA-based).
 * Readings (listed in the design notes as well): q has H heads and k, v have
 * Hkv heads, H = G * Hkv; query head h reads key/value head h / G. One block
 * selection serves each key/value head: it is scored with the group's pooled
 * query (the mean over the group's G heads of their block means), which by
 * linearity is the mean of the G heads' block scores.
 * ------------------------------------------------------------------------ */

/* The attention over the kept blocks, with Hkv key/value heads: q and o have
 * H heads, k and v have Hkv; idx and rows are per query head ([B, H, nrows, k],
 * [B, H, nrows]). For every query row n of query block i = rows[b,h,r]:
 *   l_t = scale * sum_d q[b,n,h,d] * k[b,t,g,d]  (g = h / G) for the tokens t
 *         of the kept blocks (an entry below 0 keeps nothing; with
 *         ORACLE_CAUSAL, t > n is left out),
 *   m = max_t l_t,  w_t = exp(l_t - m),  o[n] = sum_t w_t v[b,t,g,:] / sum_t w_t.
 * Each key/value head's k and v rows are first converted (exactly) to one
 * contiguous float64 array, so the sums below read plain doubles; every sum
 * runs in the order written. Parallel over query rows only. */
void oracle_sparse_attn_gqa(const void* q, const void* kmat, const void* v, int dtype, int B, int N,
                            int H, int Hkv, int D, int bs, const int* idx, int k, const int* rows,
                            int nrows, double scale, int flags, double* o) {
  long ntok = (long)k * bs;
  int G = H / Hkv;
  double* kd = (double*)malloc((size_t)N * D * sizeof(double));
  double* vd = (double*)malloc((size_t)N * D * sizeof(double));
  for (int b = 0; b < B; ++b)
    for (int g = 0; g < Hkv; ++g) {
      /* k[b, :, g, :] and v[b, :, g, :] as float64 [N, D] */
#pragma omp parallel for schedule(static)
      for (int n = 0; n < N; ++n)
        for (int d = 0; d < D; ++d) {
          kd[(size_t)n * D + d] = elem(kmat, dtype, at_bnhd(N, Hkv, D, b, n, g, d));
          vd[(size_t)n * D + d] = elem(v, dtype, at_bnhd(N, Hkv, D, b, n, g, d));
        }
#pragma omp parallel
      {
        double* logit = (double*)malloc((size_t)ntok * sizeof(double));
        double* qrow = (double*)malloc((size_t)D * sizeof(double));
#pragma omp for collapse(3) schedule(dynamic, 4)
        for (int hg = 0; hg < G; ++hg)
          for (int r = 0; r < nrows; ++r)
            for (int t_q = 0; t_q < bs; ++t_q) {
              int h = g * G + hg;
              size_t bh = (size_t)b * H + h;
              int i = rows ? rows[bh * nrows + r] : r;
              const int* sel = idx + (bh * nrows + r) * k;
              int n = i * bs + t_q;
              for (int d = 0; d < D; ++d) qrow[d] = elem(q, dtype, at_bnhd(N, H, D, b, n, h, d));
              /* logits over the tokens of the selected blocks */
              double m = -INFINITY;
              for (int s = 0; s < k; ++s)
                for (int u = 0; u < bs; ++u) {
                  double l = -INFINITY; /* masked or unselected */
                  if (sel[s] >= 0) {
                    int t = sel[s] * bs + u;
                    if (!(flags & ORACLE_CAUSAL) || t <= n) {
                      const double* kt = kd + (size_t)t * D;
                      double dot = 0.0;
                      for (int d = 0; d < D; ++d) dot += qrow[d] * kt[d];
                      l = scale * dot;
                    }
                  }
                  logit[(long)s * bs + u] = l;
                  if (l > m) m = l;
                }
              /* softmax weights and the weighted sum of v */
              double* out = o + ((bh * nrows + r) * bs + t_q) * D;
              for (int d = 0; d < D; ++d) out[d] = 0.0;
              double z = 0.0;
              for (int s = 0; s < k; ++s)
                for (int u = 0; u < bs; ++u) {
                  double l = logit[(long)s * bs + u];
                  if (l == -INFINITY) continue;
                  const double* vt = vd + (size_t)(sel[s] * bs + u) * D;
                  double w = exp(l - m);
                  z += w;
                  for (int d = 0; d < D; ++d) out[d] += w * vt[d];
                }
              for (int d = 0; d < D; ++d) out[d] /= z;
            }
        free(logit);
        free(qrow);
      }
    }
  free(kd);
  free(vd);
}

/* ------------------------------------------------------------------------
 * Backward pass. The selection is a set of indices (top-k carries no
 * gradient), so the gradients are those of the attention with the index
 * lists held fixed. For each query token n with the kept key tokens T(n) (and
 * the causal mask when flagged):
 *   p_t = softmax_t(scale q_n . k_t),  o_n = sum_t p_t v_t,
 *   D_n = dO_n . o_n,  dP_t = dO_n . v_t,  dS_t = p_t (dP_t - D_n),
 *   dq_n = scale sum_t dS_t k_t,  dk_t += scale dS_t q_n,  dv_t += p_t dO_n.
 * dq, dk, dv are [B, N, H, D] float64; do_ is read like q (same dtype).
 * rows [B, H, nrows] (NULL: every query block) restricts the query blocks
 * whose contributions are summed (a sample, for timing).
 * Parallel over (b, h) only, so every sum has a fixed order.
 * ------------------------------------------------------------------------ */
void oracle_sparse_attn_bwd(const void* q, const void* kmat, const void* v, const void* do_, int dtype,
                            int B, int N, int H, int D, int bs, const int* idx, int k, const int* rows,
                            int nrows, double scale, int flags, double* dq, double* dk, double* dv) {
  int nb = N / bs;
  long ntok = (long)k * bs;
  size_t total = (size_t)B * N * H * D;
  for (size_t e = 0; e < total; ++e) dq[e] = dk[e] = dv[e] = 0.0;
#pragma omp parallel
  {
    double* p = (double*)malloc((size_t)ntok * sizeof(double));
    int* tok = (int*)malloc((size_t)ntok * sizeof(int));
    double* qrow = (double*)malloc((size_t)D * sizeof(double));
    double* dorow = (double*)malloc((size_t)D * sizeof(double));
    double* orow = (double*)malloc((size_t)D * sizeof(double));
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h) {
        size_t bh = (size_t)b * H + h;
        for (int r = 0; r < (rows ? nrows : nb); ++r) {
          int i = rows ? rows[bh * nrows + r] : r;
          const int* sel = idx + (bh * nb + i) * k;
          for (int t_q = 0; t_q < bs; ++t_q) {
            int n = i * bs + t_q;
            for (int d = 0; d < D; ++d) {
              qrow[d] = elem(q, dtype, at_bnhd(N, H, D, b, n, h, d));
              dorow[d] = elem(do_, dtype, at_bnhd(N, H, D, b, n, h, d));
            }
            /* the softmax weights over the kept, unmasked key tokens */
            long cnt = 0;
            double m = -INFINITY;
            for (int s = 0; s < k; ++s) {
              if (sel[s] < 0) continue;
              for (int u = 0; u < bs; ++u) {
                int t = sel[s] * bs + u;
                if ((flags & ORACLE_CAUSAL) && t > n) continue;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += qrow[d] * elem(kmat, dtype, at_bnhd(N, H, D, b, t, h, d));
                p[cnt] = scale * dot;
                tok[cnt] = t;
                if (p[cnt] > m) m = p[cnt];
                ++cnt;
              }
            }
            double z = 0.0;
            for (long c = 0; c < cnt; ++c) {
              p[c] = exp(p[c] - m);
              z += p[c];
            }
            for (long c = 0; c < cnt; ++c) p[c] /= z;
            /* o_n and D_n = dO_n . o_n */
            for (int d = 0; d < D; ++d) orow[d] = 0.0;
            for (long c = 0; c < cnt; ++c)
              for (int d = 0; d < D; ++d) orow[d] += p[c] * elem(v, dtype, at_bnhd(N, H, D, b, tok[c], h, d));
            double Dn = 0.0;
            for (int d = 0; d < D; ++d) Dn += dorow[d] * orow[d];
            /* dS_t, then the three gradients */
            for (long c = 0; c < cnt; ++c) {
              int t = tok[c];
              double dP = 0.0;
              for (int d = 0; d < D; ++d) dP += dorow[d] * elem(v, dtype, at_bnhd(N, H, D, b, t, h, d));
              double dS = p[c] * (dP - Dn);
              for (int d = 0; d < D; ++d) {
                dq[at_bnhd(N, H, D, b, n, h, d)] += scale * dS * elem(kmat, dtype, at_bnhd(N, H, D, b, t, h, d));
                dk[at_bnhd(N, H, D, b, t, h, d)] += scale * dS * qrow[d];
                dv[at_bnhd(N, H, D, b, t, h, d)] += p[c] * dorow[d];
              }
            }
          }
        }
      }
    free(p);
    free(tok);
    free(qrow);
    free(dorow);
    free(orow);
  }
}
