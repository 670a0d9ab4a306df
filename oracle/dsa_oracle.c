/*
 * Plain CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only through the seeded input generators.
 *
 * Every routine is the literal definition of its step, written as scalar
 * loops with fp64 accumulation on inputs decoded exactly from their storage
 * formats (fp32, bf16, fp8 e4m3).  No blocking, fusion or reordering beyond
 * what the definition states.  Rows are distributed over host threads with
 * OpenMP; each row is computed independently, so the result does not depend
 * on the thread count.
 *
 * Sources (the pages print their formulas stripped, so the indexer formula is
 * taken in the form the method is usually written in, consistent with the
 * words of the pages):
 *  - "Linear and Sparse Attention" (yuxiangdai.com), section "DeepSeek Sparse
 *    Attention": a lightning indexer scores all tokens, then top-k selection
 *    keeps the highest-scoring tokens for attention.
 *  - "GLM sparse attention" (thethings.ai), ReLU paragraph: the indexer
 *    clips each negative similarity to zero before the weighted sum; the
 *    threshold figure: the cut-off is the k-th best score; MLA passage: one
 *    cached latent plus one decoupled rotary key per token, scored directly by
 *    absorbed queries, shared by every head; a full softmax over the
 *    selected tokens, with nothing approximated in the attention itself.
 *  - "Sparse Attention Architecture Evolution in LLMs" (intl.cloud.baidu.com),
 *    "Top-K Selection": k = 2048.
 *  - "DeepSeek Sparse Attention" (divagr.pages.dev), "The lightning
 *    indexer": scores rank positions and are not attention weights; "the
 *    risk": a token left out of the selection adds nothing to the output.
 *
 * Readings where the pages are silent (each repeated beside its code):
 *  - candidates of query t are the positions s <= t of its own sequence;
 *  - the indexer carries no scale factor beyond the head weights w;
 *  - ties in top-k go to the lower position; -0 and +0 compare equal;
 *    NaN scores rank as -inf;
 *  - when t+1 <= k every candidate is selected and the rest is -1;
 *  - the attention value vector is the first D_V columns of the cached row.
 *
 * Parity pins: tests/test_oracle.py checks each routine against closed forms,
 * library routines (matmul, stable argsort, scaled-dot-product attention) and
 * invariants the method fixes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP FP8 E4M3 (the "fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa
 * bits; no infinities; S.1111.111 is NaN; exponent 0 encodes subnormals
 * m * 2^-9. Decoded from the format definition. */
double oracle_e4m3_to_f64(uint8_t v) {
  int s = (v >> 7) & 1, e = (v >> 3) & 0xF, m = v & 7;
  double r;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0)
    r = ldexp((double)m, -9);
  else
    r = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return s ? -r : r;
}

static double load_elem(const void* base, int dtype, int64_t i) {
  switch (dtype) {
    case OR_F32: return (double)((const float*)base)[i];
    case OR_BF16: return oracle_bf16_to_f64(((const uint16_t*)base)[i]);
    default: return oracle_e4m3_to_f64(((const uint8_t*)base)[i]);
  }
}

/*
 * Lightning indexer:  I[t,s] = sum_j w[t,j] * ReLU( <q_I[t,j,:], k_I[s,:]> )
 * for s <= t, and -inf for t < s < ld.  ReLU clips each head's similarity
 * at zero before the weighted head sum ("GLM sparse attention", ReLU
 * paragraph).  Inputs are decoded exactly; an fp8 value is its decoded code
 * times the fp32 scale of its token (q_scale per (query row, head), k_scale
 * per key row), multiplied in fp64.
 *
 * Row i of the output belongs to query row qrow[i] (index into q_I, q_scale
 * and w), whose sequence starts at key row kbase[i]; tpos[i] is the query's
 * position inside that sequence.  A (optional) receives the error scale
 * sum_j |w[t,j]| * |<q_I[t,j], k_I[s]>| used by the tests' tolerance.
 */
void oracle_indexer_scores(int64_t n_rows, const int64_t* qrow, const int64_t* kbase,
                           const int64_t* tpos, int H_I, int D_I, int dtype, const void* q_I,
                           const float* q_scale, const float* w, const void* k_I,
                           const float* k_scale, int64_t ld, double* I, double* A) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    const int64_t qr = qrow[i], kb = kbase[i], t = tpos[i];
    double* q = (double*)malloc(sizeof(double) * (size_t)H_I * D_I);
    double* kv = (double*)malloc(sizeof(double) * (size_t)D_I);
    for (int j = 0; j < H_I; ++j) {
      double sc = q_scale ? (double)q_scale[qr * H_I + j] : 1.0;
      for (int d = 0; d < D_I; ++d)
        q[j * D_I + d] = load_elem(q_I, dtype, (qr * H_I + j) * D_I + d) * sc;
    }
    for (int64_t s = 0; s < ld; ++s) {
      if (s > t) {
        I[i * ld + s] = -INFINITY;
        if (A) A[i * ld + s] = 0.0;
        continue;
      }
      double ksc = k_scale ? (double)k_scale[kb + s] : 1.0;
      for (int d = 0; d < D_I; ++d) kv[d] = load_elem(k_I, dtype, (kb + s) * D_I + d) * ksc;
      double acc = 0.0, aabs = 0.0;
      for (int j = 0; j < H_I; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D_I; ++d) dot += q[j * D_I + d] * kv[d];
        double wj = (double)w[qr * H_I + j];
        acc += wj * (dot > 0.0 ? dot : 0.0);
        aabs += fabs(wj) * fabs(dot);
      }
      I[i * ld + s] = acc;
      if (A) A[i * ld + s] = aabs;
    }
    free(q);
    free(kv);
  }
}

/* Ranking key: NaN ranks as -inf; -0 == +0 falls out of double comparison. */
typedef struct {
  double v;
  int64_t s;
} cand_t;

static int cand_cmp(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->v > b->v) return -1;
  if (a->v < b->v) return 1;
  return (a->s < b->s) ? -1 : (a->s > b->s);
}

static void topk_row(cand_t* c, int64_t n, int k, int32_t* out) {
  qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
  int64_t m = n < k ? n : k;
  for (int64_t r = 0; r < m; ++r) out[r] = (int32_t)c[r].s;
  for (int64_t r = m; r < k; ++r) out[r] = -1;
}

/*
 * Top-k selection ("Sparse Attention Architecture Evolution in LLMs", Top-K
 * Selection; "GLM sparse attention",
 * threshold figure): per row, the candidates s in [0, n_valid) ordered by
 * score descending, then position ascending (ties to the lower position);
 * the first min(k, n_valid) are kept, the remaining slots are -1.  Output is
 * in that order (the library's own order is unspecified, tests compare sets).
 */
void oracle_topk_f32(int64_t n_rows, const float* scores, int64_t ld, const int64_t* n_valid,
                     int k, int32_t* idx) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t n = n_valid[i];
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t s = 0; s < n; ++s) {
      float x = scores[i * ld + s];
      c[s].v = isnan(x) ? -INFINITY : (double)x;
      c[s].s = s;
    }
    topk_row(c, n, k, idx + i * (int64_t)k);
    free(c);
  }
}

void oracle_topk_f64(int64_t n_rows, const double* scores, int64_t ld, const int64_t* n_valid,
                     int k, int32_t* idx) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t n = n_valid[i];
    cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t s = 0; s < n; ++s) {
      double x = scores[i * ld + s];
      c[s].v = isnan(x) ? -INFINITY : x;
      c[s].s = s;
    }
    topk_row(c, n, k, idx + i * (int64_t)k);
    free(c);
  }
}

/*
 * Softmax attention of one query row over a list of cached rows, for every
 * head ("GLM sparse attention", MLA passage: one latent row per token scored
 * directly by the absorbed query of each head; exact softmax).
 *   z_s = sm_scale * <q[h, 0:D_K], C[s, 0:D_K]>
 *   o[h, v] = sum_s softmax(z)_s * C[s, v]        for v < D_V
 *   lse[h]  = log sum_s exp(z_s)
 * Positions listed as -1 are empty slots.  With no position at all the
 * output is 0 and lse is -inf.
 * The cache C is stored as bf16, or as fp8 e4m3 codes with one fp32 scale per
 * token (the FP8 argument of "GLM sparse attention", ReLU paragraph, read as
 * applying to the cached latent as it does to the indexer keys): every
 * element is decoded exactly, C[s, d] = code * kv_scale[s], in fp64.
 */
static double cache_elem(const void* kv, int kv_dtype, const float* kv_scale, int64_t row,
                         int D_K, int d) {
  const double x = load_elem(kv, kv_dtype, row * D_K + d);
  return kv_scale ? x * (double)kv_scale[row] : x;
}

static void attend_row(const uint16_t* q, const void* kv, int kv_dtype, const float* kv_scale,
                       int64_t kb, const int64_t* pos, int64_t npos, int H, int D_K, int D_V,
                       double sm_scale, double* out, double* lse) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
  double* qh = (double*)malloc(sizeof(double) * (size_t)D_K);
  for (int h = 0; h < H; ++h) {
    for (int d = 0; d < D_K; ++d) qh[d] = oracle_bf16_to_f64(q[(int64_t)h * D_K + d]);
    double m = -INFINITY;
    for (int64_t r = 0; r < npos; ++r) {
      double dot = 0.0;
      for (int d = 0; d < D_K; ++d)
        dot += qh[d] * cache_elem(kv, kv_dtype, kv_scale, kb + pos[r], D_K, d);
      z[r] = sm_scale * dot;
      if (z[r] > m) m = z[r];
    }
    double* o = out + (int64_t)h * D_V;
    for (int v = 0; v < D_V; ++v) o[v] = 0.0;
    if (npos == 0) {
      lse[h] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int64_t r = 0; r < npos; ++r) {
      double p = exp(z[r] - m);
      sum += p;
      for (int v = 0; v < D_V; ++v)
        o[v] += p * cache_elem(kv, kv_dtype, kv_scale, kb + pos[r], D_K, v);
    }
    for (int v = 0; v < D_V; ++v) o[v] /= sum;
    lse[h] = m + log(sum);
  }
  free(z);
  free(qh);
}

/*
 * Sparse MLA attention: row i attends over the positions idx[i, 0:k] (local
 * to its sequence, -1 = empty) of the cache rows starting at kbase[i].
 * q: bf16 [*, H, D_K] addressed by qrow[i]; kv: [N_k, D_K] in kv_dtype (bf16,
 * or e4m3 with kv_scale [N_k]; kv_scale NULL for bf16).
 * out: [n_rows, H, D_V]; lse: [n_rows, H].
 */
void oracle_sparse_mla_attn_kv(int64_t n_rows, const int64_t* qrow, const int64_t* kbase,
                               const int32_t* idx, int k, int H, int D_K, int D_V,
                               double sm_scale, const uint16_t* q, const void* kv, int kv_dtype,
                               const float* kv_scale, double* out, double* lse) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(k > 0 ? k : 1));
    int64_t np = 0;
    for (int r = 0; r < k; ++r)
      if (idx[i * (int64_t)k + r] >= 0) pos[np++] = idx[i * (int64_t)k + r];
    attend_row(q + qrow[i] * (int64_t)H * D_K, kv, kv_dtype, kv_scale, kbase[i], pos, np, H, D_K,
               D_V, sm_scale, out + i * (int64_t)H * D_V, lse + i * (int64_t)H);
    free(pos);
  }
}

void oracle_sparse_mla_attn(int64_t n_rows, const int64_t* qrow, const int64_t* kbase,
                            const int32_t* idx, int k, int H, int D_K, int D_V, double sm_scale,
                            const uint16_t* q, const uint16_t* kv, double* out, double* lse) {
  oracle_sparse_mla_attn_kv(n_rows, qrow, kbase, idx, k, H, D_K, D_V, sm_scale, q, kv, OR_BF16,
                            NULL, out, lse);
}

/* Dense causal MLA attention of row i over every position 0..tpos[i]. */
void oracle_dense_mla_attn_kv(int64_t n_rows, const int64_t* qrow, const int64_t* kbase,
                              const int64_t* tpos, int H, int D_K, int D_V, double sm_scale,
                              const uint16_t* q, const void* kv, int kv_dtype,
                              const float* kv_scale, double* out, double* lse) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t n = tpos[i] + 1;
    int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t s = 0; s < n; ++s) pos[s] = s;
    attend_row(q + qrow[i] * (int64_t)H * D_K, kv, kv_dtype, kv_scale, kbase[i], pos, n, H, D_K,
               D_V, sm_scale, out + i * (int64_t)H * D_V, lse + i * (int64_t)H);
    free(pos);
  }
}

void oracle_dense_mla_attn(int64_t n_rows, const int64_t* qrow, const int64_t* kbase,
                           const int64_t* tpos, int H, int D_K, int D_V, double sm_scale,
                           const uint16_t* q, const uint16_t* kv, double* out, double* lse) {
  oracle_dense_mla_attn_kv(n_rows, qrow, kbase, tpos, H, D_K, D_V, sm_scale, q, kv, OR_BF16, NULL,
                           out, lse);
}
