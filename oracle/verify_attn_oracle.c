/*
 * fp64 CPU oracle for tree-verification attention — TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package's smoke check and the bench's CPU-baseline leg
 * may load or run this file's library. The CUDA product path never calls it and
 * shares no code with it.
 *
 * What it computes (LongSpec, gist.science summary, section 2C "Schnelle Tree
 * Attention"): during verification each draft-tree query attends to the cached
 * prefix with no mask ("Cached-Teil ... keine Maskierung") and to the speculative
 * tree tokens under a tree mask ("Speculative-Teil ... Baum-Maskierung"); the two
 * parts are joined by a log-sum-exp step so that the result is exact ("korrekt
 * zusammengefuehrt"), i.e. one softmax over the union of both key sets. The
 * abstracts (mlsanity arXiv v1 abstract; PaperTrail ACL record) call the method
 * lossless, so the oracle is that single softmax, written out plainly:
 *
 *   for sequence b, tree node i, query head h, kv head kh = h / (H_q / H_kv):
 *     visible(i) = { prefix keys 0 .. L_b-1 } U { tree nodes on the root->i path, i included }
 *     s_x   = scale * <q[b,i,h,:], k_x[kh,:]>                    (fp64)
 *     m     = max_x s_x
 *     lse   = m + ln( sum_x exp(s_x - m) )                        (natural log, scale included)
 *     out   = sum_x exp(s_x - lse) * v_x[kh,:]
 *
 * The tree mask is read as "ancestor or self" (the standard token-tree
 * verification mask); the root is node 0 with parent -1 and parent[i] is in
 * [0, i) for every other node. Ancestors are found by walking parent links.
 * Inputs are bf16 bit patterns widened exactly to fp64. There is no blocking,
 * no split of the key axis and no merge step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_TREE 2
#define ORACLE_NO_MEM 3

static double bf16_to_f64(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof(f));
  return (double)f;
}

/* Checks every tree of the batch: node 0 is the root (parent -1), every other
 * node's parent lies in [0, i). Returns ORACLE_OK or ORACLE_BAD_TREE. */
int oracle_check_trees(const int32_t* parent, int B, int T) {
  for (int b = 0; b < B; ++b) {
    const int32_t* p = parent + (int64_t)b * T;
    if (p[0] != -1) return ORACLE_BAD_TREE;
    for (int i = 1; i < T; ++i)
      if (p[i] < 0 || p[i] >= i) return ORACLE_BAD_TREE;
  }
  return ORACLE_OK;
}

/* vis[c] = 1 iff tree node c is node i or one of its ancestors. */
static void ancestors_or_self(const int32_t* p, int T, int i, unsigned char* vis) {
  memset(vis, 0, (size_t)T);
  for (int c = i; c >= 0; c = p[c]) vis[c] = 1;
}

/*
 * Full oracle over selected output rows.
 *   q        bf16 [B*T, Hq, d]        k_cache/v_cache bf16 [cu[B], Hkv, d]
 *   k_tree/v_tree bf16 [B*T, Hkv, d]  parent int32 [B*T]   cu_seqlens int32 [B+1]
 *   rows     row ids r = (b*T + i)*Hq + h, or NULL for all B*T*Hq rows in order
 *   out      fp64 [nrows, d]          lse fp64 [nrows]
 *   nthreads OpenMP threads (<= 0: the runtime default)
 */
int oracle_verify_attn(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                       const uint16_t* k_tree, const uint16_t* v_tree,
                       const int32_t* parent, const int32_t* cu_seqlens,
                       int B, int Hq, int Hkv, int d, int T, double scale,
                       const int64_t* rows, int64_t nrows,
                       double* out, double* lse, int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || T < 1 || Hq % Hkv != 0) return ORACLE_BAD_ARG;
  if (cu_seqlens[0] != 0) return ORACLE_BAD_ARG;
  int64_t max_L = 0;
  for (int b = 0; b < B; ++b) {
    int64_t L = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
    if (L < 0) return ORACLE_BAD_ARG;
    if (L > max_L) max_L = L;
  }
  if (oracle_check_trees(parent, B, T) != ORACLE_OK) return ORACLE_BAD_TREE;
  const int64_t total_rows = (int64_t)B * T * Hq;
  if (rows == NULL) nrows = total_rows;
  for (int64_t n = 0; rows != NULL && n < nrows; ++n)
    if (rows[n] < 0 || rows[n] >= total_rows) return ORACLE_BAD_ARG;
  const int group = Hq / Hkv;
  int failed = 0;

#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(max_L + T));
    double* qv = (double*)malloc(sizeof(double) * (size_t)d);
    unsigned char* vis = (unsigned char*)malloc((size_t)T);
    if (s == NULL || qv == NULL || vis == NULL) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int64_t n = 0; n < nrows; ++n) {
      if (failed) continue;
      const int64_t r = rows ? rows[n] : n;
      const int h = (int)(r % Hq);
      const int64_t tok = r / Hq;          /* b*T + i */
      const int b = (int)(tok / T);
      const int i = (int)(tok % T);
      const int kh = h / group;
      const int64_t L = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
      const int64_t k0 = cu_seqlens[b];

      for (int c = 0; c < d; ++c) qv[c] = bf16_to_f64(q[r * d + c]);
      ancestors_or_self(parent + (int64_t)b * T, T, i, vis);

      /* scores of every visible key: prefix first, then visible tree nodes */
      int64_t nk = 0;
      for (int64_t j = 0; j < L; ++j) {
        const uint16_t* kr = k_cache + ((k0 + j) * Hkv + kh) * (int64_t)d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qv[c] * bf16_to_f64(kr[c]);
        s[nk++] = scale * acc;
      }
      for (int t = 0; t < T; ++t) {
        if (!vis[t]) continue;
        const uint16_t* kr = k_tree + (((int64_t)b * T + t) * Hkv + kh) * (int64_t)d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qv[c] * bf16_to_f64(kr[c]);
        s[nk++] = scale * acc;
      }

      double m = -INFINITY;
      for (int64_t x = 0; x < nk; ++x) if (s[x] > m) m = s[x];
      double sum = 0.0;
      for (int64_t x = 0; x < nk; ++x) sum += exp(s[x] - m);
      const double l = m + log(sum);
      lse[n] = l;

      double* o = out + n * (int64_t)d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      nk = 0;
      for (int64_t j = 0; j < L; ++j) {
        const double w = exp(s[nk++] - l);
        const uint16_t* vr = v_cache + ((k0 + j) * Hkv + kh) * (int64_t)d;
        for (int c = 0; c < d; ++c) o[c] += w * bf16_to_f64(vr[c]);
      }
      for (int t = 0; t < T; ++t) {
        if (!vis[t]) continue;
        const double w = exp(s[nk++] - l);
        const uint16_t* vr = v_tree + (((int64_t)b * T + t) * Hkv + kh) * (int64_t)d;
        for (int c = 0; c < d; ++c) o[c] += w * bf16_to_f64(vr[c]);
      }
    }
    free(s);
    free(qv);
    free(vis);
  }
  return failed ? ORACLE_NO_MEM : ORACLE_OK;
}

/*
 * One softmax over an explicit key set: used by the tests to form partial
 * results (prefix only, tree only, a slice of the prefix) and check that the
 * log-sum-exp merge of partials reproduces the union (the "Aggregation" step of
 * section 2C). n may be 0: then lse = -inf and out = 0.
 *   q_row bf16 [d]; keys/vals bf16 rows at stride `stride` elements.
 */
void oracle_softmax_keyset(const uint16_t* q_row, const uint16_t* keys, const uint16_t* vals,
                           int64_t n, int64_t stride, int d, double scale,
                           double* out, double* lse) {
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (n <= 0) {
    *lse = -INFINITY;
    return;
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += bf16_to_f64(q_row[c]) * bf16_to_f64(keys[j * stride + c]);
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }
  double sum = 0.0;
  for (int64_t j = 0; j < n; ++j) sum += exp(s[j] - m);
  const double l = m + log(sum);
  for (int64_t j = 0; j < n; ++j) {
    const double w = exp(s[j] - l);
    for (int c = 0; c < d; ++c) out[c] += w * bf16_to_f64(vals[j * stride + c]);
  }
  *lse = l;
  free(s);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
