/*
 * xs_oracle.c -- CPU oracle for fused attention + Ulysses post-attention All-to-All.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this file:
 * only the tests, the package's smoke() and the CPU-baseline leg of bench.py do.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * What it computes, in fp64, written as the plain definitions:
 *
 *  1. Non-causal scaled dot-product softmax attention, per batch b, head h and query row i:
 *         s_j = scale * sum_d q[b,h,i,d] * k[b,h,j,d]            (j = 0 .. S-1)
 *         m   = max_j s_j
 *         p_j = exp(s_j - m)
 *         l   = sum_j p_j
 *         O[b,h,i,d] = sum_j p_j * v[b,h,j,d] / l
 *     Source: "X-Stage: An Overlooked Pipeline Stage for Communication-Computation Overlap
 *     in DiT Inference" -- abstract (Ulysses sequence-parallel attention fused with
 *     FlashAttention) and the explainer's "Technisches Resuemee", section "Zentrale
 *     Beitraege", item "FlashAttention-A2A (Piggybacking)".  The pages name the operation
 *     (FlashAttention in DiT inference) but print no formula; the formula above is the
 *     textbook definition of softmax(Q K^T * scale) V, with the row maximum subtracted
 *     before exp (which leaves the value unchanged).  Non-causal: DiT self-attention.
 *
 *  2. The Ulysses post-attention All-to-All (same page, same item: the output-tile owner
 *     stores its finished tile into the destination rank's sequence shard).  The pages do
 *     not print the layout; the reading used here: the attention output is head-major
 *     O[b,h,s,d]; virtual rank r receives the sequence shard s in [r*S/P, (r+1)*S/P) of
 *     every head, laid out as dest[r][b, s_local, h, d] with s = r*S/P + s_local and h
 *     the global head index.
 *
 *  3. The inverse exchange (sequence-sharded -> head-major), used by tests to check that
 *     the permutation round-trips.
 *
 * Parallelism: query rows are independent, so the row loop is split across OpenMP
 * threads.  Inside one row the arithmetic runs in the order written above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define XSO_OK 0
#define XSO_BAD_ARG 1

int xs_oracle_version(void) { return 1; }

/* Number of threads OpenMP would use (1 without OpenMP). */
int xs_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * One query row of attention (definition 1 above).
 *   q_row: [D], k, v: [S, D] of the same (b, h), out_row: [D], work: [S] scratch.
 */
static void attention_row(const double *q_row, const double *k, const double *v, int S, int D,
                          double scale, double *out_row, double *work) {
  double m = -INFINITY;
  for (int j = 0; j < S; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q_row[d] * k[(size_t)j * D + d];
    work[j] = dot * scale;
    if (work[j] > m) m = work[j];
  }
  double l = 0.0;
  for (int j = 0; j < S; ++j) {
    work[j] = exp(work[j] - m);
    l += work[j];
  }
  for (int d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int j = 0; j < S; ++j) acc += work[j] * v[(size_t)j * D + d];
    out_row[d] = acc / l;
  }
}

/*
 * Attention for selected query rows of every (b, h).
 *   q, k, v : [B, H, S, D] fp64, contiguous.
 *   rows    : NULL -> every row 0..S-1 (nrows must equal S);
 *             else [B*H, nrows] row indices, one list per (b, h).
 *   out     : [B, H, nrows, D] fp64.
 *   scale   : multiplier of q.k (the caller passes 1/sqrt(D) for the standard scale).
 *   nthreads: <= 0 -> OpenMP default.
 */
int xs_oracle_attention(const double *q, const double *k, const double *v, int B, int H, int S,
                        int D, double scale, const int32_t *rows, int nrows, double *out,
                        int nthreads) {
  if (!q || !k || !v || !out || B <= 0 || H <= 0 || S <= 0 || D <= 0 || nrows <= 0) return XSO_BAD_ARG;
  if (!rows && nrows != S) return XSO_BAD_ARG;
  if (rows) {
    for (long long t = 0; t < (long long)B * H * nrows; ++t)
      if (rows[t] < 0 || rows[t] >= S) return XSO_BAD_ARG;
  }
  const long long total = (long long)B * H * nrows;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int fail = 0;
#pragma omp parallel
  {
    double *work = (double *)malloc(sizeof(double) * (size_t)S);
    if (!work) {
#pragma omp atomic write
      fail = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (long long t = 0; t < total; ++t) {
        long long bh = t / nrows;
        int ii = (int)(t % nrows);
        int i = rows ? rows[bh * nrows + ii] : ii;
        const double *kb = k + (size_t)bh * S * D;
        const double *vb = v + (size_t)bh * S * D;
        attention_row(q + ((size_t)bh * S + i) * D, kb, vb, S, D, scale, out + (size_t)t * D, work);
      }
      free(work);
    }
  }
  return fail ? XSO_BAD_ARG : XSO_OK;
}

/*
 * Softmax probabilities of one query row: probs[j] = p_j / l for the row i of head (b, h).
 * Exposed so that tests can check normalisation directly.
 */
int xs_oracle_softmax_row(const double *q, const double *k, int B, int H, int S, int D,
                          double scale, int b, int h, int i, double *probs) {
  if (!q || !k || !probs || b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= S) return XSO_BAD_ARG;
  size_t bh = (size_t)b * H + h;
  const double *q_row = q + (bh * S + i) * D;
  const double *kb = k + bh * S * D;
  double m = -INFINITY;
  for (int j = 0; j < S; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q_row[d] * kb[(size_t)j * D + d];
    probs[j] = dot * scale;
    if (probs[j] > m) m = probs[j];
  }
  double l = 0.0;
  for (int j = 0; j < S; ++j) {
    probs[j] = exp(probs[j] - m);
    l += probs[j];
  }
  for (int j = 0; j < S; ++j) probs[j] /= l;
  return XSO_OK;
}

static int a2a_shape_ok(int B, int H, int S, int D, int P) {
  return B > 0 && H > 0 && S > 0 && D > 0 && P > 0 && S % P == 0 && H % P == 0;
}

/*
 * Post-attention All-to-All (definition 2), element by element.
 *   src : [B, H, S, D] elements of elem_bytes bytes each (head-major attention output).
 *   dest: [P][B][S/P][H][D] (the P slabs back to back).
 * Every destination slot is written exactly once by the explicit loop below.
 */
int xs_oracle_a2a_post(const void *src, void *dest, int B, int H, int S, int D, int P,
                       int elem_bytes) {
  if (!src || !dest || !a2a_shape_ok(B, H, S, D, P) || elem_bytes <= 0) return XSO_BAD_ARG;
  const int Sl = S / P;
  const unsigned char *s8 = (const unsigned char *)src;
  unsigned char *d8 = (unsigned char *)dest;
  for (int r = 0; r < P; ++r)
    for (int b = 0; b < B; ++b)
      for (int sl = 0; sl < Sl; ++sl)
        for (int h = 0; h < H; ++h)
          for (int d = 0; d < D; ++d) {
            int s = r * Sl + sl;
            size_t dst_idx = ((((size_t)r * B + b) * Sl + sl) * H + h) * D + d;
            size_t src_idx = (((size_t)b * H + h) * S + s) * D + d;
            memcpy(d8 + dst_idx * elem_bytes, s8 + src_idx * elem_bytes, (size_t)elem_bytes);
          }
  return XSO_OK;
}

/*
 * Inverse exchange: sequence-sharded slabs [P][B][S/P][H][D] back to head-major
 * [B, H, S, D].  (In Ulysses this is the direction of the pre-attention exchange.)
 */
int xs_oracle_a2a_pre(const void *slabs, void *dst, int B, int H, int S, int D, int P,
                      int elem_bytes) {
  if (!slabs || !dst || !a2a_shape_ok(B, H, S, D, P) || elem_bytes <= 0) return XSO_BAD_ARG;
  const int Sl = S / P;
  const unsigned char *s8 = (const unsigned char *)slabs;
  unsigned char *d8 = (unsigned char *)dst;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int s = 0; s < S; ++s)
        for (int d = 0; d < D; ++d) {
          int r = s / Sl, sl = s % Sl;
          size_t slab_idx = ((((size_t)r * B + b) * Sl + sl) * H + h) * D + d;
          size_t hm_idx = (((size_t)b * H + h) * S + s) * D + d;
          memcpy(d8 + hm_idx * elem_bytes, s8 + slab_idx * elem_bytes, (size_t)elem_bytes);
        }
  return XSO_OK;
}

/*
 * Where the row (b, h, s) of the attention output lands after the post-attention
 * exchange: rank r and the element offset of its first element inside slab r.
 */
int xs_oracle_dest_slot(int B, int H, int S, int D, int P, int b, int h, int s, int *rank,
                        long long *offset) {
  if (!rank || !offset || !a2a_shape_ok(B, H, S, D, P)) return XSO_BAD_ARG;
  if (b < 0 || b >= B || h < 0 || h >= H || s < 0 || s >= S) return XSO_BAD_ARG;
  const int Sl = S / P;
  *rank = s / Sl;
  *offset = (((long long)b * Sl + (s % Sl)) * H + h) * (long long)D;
  return XSO_OK;
}

/*
 * 4. Partial attention over one key/value shard, returning the log-sum-exp of the row
 *    (the "Route" primitive: the owner of a KV shard attends the routed query rows over its
 *    own keys and sends back a small result that the requester merges with an online
 *    softmax).  Source: page "Move the Query, Not the Cache: Characterizing Cross-Instance
 *    Latent Attention Redistribution Across GPU Fabrics", explainer "Technisches Resuemee:
 *    Den Query bewegen, nicht den Cache" -> "Methodik" -> "Primitiv-Vergleich" (Route) and
 *    "Korrektheitsverifizierung" (routed partial attention merged by online softmax
 *    reproduces single-instance attention).  The pages print no formula; the definitions
 *    below are the textbook ones.  Per (b, h) and query row i, over the Skv keys j of the
 *    shard:
 *         s_j = scale * sum_d q[b,h,i,d] * k[b,h,j,d]
 *         m   = max_j s_j
 *         l   = sum_j exp(s_j - m)
 *         O_i = sum_j exp(s_j - m) * v[b,h,j,d] / l
 *         lse = m + log(l)            (= log sum_j exp(s_j), natural log)
 *    A shard without keys (Skv = 0) has l = 0: lse = -inf, and O is set to 0 (reading: the
 *    empty part has weight zero in the merge, so its O never matters).
 *
 * 5. Merge of n partial results of the same query row (definition 4 applied to disjoint key
 *    sets K_1 .. K_n whose union is all keys):
 *         M   = max_t lse_t
 *         w_t = exp(lse_t - M)
 *         O   = sum_t w_t * O_t / sum_t w_t
 *         lse = M + log(sum_t w_t)
 *    which equals definition 1 (and 4) over the union, since w_t * O_t * exp(M) is the
 *    un-normalised sum over K_t.  Rows whose parts are all empty (M = -inf) give O = 0 and
 *    lse = -inf.
 */

/* One query row of definition 4.  k, v: [Skv, D]; work: [Skv] scratch. */
static void partial_row(const double *q_row, const double *k, const double *v, int Skv, int D,
                        double scale, double *out_row, double *lse, double *work) {
  if (Skv == 0) {
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    *lse = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int j = 0; j < Skv; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q_row[d] * k[(size_t)j * D + d];
    work[j] = dot * scale;
    if (work[j] > m) m = work[j];
  }
  double l = 0.0;
  for (int j = 0; j < Skv; ++j) {
    work[j] = exp(work[j] - m);
    l += work[j];
  }
  for (int d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int j = 0; j < Skv; ++j) acc += work[j] * v[(size_t)j * D + d];
    out_row[d] = acc / l;
  }
  *lse = m + log(l);
}

/*
 * Partial attention (definition 4) for selected query rows of every (b, h).
 *   q      : [B, H, Sq, D] fp64;  k, v: [B, H, Skv, D] fp64 (Skv may be 0: k, v unused).
 *   rows   : NULL -> every row 0..Sq-1 (nrows must equal Sq); else [B*H, nrows] indices.
 *   out    : [B, H, nrows, D];  lse: [B, H, nrows].
 */
int xs_oracle_attention_partial(const double *q, const double *k, const double *v, int B, int H,
                                int Sq, int Skv, int D, double scale, const int32_t *rows,
                                int nrows, double *out, double *lse, int nthreads) {
  if (!q || !out || !lse || B <= 0 || H <= 0 || Sq <= 0 || Skv < 0 || D <= 0 || nrows <= 0)
    return XSO_BAD_ARG;
  if (Skv > 0 && (!k || !v)) return XSO_BAD_ARG;
  if (!rows && nrows != Sq) return XSO_BAD_ARG;
  if (rows) {
    for (long long t = 0; t < (long long)B * H * nrows; ++t)
      if (rows[t] < 0 || rows[t] >= Sq) return XSO_BAD_ARG;
  }
  const long long total = (long long)B * H * nrows;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int fail = 0;
#pragma omp parallel
  {
    double *work = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
    if (!work) {
#pragma omp atomic write
      fail = 1;
    } else {
#pragma omp for schedule(dynamic, 16)
      for (long long t = 0; t < total; ++t) {
        long long bh = t / nrows;
        int ii = (int)(t % nrows);
        int i = rows ? rows[bh * nrows + ii] : ii;
        const double *kb = Skv > 0 ? k + (size_t)bh * Skv * D : NULL;
        const double *vb = Skv > 0 ? v + (size_t)bh * Skv * D : NULL;
        partial_row(q + ((size_t)bh * Sq + i) * D, kb, vb, Skv, D, scale, out + (size_t)t * D,
                    lse + t, work);
      }
      free(work);
    }
  }
  return fail ? XSO_BAD_ARG : XSO_OK;
}

/*
 * Merge (definition 5) of n partial results.
 *   o_parts  : [n, R, D] fp64;  lse_parts: [n, R] fp64 (-inf marks an empty part).
 *   out      : [R, D];  lse_out: [R] (nullable).
 */
int xs_oracle_lse_merge(const double *o_parts, const double *lse_parts, int n, long long R, int D,
                        double *out, double *lse_out) {
  if (!o_parts || !lse_parts || !out || n <= 0 || R <= 0 || D <= 0) return XSO_BAD_ARG;
  for (long long r = 0; r < R; ++r) {
    double M = -INFINITY;
    for (int t = 0; t < n; ++t)
      if (lse_parts[(size_t)t * R + r] > M) M = lse_parts[(size_t)t * R + r];
    double *o = out + (size_t)r * D;
    if (M == -INFINITY) {
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (lse_out) lse_out[r] = -INFINITY;
      continue;
    }
    double W = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int t = 0; t < n; ++t) {
      const double w = exp(lse_parts[(size_t)t * R + r] - M);
      W += w;
      const double *ot = o_parts + ((size_t)t * R + r) * D;
      for (int d = 0; d < D; ++d) o[d] += w * ot[d];
    }
    for (int d = 0; d < D; ++d) o[d] /= W;
    if (lse_out) lse_out[r] = M + log(W);
  }
  return XSO_OK;
}
