/*
 * oracle.c -- plain, slow fp64 CPU reference for exact multi-head attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes is the definition of attention, written out with no tiling,
 * fusion or reordering:
 *
 *   s_ij = scale * sum_c q_ic k_jc                       (FlashAttention saves IO, not
 *                                                          N^2 work, section 1: S = QK^T/sqrt(d))
 *   safe softmax in three passes over the row:            (Flash Attention wiki note, "Safe
 *     m_i = max_j s_ij,  l_i = sum_j exp(s_ij - m_i),      Softmax": subtract the row max,
 *     p_ij = exp(s_ij - m_i) / l_i                         then sum, then normalise)
 *   o_i = sum_j p_ij v_j,   lse_i = m_i + ln l_i          (section 1: O = PV; the saved
 *                                                          per-row statistics, "AI Bible 13",
 *                                                          section 03, second axe)
 *
 * Causal masking is bottom-right aligned: key j is visible to query i iff
 * j <= i + (Nk - Nq).  Masked terms are excluded from every sum.  A row with no
 * visible key has o = 0 and lse = -inf.
 *
 * The backward pass is the textbook vector-Jacobian product of the same
 * definition (the pages only say that the backward recomputes S and P from the
 * saved statistics; they print no gradient formula):
 *   dV_j = sum_i p_ij dO_i,   dP_ij = dO_i . v_j,   D_i = sum_j p_ij dP_ij,
 *   dS_ij = p_ij (dP_ij - D_i),   dQ_i = scale sum_j dS_ij k_j,
 *   dK_j = scale sum_i dS_ij q_i.
 *
 * The (m, l, u) row state and the merge of two states follow "FlashAttention
 * saves IO, not N^2 work", section 2 (the three-value state of a scored
 * stream) and section 3 (merging the states of two blocks).
 *
 * Layouts (all row-major, fp64):
 *   prefill  q, o, dq, do : [B][Nq][H][d]     k, v, dk, dv : [B][Nk][H][d]
 *            lse          : [B][H][Nq]
 *   decode   q, o : [B][H][d]   k, v : [total][H][d] with cu_seqlens[B+1]
 *            lse  : [B][H]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(b, n, h, c, N, H, D) ((((size_t)(b) * (N) + (n)) * (H) + (h)) * (D) + (c))

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Largest visible key index + 1 for query row i (bottom-right causal). */
static long visible_keys(long i, long Nq, long Nk, int causal) {
  if (!causal) return Nk;
  long lim = i + (Nk - Nq) + 1;
  if (lim < 0) lim = 0;
  if (lim > Nk) lim = Nk;
  return lim;
}

/*
 * One query row of one head, the three-pass definition.  s and p are scratch
 * rows of length Nk.  q_row is d values; k, v are addressed with row stride
 * `kstride` (elements between consecutive keys of this head).
 */
static void row_forward(const double* q_row, const double* k, const double* v, long kstride,
                        long nvis, int d, double scale, double* s, double* p, double* o_row,
                        double* lse_out) {
  /* scores of the visible keys; the masked tail is excluded entirely */
  for (long j = 0; j < nvis; ++j) {
    const double* kj = k + (size_t)j * kstride;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q_row[c] * kj[c];
    s[j] = scale * acc;
  }
  if (nvis == 0) {
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    *lse_out = -INFINITY;
    return;
  }
  /* pass 1: row max */
  double m = -INFINITY;
  for (long j = 0; j < nvis; ++j)
    if (s[j] > m) m = s[j];
  /* pass 2: sum of shifted exponentials */
  double l = 0.0;
  for (long j = 0; j < nvis; ++j) l += exp(s[j] - m);
  /* pass 3: normalise, then weight the values */
  for (long j = 0; j < nvis; ++j) p[j] = exp(s[j] - m) / l;
  for (int c = 0; c < d; ++c) o_row[c] = 0.0;
  for (long j = 0; j < nvis; ++j) {
    const double* vj = v + (size_t)j * kstride;
    const double pj = p[j];
    for (int c = 0; c < d; ++c) o_row[c] += pj * vj[c];
  }
  *lse_out = m + log(l);
}

/* Forward over all (b, h, row).  Returns 0, or -1 on allocation failure. */
int oracle_attn_fwd(const double* q, const double* k, const double* v, int B, int H, int Nq,
                    int Nk, int d, int causal, double scale, double* o, double* lse) {
  int fail = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    if (!s || !p) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for collapse(3) schedule(dynamic, 16)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h)
        for (int i = 0; i < Nq; ++i) {
          if (!s || !p) continue;
          const double* q_row = q + IDX4(b, i, h, 0, Nq, H, d);
          const double* kb = k + IDX4(b, 0, h, 0, Nk, H, d);
          const double* vb = v + IDX4(b, 0, h, 0, Nk, H, d);
          long nvis = visible_keys(i, Nq, Nk, causal);
          row_forward(q_row, kb, vb, (long)H * d, nvis, d, scale, s, p,
                      o + IDX4(b, i, h, 0, Nq, H, d), lse + ((size_t)b * H + h) * Nq + i);
        }
    free(s);
    free(p);
  }
  return fail ? -1 : 0;
}

/*
 * Forward for a chosen subset of query rows of one head.  q_rows: [R][d],
 * row_idx[R] gives each row's position in the full Nq-row query sequence (it
 * decides causal visibility).  k, v: [Nk][d] (one head, contiguous).
 */
int oracle_attn_fwd_rows(const double* q_rows, const int64_t* row_idx, int R, const double* k,
                         const double* v, int Nq, int Nk, int d, int causal, double scale,
                         double* o_rows, double* lse_rows) {
  int fail = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    if (!s || !p) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 4)
    for (int r = 0; r < R; ++r) {
      if (!s || !p) continue;
      long nvis = visible_keys((long)row_idx[r], Nq, Nk, causal);
      row_forward(q_rows + (size_t)r * d, k, v, d, nvis, d, scale, s, p, o_rows + (size_t)r * d,
                  lse_rows + r);
    }
    free(s);
    free(p);
  }
  return fail ? -1 : 0;
}

/* The full probability matrix of one head ([Nq][Nk], zeros where masked). */
int oracle_attn_probs(const double* q, const double* k, int Nq, int Nk, int d, int causal,
                      double scale, double* P) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
  if (!s) return -1;
  for (int i = 0; i < Nq; ++i) {
    double* prow = P + (size_t)i * Nk;
    for (int j = 0; j < Nk; ++j) prow[j] = 0.0;
    long nvis = visible_keys(i, Nq, Nk, causal);
    if (nvis == 0) continue;
    for (long j = 0; j < nvis; ++j) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * k[(size_t)j * d + c];
      s[j] = scale * acc;
    }
    double m = -INFINITY;
    for (long j = 0; j < nvis; ++j)
      if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < nvis; ++j) l += exp(s[j] - m);
    for (long j = 0; j < nvis; ++j) prow[j] = exp(s[j] - m) / l;
  }
  free(s);
  return 0;
}

/*
 * Backward for one head: q, dout: [Nq][d]; k, v: [Nk][d] (contiguous).  The
 * probabilities are rebuilt from the definition (not from a saved lse).
 * Writes dq [Nq][d], dk [Nk][d], dv [Nk][d].
 */
static int head_backward(const double* q, const double* k, const double* v, const double* dout,
                         int Nq, int Nk, int d, int causal, double scale, double* dq, double* dk,
                         double* dv, int parallel_rows) {
  memset(dq, 0, sizeof(double) * (size_t)Nq * d);
  memset(dk, 0, sizeof(double) * (size_t)Nk * d);
  memset(dv, 0, sizeof(double) * (size_t)Nk * d);
  int fail = 0;
#pragma omp parallel if (parallel_rows)
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
    double* dk_loc = (double*)calloc((size_t)Nk * d + 1, sizeof(double));
    double* dv_loc = (double*)calloc((size_t)Nk * d + 1, sizeof(double));
    int ok = s && p && dp && dk_loc && dv_loc;
    if (!ok) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 8)
    for (int i = 0; i < Nq; ++i) {
      if (!ok) continue;
      const double* qi = q + (size_t)i * d;
      const double* doi = dout + (size_t)i * d;
      long nvis = visible_keys(i, Nq, Nk, causal);
      if (nvis == 0) continue; /* fully masked row: o = 0 is constant, all gradients 0 */
      for (long j = 0; j < nvis; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qi[c] * k[(size_t)j * d + c];
        s[j] = scale * acc;
      }
      double m = -INFINITY;
      for (long j = 0; j < nvis; ++j)
        if (s[j] > m) m = s[j];
      double l = 0.0;
      for (long j = 0; j < nvis; ++j) l += exp(s[j] - m);
      for (long j = 0; j < nvis; ++j) p[j] = exp(s[j] - m) / l;
      /* dP_ij = dO_i . v_j ;  D_i = sum_j p_ij dP_ij (Jacobian form) */
      double Di = 0.0;
      for (long j = 0; j < nvis; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += doi[c] * v[(size_t)j * d + c];
        dp[j] = acc;
        Di += p[j] * acc;
      }
      double* dqi = dq + (size_t)i * d;
      for (long j = 0; j < nvis; ++j) {
        const double dsij = p[j] * (dp[j] - Di);
        const double* kj = k + (size_t)j * d;
        double* dkj = dk_loc + (size_t)j * d;
        double* dvj = dv_loc + (size_t)j * d;
        for (int c = 0; c < d; ++c) {
          dqi[c] += scale * dsij * kj[c];
          dkj[c] += scale * dsij * qi[c];
          dvj[c] += p[j] * doi[c];
        }
      }
    }
    if (ok) {
#pragma omp critical
      {
        for (size_t t = 0; t < (size_t)Nk * d; ++t) {
          dk[t] += dk_loc[t];
          dv[t] += dv_loc[t];
        }
      }
    }
    free(s);
    free(p);
    free(dp);
    free(dk_loc);
    free(dv_loc);
  }
  return fail ? -1 : 0;
}

/* Gather one head of a [B][N][H][d] tensor into a contiguous [N][d] buffer. */
static void gather_head(const double* x, int b, int h, int N, int H, int d, double* out) {
  for (int n = 0; n < N; ++n) memcpy(out + (size_t)n * d, x + IDX4(b, n, h, 0, N, H, d), sizeof(double) * d);
}
static void scatter_head(const double* in, int b, int h, int N, int H, int d, double* x) {
  for (int n = 0; n < N; ++n) memcpy(x + IDX4(b, n, h, 0, N, H, d), in + (size_t)n * d, sizeof(double) * d);
}

/* Backward over all (b, h).  Layouts as in the header comment. */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout, int B,
                    int H, int Nq, int Nk, int d, int causal, double scale, double* dq, double* dk,
                    double* dv) {
  const int nheads = B * H;
  int nthreads = oracle_num_threads();
  /* parallel over heads when there are enough of them, otherwise over rows */
  int per_head_parallel = nheads < nthreads;
  int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) if (!per_head_parallel)
  for (int bh = 0; bh < nheads; ++bh) {
    int b = bh / H, h = bh % H;
    size_t nq = (size_t)Nq * d, nk = (size_t)Nk * d;
    double* buf = (double*)malloc(sizeof(double) * (2 * nq + 2 * nk + nq + 2 * nk + 1));
    if (!buf) {
#pragma omp atomic write
      fail = 1;
      continue;
    }
    double *qh = buf, *doh = qh + nq, *kh = doh + nq, *vh = kh + nk;
    double *dqh = vh + nk, *dkh = dqh + nq, *dvh = dkh + nk;
    gather_head(q, b, h, Nq, H, d, qh);
    gather_head(dout, b, h, Nq, H, d, doh);
    gather_head(k, b, h, Nk, H, d, kh);
    gather_head(v, b, h, Nk, H, d, vh);
    if (head_backward(qh, kh, vh, doh, Nq, Nk, d, causal, scale, dqh, dkh, dvh, per_head_parallel)) {
#pragma omp atomic write
      fail = 1;
    }
    scatter_head(dqh, b, h, Nq, H, d, dq);
    scatter_head(dkh, b, h, Nk, H, d, dk);
    scatter_head(dvh, b, h, Nk, H, d, dv);
    free(buf);
  }
  return fail ? -1 : 0;
}

/*
 * Decode: one query per (b, h), attending to that sequence's L_b keys, where
 * the keys of sequence b are rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of the
 * packed k, v.  With one query, bottom-right causal alignment makes every key
 * visible, so the mask is a no-op.
 */
int oracle_decode(const double* q, const double* k, const double* v, const int32_t* cu_seqlens,
                  int B, int H, int d, double scale, double* o, double* lse) {
  long maxlen = 0;
  for (int b = 0; b < B; ++b) {
    long L = (long)cu_seqlens[b + 1] - cu_seqlens[b];
    if (L > maxlen) maxlen = L;
  }
  int fail = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
    if (!s || !p) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
      for (int h = 0; h < H; ++h) {
        if (!s || !p) continue;
        long start = cu_seqlens[b];
        long L = (long)cu_seqlens[b + 1] - start;
        const double* kb = k + ((size_t)start * H + h) * d;
        const double* vb = v + ((size_t)start * H + h) * d;
        row_forward(q + ((size_t)b * H + h) * d, kb, vb, (long)H * d, L, d, scale, s, p,
                    o + ((size_t)b * H + h) * d, lse + (size_t)b * H + h);
      }
    free(s);
    free(p);
  }
  return fail ? -1 : 0;
}

/*
 * The three-value state of a stream of (score, value) pairs: m = max score,
 * l = sum exp(s - m), u = sum exp(s - m) v.  An empty stream is (-inf, 0, 0).
 */
void oracle_row_state(const double* s, const double* v, int n, int dv, double* m, double* l,
                      double* u) {
  double mm = -INFINITY;
  for (int j = 0; j < n; ++j)
    if (s[j] > mm) mm = s[j];
  double ll = 0.0;
  for (int c = 0; c < dv; ++c) u[c] = 0.0;
  if (n > 0) {
    for (int j = 0; j < n; ++j) {
      double w = exp(s[j] - mm);
      ll += w;
      for (int c = 0; c < dv; ++c) u[c] += w * v[(size_t)j * dv + c];
    }
  }
  *m = mm;
  *l = ll;
}

/*
 * Merge of two block states (A, B) into one: m = max(mA, mB), each side
 * rescaled by exp(m_side - m).  A side that is empty (m = -inf) contributes
 * nothing (its scale is taken as 0 rather than exp(-inf - -inf)).
 */
void oracle_merge_state(double ma, double la, const double* ua, double mb, double lb,
                        const double* ub, int dv, double* m, double* l, double* u) {
  double mm = ma > mb ? ma : mb;
  double sa = (ma == -INFINITY) ? 0.0 : exp(ma - mm);
  double sb = (mb == -INFINITY) ? 0.0 : exp(mb - mm);
  *m = mm;
  *l = sa * la + sb * lb;
  for (int c = 0; c < dv; ++c) u[c] = sa * ua[c] + sb * ub[c];
}
