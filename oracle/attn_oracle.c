/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (the pages' definition, written out directly):
 *   "FlashAttention 1-4 详解", section 原算法 (standard attention):
 *       Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V
 *   with the scale passed in by the caller (the pages use 1/sqrt(d)), a causal
 *   option (the lower-triangle mask: key j visible to query i iff j <= i, section
 *   其他优化 / FlashAttention 2 的工程优化, causal mask), and packed variable-length
 *   batches (sequence b owns tokens [cu[b], cu[b+1]); indices are local to it).
 *
 * Layout of every tensor: token-major, q/k/v/o/dq/dk/dv[T][H][d] in fp64, where T
 * is the number of packed tokens.  lse is [H][T] (natural log, includes the scale).
 *
 * Functions:
 *   oracle_fwd         explicit score row, two-pass softmax, P.V, LSE (definition)
 *   oracle_fwd_rows    the same for a list of (token, head) rows only
 *   oracle_probs       the full probability matrix P of one (sequence, head)
 *   *_masked           the three above with a sliding-window mask added to the
 *                      causal option (see visible_range)
 *   oracle_online_fwd  the tiled online-softmax algorithm in the pages' steps
 *                      (FlashAttention 1 recurrences, FlashAttention 2 deferred
 *                      normalisation, FlashAttention 4 conditional rescale)
 *   oracle_bwd         the textbook backward pass (recomputes P); *_masked adds
 *                      the sliding window
 *   oracle_bwd_sampled the same gradients for selected query rows (dQ) and key
 *                      rows (dK, dV) of one (sequence, head), for full-size checks
 *
 * Empty rows cannot occur: a causal row always sees its own key, a non-causal row
 * sees every key of a non-empty sequence, and a window never excludes the row's
 * own key.  Zero-length sequences are skipped.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of keys visible to local query row i of a sequence of length L. */
static int visible_keys(int i, int L, int causal) { return causal ? i + 1 : L; }

/* Keys visible to local query row i, as the half-open range [*lo, *hi).
 * Causal ("FlashAttention 1-4 详解", 其他优化, lower triangle): j <= i.
 * Sliding window, the mask added beside causal (the pages name FlexAttention's
 * masks as the interface FA4 serves -- "FlashAttention V4 deep-dive" section 5,
 * FA-4 summary item [27] -- but print no mask other than causal; reading:
 * local attention): j >= i - wl when wl >= 0 and j <= i + wr when wr >= 0; a
 * negative bound means that side is unbounded.  With wl, wr >= 0 the range always
 * holds j = i. */
static void visible_range(int i, int L, int causal, int wl, int wr, int* lo, int* hi) {
  int a = 0, b = L;
  if (wl >= 0 && i - wl > a) a = i - wl;
  if (causal && i + 1 < b) b = i + 1;
  if (wr >= 0 && i + wr + 1 < b) b = i + wr + 1;
  *lo = a;
  *hi = b;
}

/* One query row of one head: scores, two-pass softmax, output row and LSE over the
 * visible keys [lo, hi).
 * "FlashAttention 1-4 详解", 原算法 (S = Q K^T, P = softmax(S scaled), O = P V) and
 * Online Softmax 数学推导 (two-pass stable softmax: subtract the row max m, divide
 * by the sum of e^{x_j - m}).  srow is caller scratch of length >= L. */
static void attend_row(const double* k, const double* v, double* o_row, double* lse_out,
                       const double* q_row, int64_t seq_base, int lo, int hi, int H, int d,
                       int h, double scale, double* srow) {
  /* Pass 0: scores s_j = scale * <q_i, k_j>. */
  for (int j = lo; j < hi; ++j) {
    const double* k_row = k + ((seq_base + j) * H + h) * (int64_t)d;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q_row[c] * k_row[c];
    srow[j - lo] = scale * acc;
  }
  const int nvis = hi - lo;
  /* Pass 1: row max. */
  double m = -INFINITY;
  for (int j = 0; j < nvis; ++j) if (srow[j] > m) m = srow[j];
  /* Pass 2: exponentials and their sum. */
  double l = 0.0;
  for (int j = 0; j < nvis; ++j) { srow[j] = exp(srow[j] - m); l += srow[j]; }
  /* Normalise and contract with V. */
  for (int c = 0; c < d; ++c) o_row[c] = 0.0;
  for (int j = 0; j < nvis; ++j) {
    const double p = srow[j] / l;
    const double* v_row = v + ((seq_base + lo + j) * H + h) * (int64_t)d;
    for (int c = 0; c < d; ++c) o_row[c] += p * v_row[c];
  }
  *lse_out = m + log(l);
}

static int set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
  return omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

/* Exact forward pass over every row.  Returns the number of threads used, or -1 on
 * bad arguments.  cu has nseq+1 entries (token offsets, cu[0] = 0).  wl / wr are
 * the sliding-window bounds of visible_range (negative: unbounded). */
int oracle_fwd_masked(const double* q, const double* k, const double* v, double* o,
                      double* lse, int nseq, const int64_t* cu, int H, int d, int causal,
                      int wl, int wr, double scale, int nthreads) {
  if (nseq < 0 || H <= 0 || d <= 0 || !cu) return -1;
  const int used = set_threads(nthreads);
  const int64_t T = cu[nseq];
  int Lmax = 0;
  for (int b = 0; b < nseq; ++b) {
    const int64_t L = cu[b + 1] - cu[b];
    if (L < 0) return -1;
    if (L > Lmax) Lmax = (int)L;
  }
  const int64_t units = (int64_t)nseq * H;
#pragma omp parallel
  {
    double* srow = (double*)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      const int b = (int)(u / H), h = (int)(u % H);
      const int64_t base = cu[b];
      const int L = (int)(cu[b + 1] - cu[b]);
      for (int i = 0; i < L; ++i) {
        const int64_t tok = base + i;
        int lo, hi;
        visible_range(i, L, causal, wl, wr, &lo, &hi);
        attend_row(k, v, o + (tok * H + h) * (int64_t)d, lse + (int64_t)h * T + tok,
                   q + (tok * H + h) * (int64_t)d, base, lo, hi, H, d, h, scale, srow);
      }
    }
    free(srow);
  }
  return used;
}

int oracle_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
               int nseq, const int64_t* cu, int H, int d, int causal, double scale,
               int nthreads) {
  return oracle_fwd_masked(q, k, v, o, lse, nseq, cu, H, d, causal, -1, -1, scale, nthreads);
}

/* Exact forward pass for selected rows only: rows[r] is a packed token index and
 * heads[r] its head.  o_rows is [nrows][d], lse_rows [nrows]. */
int oracle_fwd_rows_masked(const double* q, const double* k, const double* v, int nseq,
                           const int64_t* cu, int H, int d, int causal, int wl, int wr,
                           double scale, const int64_t* rows, const int* heads, int nrows,
                           double* o_rows, double* lse_rows, int nthreads) {
  if (nseq <= 0 || H <= 0 || d <= 0 || !cu) return -1;
  const int used = set_threads(nthreads);
  const int64_t T = cu[nseq];
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int r = 0; r < nrows; ++r) {
    const int64_t tok = rows[r];
    const int h = heads[r];
    if (tok < 0 || tok >= T || h < 0 || h >= H) { bad = 1; continue; }
    int b = 0;
    while (cu[b + 1] <= tok) ++b;
    const int64_t base = cu[b];
    const int L = (int)(cu[b + 1] - cu[b]);
    int lo, hi;
    visible_range((int)(tok - base), L, causal, wl, wr, &lo, &hi);
    double* srow = (double*)malloc(sizeof(double) * L);
    attend_row(k, v, o_rows + (int64_t)r * d, lse_rows + r, q + (tok * H + h) * (int64_t)d,
               base, lo, hi, H, d, h, scale, srow);
    free(srow);
  }
  return bad ? -1 : used;
}

int oracle_fwd_rows(const double* q, const double* k, const double* v, int nseq,
                    const int64_t* cu, int H, int d, int causal, double scale,
                    const int64_t* rows, const int* heads, int nrows, double* o_rows,
                    double* lse_rows, int nthreads) {
  return oracle_fwd_rows_masked(q, k, v, nseq, cu, H, d, causal, -1, -1, scale, rows, heads,
                                nrows, o_rows, lse_rows, nthreads);
}

/* Probability matrix P[L][L] of sequence b, head h (zeros where masked).
 * "FlashAttention 1-4 详解", 原算法: P = softmax(S / sqrt(d)), row-wise. */
int oracle_probs_masked(const double* q, const double* k, int nseq, const int64_t* cu, int H,
                        int d, int causal, int wl, int wr, double scale, int b, int h,
                        double* P) {
  if (b < 0 || b >= nseq || h < 0 || h >= H) return -1;
  const int64_t base = cu[b];
  const int L = (int)(cu[b + 1] - cu[b]);
  for (int i = 0; i < L; ++i) {
    double* prow = P + (int64_t)i * L;
    const double* q_row = q + ((base + i) * H + h) * (int64_t)d;
    int lo, hi;
    visible_range(i, L, causal, wl, wr, &lo, &hi);
    double m = -INFINITY;
    for (int j = 0; j < L; ++j) {
      if (j < lo || j >= hi) { prow[j] = 0.0; continue; }
      const double* k_row = k + ((base + j) * H + h) * (int64_t)d;
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += q_row[c] * k_row[c];
      prow[j] = scale * acc;
      if (prow[j] > m) m = prow[j];
    }
    double l = 0.0;
    for (int j = lo; j < hi; ++j) { prow[j] = exp(prow[j] - m); l += prow[j]; }
    for (int j = lo; j < hi; ++j) prow[j] /= l;
  }
  return 0;
}

int oracle_probs(const double* q, const double* k, int nseq, const int64_t* cu, int H, int d,
                 int causal, double scale, int b, int h, double* P) {
  return oracle_probs_masked(q, k, nseq, cu, H, d, causal, -1, -1, scale, b, h, P);
}

/* Tiled online softmax, in the order the pages give the steps.
 *  - "FlashAttention 1-4 详解", FlashAttention 1 / Online Softmax 数学推导: per key
 *    tile, m_new = max(m, rowmax(S_ij)), P~ = exp(S_ij - m_new),
 *    l_new = e^{m - m_new} l + sum P~, O_new = e^{m - m_new} O + P~ V_j.
 *  - same page, FlashAttention 2 / 减少非矩阵乘运算占比: O is divided by l once,
 *    after the last key tile.
 *  - same page, FlashAttention 4 / 三项核心技术 (2), and "FlashAttention V4 deep-dive"
 *    section 3.2 (conditional rescale): the correction is applied only when the
 *    running maximum has grown.  Reading: the reference maximum m is replaced (and
 *    O, l rescaled) only when rowmax exceeds it by more than tau (natural-log units
 *    here); otherwise the stale m is kept and P~ = exp(S - m) may exceed 1.
 *    tau = 0 is the page's "only when m_new > m" rule.
 * Scores are scaled by `scale` before the recurrences (section 原算法 puts 1/sqrt(d)
 * on S).  Queries are processed in tiles of Br rows, keys in tiles of Bc; a causal
 * row only takes keys j <= i.  lse = m + ln l.  Returns the number of rescales
 * performed (first tile excluded) or -1. */
int64_t oracle_online_fwd(const double* q, const double* k, const double* v, double* o,
                          double* lse, int nseq, const int64_t* cu, int H, int d, int causal,
                          double scale, int Br, int Bc, double tau) {
  if (Br <= 0 || Bc <= 0 || nseq < 0 || !cu) return -1;
  const int64_t T = cu[nseq];
  int64_t rescales = 0;
  double* Sblk = (double*)malloc(sizeof(double) * (size_t)Br * Bc);
  double* m = (double*)malloc(sizeof(double) * Br);
  double* l = (double*)malloc(sizeof(double) * Br);
  double* Oblk = (double*)malloc(sizeof(double) * (size_t)Br * d);
  for (int b = 0; b < nseq; ++b) {
    const int64_t base = cu[b];
    const int L = (int)(cu[b + 1] - cu[b]);
    for (int h = 0; h < H; ++h) {
      for (int i0 = 0; i0 < L; i0 += Br) {
        const int br = (L - i0 < Br) ? L - i0 : Br;
        for (int r = 0; r < br; ++r) { m[r] = -INFINITY; l[r] = 0.0; }
        memset(Oblk, 0, sizeof(double) * (size_t)Br * d);
        for (int j0 = 0; j0 < L; j0 += Bc) {
          const int bc = (L - j0 < Bc) ? L - j0 : Bc;
          for (int r = 0; r < br; ++r) {
            const int i = i0 + r;
            const double* q_row = q + ((base + i) * H + h) * (int64_t)d;
            /* S_ij for this tile (masked entries left out of every step). */
            double rowmax = -INFINITY;
            int any = 0;
            for (int c = 0; c < bc; ++c) {
              const int j = j0 + c;
              double s = -INFINITY;
              if (!causal || j <= i) {
                const double* k_row = k + ((base + j) * H + h) * (int64_t)d;
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += q_row[e] * k_row[e];
                s = scale * acc;
                any = 1;
                if (s > rowmax) rowmax = s;
              }
              Sblk[(size_t)r * Bc + c] = s;
            }
            if (!any) continue; /* tile fully masked for this row: skipped */
            /* m_new and the conditional correction. */
            if (m[r] == -INFINITY) {
              m[r] = rowmax;
            } else if (rowmax - m[r] > tau) {
              const double alpha = exp(m[r] - rowmax);
              l[r] *= alpha;
              for (int e = 0; e < d; ++e) Oblk[(size_t)r * d + e] *= alpha;
              m[r] = rowmax;
              ++rescales;
            }
            /* P~ = exp(S - m), l += sum P~, O += P~ V_j. */
            for (int c = 0; c < bc; ++c) {
              const double s = Sblk[(size_t)r * Bc + c];
              if (s == -INFINITY) continue;
              const double p = exp(s - m[r]);
              l[r] += p;
              const double* v_row = v + ((base + j0 + c) * H + h) * (int64_t)d;
              for (int e = 0; e < d; ++e) Oblk[(size_t)r * d + e] += p * v_row[e];
            }
          }
        }
        /* Deferred normalisation. */
        for (int r = 0; r < br; ++r) {
          const int64_t tok = base + i0 + r;
          for (int e = 0; e < d; ++e) o[(tok * H + h) * (int64_t)d + e] = Oblk[(size_t)r * d + e] / l[r];
          lse[(int64_t)h * T + tok] = m[r] + log(l[r]);
        }
      }
    }
  }
  free(Sblk); free(m); free(l); free(Oblk);
  return rescales;
}

/* Textbook backward pass of the forward above (the pages only say that the
 * backward recomputes P instead of storing it: "FlashAttention 1-4 详解", 总结 table,
 * 反向传播重计算).  With P from the definition, O = P V and upstream gradient dO:
 *   D_i   = sum_c dO_ic O_ic
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij k_j
 *   dK_j  = scale sum_i dS_ij q_i
 * O is recomputed here from the definition (not taken from the caller).  One
 * thread owns a whole (sequence, head), so the accumulations do not race. */
int oracle_bwd_masked(const double* q, const double* k, const double* v, const double* dout,
                      double* dq, double* dk, double* dv, int nseq, const int64_t* cu, int H,
                      int d, int causal, int wl, int wr, double scale, int nthreads) {
  if (nseq < 0 || H <= 0 || d <= 0 || !cu) return -1;
  const int used = set_threads(nthreads);
  const int64_t T = cu[nseq];
  memset(dq, 0, sizeof(double) * (size_t)T * H * d);
  memset(dk, 0, sizeof(double) * (size_t)T * H * d);
  memset(dv, 0, sizeof(double) * (size_t)T * H * d);
  int Lmax = 0;
  for (int b = 0; b < nseq; ++b) if (cu[b + 1] - cu[b] > Lmax) Lmax = (int)(cu[b + 1] - cu[b]);
  const int64_t units = (int64_t)nseq * H;
#pragma omp parallel
  {
    double* prow = (double*)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
    double* orow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
      const int b = (int)(u / H), h = (int)(u % H);
      const int64_t base = cu[b];
      const int L = (int)(cu[b + 1] - cu[b]);
      for (int i = 0; i < L; ++i) {
        const int64_t ti = base + i;
        const double* q_row = q + (ti * H + h) * (int64_t)d;
        const double* do_row = dout + (ti * H + h) * (int64_t)d;
        int lo, hi;
        visible_range(i, L, causal, wl, wr, &lo, &hi);
        /* P row by the definition (entries [lo, hi) of prow). */
        double mx = -INFINITY;
        for (int j = lo; j < hi; ++j) {
          const double* k_row = k + ((base + j) * H + h) * (int64_t)d;
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += q_row[c] * k_row[c];
          prow[j] = scale * acc;
          if (prow[j] > mx) mx = prow[j];
        }
        double l = 0.0;
        for (int j = lo; j < hi; ++j) { prow[j] = exp(prow[j] - mx); l += prow[j]; }
        for (int j = lo; j < hi; ++j) prow[j] /= l;
        /* O row and D_i. */
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        for (int j = lo; j < hi; ++j) {
          const double* v_row = v + ((base + j) * H + h) * (int64_t)d;
          for (int c = 0; c < d; ++c) orow[c] += prow[j] * v_row[c];
        }
        double Di = 0.0;
        for (int c = 0; c < d; ++c) Di += do_row[c] * orow[c];
        double* dq_row = dq + (ti * H + h) * (int64_t)d;
        for (int j = lo; j < hi; ++j) {
          const int64_t tj = base + j;
          const double* k_row = k + (tj * H + h) * (int64_t)d;
          const double* v_row = v + (tj * H + h) * (int64_t)d;
          double* dk_row = dk + (tj * H + h) * (int64_t)d;
          double* dv_row = dv + (tj * H + h) * (int64_t)d;
          double dp = 0.0;
          for (int c = 0; c < d; ++c) dp += do_row[c] * v_row[c];
          const double ds = prow[j] * (dp - Di);
          for (int c = 0; c < d; ++c) {
            dv_row[c] += prow[j] * do_row[c];
            dq_row[c] += scale * ds * k_row[c];
            dk_row[c] += scale * ds * q_row[c];
          }
        }
      }
    }
    free(prow);
    free(orow);
  }
  return used;
}

int oracle_bwd(const double* q, const double* k, const double* v, const double* dout,
               double* dq, double* dk, double* dv, int nseq, const int64_t* cu, int H, int d,
               int causal, double scale, int nthreads) {
  return oracle_bwd_masked(q, k, v, dout, dq, dk, dv, nseq, cu, H, d, causal, -1, -1, scale,
                           nthreads);
}

/* The textbook backward of oracle_bwd, for one (sequence b, head h), evaluated only
 * at selected positions so that long sequences stay affordable:
 *   dQ_i for the local query rows qi[0..nq), dK_j and dV_j for the local key rows
 *   kj[0..nk).
 * Per query row it first computes, from the definition, m_i, l_i (so P_ij =
 * exp(s_ij - m_i) / l_i), the exact O_i and D_i = <dO_i, O_i> (rows in parallel).
 * Then dQ_i = scale sum_j P_ij (<dO_i, v_j> - D_i) k_j, and for a key j
 * dV_j = sum_i P_ij dO_i and dK_j = scale sum_i P_ij (<dO_i, v_j> - D_i) q_i over the
 * query rows that see key j.  dq_out is [nq][d], dk_out and dv_out [nk][d]. */
int oracle_bwd_sampled(const double* q, const double* k, const double* v, const double* dout,
                       int nseq, const int64_t* cu, int H, int d, int causal, double scale,
                       int b, int h, const int* qi, int nq, const int* kj, int nk,
                       double* dq_out, double* dk_out, double* dv_out, int nthreads) {
  if (b < 0 || b >= nseq || h < 0 || h >= H || d <= 0) return -1;
  const int used = set_threads(nthreads);
  const int64_t base = cu[b];
  const int L = (int)(cu[b + 1] - cu[b]);
  for (int r = 0; r < nq; ++r) if (qi[r] < 0 || qi[r] >= L) return -1;
  for (int r = 0; r < nk; ++r) if (kj[r] < 0 || kj[r] >= L) return -1;
  double* m = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
  double* l = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
  double* Dv = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
#define QROW(i) (q + ((base + (i)) * H + h) * (int64_t)d)
#define KROW(j) (k + ((base + (j)) * H + h) * (int64_t)d)
#define VROW(j) (v + ((base + (j)) * H + h) * (int64_t)d)
#define DOROW(i) (dout + ((base + (i)) * H + h) * (int64_t)d)
  /* Pass 1: per query row, the softmax statistics, O_i and D_i. */
#pragma omp parallel
  {
    double* srow = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
    double* orow = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 16)
    for (int i = 0; i < L; ++i) {
      const int nvis = visible_keys(i, L, causal);
      double mi = -INFINITY;
      for (int j = 0; j < nvis; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += QROW(i)[c] * KROW(j)[c];
        srow[j] = scale * acc;
        if (srow[j] > mi) mi = srow[j];
      }
      double li = 0.0;
      for (int j = 0; j < nvis; ++j) { srow[j] = exp(srow[j] - mi); li += srow[j]; }
      for (int c = 0; c < d; ++c) orow[c] = 0.0;
      for (int j = 0; j < nvis; ++j)
        for (int c = 0; c < d; ++c) orow[c] += (srow[j] / li) * VROW(j)[c];
      double di = 0.0;
      for (int c = 0; c < d; ++c) di += DOROW(i)[c] * orow[c];
      m[i] = mi; l[i] = li; Dv[i] = di;
    }
    free(srow);
    free(orow);
  }
  /* P_ij and dS_ij from the statistics. */
#define P_OF(i, j, pij, dsij)                                        \
  do {                                                                \
    double acc_ = 0.0, dp_ = 0.0;                                     \
    for (int c = 0; c < d; ++c) acc_ += QROW(i)[c] * KROW(j)[c];      \
    pij = exp(scale * acc_ - m[i]) / l[i];                            \
    for (int c = 0; c < d; ++c) dp_ += DOROW(i)[c] * VROW(j)[c];      \
    dsij = pij * (dp_ - Dv[i]);                                       \
  } while (0)
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < nq; ++r) {
    const int i = qi[r];
    double* out = dq_out + (int64_t)r * d;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int j = 0; j < visible_keys(i, L, causal); ++j) {
      double pij, dsij;
      P_OF(i, j, pij, dsij);
      for (int c = 0; c < d; ++c) out[c] += scale * dsij * KROW(j)[c];
    }
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < nk; ++r) {
    const int j = kj[r];
    double* dko = dk_out + (int64_t)r * d;
    double* dvo = dv_out + (int64_t)r * d;
    for (int c = 0; c < d; ++c) { dko[c] = 0.0; dvo[c] = 0.0; }
    for (int i = causal ? j : 0; i < L; ++i) {
      double pij, dsij;
      P_OF(i, j, pij, dsij);
      for (int c = 0; c < d; ++c) {
        dvo[c] += pij * DOROW(i)[c];
        dko[c] += scale * dsij * QROW(i)[c];
      }
    }
  }
#undef P_OF
#undef QROW
#undef KROW
#undef VROW
#undef DOROW
  free(m); free(l); free(Dv);
  return used;
}
