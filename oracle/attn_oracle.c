/*
 * Reference oracle for exact scaled-dot-product attention -- TEST INFRASTRUCTURE.
 *
 * Only the test suite, the package smoke check and the benchmark's CPU-baseline
 * leg may load this library.  The product path (the CUDA library and its Python
 * binding) never calls it and shares no code with it.
 *
 * Everything is plain fp64, one query row at a time, written straight from the
 * definitions on the pages:
 *
 *   s_j = scale * q . k_j + B[i, j]                  ("Understanding FlashAttention
 *                                                      Pt 1", 0.2 Notation: S = QK^T/sqrt(d) + B)
 *   m   = max_j s_j,  l = sum_j exp(s_j - m),        ("Softmax does not need the matrix",
 *   o   = sum_j exp(s_j - m) v_j / l                   section "Carry the Normalizer")
 *   LSE = m + ln l                                    (natural log; kept for the backward)
 *
 * The backward is the exact gradient of that function.  The pages name the
 * recompute-from-row-statistics scheme but print no formulas, so the oracle
 * uses the textbook softmax Jacobian:
 *   dV_j = sum_i P_ij dO_i,  dP_ij = dO_i . v_j,  D_i = dO_i . o_i,
 *   dS_ij = P_ij (dP_ij - D_i),  dQ_i = scale sum_j dS_ij k_j,
 *   dK_j = scale sum_i dS_ij q_i;  GQA heads sum into their shared KV head.
 *
 * Readings where the pages are silent:
 *   causal: key j is visible from query i iff j <= i + (Nk - Nq) (bottom-right
 *           alignment, so j <= i when Nq == Nk);
 *   local (sliding-window) attention ("Understanding FlashAttention Pt 1",
 *           contents 4.2, title only): with a = i + (Nk - Nq), key j is visible
 *           iff a - window_left <= j <= a + window_right; a negative window is
 *           unbounded on that side, and causal caps the right side at 0;
 *   a row with no visible key (or every score -inf) has o = 0, LSE = -inf and
 *           zero gradients;
 *   GQA: query head h reads KV head h / (Hq / Hkv).
 *
 * Layouts (row-major, innermost last):
 *   q, o, dout, dq : [B, Nq, Hq, d]      k, v, dk, dv : [B, Nk, Hkv, d]
 *   (the forward also takes a value width dv != d: v [B, Nk, Hkv, dv] and
 *   o [B, Nq, Hq, dv], "Understanding FlashAttention Pt 1", 0.2 Notation, which
 *   gives V its own width d_v)
 *   lse            : [B, Hq, Nq]         bias         : [Hq, Nq, Nk] + b * bias_bstride
 *
 * ORACLE_MUTANT (compile-time, default 0) plants one known mistake; the test
 * suite builds such variants to show that the pins catch each of them.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

static inline long long idx4(long long b, long long n, long long h, long long c,
                             long long N, long long H, long long D) {
  return ((b * N + n) * H + h) * D + c;
}

/* Keys *lo .. *lo + count - 1 are visible from query row i; returns count. */
static inline long long key_range(long long i, long long Nq, long long Nk, int causal,
                                  int wl, int wr, long long* lo) {
  const long long a = i + (Nk - Nq); /* the key aligned with row i */
  long long first = 0, end = Nk;
  if (causal) {
#if ORACLE_MUTANT == 3
    const long long last = a - 1; /* planted: off-by-one diagonal */
#else
    const long long last = a;
#endif
    if (last + 1 < end) end = last + 1;
  }
  if (wr >= 0 && a + wr + 1 < end) end = a + wr + 1;
#if ORACLE_MUTANT == 11
  if (wl >= 0 && a - wl + 1 > first) first = a - wl + 1; /* planted: window one key short */
#else
  if (wl >= 0 && a - wl > first) first = a - wl;
#endif
  *lo = first;
  return end > first ? end - first : 0;
}

/* The same range as [*lo, end): returns end. */
static inline long long lo_end(long long i, long long Nq, long long Nk, int causal, int wl, int wr,
                               long long* lo) {
  const long long n = key_range(i, Nq, Nk, causal, wl, wr, lo);
  return *lo + n;
}

static inline int kv_head_of(int h, int Hq, int Hkv) {
#if ORACLE_MUTANT == 4
  return h % Hkv; /* planted: interleaved instead of contiguous groups */
#else
  return h / (Hq / Hkv);
#endif
}

/* Scores of one row: s[j] for the visible keys, returns the row max. */
static double row_scores(const double* qi, const double* kbase, long long kstride,
                         const double* brow, long long nvis, int d, double scale,
                         double* s) {
  double m = -INFINITY;
  for (long long j = 0; j < nvis; ++j) {
    const double* kj = kbase + j * kstride;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
#if ORACLE_MUTANT == 1
    double sj = dot; /* planted: scale dropped */
#else
    double sj = scale * dot;
#endif
    if (brow) {
#if ORACLE_MUTANT == 2
      sj -= brow[j]; /* planted: bias subtracted */
#else
      sj += brow[j];
#endif
    }
    s[j] = sj;
    if (sj > m) m = sj;
  }
  return m;
}

/*
 * One query row of the forward: the plain definition (materialise the row's
 * scores, subtract the max, exponentiate, normalise).  p[] receives the
 * normalised probabilities of the visible keys when non-NULL.
 */
static void fwd_row(const double* qi, const double* kbase, long long kstride, const double* vbase,
                    long long vstride, const double* brow, long long nvis, int d, int dv,
                    double scale, double* s, double* p, double* oi, double* lse_i) {
  for (int c = 0; c < dv; ++c) oi[c] = 0.0;
  if (nvis == 0) { *lse_i = -INFINITY; return; }
  double m = row_scores(qi, kbase, kstride, brow, nvis, d, scale, s);
  if (m == -INFINITY) { *lse_i = -INFINITY; if (p) for (long long j = 0; j < nvis; ++j) p[j] = 0.0; return; }
  double l = 0.0;
  for (long long j = 0; j < nvis; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
  for (long long j = 0; j < nvis; ++j) {
    const double w = s[j] / l;
    if (p) p[j] = w;
    const double* vj = vbase + j * vstride;
#if ORACLE_MUTANT == 10
    const double* kj = kbase + j * kstride; /* planted: K used in place of V */
    for (int c = 0; c < dv; ++c) oi[c] += w * kj[c % d];
#else
    for (int c = 0; c < dv; ++c) oi[c] += w * vj[c];
#endif
  }
#if ORACLE_MUTANT == 5
  *lse_i = log(l); /* planted: max dropped from LSE */
#else
  *lse_i = m + log(l);
#endif
}

void oracle_attn_fwd(const double* q, const double* k, const double* v,
                     const double* bias, long long bias_bstride,
                     double* o, double* lse, int B, int Hq, int Hkv, int Nq, int Nk,
                     int d, int dv, double scale, int causal, int wl, int wr) {
  const long long nbh = (long long)B * Hq;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
#pragma omp for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
      const int b = (int)(bh / Hq), h = (int)(bh % Hq);
      const int hk = kv_head_of(h, Hq, Hkv);
      const double* kb = k + idx4(b, 0, hk, 0, Nk, Hkv, d);
      const double* vb = v + idx4(b, 0, hk, 0, Nk, Hkv, dv);
      for (long long i = 0; i < Nq; ++i) {
        const double* brow = bias ? bias + b * bias_bstride + ((long long)h * Nq + i) * Nk : NULL;
        long long lo;
        const long long nvis = key_range(i, Nq, Nk, causal, wl, wr, &lo);
        const long long ks = (long long)Hkv * d, vs = (long long)Hkv * dv;
        fwd_row(q + idx4(b, i, h, 0, Nq, Hq, d), kb + lo * ks, ks, vb + lo * vs, vs, brow ? brow + lo : NULL,
                nvis, d, dv, scale, s, NULL, o + idx4(b, i, h, 0, Nq, Hq, dv),
                lse + ((long long)b * Hq + h) * Nq + i);
      }
    }
    free(s);
  }
}

/*
 * Forward for a chosen subset of rows of ONE (batch, head): used to check
 * full-size launches on sampled outputs.  q_rows[r] is query row rows[r];
 * k_head / v_head hold that head's keys/values densely as [Nk, d];
 * bias_rows[r] (optional) is bias row rows[r] over all Nk keys.
 */
void oracle_attn_fwd_rows(const double* q_rows, const double* k_head, const double* v_head,
                          const double* bias_rows, const long long* rows, int R,
                          double* o_rows, double* lse_rows, int Nq, int Nk, int d, int dv,
                          double scale, int causal, int wl, int wr) {
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < R; ++r) {
      long long lo;
      const long long nvis = key_range(rows[r], Nq, Nk, causal, wl, wr, &lo);
      fwd_row(q_rows + (long long)r * d, k_head + lo * d, d, v_head + lo * dv, dv,
              bias_rows ? bias_rows + (long long)r * Nk + lo : NULL, nvis, d, dv, scale, s, NULL,
              o_rows + (long long)r * dv, lse_rows + r);
    }
    free(s);
  }
}

/* Packed variable-length forward: sequence z owns query rows cu_q[z]..cu_q[z+1]-1
 * and key rows cu_k[z]..cu_k[z+1]-1.  q: [Tq, Hq, d], k/v: [Tk, Hkv, d],
 * lse: [Hq, Tq].  Causal masking applies inside each sequence only. */
void oracle_attn_fwd_varlen(const double* q, const double* k, const double* v,
                            const int* cu_q, const int* cu_k, int nseq,
                            double* o, double* lse, int Hq, int Hkv, int d,
                            double scale, int causal, int wl, int wr) {
  const long long Tq = cu_q[nseq];
  int maxk = 1;
  for (int z = 0; z < nseq; ++z) if (cu_k[z + 1] - cu_k[z] > maxk) maxk = cu_k[z + 1] - cu_k[z];
  const long long nzh = (long long)nseq * Hq;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * maxk);
#pragma omp for schedule(dynamic, 1)
    for (long long zh = 0; zh < nzh; ++zh) {
      const int z = (int)(zh / Hq), h = (int)(zh % Hq);
      const int hk = kv_head_of(h, Hq, Hkv);
      const long long q0 = cu_q[z], nq = cu_q[z + 1] - cu_q[z];
      const long long k0 = cu_k[z], nk = cu_k[z + 1] - cu_k[z];
      const double* kb = k + (k0 * Hkv + hk) * d;
      const double* vb = v + (k0 * Hkv + hk) * d;
      for (long long i = 0; i < nq; ++i) {
        long long lo;
        const long long nvis = key_range(i, nq, nk, causal, wl, wr, &lo);
        const long long kvs = (long long)Hkv * d;
        fwd_row(q + ((q0 + i) * Hq + h) * d, kb + lo * kvs, kvs, vb + lo * kvs, kvs, NULL, nvis, d, d, scale, s,
                NULL, o + ((q0 + i) * Hq + h) * d, lse + (long long)h * Tq + q0 + i);
      }
    }
    free(s);
  }
}

/*
 * Streaming replay of the forward: the keys of each row are visited in blocks
 * of `block` and only the state (m, l, a) is carried, with the rescale by
 * exp(m - m') whenever a block raises the maximum, then one normalisation at
 * the end ("Softmax does not need the matrix", "Carry the Normalizer" and the
 * lab's online-tiled row).  *rescales counts the blocks that raised an
 * already-finite running max (the rescale events the lab plots).
 */
void oracle_attn_fwd_stream(const double* q, const double* k, const double* v,
                            const double* bias, long long bias_bstride,
                            double* o, double* lse, int B, int Hq, int Hkv, int Nq, int Nk,
                            int d, double scale, int causal, int wl, int wr, int block,
                            long long* rescales) {
  const long long nbh = (long long)B * Hq;
  long long total = 0;
#pragma omp parallel reduction(+ : total)
  {
    double* a = (double*)malloc(sizeof(double) * d);
    double* sb = (double*)malloc(sizeof(double) * block);
#pragma omp for schedule(dynamic, 1)
    for (long long bh = 0; bh < nbh; ++bh) {
      const int b = (int)(bh / Hq), h = (int)(bh % Hq);
      const int hk = kv_head_of(h, Hq, Hkv);
      for (long long i = 0; i < Nq; ++i) {
        const double* qi = q + idx4(b, i, h, 0, Nq, Hq, d);
        const double* brow = bias ? bias + b * bias_bstride + ((long long)h * Nq + i) * Nk : NULL;
        long long lo;
        const long long end = lo_end(i, Nq, Nk, causal, wl, wr, &lo);
        double m = -INFINITY, l = 0.0;
        for (int c = 0; c < d; ++c) a[c] = 0.0;
        for (long long j0 = lo; j0 < end; j0 += block) {
          const long long nb = end - j0 < block ? end - j0 : block;
          const double mb = row_scores(qi, k + idx4(b, j0, hk, 0, Nk, Hkv, d), (long long)Hkv * d,
                                       brow ? brow + j0 : NULL, nb, d, scale, sb);
          const double mnew = mb > m ? mb : m;
          if (mnew == -INFINITY) continue; /* nothing finite seen yet */
          if (m != -INFINITY && mnew > m) ++total;
          const double alpha = (m == -INFINITY) ? 0.0 : exp(m - mnew);
#if ORACLE_MUTANT == 9
          l = l + 0.0 * alpha; /* planted: old state not rescaled */
#else
          l *= alpha;
          for (int c = 0; c < d; ++c) a[c] *= alpha;
#endif
          for (long long j = 0; j < nb; ++j) {
            const double e = exp(sb[j] - mnew);
            l += e;
            const double* vj = v + idx4(b, j0 + j, hk, 0, Nk, Hkv, d);
            for (int c = 0; c < d; ++c) a[c] += e * vj[c];
          }
          m = mnew;
        }
        double* oi = o + idx4(b, i, h, 0, Nq, Hq, d);
        double* li = lse + ((long long)b * Hq + h) * Nq + i;
        if (m == -INFINITY) {
          for (int c = 0; c < d; ++c) oi[c] = 0.0;
          *li = -INFINITY;
        } else {
          for (int c = 0; c < d; ++c) oi[c] = a[c] / l;
          *li = m + log(l);
        }
      }
    }
    free(a);
    free(sb);
  }
  if (rescales) *rescales = total;
}

/*
 * Backward: exact gradient of the forward above.  Work is split over
 * (batch, KV head) so that every dK/dV row has a single writer; the G query
 * heads of a group are visited one after another.
 */
void oracle_attn_bwd(const double* q, const double* k, const double* v,
                     const double* bias, long long bias_bstride, const double* dout,
                     double* dq, double* dk, double* dv, int B, int Hq, int Hkv, int Nq,
                     int Nk, int d, int dvw, double scale, int causal, int wl, int wr) {
  /* dvw: width of V, O, dO and dV (d_v); d: width of Q, K, dQ and dK */
  const int G = Hq / Hkv;
  const long long nbk = (long long)B * Hkv;
  memset(dk, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
  memset(dv, 0, sizeof(double) * (size_t)B * Nk * Hkv * dvw);
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* p = (double*)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
    double* oi = (double*)malloc(sizeof(double) * dvw);
#pragma omp for schedule(dynamic, 1)
    for (long long bk = 0; bk < nbk; ++bk) {
      const int b = (int)(bk / Hkv), hk = (int)(bk % Hkv);
      for (int g = 0; g < G; ++g) {
        int h = hk * G + g;
#if ORACLE_MUTANT == 4
        h = g * Hkv + hk; /* planted: interleaved groups (matches kv_head_of above) */
#endif
        const double* kb = k + idx4(b, 0, hk, 0, Nk, Hkv, d);
        const double* vb = v + idx4(b, 0, hk, 0, Nk, Hkv, dvw);
        for (long long i = 0; i < Nq; ++i) {
          const double* qi = q + idx4(b, i, h, 0, Nq, Hq, d);
          const double* doi = dout + idx4(b, i, h, 0, Nq, Hq, dvw);
          double* dqi = dq + idx4(b, i, h, 0, Nq, Hq, d);
          const double* brow = bias ? bias + b * bias_bstride + ((long long)h * Nq + i) * Nk : NULL;
          long long lo;
          const long long nvis = key_range(i, Nq, Nk, causal, wl, wr, &lo);
          const long long kvs = (long long)Hkv * d, vvs = (long long)Hkv * dvw;
          double lse_i;
          fwd_row(qi, kb + lo * kvs, kvs, vb + lo * vvs, vvs, brow ? brow + lo : NULL, nvis, d, dvw, scale, s, p,
                  oi, &lse_i);
          for (int c = 0; c < d; ++c) dqi[c] = 0.0;
          if (lse_i == -INFINITY) continue;
          double Di = 0.0;
          for (int c = 0; c < dvw; ++c) Di += doi[c] * oi[c];
          for (long long j = 0; j < nvis; ++j) { /* key lo + j; p[j] is its probability */
            const double* kj = kb + (lo + j) * kvs;
            const double* vj = vb + (lo + j) * vvs;
            double* dkj = dk + idx4(b, lo + j, hk, 0, Nk, Hkv, d);
            double* dvj = dv + idx4(b, lo + j, hk, 0, Nk, Hkv, dvw);
            double dP = 0.0;
            for (int c = 0; c < dvw; ++c) dP += doi[c] * vj[c];
#if ORACLE_MUTANT == 6
            const double dS = p[j] * (dP + Di); /* planted: wrong sign */
#else
            const double dS = p[j] * (dP - Di);
#endif
#if ORACLE_MUTANT == 8
            for (int c = 0; c < dvw; ++c) dvj[c] += dS * doi[c]; /* planted: dS in place of P */
#else
            for (int c = 0; c < dvw; ++c) dvj[c] += p[j] * doi[c];
#endif
#if ORACLE_MUTANT == 7
            for (int c = 0; c < d; ++c) dqi[c] += dS * kj[c]; /* planted: scale dropped */
#else
            for (int c = 0; c < d; ++c) dqi[c] += scale * dS * kj[c];
#endif
            for (int c = 0; c < d; ++c) dkj[c] += scale * dS * qi[c];
          }
        }
      }
    }
    free(s);
    free(p);
    free(oi);
  }
}

/*
 * FP8 inputs (the handbook's contents name FlashAttention-3's FP8 path, 5.4 to
 * 5.6, without a definition): the oracle for an FP8 forward is the exact
 * attention of the quantised-then-dequantised inputs, so only the rounding to
 * e4m3 is defined here.  e4m3 (the OCP 8-bit floating-point format): 4
 * exponent bits with bias 7, 3 mantissa bits, no infinities, largest finite
 * value 448, subnormals m * 2^-9.  Rounding is to nearest with ties to an even
 * mantissa; magnitudes at or above 448 saturate to 448.  out = q(x / scale) *
 * scale for a positive per-tensor scale.
 */
static double round_e4m3(double x) {
  if (x != x) return x;
  const double a = fabs(x);
  if (a >= 448.0) return copysign(448.0, x);
  int ex;
  frexp(a, &ex);                              /* a = f * 2^ex, f in [0.5, 1) */
  int e = ex - 1;                             /* a in [2^e, 2^(e+1)) */
  if (a == 0.0 || e < -6) e = -6;             /* subnormal range: same spacing as 2^-6 */
  const double spacing = ldexp(1.0, e - 3);   /* 3 mantissa bits */
  const double r = nearbyint(a / spacing);    /* default rounding mode: ties to even */
  return copysign(r * spacing, x);
}

void oracle_quantize_e4m3(const double* x, long long n, double scale, double* out) {
  for (long long i = 0; i < n; ++i) out[i] = round_e4m3(x[i] / scale) * scale;
}

/*
 * Per-head quantisation of x [B, N, H, d] for the FP8 forward: for each
 * (batch b, head h), amax = max |x| over that head's rows, scale = amax / 448
 * (1 when amax = 0), and each element becomes e4m3(x / scale) * scale.  The
 * scale and the quotient are taken in fp32 (IEEE division), the precision in
 * which the kernel decides each e4m3 code, so that both sides pick the same
 * code; the returned values and scales are exact in fp64.
 */
void oracle_quantize_e4m3_heads(const double* x, int B, int N, int H, int d, double* out, double* scales) {
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      double amax = 0.0;
      for (int n = 0; n < N; ++n) {
        const double* row = x + (((long long)b * N + n) * H + h) * d;
        for (int c = 0; c < d; ++c) if (fabs(row[c]) > amax) amax = fabs(row[c]);
      }
      const float scale = amax > 0.0 ? (float)amax / 448.0f : 1.0f;
      scales[b * H + h] = scale;
      for (int n = 0; n < N; ++n) {
        const long long o = (((long long)b * N + n) * H + h) * d;
        for (int c = 0; c < d; ++c) {
          const float qf = (float)x[o + c] / scale;
          out[o + c] = round_e4m3((double)qf) * (double)scale;
        }
      }
    }
}

/*
 * Merge of partial results over disjoint key shards: shard t holds the exact
 * attention (o_t, lse_t) of the row over its own keys only.  The combined row
 * follows from the same rescale-and-add recurrence as the streaming forward:
 * weights exp(lse_t - lse), lse = m + ln sum_t exp(lse_t - m).
 * o_parts: [T, R, d], lse_parts: [T, R].
 */
void oracle_merge_partials(const double* o_parts, const double* lse_parts, int T, int R, int d,
                           double* o, double* lse) {
  for (int r = 0; r < R; ++r) {
    double m = -INFINITY;
    for (int t = 0; t < T; ++t) if (lse_parts[(long long)t * R + r] > m) m = lse_parts[(long long)t * R + r];
    double* orow = o + (long long)r * d;
    for (int c = 0; c < d; ++c) orow[c] = 0.0;
    if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
    double l = 0.0;
    for (int t = 0; t < T; ++t) l += exp(lse_parts[(long long)t * R + r] - m);
    for (int t = 0; t < T; ++t) {
      const double w = exp(lse_parts[(long long)t * R + r] - m) / l;
      const double* op = o_parts + ((long long)t * R + r) * d;
      for (int c = 0; c < d; ++c) orow[c] += w * op[c];
    }
    lse[r] = m + log(l);
  }
}
