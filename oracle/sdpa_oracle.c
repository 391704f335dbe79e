/*
 * Oracle for the fused scaled-dot-product-attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
 * fp64 CPU definition the CUDA library is checked against.  Only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark may load it; the
 * library never does, and the two share no code.
 *
 * What it computes (for every batch b, query head h, query row i):
 *
 *   s[j]  = scale * sum_c q[b,h,i,c] * k[b,hk,j,c]            (Axon PR "Add
 *           scaled_dot_product_attention", description: softmax(Q.K^T*scale
 *           + mask).V)
 *         + rel_h[i, kh(j)] + rel_w[i, kw(j)]                   (mlx-examples
 *           issue "segment_anything: fuse attention ...": the SAM image
 *           encoder adds add_decomposed_rel_pos's bias to (q*scale)@k^T
 *           before the softmax)
 *         + mask term                                           (Axon PR, the
 *           :mask option: causal, {causal, offset}, {sliding_window, w},
 *           {sliding_window, w, offset}, runtime boolean/float tensor; the
 *           mlx issue: the mask is an additive array broadcast to
 *           [B, N, T_q, T_kv])
 *   m     = max_j s[j];  p[j] = exp(s[j] - m);  l = sum_j p[j]
 *   out   = sum_j (p[j] / l) * v[b,hk,j,:];   lse = m + log(l)
 *
 * with the decomposed relative-position terms of the SAM image encoder
 * (the candle PR "SDPA with Relative Positional Embeddings": term_h and
 * term_w injected into the scores), computed from the UNSCALED query:
 *
 *   rel_h[i, kh] = sum_c q[i,c] * Rh[qh(i) - kh + Kh - 1, c]
 *   rel_w[i, kw] = sum_c q[i,c] * Rw[qw(i) - kw + Kw - 1, c]
 *   qh(i) = i / Qw, qw(i) = i % Qw, kh(j) = j / Kw, kw(j) = j % Kw
 *
 * (Qh, Qw) is the query patch grid and (Kh, Kw) the key patch grid.  They may
 * differ: the formula is read with each coordinate taken from its own grid
 * and the shift from the key grid, so the offset qh - kh runs from -(Kh - 1)
 * to Qh - 1 and Rh needs Qh + Kh - 1 rows (Rw: Qw + Kw - 1); with equal grids
 * that is the 2*K - 1 rows of SAM's tables.
 *
 * Readings of what the pages leave open (each one stated where it is used):
 *   - GQA/MQA "repeat key/value heads to match the query": each kv head is
 *     repeated g = Hq/Hkv times consecutively, so hk = h / g.
 *   - {causal, offset}: key j is visible from row i iff j <= i + offset.
 *   - {sliding_window, w, offset}: visible iff i + offset - w < j <= i + offset
 *     (w keys, the diagonal included).
 *   - boolean mask: nonzero = attend, zero = excluded (-inf).
 *   - a row with no visible key: output 0, lse = -inf.
 *
 * Everything is double precision; the inputs are the already-rounded values
 * of whatever I/O type the device path uses, widened to double by the caller.
 * The score row of each query is materialised in full, as in the unfused
 * matmul -> +bias -> softmax -> matmul formulation the mlx issue describes.
 *
 * ORACLE_PLANT (compile-time, default 0) exists only so that a test can build
 * a deliberately wrong copy of this file and check that the oracle's pins
 * reject it; the shipped build never defines it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

enum { MASK_NONE = 0, MASK_CAUSAL = 1, MASK_SLIDING = 2, MASK_FLOAT = 3, MASK_BOOL = 4 };

/* Visibility of key j from query row i under the causal / sliding readings. */
static int visible(int kind, long long i, long long j, long long offset, long long window) {
  if (kind == MASK_CAUSAL) {
#if ORACLE_PLANT == 7
    return j < i + offset;
#else
    return j <= i + offset;
#endif
  }
  if (kind == MASK_SLIDING) {
#if ORACLE_PLANT == 8
    return (i + offset - window <= j) && (j <= i + offset);
#else
    return (i + offset - window < j) && (j <= i + offset);
#endif
  }
  return 1;
}

static double dot(const double* a, const double* b, int n) {
  double acc = 0.0;
  for (int c = 0; c < n; ++c) acc += a[c] * b[c];
  return acc;
}

/*
 * Computes the rows listed in `rows` (all Tq rows when rows == NULL) for every
 * (b, h).  Shapes (contiguous, row-major):
 *   q   [B, Hq,  Tq,  d]      k, v [B, Hkv, Tkv, d]
 *   out [B, Hq,  nrows, d]    lse  [B, Hq, nrows]      (lse may be NULL)
 *   weights [B, Hq, nrows, Tkv] (may be NULL; the softmax weights p/l)
 *   fmask / bmask: element (b, h, i, j) at b*msb + h*msh + i*msq + j
 *   rel_h [q_h + k_h - 1, d], rel_w [q_w + k_w - 1, d]  (both NULL: no rel-pos term)
 * Returns 0, or -1 on an inconsistent argument.
 */
int oracle_sdpa_rows(const double* q, const double* k, const double* v,
                     int B, int Hq, int Hkv, int Tq, int Tkv, int d, double scale,
                     int mask_kind, long long offset, long long window,
                     const double* fmask, const unsigned char* bmask,
                     long long msb, long long msh, long long msq,
                     const double* rel_h, const double* rel_w,
                     int q_h, int q_w, int k_h, int k_w,
                     const long long* rows, long long nrows,
                     double* out, double* lse, double* weights) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Tq < 0 || Tkv < 0 || d <= 0) return -1;
  if (Hq % Hkv != 0) return -1;
  const int use_rel = (rel_h != NULL) && (rel_w != NULL);
  if ((rel_h != NULL) != (rel_w != NULL)) return -1;
  if (use_rel && ((long long)q_h * q_w != Tq || (long long)k_h * k_w != Tkv)) return -1;
  if (mask_kind == MASK_FLOAT && fmask == NULL) return -1;
  if (mask_kind == MASK_BOOL && bmask == NULL) return -1;
  if (rows == NULL) nrows = Tq;
  const int g = Hq / Hkv;
  const long long total = (long long)B * Hq * nrows;

#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Tkv > 0 ? Tkv : 1));
    double* relh = (double*)malloc(sizeof(double) * (size_t)(k_h > 0 ? k_h : 1));
    double* relw = (double*)malloc(sizeof(double) * (size_t)(k_w > 0 ? k_w : 1));
#pragma omp for schedule(dynamic, 4)
    for (long long task = 0; task < total; ++task) {
      const long long r = task % nrows;
      const long long bh = task / nrows;
      const int h = (int)(bh % Hq);
      const int b = (int)(bh / Hq);
      const long long i = rows ? rows[r] : r;
#if ORACLE_PLANT == 6
      const int hk = h % Hkv;
#else
      const int hk = h / g;
#endif
      const double* qi = q + (((long long)b * Hq + h) * Tq + i) * d;
      const double* kb = k + ((long long)b * Hkv + hk) * (long long)Tkv * d;
      const double* vb = v + ((long long)b * Hkv + hk) * (long long)Tkv * d;
      double* o = out + task * d;

      if (use_rel) {
        /* SAM add_decomposed_rel_pos: project the unscaled query onto the
           rows of each table picked by the relative offset. */
#if ORACLE_PLANT == 4
        const long long qh = i % q_w, qw = i / q_w;
#else
        const long long qh = i / q_w, qw = i % q_w;
#endif
        const double* th = rel_h;
        const double* tw = rel_w;
#if ORACLE_PLANT == 3
        th = rel_w; tw = rel_h;
#endif
        for (int a = 0; a < k_h; ++a) {
#if ORACLE_PLANT == 1
          const long long idx = a - qh + k_h - 1;
#elif ORACLE_PLANT == 13
          const long long idx = (qh - a + q_h - 1 + (q_h + k_h - 1)) % (q_h + k_h - 1);
#else
          const long long idx = qh - a + k_h - 1;
#endif
#if ORACLE_PLANT == 3
          relh[a] = dot(qi, th + (idx % (2 * k_w - 1)) * d, d); /* swapped tables differ in size */
#else
          relh[a] = dot(qi, th + idx * d, d);
#endif
        }
        for (int a = 0; a < k_w; ++a) {
#if ORACLE_PLANT == 13
          const long long idx = (qw - a + q_w - 1 + (q_w + k_w - 1)) % (q_w + k_w - 1);
#else
          const long long idx = qw - a + k_w - 1;
#endif
#if ORACLE_PLANT == 2
          relw[a] = 0.0;
#else
#if ORACLE_PLANT == 3
          relw[a] = dot(qi, tw + (idx % (2 * k_h - 1)) * d, d);
#else
          relw[a] = dot(qi, tw + idx * d, d);
#endif
#endif
        }
      }

      double m = -INFINITY;
      for (long long j = 0; j < Tkv; ++j) {
        double x = scale * dot(qi, kb + j * d, d);
        if (use_rel) {
#if ORACLE_PLANT == 5
          x += scale * (relh[j / k_w] + relw[j % k_w]);
#else
          x += relh[j / k_w] + relw[j % k_w];
#endif
        }
        if (mask_kind == MASK_CAUSAL || mask_kind == MASK_SLIDING) {
          if (!visible(mask_kind, i, j, offset, window)) x = -INFINITY;
        } else if (mask_kind == MASK_FLOAT) {
#if ORACLE_PLANT == 11
          x += fmask[h * msh + i * msq + j];
#else
          x += fmask[b * msb + h * msh + i * msq + j];
#endif
        } else if (mask_kind == MASK_BOOL) {
          const unsigned char keep = bmask[b * msb + h * msh + i * msq + j];
#if ORACLE_PLANT == 12
          if (keep) x = -INFINITY;
#else
          if (!keep) x = -INFINITY;
#endif
        }
        s[j] = x;
        if (x > m) m = x;
      }

      memset(o, 0, sizeof(double) * (size_t)d);
      if (m == -INFINITY) {
        /* No visible key: the reading is a zero row with lse = -inf. */
        if (lse) lse[task] = -INFINITY;
        if (weights) for (long long j = 0; j < Tkv; ++j) weights[task * Tkv + j] = 0.0;
        continue;
      }
      double l = 0.0;
      for (long long j = 0; j < Tkv; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
      }
      for (long long j = 0; j < Tkv; ++j) {
#if ORACLE_PLANT == 10
        const double w = s[j];
#else
        const double w = s[j] / l;
#endif
        if (weights) weights[task * Tkv + j] = w;
        if (w == 0.0) continue;
        const double* vj = vb + j * d;
        for (int c = 0; c < d; ++c) o[c] += w * vj[c];
      }
      if (lse) lse[task] = m + log(l);
    }
    free(s);
    free(relh);
    free(relw);
  }
  return 0;
}

/* Number of OpenMP threads the oracle will use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
