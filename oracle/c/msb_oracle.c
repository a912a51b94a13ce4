/*
 * msb_oracle.c -- plain C99 restatement of one sparse-MoE block decode step, in double
 * precision.  TEST INFRASTRUCTURE: only the tests load it (to cross-check the numpy
 * oracle); it shares no code with the CUDA library and includes none of its headers.
 *
 * Per token t, in the order of "KAIST drops calibration from MoE decoding, speeds up
 * blocks by up to 2.69x over vLLM" (opening paragraph, "Top-k instead of a threshold",
 * "A reader built from weights alone") and "MoE top_k override (--moe-top-k)" ("Ce que
 * ca fait"):
 *   1. router: logits = x . W_router, softmax over E, the K largest logits (ties to the
 *      lower expert index); weights = their probabilities, renormalised if asked;
 *   2. per routed expert: ternary sketch of each gate row (Ternary Weight Networks:
 *      T = sign(W) [|W| > 0.7 mean|W|], alpha = mean |W| over the kept entries, stored
 *      as float), scores s_j = alpha_j |T_j . x|;
 *   3. selection: the k channels of highest score (ties to the lower index), or
 *      {j : s_j > tau} (threshold comparator), or every channel (dense);
 *   4. y_e = sum over the selected j of silu(gate_j . x) (up_j . x) down[:, j], plus
 *      A_e (B_e x) unless dense;
 *   5. y = sum_e w_e y_e.
 * Every sum is a plain left-to-right loop in double; weights and x are BF16 bit
 * patterns, widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf(uint16_t b) {
  union {
    uint32_t u;
    float f;
  } v;
  v.u = (uint32_t)b << 16;
  return (double)v.f;
}

/* Ternary sketch of one row (length d): t[i] in {-1, 0, 1}; returns alpha (as float). */
static float sketch_row(const uint16_t* row, int d, int8_t* t) {
  double total = 0.0, kept = 0.0;
  int n = 0;
  for (int i = 0; i < d; ++i) total += fabs(bf(row[i]));
  for (int i = 0; i < d; ++i) {
    const double w = bf(row[i]);
    t[i] = 0;
    if (10.0 * d * fabs(w) > 7.0 * total) { /* |w| > 0.7 * total / d, exactly */
      t[i] = w > 0 ? 1 : -1;
      kept += fabs(w);
      ++n;
    }
  }
  return n ? (float)(kept / n) : 0.0f;
}

/* key (score desc, index asc): does channel a come before channel b? */
static int before(const double* s, int a, int b) { return s[a] > s[b] || (s[a] == s[b] && a < b); }

/*
 * One block step for B tokens.
 *   x        [B][d] BF16            router [d][E] BF16
 *   gate, up [E][I][d] BF16         down [E][d][I] BF16
 *   lr_a     [E][d][r] BF16         lr_b [E][r][d] BF16 (may be NULL when r == 0)
 *   mode     0: top-k (k channels), 1: threshold (s > tau), 2: dense (all channels, no
 *            low-rank term)
 * Outputs: y [B][d], ids [B][K], w [B][K], sel [B][K][I] (the selected channels,
 * ascending; nsel [B][K] of them), scores [B][K][I] (0 in dense mode).
 * Returns 0, or -1 on a bad argument.
 */
int msb_oracle_block(const uint16_t* x, int B, const uint16_t* router, const uint16_t* gate,
                     const uint16_t* up, const uint16_t* down, const uint16_t* lr_a,
                     const uint16_t* lr_b, int d, int I, int E, int K, int r, int renorm, int mode,
                     int k, double tau, double* y, int32_t* ids, double* w, int32_t* sel,
                     int32_t* nsel, double* scores) {
  if (B < 1 || d < 1 || I < 1 || E < 1 || K < 1 || K > E || r < 0 || mode < 0 || mode > 2 ||
      (mode == 0 && (k < 1 || k > I)) || (r > 0 && mode != 2 && (!lr_a || !lr_b)))
    return -1;
  double* xv = malloc(sizeof(double) * d);
  double* logits = malloc(sizeof(double) * E);
  double* p = malloc(sizeof(double) * E);
  int8_t* t = malloc((size_t)d);
  double* s = malloc(sizeof(double) * I);
  double* ye = malloc(sizeof(double) * d);
  double* z = malloc(sizeof(double) * (r > 0 ? r : 1));
  char* taken = malloc((size_t)E);
  if (!xv || !logits || !p || !t || !s || !ye || !z || !taken) {
    free(xv); free(logits); free(p); free(t); free(s); free(ye); free(z); free(taken);
    return -1;
  }
  for (int tok = 0; tok < B; ++tok) {
    for (int i = 0; i < d; ++i) xv[i] = bf(x[(size_t)tok * d + i]);
    /* 1. router */
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += xv[i] * bf(router[(size_t)i * E + e]);
      logits[e] = acc;
      if (acc > mx) mx = acc;
    }
    double psum = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp(logits[e] - mx);
      psum += p[e];
    }
    memset(taken, 0, (size_t)E);
    double wsum = 0.0;
    for (int q = 0; q < K; ++q) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || logits[e] > logits[best])) best = e; /* ties: lower e */
      taken[best] = 1;
      ids[tok * K + q] = best;
      w[tok * K + q] = p[best] / psum;
      wsum += w[tok * K + q];
    }
    if (renorm)
      for (int q = 0; q < K; ++q) w[tok * K + q] /= wsum;
    for (int i = 0; i < d; ++i) y[(size_t)tok * d + i] = 0.0;

    for (int q = 0; q < K; ++q) {
      const int e = ids[tok * K + q];
      const uint16_t* G = gate + (size_t)e * I * d;
      const uint16_t* U = up + (size_t)e * I * d;
      const uint16_t* D = down + (size_t)e * d * I;
      double* sc = scores + ((size_t)tok * K + q) * I;
      int32_t* sl = sel + ((size_t)tok * K + q) * I;
      /* 2. scores */
      for (int j = 0; j < I; ++j) {
        sc[j] = 0.0;
        if (mode == 2) continue;
        const float alpha = sketch_row(G + (size_t)j * d, d, t);
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += t[i] * xv[i];
        sc[j] = (double)alpha * fabs(acc);
      }
      memcpy(s, sc, sizeof(double) * I);
      /* 3. selection (ascending channel order) */
      int n = 0;
      for (int j = 0; j < I; ++j) {
        int keep;
        if (mode == 2) {
          keep = 1;
        } else if (mode == 1) {
          keep = s[j] > tau;
        } else {
          int rank = 0; /* channels ahead of j under the key */
          for (int i = 0; i < I; ++i) rank += before(s, i, j);
          keep = rank < k;
        }
        if (keep) sl[n++] = j;
      }
      nsel[tok * K + q] = n;
      /* 4. gathered SwiGLU expert over the selected channels, then the low-rank term */
      for (int i = 0; i < d; ++i) ye[i] = 0.0;
      for (int m = 0; m < n; ++m) {
        const int j = sl[m];
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) {
          g += bf(G[(size_t)j * d + i]) * xv[i];
          u += bf(U[(size_t)j * d + i]) * xv[i];
        }
        const double h = g / (1.0 + exp(-g)) * u;
        for (int i = 0; i < d; ++i) ye[i] += h * bf(D[(size_t)i * I + j]);
      }
      if (r > 0 && mode != 2) {
        for (int c = 0; c < r; ++c) {
          double acc = 0.0;
          for (int i = 0; i < d; ++i) acc += bf(lr_b[((size_t)e * r + c) * d + i]) * xv[i];
          z[c] = acc;
        }
        for (int i = 0; i < d; ++i) {
          double acc = 0.0;
          for (int c = 0; c < r; ++c) acc += bf(lr_a[((size_t)e * d + i) * r + c]) * z[c];
          ye[i] += acc;
        }
      }
      /* 5. combine */
      for (int i = 0; i < d; ++i) y[(size_t)tok * d + i] += w[tok * K + q] * ye[i];
    }
  }
  free(xv); free(logits); free(p); free(t); free(s); free(ye); free(z); free(taken);
  return 0;
}
