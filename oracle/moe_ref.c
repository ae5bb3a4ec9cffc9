/* moe_ref.c -- a second CPU oracle of the sparse MoE FFN layer forward, in
 * plain C loops and float64.  TEST INFRASTRUCTURE ONLY: loaded by tests/ (and
 * compiled by the build entry point); the library never links or calls it.
 *
 * It computes the same definition as oracle/moe_oracle.py, written again
 * from the sources so the two can check each other:
 *   1. r_t = 1 / sqrt((1/d) sum_i x_ti^2 + eps)            (CODA thread, RMSNorm)
 *   2. l_te = fp32( r_t * sum_i (x_ti gamma_i) Wr_ie + b_e ) (CODA thread: r after
 *      the router GEMM, before the top-k; MoE glossary, gating network)
 *   3. the k largest logits, largest first, ties to the lower expert; gate =
 *      softmax over all E at the chosen experts, optionally renormalised over
 *      the k chosen                                           (MoE glossary, Top-k Gating)
 *   4. capacity C = floor((T*k)/E * capacity_factor); an expert keeps its
 *      first C assignments in assignment order t*k + j       (MoE glossary, Expert Capacity)
 *   5. kept assignments grouped by expert, assignment order inside a group;
 *      perm[offsets[e] + rank] = a, inv_perm[a] = that position or -1
 *                                                            (OmniMoE summary, section 2.2)
 *   6. y_a = (silu(r_t (x_t gamma) W1_e) * (r_t (x_t gamma) W3_e)) W2_e, expert e's
 *      columns [offs[e], offs[e+1]) of W1, W3 and rows of W2 (nanoMOE notes,
 *      "Offset Calculation")                                 (CODA thread: r in GEMM 1)
 *   7. out_t = sum over kept slots j, in slot order, of gate_tj * y_(t*k+j)
 *
 * bf16 inputs are bit patterns (uint16), widened exactly; every sum and
 * product is float64; the logits are rounded once to float32 and the top-k
 * is decided on those values.  Sums run in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Returns 0 on success, 1 on an expert id out of range, 2 on an allocation failure. */
int moe_ref_layer(const uint16_t* x, const uint16_t* gamma, const uint16_t* Wr, const double* bias,
                  const uint16_t* W1, const uint16_t* W3, const uint16_t* W2, const int32_t* offs,
                  int32_t T, int32_t d, int32_t E, int32_t k, double eps, double capacity_factor,
                  int32_t renormalize, const int32_t* idx_override,
                  double* r, float* logits, int32_t* idx, double* gate, int32_t* counts, int32_t* offsets,
                  int32_t* perm, int32_t* inv_perm, double* out) {
  const int32_t F = offs[E];
  const int64_t nA = (int64_t)T * k;
  double* xg = (double*)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
  double* h = (double*)malloc(sizeof(double) * (size_t)(F > 0 ? F : 1));
  double* p = (double*)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
  int32_t* rank = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nA > 0 ? nA : 1));
  int32_t* run = (int32_t*)calloc((size_t)(E > 0 ? E : 1), sizeof(int32_t));
  if (!xg || !h || !p || !rank || !run) {
    free(xg); free(h); free(p); free(rank); free(run);
    return 2;
  }
  int status = 0;

  /* 1.-3. statistic, router, top-k, gates */
  for (int32_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      const double v = bf(x[(int64_t)t * d + i]);
      ss += v * v;
    }
    r[t] = 1.0 / sqrt(ss / (double)d + eps);
    for (int32_t i = 0; i < d; ++i) xg[i] = bf(x[(int64_t)t * d + i]) * bf(gamma[i]);
    for (int32_t e = 0; e < E; ++e) {
      double s = 0.0;
      for (int32_t i = 0; i < d; ++i) s += xg[i] * bf(Wr[(int64_t)i * E + e]);
      double l = r[t] * s;
      if (bias) l += bias[e];
      logits[(int64_t)t * E + e] = (float)l;
    }
    const float* lt = logits + (int64_t)t * E;
    if (idx_override) {
      for (int32_t j = 0; j < k; ++j) idx[(int64_t)t * k + j] = idx_override[(int64_t)t * k + j];
    } else {
      for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
          int used = 0;
          for (int32_t q = 0; q < j; ++q) used |= idx[(int64_t)t * k + q] == e;
          if (!used && (best < 0 || (double)lt[e] > (double)lt[best])) best = e;
        }
        idx[(int64_t)t * k + j] = best;
      }
    }
    double m = (double)lt[0];
    for (int32_t e = 1; e < E; ++e)
      if ((double)lt[e] > m) m = (double)lt[e];
    double z = 0.0;
    for (int32_t e = 0; e < E; ++e) {
      p[e] = exp((double)lt[e] - m);
      z += p[e];
    }
    double gs = 0.0;
    for (int32_t j = 0; j < k; ++j) {
      const int32_t e = idx[(int64_t)t * k + j];
      if (e < 0 || e >= E) {
        status = 1;
        gate[(int64_t)t * k + j] = 0.0;
        continue;
      }
      gate[(int64_t)t * k + j] = p[e] / z;
      gs += gate[(int64_t)t * k + j];
    }
    if (renormalize)
      for (int32_t j = 0; j < k; ++j) gate[(int64_t)t * k + j] /= gs;
  }
  if (status) goto done;

  /* 4.-5. counts, ranks in assignment order, capacity, expert-centric order */
  {
    const int capped = capacity_factor > 0.0;
    const int64_t C = capped ? (int64_t)floor((double)nA / (double)E * capacity_factor) : nA;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < nA; ++a) {
      const int32_t e = idx[a];
      rank[a] = run[e]++;
      counts[e] += 1;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) {
      const int64_t kept = counts[e] < C ? counts[e] : C;
      offsets[e + 1] = offsets[e] + (int32_t)kept;
    }
    for (int64_t a = 0; a < nA; ++a) {
      if (rank[a] < C) {
        const int32_t pos = offsets[idx[a]] + rank[a];
        perm[pos] = (int32_t)a;
        inv_perm[a] = pos;
      } else {
        inv_perm[a] = -1;
      }
    }
  }

  /* 6.-7. experts and combine, slot order */
  for (int64_t i = 0; i < (int64_t)T * d; ++i) out[i] = 0.0;
  for (int32_t t = 0; t < T; ++t) {
    for (int32_t i = 0; i < d; ++i) xg[i] = bf(x[(int64_t)t * d + i]) * bf(gamma[i]);
    for (int32_t j = 0; j < k; ++j) {
      const int64_t a = (int64_t)t * k + j;
      if (inv_perm[a] < 0) continue;
      const int32_t e = idx[a];
      const int32_t o0 = offs[e], o1 = offs[e + 1];
      for (int32_t n = o0; n < o1; ++n) {
        double u = 0.0, v = 0.0;
        for (int32_t i = 0; i < d; ++i) {
          u += xg[i] * bf(W1[(int64_t)i * F + n]);
          v += xg[i] * bf(W3[(int64_t)i * F + n]);
        }
        h[n - o0] = silu(r[t] * u) * (r[t] * v);
      }
      for (int32_t c = 0; c < d; ++c) {
        double y = 0.0;
        for (int32_t n = o0; n < o1; ++n) y += h[n - o0] * bf(W2[(int64_t)n * d + c]);
        out[(int64_t)t * d + c] += gate[a] * y;
      }
    }
  }

done:
  free(xg); free(h); free(p); free(rank); free(run);
  return status;
}
