/*
 * CPU oracle for one decode step of a Kimi-K3-style mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, header,
 * table or helper with the CUDA library; both sides receive the same bf16
 * input bits from the seeded generator and nothing else.
 *
 * What it computes, in plain loops and in double precision (fp64), in the
 * order the layer is defined:
 *   1. h = residual_in + W_o . attn_out                     (o_proj + residual)
 *   2. rstd = 1 / sqrt(mean(h^2) + eps);  x = h * rstd * gamma      (RMSNorm)
 *   3. logits = W_r . x                                          (router GEMV)
 *   4. idx = the k largest logits, descending, ties to the lower expert index;
 *      gate = softmax over the k selected logits                 (top-k gates)
 *   5. per selected expert e: g = W_gu[e][0:I] . x, u = W_gu[e][I:2I] . x,
 *      a = silu(g) * u,  y = W_down[e] . a                        (SwiGLU expert)
 *   6. out = bf16_rne(h + sum_j gate_j * y_j)                 (gate-weighted combine)
 *
 * Sources.  "vLLM speeds up Kimi K3 up to 1.9x on NVIDIA GB300 with
 * agent-assisted kernels", section "How the specialised decode path works":
 * 16 of 896 experts are active per token; the attention output projection is
 * followed by the residual step; the expert work is the dense per-expert
 * kernels chosen by batch size.  The remaining definitions (RMSNorm with eps
 * 1e-6, router in fp32 accumulation, softmax gates renormalised over the
 * selected experts, SwiGLU experts, gate-weighted combine into the residual,
 * bf16 output) are the layer's stated configuration; the pages are silent on
 * them.
 *
 * Precision readings (the pages fix none):
 *   - every sum, product and transcendental is fp64;
 *   - the top-k decision is taken on logits rounded to fp32, the precision the
 *     router accumulates in, with ties going to the lower expert index;
 *   - gates are computed in fp64 from those fp32 logits, max-subtracted;
 *   - the output is rounded once, fp64 -> bf16, round to nearest even.
 *
 * Parity: every function is pinned by tests that do not call it through
 * itself (closed forms, invariants, brute force on tiny inputs); see
 * tests/test_oracle_pins.py.  ORACLE_MUTANT (default 0) builds deliberately
 * wrong variants used only by the test that checks those pins catch them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUT(n) (ORACLE_MUTANT == (n))

#define OK 0
#define BAD_ARG (-1)

static double bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even. */
uint16_t oracle_bf16_rne(double v) {
  if (isnan(v)) return 0x7FC0;
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  double a = fabs(v);
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
  int e = ex - 8;
  if (e < -133) e = -133; /* subnormal bf16 spacing */
  double ulp = ldexp(1.0, e);
  double q = a / ulp; /* exact: power-of-two scaling */
  double r;
#if MUT(18)
  r = floor(q); /* mutant: truncation */
#else
  r = nearbyint(q); /* current rounding mode: to nearest, ties to even */
#endif
  double m = r * ulp;
  if (m > 3.3895313892515355e38) m = INFINITY; /* beyond the largest finite bf16 */
  float f = (float)(signbit(v) ? -m : m);      /* exact: m has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* Step 1: h[b][i] = residual[b][i] + sum_j W_o[i][j] * attn[b][j]. */
int oracle_oproj_residual(int B, int d, int d_o, const uint16_t* W_o, const uint16_t* attn,
                          const uint16_t* resid, double* h) {
  if (B < 0 || d <= 0 || d_o <= 0 || !W_o || !attn || !resid || !h) return BAD_ARG;
  long n = (long)B * d;
#pragma omp parallel for schedule(static)
  for (long bi = 0; bi < n; ++bi) {
    long b = bi / d, i = bi % d;
    double s = 0.0;
    for (long j = 0; j < d_o; ++j) {
      long w;
#if MUT(2)
      w = (d == d_o) ? j * d_o + i : i * d_o + j; /* mutant: transposed operand */
#elif MUT(3)
      w = ((i + 1) % d) * d_o + j; /* mutant: wrong row */
#else
      w = i * d_o + j;
#endif
      s += bf16(W_o[w]) * bf16(attn[b * d_o + j]);
    }
#if MUT(1)
    h[bi] = s; /* mutant: residual dropped */
#else
    h[bi] = bf16(resid[bi]) + s;
#endif
  }
  return OK;
}

/* Step 2: rstd[b] = 1/sqrt(sum_i h^2 / d + eps); x[b][i] = h[b][i] * rstd[b] * gamma[i]. */
int oracle_rmsnorm(int B, int d, const double* h, const uint16_t* gamma, double eps, double* rstd,
                   double* x) {
  if (B < 0 || d <= 0 || !h || !gamma || !rstd || !x) return BAD_ARG;
  for (long b = 0; b < B; ++b) {
    double ss = 0.0;
    for (long i = 0; i < d; ++i) ss += h[b * d + i] * h[b * d + i];
    double ms = ss / d;
#if MUT(4)
    rstd[b] = 1.0 / sqrt(ms); /* mutant: eps dropped */
#elif MUT(6)
    rstd[b] = 1.0 / (ms + eps); /* mutant: square root missing */
#else
    rstd[b] = 1.0 / sqrt(ms + eps);
#endif
    for (long i = 0; i < d; ++i) {
#if MUT(5)
      x[b * d + i] = h[b * d + i] * rstd[b]; /* mutant: scale dropped */
#else
      x[b * d + i] = h[b * d + i] * rstd[b] * bf16(gamma[i]);
#endif
    }
  }
  return OK;
}

/* Step 3: logits[b][e] = sum_i W_r[e][i] * x[b][i]. */
int oracle_router(int B, int d, int E, const uint16_t* W_r, const double* x, double* logits) {
  if (B < 0 || d <= 0 || E <= 0 || !W_r || !x || !logits) return BAD_ARG;
  long n = (long)B * E;
#pragma omp parallel for schedule(static)
  for (long be = 0; be < n; ++be) {
    long b = be / E, e = be % E;
    double s = 0.0;
    for (long i = 0; i < d; ++i) {
#if MUT(7)
      s += bf16(W_r[i * E + e]) * x[b * d + i]; /* mutant: transposed operand */
#else
      s += bf16(W_r[e * d + i]) * x[b * d + i];
#endif
    }
    logits[be] = s;
  }
  return OK;
}

/* Order used by the selection: larger logit first; equal logits, lower index first. */
static int before(float la, int ia, float lb, int ib) {
#if MUT(8)
  if (la != lb) return la < lb; /* mutant: ascending */
#else
  if (la != lb) return la > lb;
#endif
#if MUT(9)
  return ia > ib; /* mutant: ties to the higher index */
#else
  return ia < ib;
#endif
}

/* Step 4: selection of the k best fp32 logits per token, then softmax over them.
 * Plain repeated scan: pick the best not-yet-chosen expert k times. */
int oracle_topk_gates(int B, int E, int k, const float* logits, int32_t* idx, double* gate) {
  if (B < 0 || E <= 0 || k <= 0 || k > E || !logits || !idx || !gate) return BAD_ARG;
  char* taken = (char*)malloc((size_t)E);
  if (!taken) return BAD_ARG;
  for (long b = 0; b < B; ++b) {
    const float* l = logits + b * E;
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || before(l[e], e, l[best], best)) best = e;
      }
      taken[best] = 1;
      idx[b * k + j] = best;
    }
    double m = (double)l[idx[b * k]];
    double sum = 0.0;
#if MUT(10)
    for (int e = 0; e < E; ++e) sum += exp((double)l[e] - m); /* mutant: all experts */
#else
    for (int j = 0; j < k; ++j) sum += exp((double)l[idx[b * k + j]] - m);
#endif
    for (int j = 0; j < k; ++j) {
#if MUT(11)
      gate[b * k + j] = exp(m - (double)l[idx[b * k + j]]) / sum; /* mutant: sign */
#else
      gate[b * k + j] = exp((double)l[idx[b * k + j]] - m) / sum;
#endif
    }
  }
  free(taken);
  return OK;
}

static double silu(double g) {
#if MUT(17)
  return g / (1.0 + exp(g)); /* mutant: sign */
#else
  return g / (1.0 + exp(-g));
#endif
}

/* Step 5 for one expert and one token: a[t] = silu(g_t) * u_t, y = W_down . a.
 * W_gu is [2I][d] (gate rows 0..I-1, up rows I..2I-1); W_down is [d][I]. */
int oracle_expert(int d, int I, const uint16_t* W_gu, const uint16_t* W_down, const double* x,
                  double* a, double* y) {
  if (d <= 0 || I <= 0 || !W_gu || !W_down || !x || !a || !y) return BAD_ARG;
  for (long t = 0; t < I; ++t) {
    double g = 0.0, u = 0.0;
    for (long i = 0; i < d; ++i) {
#if MUT(13)
      g += bf16(W_gu[(I + t) * d + i]) * x[i]; /* mutant: gate/up rows swapped */
      u += bf16(W_gu[t * d + i]) * x[i];
#else
      g += bf16(W_gu[t * d + i]) * x[i];
      u += bf16(W_gu[(I + t) * d + i]) * x[i];
#endif
    }
#if MUT(12)
    a[t] = silu(u) * g; /* mutant: activation on the wrong projection */
#else
    a[t] = silu(g) * u;
#endif
  }
#pragma omp parallel for schedule(static)
  for (long i = 0; i < d; ++i) {
    double s = 0.0;
    for (long t = 0; t < I; ++t) {
#if MUT(14)
      s += bf16(W_down[t * d + i]) * a[t]; /* mutant: transposed operand */
#else
      s += bf16(W_down[i * I + t]) * a[t];
#endif
    }
    y[i] = s;
  }
  return OK;
}

/* Step 6 for one token: out_ref[i] = h[i] + sum_j gate[j] * y_j[i] (j ascending),
 * out_bf16 = bf16_rne(out_ref).  ys holds k pointers to the experts' y. */
int oracle_combine(int d, int k, const double* h, const double* gate, const double* const* ys,
                   double* out_ref, uint16_t* out_bf16) {
  if (d <= 0 || k <= 0 || !h || !gate || !ys || !out_ref) return BAD_ARG;
  for (long i = 0; i < d; ++i) {
    double s = 0.0;
    for (int j = 0; j < k; ++j) {
#if MUT(16)
      s += ys[j][i]; /* mutant: gate factor dropped */
#else
      s += gate[j] * ys[j][i];
#endif
    }
#if MUT(15)
    out_ref[i] = s; /* mutant: residual dropped */
#else
    out_ref[i] = h[i] + s;
#endif
    if (out_bf16) out_bf16[i] = oracle_bf16_rne(out_ref[i]);
  }
  return OK;
}

/* Steps 1-4 for B tokens.  logits64 is optional; logits32 receives the fp32
 * logits on which the selection is decided. */
int oracle_front(int B, int d, int d_o, int E, int k, double eps, const uint16_t* W_o,
                 const uint16_t* gamma, const uint16_t* W_r, const uint16_t* attn,
                 const uint16_t* resid, double* h, double* rstd, double* x, double* logits64,
                 float* logits32, int32_t* idx, double* gate) {
  if (!logits32) return BAD_ARG;
  int rc = oracle_oproj_residual(B, d, d_o, W_o, attn, resid, h);
  if (rc) return rc;
  rc = oracle_rmsnorm(B, d, h, gamma, eps, rstd, x);
  if (rc) return rc;
  double* l = logits64 ? logits64 : (double*)malloc(sizeof(double) * (size_t)B * E);
  if (!l) return BAD_ARG;
  rc = oracle_router(B, d, E, W_r, x, l);
  if (!rc) {
    for (long n = 0; n < (long)B * E; ++n) logits32[n] = (float)l[n];
    rc = oracle_topk_gates(B, E, k, logits32, idx, gate);
  }
  if (!logits64) free(l);
  return rc;
}

/* Steps 5-6 for one token, given its k selected experts' weights. */
int oracle_moe_token(int d, int I, int k, const uint16_t* const* W_gu_sel,
                     const uint16_t* const* W_down_sel, const double* x, const double* h,
                     const double* gate, double* a_out /* [k][I] or NULL */, double* out_ref,
                     uint16_t* out_bf16) {
  if (d <= 0 || I <= 0 || k <= 0 || !W_gu_sel || !W_down_sel) return BAD_ARG;
  double* y = (double*)malloc(sizeof(double) * (size_t)k * d);
  double* a = (double*)malloc(sizeof(double) * (size_t)k * I);
  const double** ys = (const double**)malloc(sizeof(double*) * (size_t)k);
  int rc = (y && a && ys) ? OK : BAD_ARG;
  for (int j = 0; j < k && !rc; ++j) {
    rc = oracle_expert(d, I, W_gu_sel[j], W_down_sel[j], x, a + (long)j * I, y + (long)j * d);
    ys[j] = y + (long)j * d;
  }
  if (!rc) rc = oracle_combine(d, k, h, gate, ys, out_ref, out_bf16);
  if (!rc && a_out) memcpy(a_out, a, sizeof(double) * (size_t)k * I);
  free(y);
  free(a);
  free(ys);
  return rc;
}

int oracle_mutant(void) { return ORACLE_MUTANT; }

int oracle_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
