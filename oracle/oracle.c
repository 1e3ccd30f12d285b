/*
 * oracle.c -- CPU reference of the quantised MoE expert forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check
 * and the benchmark's CPU-baseline leg may load or call this file.  The
 * product path never does: it shares no code, header, table or helper with
 * this file, and it never falls back to it.
 *
 * Plain, slow, obviously correct: fp64 arithmetic throughout, one output at
 * a time, on the logical (unpacked) layout -- one code per byte, bf16 scale
 * and bias per group of `G` consecutive inputs of a row.  No blocking, no
 * fusion, no reordering beyond the definitions.
 *
 * Source pages: "What is Flash-MoE? Running 397B-parameter AI models on a
 * laptop" (a2a-mcp.org, in German, Chinese, Hindi and Portuguese editions)
 * and the news.hada.io summary "Flash-MoE - running a 397-billion-parameter
 * model on a notebook".  Section names below are those pages' headings.
 *
 * Every function also returns an error scale S per output (S = sum of the
 * absolute values of the terms that make up the output, propagated to first
 * order through the later steps); the parity tests accept a device result d
 * for oracle value v when |d - v| <= 1e-3 * S + 1e-5.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - group size 64, bf16 scale and bias, one shared expert alongside the
 *     top-4 routed ones (the pages give 4 routed + 1 shared of 512);
 *   - top-k is taken on the logits, ties to the lower expert index, NaN
 *     treated as -inf (and reported); gate weights are the softmax of the
 *     k selected logits (softmax, top-k and renormalisation select the same
 *     experts and give the same weights);
 *   - the shared expert's output is scaled by sigmoid(w_sg . xn);
 *   - RMSNorm: xn' = h' * (mean(h'^2) + eps)^(-1/2) * w.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* Timing build only (ORACLE_OMP, used by the benchmark's CPU baseline on all
 * host cores): the independent output rows of the matrix-vector products
 * are spread over threads.  Each row is still computed by one thread in the
 * same order, so the results are those of the plain build bit for bit.  The
 * checks use the plain build. */
#ifdef ORACLE_OMP
#include <omp.h>
#define ORACLE_ROWS_PARALLEL _Pragma("omp parallel for schedule(static)")
void oracle_set_threads(int n) { omp_set_num_threads(n); }
#else
#define ORACLE_ROWS_PARALLEL
#endif

/* Exact value of a bf16 bit pattern (bf16 is the top half of an IEEE fp32). */
double oracle_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Group-affine dequantised matrix-vector product (pages: "FMA-optimised
 * dequantisation kernels" -- each weight is code * scale + bias; "hand-tuned
 * Metal compute shaders" -- 4-bit / 2-bit matrix-vector multiply).
 *   y[r] = sum_j (q[r][j] * s[r][j/G] + b[r][j/G]) * x[j]
 *   S[r] = sum_j |(q[r][j] * s[r][j/G] + b[r][j/G]) * x[j]|          */
void oracle_qgemv(const uint8_t* q, const uint16_t* s, const uint16_t* b, int rows, int cols,
                  int G, const double* x, double* y, double* S) {
  int ng = cols / G;
  ORACLE_ROWS_PARALLEL
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0, mag = 0.0;
    for (int j = 0; j < cols; ++j) {
      double w = (double)q[(size_t)r * cols + j] * oracle_bf16(s[(size_t)r * ng + j / G]) +
                 oracle_bf16(b[(size_t)r * ng + j / G]);
      acc += w * x[j];
      mag += fabs(w * x[j]);
    }
    y[r] = acc;
    if (S) S[r] = mag;
  }
}

/* Dense fp32-weight matrix-vector product: the router (pages: "Understanding
 * Mixture-of-Experts" -- a router picks experts per layer) and the shared
 * expert's gate logit.  y[r] = sum_j W[r][j] x[j], S[r] = sum_j |W[r][j] x[j]|. */
void oracle_gemv_f32(const float* W, int rows, int cols, const double* x, double* y, double* S) {
  ORACLE_ROWS_PARALLEL
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0, mag = 0.0;
    for (int j = 0; j < cols; ++j) {
      double t = (double)W[(size_t)r * cols + j] * x[j];
      acc += t;
      mag += fabs(t);
    }
    y[r] = acc;
    if (S) S[r] = mag;
  }
}

/* Routing (pages: "Understanding Mixture-of-Experts" -- 4 routed experts of
 * 512 per layer, plus 1 shared).  Selects the k largest logits, ties to the
 * lower index, NaN ordered below every number; p = softmax over the k
 * selected logits.  ids/p are in selection order (largest first).
 * Returns 1 if any logit was NaN, else 0. */
int oracle_topk_softmax(const double* logits, int E, int k, int32_t* ids, double* p) {
  int nan_seen = 0;
  for (int e = 0; e < E; ++e)
    if (isnan(logits[e])) nan_seen = 1;
  for (int t = 0; t < k; ++t) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      int taken = 0;
      for (int u = 0; u < t; ++u)
        if (ids[u] == e) taken = 1;
      if (taken) continue;
      if (best < 0) { best = e; continue; }
      double le = logits[e], lb = logits[best];
      int better;
      if (isnan(le)) better = 0;
      else if (isnan(lb)) better = 1;
      else better = le > lb; /* equal values keep the lower index */
      if (better) best = e;
    }
    ids[t] = best;
  }
  double m = -INFINITY;
  for (int t = 0; t < k; ++t) {
    double l = logits[ids[t]];
    if (!isnan(l) && l > m) m = l;
  }
  double z = 0.0;
  for (int t = 0; t < k; ++t) {
    double l = logits[ids[t]];
    p[t] = isnan(l) ? 0.0 : exp(l - m);
    z += p[t];
  }
  for (int t = 0; t < k; ++t) p[t] /= z;
  return nan_seen;
}

double oracle_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* SwiGLU (pages: "hand-tuned Metal compute shaders" -- fused SwiGLU
 * activation): a = silu(g) * u, silu(g) = g * sigmoid(g). */
double oracle_swiglu(double g, double u) { return g * oracle_sigmoid(g) * u; }

typedef struct {
  const uint8_t* q;      /* gate [I][H], up [I][H], down [H][I] codes, one per byte */
  const uint16_t* scale; /* bf16 bits, [rows][cols / G] per matrix, same order */
  const uint16_t* bias;
} oracle_expert_t;

/* One expert's feed-forward on input x[H] (pages: gate and up projections,
 * SwiGLU, down projection, all as dequantised matrix-vector products):
 *   g = Wg x, u = Wu x, a = silu(g) u, y = Wd a.
 * Outputs a[I], y[H] and their error scales (first-order propagation of the
 * gate/up scales through SwiGLU, and of a's scale through the down product). */
void oracle_expert_ffn(const oracle_expert_t* ex, int H, int I, int G, const double* x,
                       double* g, double* u, double* a, double* y, double* S_g, double* S_u,
                       double* S_a, double* S_y) {
  size_t n = (size_t)H * I, ng = n / G;
  oracle_qgemv(ex->q, ex->scale, ex->bias, I, H, G, x, g, S_g);
  oracle_qgemv(ex->q + n, ex->scale + ng, ex->bias + ng, I, H, G, x, u, S_u);
  for (int i = 0; i < I; ++i) {
    double sg = oracle_sigmoid(g[i]);
    a[i] = oracle_swiglu(g[i], u[i]);
    /* d a = u (sg + g sg (1 - sg)) d g + g sg d u */
    S_a[i] = fabs(u[i] * (sg + g[i] * sg * (1.0 - sg))) * S_g[i] + fabs(g[i] * sg) * S_u[i];
  }
  const uint8_t* qd = ex->q + 2 * n;
  const uint16_t* sd = ex->scale + 2 * ng;
  const uint16_t* bd = ex->bias + 2 * ng;
  oracle_qgemv(qd, sd, bd, H, I, G, a, y, S_y);
  /* add |Wd| S_a: the down product sees a with its own error */
  int ngd = I / G;
  ORACLE_ROWS_PARALLEL
  for (int r = 0; r < H; ++r) {
    double prop = 0.0;
    for (int j = 0; j < I; ++j) {
      double w = (double)qd[(size_t)r * I + j] * oracle_bf16(sd[(size_t)r * ngd + j / G]) +
                 oracle_bf16(bd[(size_t)r * ngd + j / G]);
      prop += fabs(w) * S_a[j];
    }
    S_y[r] += prop;
  }
}

/* Weighted combine + residual + shared-expert sigmoid gate, then two-pass
 * RMSNorm (pages: "hand-tuned Metal compute shaders" -- MoE combine +
 * residual + sigmoid gating in one pass; two-pass RMSNorm, sum of squares
 * then apply; the result feeds the next layer directly):
 *   h'  = h + sum_k p[k] y[k] + gamma y[shared]
 *   r   = (sum_i h'_i^2 / H + eps)^(-1/2)
 *   xn' = h' * r * w
 * y is [(k+1)][H], the shared expert last.  S_y (may be NULL) are the
 * error scales of y, S_gamma that of gamma (tolerance 1e-3 * S each).
 * S_h and S_xn are the error scales of the outputs in the same units:
 *   S_h  = |h| + sum_k |p_k y_k| + |gamma y_s|          (the sum's own terms)
 *        + sum_k p_k S_y,k + gamma S_y,s + |y_s| S_gamma  (inputs' errors)
 *        + 1e-2                                         (inputs' 1e-5 slack)
 *   S_xn = |w| r S_h + |xn'| (rho + 1e-3),
 *   rho  = sum_j |h'_j| S_h,j / (H (mean(h'^2) + eps))   (first-order error of r);
 * the 1e-3 |xn'| term puts 1e-6 |xn'| into the tolerance: the fp32 rounding
 * of r and of the two products that form xn'. */
void oracle_combine_rmsnorm(int H, int k, const double* y, const double* S_y, const double* p,
                            double gamma, double S_gamma, const double* h, const float* w,
                            double eps, double* h_out, double* xn_out, double* S_h,
                            double* S_xn) {
  double ss = 0.0;
  for (int i = 0; i < H; ++i) {
    double v = h[i], mag = fabs(h[i]);
    for (int t = 0; t < k; ++t) {
      double yt = y[(size_t)t * H + i];
      v += p[t] * yt;
      mag += fabs(p[t] * yt);
      if (S_y) mag += p[t] * S_y[(size_t)t * H + i];
    }
    double ys = y[(size_t)k * H + i];
    v += gamma * ys;
    mag += fabs(gamma * ys) + fabs(ys) * S_gamma;
    if (S_y) mag += gamma * S_y[(size_t)k * H + i];
    h_out[i] = v;
    S_h[i] = mag + 1e-2;
    ss += v * v;
  }
  double ms = ss / H;
  double r = 1.0 / sqrt(ms + eps);
  double rho = 0.0;
  for (int i = 0; i < H; ++i) rho += fabs(h_out[i]) * S_h[i];
  rho /= (double)H * (ms + eps);
  for (int i = 0; i < H; ++i) {
    xn_out[i] = h_out[i] * r * (double)w[i];
    S_xn[i] = fabs((double)w[i]) * r * S_h[i] + fabs(xn_out[i]) * (rho + 1e-3);
  }
}

typedef struct {
  int H, I, E, k, G;
  double eps;
  const float* w_router;           /* [E][H] */
  const float* w_shared_gate;      /* [H] */
  const float* norm_w;             /* [H] */
  const oracle_expert_t* experts;  /* [E + 1], last = shared; unselected entries may be NULL q */
} oracle_layer_t;

/* One token through one MoE layer (all the steps above in the pages' order).
 * h, xn: the token's residual stream and normed input.  If logits_in is not
 * NULL the router product is skipped and those (fp32) logits are used, as
 * for externally supplied routing.  Outputs: logits[E], S_l[E], ids[k],
 * p[k], gamma, S_gamma, y[(k+1) H], S_y, h_out, xn_out, S_h, S_xn.
 * Returns 0, 1 if a NaN logit was seen, or -1 if a selected expert's
 * tensors were not supplied. */
int oracle_layer_token(const oracle_layer_t* L, const double* h, const double* xn,
                       const float* logits_in, double* logits, double* S_l, int32_t* ids,
                       double* p, double* gamma_out, double* S_gamma_out, double* y, double* S_y,
                       double* h_out, double* xn_out, double* S_h, double* S_xn,
                       double* work /* 6 * I doubles */) {
  int H = L->H, I = L->I, E = L->E, k = L->k;
  if (logits_in) {
    for (int e = 0; e < E; ++e) { logits[e] = (double)logits_in[e]; S_l[e] = 0.0; }
  } else {
    oracle_gemv_f32(L->w_router, E, H, xn, logits, S_l);
  }
  int nan_seen = oracle_topk_softmax(logits, E, k, ids, p);
  double z, S_z;
  oracle_gemv_f32(L->w_shared_gate, 1, H, xn, &z, &S_z);
  double gamma = oracle_sigmoid(z);
  double S_gamma = gamma * (1.0 - gamma) * S_z;
  double *g = work, *u = work + I, *a = work + 2 * I, *Sg = work + 3 * I, *Su = work + 4 * I,
         *Sa = work + 5 * I;
  for (int t = 0; t <= k; ++t) {
    int slot = (t < k) ? ids[t] : E;
    const oracle_expert_t* ex = &L->experts[slot];
    if (!ex->q) return -1;
    oracle_expert_ffn(ex, H, I, L->G, xn, g, u, a, y + (size_t)t * H, Sg, Su, Sa,
                      S_y + (size_t)t * H);
  }
  oracle_combine_rmsnorm(H, k, y, S_y, p, gamma, S_gamma, h, L->norm_w, L->eps, h_out, xn_out,
                         S_h, S_xn);
  *gamma_out = gamma;
  *S_gamma_out = S_gamma;
  return nan_seen;
}

/* Group-affine min/max quantiser (the offline weight conversion the pages'
 * conclusion mentions): per group of G values, s = (max - min) / (2^bits - 1),
 * b = min, q = round((w - b) / s) clamped to [0, 2^bits - 1]; s = 0 gives q = 0.
 * Used to pin the dequantisation by round trip. */
void oracle_quantize(const double* w, size_t n, int G, int bits, uint8_t* q, double* s,
                     double* b) {
  int qmax = (1 << bits) - 1;
  for (size_t g0 = 0; g0 < n; g0 += (size_t)G) {
    double lo = w[g0], hi = w[g0];
    for (int j = 1; j < G; ++j) {
      if (w[g0 + j] < lo) lo = w[g0 + j];
      if (w[g0 + j] > hi) hi = w[g0 + j];
    }
    double sc = (hi - lo) / qmax;
    s[g0 / G] = sc;
    b[g0 / G] = lo;
    for (int j = 0; j < G; ++j) {
      double c = sc > 0.0 ? nearbyint((w[g0 + j] - lo) / sc) : 0.0;
      if (c < 0) c = 0;
      if (c > qmax) c = qmax;
      q[g0 + j] = (uint8_t)c;
    }
  }
}

/* fp32 -> bf16 bit pattern, round to nearest, ties to even (finite inputs). */
static uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static float oracle_bf16_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* The stored-format quantiser (fp32 weights -> codes + bf16 scale/bias),
 * the offline conversion step the pages' conclusion mentions, with every
 * decision taken in fp32 exactly as written here: per group of G values
 * lo = min (+0 for a -0 minimum), hi = max; s = (hi - lo) / (2^bits - 1)
 * (one fp32 division),
 * stored as bf16 (round to nearest even), b = lo stored as bf16; with the
 * stored values S and B, q = rint((w - B) / S) (fp32 subtraction and
 * division, ties to even) clamped to [0, 2^bits - 1], and q = 0 where S = 0.
 * Finite inputs only. */
void oracle_quantize_f32(const float* w, size_t n_groups, int G, int bits, uint8_t* q, uint16_t* s,
                         uint16_t* b) {
  const int qmax = (1 << bits) - 1;
  for (size_t g = 0; g < n_groups; ++g) {
    const float* x = w + g * (size_t)G;
    float lo = x[0], hi = x[0];
    for (int j = 1; j < G; ++j) {
      if (x[j] < lo) lo = x[j];
      if (x[j] > hi) hi = x[j];
    }
    lo = lo + 0.0f;  /* a -0 minimum is stored as +0 */
    const float sc = (hi - lo) / (float)qmax;
    s[g] = oracle_f32_to_bf16(sc);
    b[g] = oracle_f32_to_bf16(lo);
    const float S = oracle_bf16_f32(s[g]), B = oracle_bf16_f32(b[g]);
    for (int j = 0; j < G; ++j) {
      float c = 0.0f;
      if (S > 0.0f) {
        const float t = (x[j] - B) / S;
        c = nearbyintf(t);
        if (c < 0.0f) c = 0.0f;
        if (c > (float)qmax) c = (float)qmax;
      }
      q[g * (size_t)G + j] = (uint8_t)c;
    }
  }
}

/* Dequantise a whole matrix: w[r][j] = q[r][j] * s[r][j/G] + b[r][j/G]. */
void oracle_dequantize(const uint8_t* q, const uint16_t* s, const uint16_t* b, int rows,
                       int cols, int G, double* w) {
  int ng = cols / G;
  for (int r = 0; r < rows; ++r)
    for (int j = 0; j < cols; ++j)
      w[(size_t)r * cols + j] = (double)q[(size_t)r * cols + j] *
                                    oracle_bf16(s[(size_t)r * ng + j / G]) +
                                oracle_bf16(b[(size_t)r * ng + j / G]);
}
