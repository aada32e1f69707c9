/* oracle.c -- plain, slow, fp64 CPU oracle of the batch-invariant decoder
 * forward and its LM-head log-probability.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call this file:
 * only the tests, the package smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code with the CUDA path; the two meet only through the
 * seeded generator in synth/ (data, no arithmetic of the method).
 *
 * What it computes is the plain definition of a pre-norm decoder's token
 * log-probabilities.  The method on the pages ("Meituan bitwise train/infer
 * consistency", section on the root cause: attention score sums, softmax
 * denominators, matrix reductions and logprob accumulation are the reduced
 * quantities) reaches the same values up to rounding order; the oracle
 * therefore writes the definition out in fp64, row by row, with no blocking,
 * chunking or reordering.
 *
 * Two modes (mode argument):
 *   OR_EXACT (0): every value fp64; weights are the bf16 values upcast
 *     exactly.  Reference for the LayerCast / FP32-compute path ("Give Me
 *     FP32 or Give Me Death?", LayerCast section: bf16-stored weights, all
 *     core ops in FP32).
 *   OR_BF16  (1): the same, but the values the bf16 path stores are rounded
 *     to bf16 (round-to-nearest-even) at the same points: residual after each
 *     add, norm outputs, q/k/v after RoPE, attention output, each linear
 *     layer's output, SwiGLU output and the LM-head input h.  Everything in
 *     between stays fp64.
 *
 * LM head ("Greedy Decoding Is Not Precision-Invariant", abstract and method
 * section): logits z = h . W^T; lse = max + ln sum exp(z - max);
 * logprob(t) = z_t - lse; greedy token = argmax (lowest id on ties);
 * margin = top-1 logit minus top-2 logit, with the two largest taken as
 * positions (a duplicated maximum gives margin 0).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
  double eps, rope_theta;
} or_cfg;

/* Logical (unfused) weights, bf16 bit patterns, row-major:
 *   embed [V][H], lm_head [V][H], final_norm [H],
 *   per layer l (stacked along a leading L axis):
 *   attn_norm [H], wq [Hq*d][H], wk [Hkv*d][H], wv [Hkv*d][H], wo [H][Hq*d],
 *   ffn_norm [H], wg [F][H], wu [F][H], wd [H][F]. */
typedef struct {
  const uint16_t *embed, *attn_norm, *wq, *wk, *wv, *wo, *ffn_norm, *wg, *wu, *wd, *final_norm, *lm_head;
} or_weights;

enum { OR_EXACT = 0, OR_BF16 = 1 };

static double bfv(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a double to the nearest bf16 value (ties to even), returned as a
 * double.  bf16 = 1 sign bit, 8 exponent bits, 7 stored mantissa bits
 * ("Give Me FP32 or Give Me Death?", floating-point formats section). */
double or_round_bf16(double x) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e;
  frexp(x, &e);                 /* x = m * 2^e, 0.5 <= |m| < 1 */
  if (e < -125) e = -125;       /* bf16 subnormal range: fixed quantum 2^-133 */
  double q = ldexp(x, 8 - e);   /* 8 significant bits in front of the point */
  double r = nearbyint(q);      /* default rounding mode: nearest, ties to even */
  double y = ldexp(r, e - 8);
  if (fabs(y) >= 0x1p128) y = copysign(INFINITY, x);
  return y;
}

static double rb(int mode, double x) { return mode == OR_BF16 ? or_round_bf16(x) : x; }

/* y[m][n] = sum_k x[m][k] * w[n][k]  (w: bf16 [N][K]) */
void or_gemm(const double* x, const uint16_t* w, double* y, int M, int N, int K) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint16_t* wr = w + (size_t)n * K;
    for (int m = 0; m < M; ++m) {
      const double* xr = x + (size_t)m * K;
      double s = 0.0;
      for (int k = 0; k < K; ++k) s += xr[k] * bfv(wr[k]);
      y[(size_t)m * N + n] = s;
    }
  }
}

/* RMSNorm: y = x / sqrt(mean(x^2) + eps) * gamma  (per row) */
void or_rmsnorm(const double* x, const uint16_t* gamma, double* y, int M, int H, double eps) {
  for (int m = 0; m < M; ++m) {
    const double* xr = x + (size_t)m * H;
    double ss = 0.0;
    for (int i = 0; i < H; ++i) ss += xr[i] * xr[i];
    double inv = 1.0 / sqrt(ss / H + eps);
    for (int i = 0; i < H; ++i) y[(size_t)m * H + i] = xr[i] * inv * bfv(gamma[i]);
  }
}

/* Rotary embedding, rotate-half pairing (i, i + d/2), frequency theta^(-2i/d),
 * angle = pos * frequency; applied in place to n_heads vectors of size d. */
void or_rope(double* x, int n_heads, int d, int pos, double theta) {
  int half = d / 2;
  for (int h = 0; h < n_heads; ++h) {
    double* v = x + (size_t)h * d;
    for (int i = 0; i < half; ++i) {
      double ang = (double)pos * pow(theta, -2.0 * i / d);
      double c = cos(ang), s = sin(ang);
      double a = v[i], b = v[i + half];
      v[i] = a * c - b * s;
      v[i + half] = b * c + a * s;
    }
  }
}

/* One query against n keys: s_j = scale * q.k_j ; p = softmax(s) (max
 * subtracted); out = sum_j p_j v_j.  K, V: [n][d]. */
void or_attention_query(const double* q, const double* K, const double* V, int n, int d, double scale,
                        double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY;
  for (int j = 0; j < n; ++j) {
    double a = 0.0;
    for (int c = 0; c < d; ++c) a += q[c] * K[(size_t)j * d + c];
    s[j] = a * scale;
    if (s[j] > mx) mx = s[j];
  }
  double den = 0.0;
  for (int j = 0; j < n; ++j) {
    s[j] = exp(s[j] - mx);
    den += s[j];
  }
  for (int c = 0; c < d; ++c) {
    double a = 0.0;
    for (int j = 0; j < n; ++j) a += s[j] * V[(size_t)j * d + c];
    out[c] = a / den;
  }
  free(s);
}

/* LM-head statistics of one logit row z[V]:
 *   res[0] = lse, res[1] = logprob(target) (target < 0: of the argmax),
 *   res[2] = argmax (lowest id among equal maxima), res[3] = margin,
 *   res[4] = index of the second-largest position. */
void or_logit_stats(const double* z, int V, int target, double* res) {
  int i1 = 0;
  for (int v = 1; v < V; ++v)
    if (z[v] > z[i1]) i1 = v;
  int i2 = -1;
  for (int v = 0; v < V; ++v) {
    if (v == i1) continue;
    if (i2 < 0 || z[v] > z[i2]) i2 = v;
  }
  double mx = z[i1];
  double s = 0.0;
  for (int v = 0; v < V; ++v) s += exp(z[v] - mx);
  double lse = mx + log(s);
  int t = target >= 0 ? target : i1;
  res[0] = lse;
  res[1] = z[t] - lse;
  res[2] = (double)i1;
  res[3] = i2 >= 0 ? z[i1] - z[i2] : INFINITY;
  res[4] = (double)i2;
}

/* LM head for B rows: z = h . W^T, then the statistics above.
 * h: [B][H] doubles, W: bf16 [V][H]; res: [B][5]; logits_opt: [B][V] or NULL. */
void or_lmhead(const double* h, const uint16_t* W, const int* target, int B, int H, int V, double* res,
               double* logits_opt) {
  double* z = (double*)malloc(sizeof(double) * (size_t)B * V);
  or_gemm(h, W, z, B, V, H);
  for (int b = 0; b < B; ++b) {
    or_logit_stats(z + (size_t)b * V, V, target ? target[b] : -1, res + (size_t)b * 5);
    if (logits_opt) memcpy(logits_opt + (size_t)b * V, z + (size_t)b * V, sizeof(double) * V);
  }
  free(z);
}

static double silu(double x) { return x / (1.0 + exp(-x)); }

/* Forward of ONE sequence: n new tokens at positions n_ctx .. n_ctx+n-1 that
 * follow n_ctx earlier positions whose per-layer keys and values (after RoPE,
 * as stored: rounded to bf16 in OR_BF16) are given in k_ctx, v_ctx
 * ([L][n_ctx][Hkv*d], NULL when n_ctx == 0).  Causal: new token t attends to
 * the n_ctx earlier positions and to new tokens 0..t, in ascending position
 * order.  For each new token t: res[t][0..4] as in or_logit_stats for
 * target[t] (target NULL or < 0: the argmax).  h_out (optional, [n][H]): the
 * final norm output before any bf16 rounding (the FP32-recompute input).
 * k_out, v_out (optional, [L][n][Hkv*d]): the new tokens' stored keys and
 * values, which a later call can take as its context.
 * Returns 0 on success, -1 on allocation failure. */
int or_forward_ctx(const or_cfg* c, const or_weights* w, int mode, const int* tokens, int n, int n_ctx,
                   const double* k_ctx, const double* v_ctx, const int* target, double* res, double* h_out,
                   double* k_out, double* v_out) {
  const int H = c->hidden, Hq = c->n_heads, Hkv = c->n_kv_heads, d = c->head_dim, F = c->ffn, V = c->vocab;
  const int QD = Hq * d, KD = Hkv * d, group = Hq / Hkv;
  const int nt = n_ctx + n; /* positions visible to the last new token */
  const double scale = 1.0 / sqrt((double)d);
  size_t big = (size_t)n * (size_t)(F > H ? F : H);
  double *r = calloc((size_t)n * H, 8), *u = calloc((size_t)n * H, 8), *q = calloc((size_t)n * QD, 8),
         *k = calloc((size_t)n * KD, 8), *vv = calloc((size_t)n * KD, 8), *o = calloc((size_t)n * QD, 8),
         *y = calloc(big, 8), *g = calloc((size_t)n * F, 8), *up = calloc((size_t)n * F, 8),
         *kh = calloc((size_t)nt * d, 8), *vh = calloc((size_t)nt * d, 8);
  if (!r || !u || !q || !k || !vv || !o || !y || !g || !up || !kh || !vh) return -1;

  for (int t = 0; t < n; ++t)
    for (int i = 0; i < H; ++i) r[(size_t)t * H + i] = bfv(w->embed[(size_t)tokens[t] * H + i]);

  for (int l = 0; l < c->n_layers; ++l) {
    const uint16_t* an = w->attn_norm + (size_t)l * H;
    const uint16_t* fn = w->ffn_norm + (size_t)l * H;
    const uint16_t* wq = w->wq + (size_t)l * QD * H;
    const uint16_t* wk = w->wk + (size_t)l * KD * H;
    const uint16_t* wv = w->wv + (size_t)l * KD * H;
    const uint16_t* wo = w->wo + (size_t)l * H * QD;
    const uint16_t* wg = w->wg + (size_t)l * F * H;
    const uint16_t* wu = w->wu + (size_t)l * F * H;
    const uint16_t* wd = w->wd + (size_t)l * H * F;

    /* attention block */
    or_rmsnorm(r, an, u, n, H, c->eps);
    for (size_t i = 0; i < (size_t)n * H; ++i) u[i] = rb(mode, u[i]);
    or_gemm(u, wq, q, n, QD, H);
    or_gemm(u, wk, k, n, KD, H);
    or_gemm(u, wv, vv, n, KD, H);
    for (int t = 0; t < n; ++t) {
      or_rope(q + (size_t)t * QD, Hq, d, n_ctx + t, c->rope_theta);
      or_rope(k + (size_t)t * KD, Hkv, d, n_ctx + t, c->rope_theta);
    }
    for (size_t i = 0; i < (size_t)n * QD; ++i) q[i] = rb(mode, q[i]);
    for (size_t i = 0; i < (size_t)n * KD; ++i) {
      k[i] = rb(mode, k[i]);
      vv[i] = rb(mode, vv[i]);
    }
    if (k_out) memcpy(k_out + (size_t)l * n * KD, k, sizeof(double) * (size_t)n * KD);
    if (v_out) memcpy(v_out + (size_t)l * n * KD, vv, sizeof(double) * (size_t)n * KD);
    const double* kc = k_ctx ? k_ctx + (size_t)l * n_ctx * KD : NULL;
    const double* vc = v_ctx ? v_ctx + (size_t)l * n_ctx * KD : NULL;
    for (int hk = 0; hk < Hkv; ++hk) {
      for (int j = 0; j < nt; ++j) /* keys in position order: the context, then the new tokens */
        for (int e = 0; e < d; ++e) {
          const int jn = j - n_ctx;
          kh[(size_t)j * d + e] = jn < 0 ? kc[(size_t)j * KD + hk * d + e] : k[(size_t)jn * KD + hk * d + e];
          vh[(size_t)j * d + e] = jn < 0 ? vc[(size_t)j * KD + hk * d + e] : vv[(size_t)jn * KD + hk * d + e];
        }
      for (int hq = hk * group; hq < (hk + 1) * group; ++hq)
        for (int t = 0; t < n; ++t) /* query at position n_ctx + t sees keys 0..n_ctx + t */
          or_attention_query(q + (size_t)t * QD + hq * d, kh, vh, n_ctx + t + 1, d, scale,
                             o + (size_t)t * QD + hq * d);
    }
    for (size_t i = 0; i < (size_t)n * QD; ++i) o[i] = rb(mode, o[i]);
    or_gemm(o, wo, y, n, H, QD);
    for (size_t i = 0; i < (size_t)n * H; ++i) r[i] = rb(mode, r[i] + rb(mode, y[i]));

    /* MLP block: SwiGLU */
    or_rmsnorm(r, fn, u, n, H, c->eps);
    for (size_t i = 0; i < (size_t)n * H; ++i) u[i] = rb(mode, u[i]);
    or_gemm(u, wg, g, n, F, H);
    or_gemm(u, wu, up, n, F, H);
    for (size_t i = 0; i < (size_t)n * F; ++i) g[i] = rb(mode, silu(g[i]) * up[i]);
    or_gemm(g, wd, y, n, H, F);
    for (size_t i = 0; i < (size_t)n * H; ++i) r[i] = rb(mode, r[i] + rb(mode, y[i]));
  }

  or_rmsnorm(r, w->final_norm, u, n, H, c->eps);
  if (h_out) memcpy(h_out, u, sizeof(double) * (size_t)n * H);
  for (size_t i = 0; i < (size_t)n * H; ++i) u[i] = rb(mode, u[i]);
  int* tg = (int*)malloc(sizeof(int) * (size_t)n);
  for (int t = 0; t < n; ++t) tg[t] = target ? target[t] : -1;
  or_lmhead(u, w->lm_head, tg, n, H, V, res, NULL);
  free(tg);
  free(r); free(u); free(q); free(k); free(vv); free(o); free(y); free(g); free(up); free(kh); free(vh);
  return 0;
}

/* Full forward of ONE sequence of n tokens (positions 0..n-1, causal): the
 * call above with no earlier positions. */
int or_forward(const or_cfg* c, const or_weights* w, int mode, const int* tokens, int n, const int* target,
               double* res, double* h_out) {
  return or_forward_ctx(c, w, mode, tokens, n, 0, NULL, NULL, target, res, h_out, NULL, NULL);
}
