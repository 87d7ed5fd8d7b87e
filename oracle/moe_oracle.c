/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the latent-MoE decode block.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library; the product path
 * never does.  It shares no code, header, table or constant with the CUDA
 * path under mxfp4_latent_moe_router_b200/csrc.
 *
 * What it computes, for every token b (all sums in fp64, in increasing index
 * order, from the exact values the inputs encode):
 *
 *   1. logits  l_e = sum_h x[h] * W_r[h][e]
 *      (page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly",
 *       section 从算子之间找时间 / "finding time between operators": router
 *       scores and the latent input projection are one matmul over the same
 *       token activations x.)
 *   2. scores   softmax: p_e = exp(l_e - max l) / sum exp(.)   key = p_e, src = p_e
 *               sigmoid: s_e = 1 / (1 + exp(-l_e))            key = s_e + bias_e, src = s_e
 *   3. top-k    experts ordered by (key descending, index ascending), first k taken;
 *               w_j = src_j / sum_sel src  (when renormalising), times routed_scale.
 *   4. latent   z[l] = sum_h x[h] * W_in[h][l]
 *   5. experts  for slot j, e = ids[j]:  g = z . Wg_e,  u = z . Wu_e,
 *               h = silu(g) * u,  silu(t) = t / (1 + exp(-t)),  y_j = h . Wd_e
 *               with W = e2m1(code) * 2^(scale - 127)  (OCP Microscaling v1.0,
 *               FP4 E2M1 element and E8M0 shared scale, block of 32 along K).
 *   6. finalize c[l] = sum_j w_j * y_j[l]
 *      (page "Kimi K3 在 vLLM 中的性能优化", section 延迟 MXFP4 最终化 /
 *       "deferred MXFP4 finalize": the top-k weighted combine of the MXFP4
 *       expert outputs feeds the latent-tail up-projection.)
 *   7. shared   h_s = silu(x . W_sg) * (x . W_su),  o_s = h_s . W_sd
 *      (page "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly",
 *       section 从算子之间找时间: the shared expert is independent of routing.)
 *   8. output   out[n] = sum_l c[l] * W_out[l][n] + o_s[n]
 *
 * Readings where the pages are silent:
 *   - nibble order: element 2t is the low nibble of byte t, 2t+1 the high one;
 *   - MXFP4 tensors are stored output-row-major with K contiguous; the gate/up
 *     tensor holds the I gate rows first, then the I up rows;
 *   - no linear-layer biases; the selection bias changes selection only;
 *   - the shared expert reads x (hidden size H), not the latent z;
 *   - the block output carries no residual add and no normalisation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

typedef struct {
  int32_t hidden, latent, num_experts, top_k, expert_inter, shared_inter;
  int32_t score_fn; /* 0 softmax, 1 sigmoid */
  int32_t renormalize;
  double routed_scale;
} oracle_cfg;

typedef struct {
  const uint16_t *router_w;  /* bf16 [H][E] */
  const float *router_bias;  /* f32 [E] or NULL */
  const uint16_t *w_in;      /* bf16 [H][L] */
  const uint16_t *w_out;     /* bf16 [L][H] */
  const uint8_t *gu_codes;   /* [E][2I][L/2] */
  const uint8_t *gu_scales;  /* [E][2I][L/32] */
  const uint8_t *dn_codes;   /* [E][L][I/2] */
  const uint8_t *dn_scales;  /* [E][L][I/32] */
  const uint16_t *sh_gate;   /* bf16 [H][I_s] */
  const uint16_t *sh_up;     /* bf16 [H][I_s] */
  const uint16_t *sh_down;   /* bf16 [I_s][H] */
} oracle_weights;

/* Every output pointer may be NULL except out. */
typedef struct {
  double *logits;  /* [B][E]   */
  double *keys;    /* [B][E]   selection keys */
  int32_t *ids;    /* [B][k]   selected experts, key-descending */
  double *weights; /* [B][k]   combine weights */
  double *margin;  /* [B]      key of k-th minus key of (k+1)-th selected, +inf if k == E */
  double *z;       /* [B][L]   */
  double *h;       /* [B][k][I] */
  double *y;       /* [B][k][L] */
  double *c;       /* [B][L]   */
  double *h_s;     /* [B][I_s] */
  double *o_s;     /* [B][H]   */
  double *out;     /* [B][H]   */
} oracle_outputs;

/* bf16: the upper 16 bits of an IEEE-754 binary32. */
double oracle_bf16_value(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP MX v1.0 FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit,
 * no Inf/NaN.  Exponent field 0 is subnormal: 0.m * 2^(1-1). */
double oracle_e2m1_value(uint8_t code) {
  int sign = (code >> 3) & 1;
  int exp_field = (code >> 1) & 3;
  int mant = code & 1;
  double mag;
  if (exp_field == 0)
    mag = 0.5 * mant; /* subnormal: m/2 * 2^0 */
  else
    mag = ldexp(1.0 + 0.5 * mant, exp_field - 1);
  return sign ? -mag : mag;
}

/* OCP MX v1.0 E8M0 shared scale: 2^(s - 127); 0xFF encodes NaN. */
double oracle_e8m0_value(uint8_t s) {
  if (s == 0xFF) return NAN;
  return ldexp(1.0, (int)s - 127);
}

/* One MXFP4 element of a row-major [rows][K] tensor. */
static double mx_element(const uint8_t *codes, const uint8_t *scales, int64_t K,
                         int64_t row, int64_t k) {
  uint8_t byte = codes[row * (K / 2) + k / 2];
  uint8_t code = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
  uint8_t s = scales[row * (K / 32) + k / 32];
  return oracle_e2m1_value(code) * oracle_e8m0_value(s);
}

/* Dequantise a whole [rows][K] MXFP4 tensor (used by the tests' pins). */
void oracle_dequant_mx(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                       int64_t K, double *out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) out[r * K + k] = mx_element(codes, scales, K, r, k);
}

static double silu(double t) { return t / (1.0 + exp(-t)); }

/* y[n] = sum_k a[k] * W[k][n] for a bf16 [K][N] weight, sums in increasing k. */
static void vec_mat_bf16(const double *a, const uint16_t *W, int64_t K, int64_t N, double *y) {
  for (int64_t n = 0; n < N; ++n) y[n] = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    double ak = a[k];
    const uint16_t *row = W + k * N;
    for (int64_t n = 0; n < N; ++n) y[n] += ak * oracle_bf16_value(row[n]);
  }
}

/* y[r] = sum_k a[k] * W[r][k] for an MXFP4 [rows][K] weight (rows r0..r0+nr). */
static void mx_mat_vec(const double *a, const uint8_t *codes, const uint8_t *scales,
                       int64_t K, int64_t r0, int64_t nr, double *y) {
  for (int64_t r = 0; r < nr; ++r) {
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) acc += a[k] * mx_element(codes, scales, K, r0 + r, k);
    y[r] = acc;
  }
}

/* Selection: experts ordered by key descending, ties to the lower index. */
static void select_top_k(const double *key, int E, int k, int32_t *ids, double *margin) {
  char *taken = (char *)calloc((size_t)E, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || key[e] > key[best]) best = e; /* strict: equal keys keep the lower index */
    }
    taken[best] = 1;
    ids[j] = best;
  }
  if (margin) {
    if (k >= E) {
      *margin = INFINITY;
    } else {
      int next = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (next < 0 || key[e] > key[next]) next = e;
      }
      *margin = key[ids[k - 1]] - key[next];
    }
  }
  free(taken);
}

static int check_cfg(const oracle_cfg *c) {
  if (!c) return 0;
  if (c->hidden <= 0 || c->latent <= 0 || c->num_experts <= 0 || c->expert_inter <= 0) return 0;
  if (c->top_k <= 0 || c->top_k > c->num_experts) return 0;
  if (c->shared_inter < 0) return 0;
  if (c->latent % 32 || c->expert_inter % 32) return 0;
  if (c->score_fn != 0 && c->score_fn != 1) return 0;
  return 1;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the token loops from here on (timing only; results do not
 * depend on it: every token is computed by one thread in the same order). */
void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Full block for B tokens.  x: bf16 [B][H]. */
int oracle_forward(const oracle_cfg *cfg, const oracle_weights *w, const uint16_t *x,
                   int32_t B, oracle_outputs *o) {
  if (!check_cfg(cfg) || !w || !x || !o || !o->out || B < 0) return ORACLE_BAD_ARG;
  const int64_t H = cfg->hidden, L = cfg->latent, E = cfg->num_experts, K = cfg->top_k;
  const int64_t I = cfg->expert_inter, Is = cfg->shared_inter;

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b) {
    double *xb = (double *)malloc(sizeof(double) * H);
    double *lg = (double *)malloc(sizeof(double) * E);
    double *key = (double *)malloc(sizeof(double) * E);
    double *src = (double *)malloc(sizeof(double) * E);
    double *z = (double *)malloc(sizeof(double) * L);
    double *gu = (double *)malloc(sizeof(double) * 2 * I);
    double *h = (double *)malloc(sizeof(double) * I);
    double *y = (double *)malloc(sizeof(double) * K * L);
    double *c = (double *)malloc(sizeof(double) * L);
    double *out = (double *)malloc(sizeof(double) * H);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * K);
    double *wt = (double *)malloc(sizeof(double) * K);

    for (int64_t i = 0; i < H; ++i) xb[i] = oracle_bf16_value(x[b * H + i]);

    /* 1. router logits */
    vec_mat_bf16(xb, w->router_w, H, E, lg);

    /* 2. scores and selection keys */
    if (cfg->score_fn == 0) {
      double mx = lg[0];
      for (int64_t e = 1; e < E; ++e)
        if (lg[e] > mx) mx = lg[e];
      double den = 0.0;
      for (int64_t e = 0; e < E; ++e) den += exp(lg[e] - mx);
      for (int64_t e = 0; e < E; ++e) {
        src[e] = exp(lg[e] - mx) / den;
        key[e] = src[e];
      }
    } else {
      for (int64_t e = 0; e < E; ++e) {
        src[e] = 1.0 / (1.0 + exp(-lg[e]));
        key[e] = src[e] + (w->router_bias ? (double)w->router_bias[e] : 0.0);
      }
    }

    /* 3. top-k and combine weights */
    double margin;
    select_top_k(key, (int)E, (int)K, ids, &margin);
    double sel = 0.0;
    for (int64_t j = 0; j < K; ++j) sel += src[ids[j]];
    for (int64_t j = 0; j < K; ++j) {
      double v = cfg->renormalize ? src[ids[j]] / sel : src[ids[j]];
      wt[j] = v * cfg->routed_scale;
    }

    /* 4. latent input projection */
    vec_mat_bf16(xb, w->w_in, H, L, z);

    /* 5. routed experts */
    for (int64_t j = 0; j < K; ++j) {
      int64_t e = ids[j];
      const uint8_t *gc = w->gu_codes + e * (2 * I) * (L / 2);
      const uint8_t *gs = w->gu_scales + e * (2 * I) * (L / 32);
      const uint8_t *dc = w->dn_codes + e * L * (I / 2);
      const uint8_t *ds = w->dn_scales + e * L * (I / 32);
      mx_mat_vec(z, gc, gs, L, 0, 2 * I, gu); /* rows [0,I) gate, [I,2I) up */
      for (int64_t i = 0; i < I; ++i) h[i] = silu(gu[i]) * gu[I + i];
      mx_mat_vec(h, dc, ds, I, 0, L, y + j * L);
      if (o->h)
        for (int64_t i = 0; i < I; ++i) o->h[(b * K + j) * I + i] = h[i];
    }

    /* 6. finalize: top-k weighted combine */
    for (int64_t l = 0; l < L; ++l) {
      double acc = 0.0;
      for (int64_t j = 0; j < K; ++j) acc += wt[j] * y[j * L + l];
      c[l] = acc;
    }

    /* 8. latent tail */
    vec_mat_bf16(c, w->w_out, L, H, out);

    /* 7. shared expert */
    if (Is > 0) {
      double *g = (double *)malloc(sizeof(double) * Is);
      double *u = (double *)malloc(sizeof(double) * Is);
      double *hs = (double *)malloc(sizeof(double) * Is);
      double *os = (double *)malloc(sizeof(double) * H);
      vec_mat_bf16(xb, w->sh_gate, H, Is, g);
      vec_mat_bf16(xb, w->sh_up, H, Is, u);
      for (int64_t i = 0; i < Is; ++i) hs[i] = silu(g[i]) * u[i];
      vec_mat_bf16(hs, w->sh_down, Is, H, os);
      for (int64_t n = 0; n < H; ++n) out[n] += os[n];
      if (o->h_s) memcpy(o->h_s + b * Is, hs, sizeof(double) * Is);
      if (o->o_s) memcpy(o->o_s + b * H, os, sizeof(double) * H);
      free(g);
      free(u);
      free(hs);
      free(os);
    }

    memcpy(o->out + b * H, out, sizeof(double) * H);
    if (o->logits) memcpy(o->logits + b * E, lg, sizeof(double) * E);
    if (o->keys) memcpy(o->keys + b * E, key, sizeof(double) * E);
    if (o->ids) memcpy(o->ids + b * K, ids, sizeof(int32_t) * K);
    if (o->weights) memcpy(o->weights + b * K, wt, sizeof(double) * K);
    if (o->margin) o->margin[b] = margin;
    if (o->z) memcpy(o->z + b * L, z, sizeof(double) * L);
    if (o->y) memcpy(o->y + b * K * L, y, sizeof(double) * K * L);
    if (o->c) memcpy(o->c + b * L, c, sizeof(double) * L);

    free(xb);
    free(lg);
    free(key);
    free(src);
    free(z);
    free(gu);
    free(h);
    free(y);
    free(c);
    free(out);
    free(ids);
    free(wt);
  }
  return ORACLE_OK;
}

/* Router only (steps 1-3), for cheap checks of the selection on many tokens. */
int oracle_route(const oracle_cfg *cfg, const oracle_weights *w, const uint16_t *x, int32_t B,
                 double *logits, double *keys, int32_t *ids, double *weights, double *margin) {
  if (!check_cfg(cfg) || !w || !x || !ids || B < 0) return ORACLE_BAD_ARG;
  const int64_t H = cfg->hidden, E = cfg->num_experts, K = cfg->top_k;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < B; ++b) {
    double *xb = (double *)malloc(sizeof(double) * H);
    double *lg = (double *)malloc(sizeof(double) * E);
    double *key = (double *)malloc(sizeof(double) * E);
    double *src = (double *)malloc(sizeof(double) * E);
    for (int64_t i = 0; i < H; ++i) xb[i] = oracle_bf16_value(x[b * H + i]);
    vec_mat_bf16(xb, w->router_w, H, E, lg);
    if (cfg->score_fn == 0) {
      double mx = lg[0];
      for (int64_t e = 1; e < E; ++e)
        if (lg[e] > mx) mx = lg[e];
      double den = 0.0;
      for (int64_t e = 0; e < E; ++e) den += exp(lg[e] - mx);
      for (int64_t e = 0; e < E; ++e) key[e] = src[e] = exp(lg[e] - mx) / den;
    } else {
      for (int64_t e = 0; e < E; ++e) {
        src[e] = 1.0 / (1.0 + exp(-lg[e]));
        key[e] = src[e] + (w->router_bias ? (double)w->router_bias[e] : 0.0);
      }
    }
    double m;
    select_top_k(key, (int)E, (int)K, ids + b * K, &m);
    double sel = 0.0;
    for (int64_t j = 0; j < K; ++j) sel += src[ids[b * K + j]];
    if (weights)
      for (int64_t j = 0; j < K; ++j)
        weights[b * K + j] =
            (cfg->renormalize ? src[ids[b * K + j]] / sel : src[ids[b * K + j]]) * cfg->routed_scale;
    if (logits) memcpy(logits + b * E, lg, sizeof(double) * E);
    if (keys) memcpy(keys + b * E, key, sizeof(double) * E);
    if (margin) margin[b] = m;
    free(xb);
    free(lg);
    free(key);
    free(src);
  }
  return ORACLE_OK;
}
