/*
 * beam_moe_oracle.c - plain fp64 CPU oracle of the Beam MoE block forward.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
 *
 * Follows, step by step, the Hugging Face launch post "Welcome Beam",
 * section "Mixture of Experts" (router and experts) and section "Residual
 * Stream" (the router and the SwiGLU product are computed in FP32 there; this
 * oracle computes everything in fp64, which is at least as precise). The same
 * steps are restated in the Russian summary of the launch (section
 * "Экспертные блоки Mixture of Experts") and in the Miles "Beam 1.0" page,
 * section 1. One token at a time, no grouping of tokens by expert, no
 * blocking or fusion: OpenMP only splits the loop over tokens.
 */
#include "beam_moe_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static int cfg_ok(const oracle_cfg* c) {
  if (!c) return 0;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->n_group <= 0) return 0;
  if (c->n_experts % c->n_group != 0) return 0;
  if (c->topk_group <= 0 || c->topk_group > c->n_group) return 0;
  if (c->top_k <= 0 || c->top_k > c->topk_group * (c->n_experts / c->n_group)) return 0;
  if (c->bias_mode != 0 && c->bias_mode != 1) return 0;
  return 1;
}

/* "a beats b": larger value first, ties to the lower index. */
static int beats(double va, int ia, double vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

int oracle_route(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const float* w_router,
                 const float* bias, int32_t* ids, double* weights, double* scores, int32_t* kept,
                 double* margins, double* all_s) {
  if (!cfg_ok(cfg) || T < 0 || (T > 0 && (!x || !w_router))) return -1;
  const int H = cfg->hidden, E = cfg->n_experts, G = cfg->n_group;
  const int Gk = cfg->topk_group, K = cfg->top_k, per = E / G;
  int bad = 0;

#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)E);      /* sigmoid scores  */
    double* c = (double*)malloc(sizeof(double) * (size_t)E);      /* choice scores   */
    double* gs = (double*)malloc(sizeof(double) * (size_t)G);     /* group scores    */
    int* gkept = (int*)malloc(sizeof(int) * (size_t)G);
    int* taken = (int*)malloc(sizeof(int) * (size_t)E);
    int* sel = (int*)malloc(sizeof(int) * (size_t)K);
    if (!s || !c || !gs || !gkept || !taken || !sel) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t t = 0; t < T; ++t) {
        const uint16_t* xt = x + t * (int64_t)H;
        /* 1. router logits and sigmoid scores, all experts */
        for (int e = 0; e < E; ++e) {
          const float* we = w_router + (int64_t)e * H;
          double l = 0.0;
          for (int h = 0; h < H; ++h) l += bf16_to_double(xt[h]) * (double)we[h];
          if (bias && cfg->bias_mode == 0) l += (double)bias[e];
          s[e] = 1.0 / (1.0 + exp(-l));
          c[e] = s[e] + ((bias && cfg->bias_mode == 1) ? (double)bias[e] : 0.0);
          if (all_s) all_s[t * E + e] = s[e];
        }
        /* 2. group score: sum of the two best choice scores in the group */
        for (int g = 0; g < G; ++g) {
          int b1 = -1, b2 = -1;
          for (int j = 0; j < per; ++j) {
            int e = g * per + j;
            if (b1 < 0 || beats(c[e], e, c[b1], b1)) {
              b2 = b1;
              b1 = e;
            } else if (b2 < 0 || beats(c[e], e, c[b2], b2)) {
              b2 = e;
            }
          }
          gs[g] = c[b1] + (b2 >= 0 ? c[b2] : 0.0);
          gkept[g] = 0;
        }
        /* 3. keep the Gk best groups */
        for (int r = 0; r < Gk; ++r) {
          int best = -1;
          for (int g = 0; g < G; ++g)
            if (!gkept[g] && (best < 0 || beats(gs[g], g, gs[best], best))) best = g;
          gkept[best] = 1;
          if (kept) kept[t * Gk + r] = best;
        }
        double mg = INFINITY;
        if (Gk < G) {
          double lastk = INFINITY, bestu = -INFINITY;
          for (int g = 0; g < G; ++g) {
            if (gkept[g] && gs[g] < lastk) lastk = gs[g];
            if (!gkept[g] && gs[g] > bestu) bestu = gs[g];
          }
          mg = lastk - bestu;
        }
        /* 4. top-K experts inside the kept groups */
        for (int e = 0; e < E; ++e) taken[e] = 0;
        for (int k = 0; k < K; ++k) {
          int best = -1;
          for (int e = 0; e < E; ++e)
            if (gkept[e / per] && !taken[e] && (best < 0 || beats(c[e], e, c[best], best)))
              best = e;
          taken[best] = 1;
          sel[k] = best;
        }
        double me = INFINITY;
        {
          double bestu = -INFINITY;
          for (int e = 0; e < E; ++e)
            if (gkept[e / per] && !taken[e] && c[e] > bestu) bestu = c[e];
          if (bestu > -INFINITY) me = c[sel[K - 1]] - bestu;
        }
        /* 5. combine weights: normalized over the selected, times the scale */
        double sum = 0.0;
        for (int k = 0; k < K; ++k) sum += s[sel[k]];
        for (int k = 0; k < K; ++k) {
          double w = cfg->renormalize ? s[sel[k]] / sum : s[sel[k]];
          if (ids) ids[t * K + k] = sel[k];
          if (weights) weights[t * K + k] = cfg->routed_scale * w;
          if (scores) scores[t * K + k] = s[sel[k]];
        }
        if (margins) {
          margins[t * 2 + 0] = mg;
          margins[t * 2 + 1] = me;
        }
      }
    }
    free(s);
    free(c);
    free(gs);
    free(gkept);
    free(taken);
    free(sel);
  }
  return bad ? -2 : 0;
}

/* a = silu(Wg x) * (Wu x) for one token: the expert's hidden activations. */
static void swiglu_hidden(int32_t H, int32_t I, const double* x, const uint16_t* w13, double* a) {
  for (int i = 0; i < I; ++i) {
    const uint16_t* wg = w13 + (int64_t)i * H;
    const uint16_t* wu = w13 + (int64_t)(I + i) * H;
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      g += bf16_to_double(wg[h]) * x[h];
      u += bf16_to_double(wu[h]) * x[h];
    }
    a[i] = g / (1.0 + exp(-g)) * u; /* silu(g) * u */
  }
}

int oracle_swiglu_expert(int32_t H, int32_t I, const double* x, const uint16_t* w13,
                         const uint16_t* w2, double* y) {
  if (H <= 0 || I <= 0 || !x || !w13 || !w2 || !y) return -1;
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  if (!a) return -2;
  swiglu_hidden(H, I, x, w13, a);
  for (int j = 0; j < H; ++j) {
    const uint16_t* wd = w2 + (int64_t)j * I;
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += bf16_to_double(wd[i]) * a[i];
    y[j] = acc;
  }
  free(a);
  return 0;
}

int oracle_hidden(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                  const uint16_t* const* w13, double* a) {
  if (!cfg_ok(cfg) || T < 0) return -1;
  if (T == 0) return 0;
  if (!x || !ids || !w13 || !a) return -1;
  const int H = cfg->hidden, I = cfg->inter, E = cfg->n_experts, K = cfg->top_k;
  int bad = 0;
#pragma omp parallel
  {
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    if (!xd) {
#pragma omp atomic write
      bad = -2;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h) xd[h] = bf16_to_double(x[t * (int64_t)H + h]);
        for (int k = 0; k < K; ++k) {
          const int e = ids[t * K + k];
          if (e < 0 || e >= E || !w13[e]) {
#pragma omp atomic write
            bad = -3;
            continue;
          }
          swiglu_hidden(H, I, xd, w13[e], a + (t * K + k) * (int64_t)I);
        }
      }
    }
    free(xd);
  }
  return bad;
}

int oracle_experts(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                   const double* weights, const uint16_t* const* w13, const uint16_t* const* w2,
                   double* out) {
  if (!cfg_ok(cfg) || T < 0) return -1;
  if (T == 0) return 0;
  if (!x || !ids || !weights || !w13 || !w2 || !out) return -1;
  const int H = cfg->hidden, I = cfg->inter, E = cfg->n_experts, K = cfg->top_k;
  int bad = 0;
#pragma omp parallel
  {
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    if (!xd || !y) {
#pragma omp atomic write
      bad = -2;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t t = 0; t < T; ++t) {
        double* ot = out + t * (int64_t)H;
        for (int h = 0; h < H; ++h) {
          xd[h] = bf16_to_double(x[t * (int64_t)H + h]);
          ot[h] = 0.0;
        }
        for (int k = 0; k < K; ++k) {
          int e = ids[t * K + k];
          if (e < 0 || e >= E || !w13[e] || !w2[e]) {
#pragma omp atomic write
            bad = -3;
            continue;
          }
          oracle_swiglu_expert(H, I, xd, w13[e], w2[e], y);
          for (int h = 0; h < H; ++h) ot[h] += weights[t * K + k] * y[h];
        }
      }
    }
    free(xd);
    free(y);
  }
  return bad;
}

/* ------------------------------------------------------------------ NVFP4 */

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static double e2m1_value(uint8_t code) {
  double v = kE2M1[code & 7];
  return (code & 8) ? -v : v;
}

double oracle_e2m1_value(uint8_t code) { return e2m1_value(code); }

double oracle_e4m3_value(uint8_t b) {
  int E = (b >> 3) & 15, f = b & 7;
  double v = E ? ldexp(1.0 + f / 8.0, E - 7) : ldexp(f / 8.0, -6);
  return (b & 0x80) ? -v : v;
}

uint8_t oracle_e4m3_encode(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  int e;
  double m = frexp((double)v, &e); /* v = m 2^e, m in [0.5, 1) */
  if (e >= -5) {                    /* v >= 2^-6: normal */
    double r = rint(m * 16.0);      /* 1.fff x 8, nearest, ties to even */
    int E = e - 1 + 7;
    if (r == 16.0) {
      r = 8.0;
      E += 1;
    }
    if (E > 15 || (E == 15 && r > 14.0)) return 0x7E;
    return (uint8_t)((E << 3) | ((int)r - 8));
  }
  double r = rint(ldexp((double)v, 9)); /* subnormal: multiples of 2^-9 */
  if (r >= 8.0) return 0x08;
  return (uint8_t)r;
}

uint8_t oracle_e2m1_encode(float v) {
  double a = fabs((double)v);
  uint8_t c;
  /* nearest grid value; at a midpoint the even code (0, 2, 4, 6) wins */
  if (a <= 0.25) c = 0;
  else if (a < 0.75) c = 1;
  else if (a <= 1.25) c = 2;
  else if (a < 1.75) c = 3;
  else if (a <= 2.5) c = 4;
  else if (a < 3.5) c = 5;
  else if (a <= 5.0) c = 6;
  else c = 7;
  return (uint8_t)(c | (v < 0.0f ? 8u : 0u));
}

int oracle_nvfp4_quantize(const float* v, int64_t K, float g, uint8_t* codes, uint8_t* sf) {
  if (!v || !codes || !sf || K <= 0 || K % 16 != 0 || !(g > 0.0f)) return -1;
  for (int64_t b = 0; b < K / 16; ++b) {
    const float* vb = v + b * 16;
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(vb[i]));
    const float sd = amax / (6.0f * g);
    const uint8_t s8 = oracle_e4m3_encode(sd);
    const float d = (float)oracle_e4m3_value(s8) * g;
    sf[b] = s8;
    for (int i = 0; i < 16; i += 2) {
      uint8_t lo = s8 ? oracle_e2m1_encode(vb[i] / d) : 0;
      uint8_t hi = s8 ? oracle_e2m1_encode(vb[i + 1] / d) : 0;
      codes[(b * 16 + i) / 2] = (uint8_t)(lo | (hi << 4));
    }
  }
  return 0;
}

/* Every E4M3 byte's value, filled once from oracle_e4m3_value so that the
 * decoder below need not recompute it for each of the billions of elements a
 * Beam-sized expert path reads; the values are oracle_e4m3_value's exactly. */
static double g_e4m3[256];
static pthread_once_t g_e4m3_once = PTHREAD_ONCE_INIT;
static void fill_e4m3(void) {
  for (int b = 0; b < 256; ++b) g_e4m3[b] = oracle_e4m3_value((uint8_t)b);
}

/* Element i of a packed row (the decoder every NVFP4 operand goes through). */
static double nvfp4_value(const uint8_t* codes, const uint8_t* sf, int64_t i, double g) {
  uint8_t byte = codes[i / 2];
  uint8_t code = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
  return e2m1_value(code) * g_e4m3[sf[i / 16]] * g;
}

double oracle_nvfp4_value(const uint8_t* codes, const uint8_t* sf, int64_t i, double g) {
  pthread_once(&g_e4m3_once, fill_e4m3);
  return nvfp4_value(codes, sf, i, g);
}

int oracle_experts_nvfp4(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                         const double* weights, const uint8_t* const* w13_codes,
                         const uint8_t* const* w13_sf, const uint8_t* const* w2_codes,
                         const uint8_t* const* w2_sf, double g_w13, double g_w2, float g_x,
                         float g_h, double* out) {
  if (!cfg_ok(cfg) || T < 0) return -1;
  if (T == 0) return 0;
  if (!x || !ids || !weights || !w13_codes || !w13_sf || !w2_codes || !w2_sf || !out) return -1;
  const int H = cfg->hidden, I = cfg->inter, E = cfg->n_experts, K = cfg->top_k;
  if (H % 16 || I % 16) return -1;
  pthread_once(&g_e4m3_once, fill_e4m3);
  int bad = 0;
#pragma omp parallel
  {
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    uint8_t* xc = (uint8_t*)malloc((size_t)H / 2);
    uint8_t* xs = (uint8_t*)malloc((size_t)H / 16);
    float* af = (float*)malloc(sizeof(float) * (size_t)I);
    double* ad = (double*)malloc(sizeof(double) * (size_t)I);
    uint8_t* ac = (uint8_t*)malloc((size_t)I / 2);
    uint8_t* as = (uint8_t*)malloc((size_t)I / 16);
    if (!xf || !xd || !xc || !xs || !af || !ad || !ac || !as) {
#pragma omp atomic write
      bad = -2;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t t = 0; t < T; ++t) {
        double* ot = out + t * (int64_t)H;
        for (int h = 0; h < H; ++h) {
          xf[h] = (float)bf16_to_double(x[t * (int64_t)H + h]);
          ot[h] = 0.0;
        }
        oracle_nvfp4_quantize(xf, H, g_x, xc, xs);
        for (int h = 0; h < H; ++h) xd[h] = nvfp4_value(xc, xs, h, (double)g_x);
        for (int k = 0; k < K; ++k) {
          const int e = ids[t * K + k];
          if (e < 0 || e >= E || !w13_codes[e] || !w13_sf[e] || !w2_codes[e] || !w2_sf[e]) {
#pragma omp atomic write
            bad = -3;
            continue;
          }
          for (int i = 0; i < I; ++i) {
            const uint8_t* gc = w13_codes[e] + (int64_t)i * (H / 2);
            const uint8_t* gs = w13_sf[e] + (int64_t)i * (H / 16);
            const uint8_t* uc = w13_codes[e] + (int64_t)(I + i) * (H / 2);
            const uint8_t* us = w13_sf[e] + (int64_t)(I + i) * (H / 16);
            double g = 0.0, u = 0.0;
            for (int h = 0; h < H; ++h) {
              g += nvfp4_value(gc, gs, h, g_w13) * xd[h];
              u += nvfp4_value(uc, us, h, g_w13) * xd[h];
            }
            af[i] = (float)(g / (1.0 + exp(-g)) * u); /* silu(g) * u, then fp32 */
          }
          oracle_nvfp4_quantize(af, I, g_h, ac, as);
          for (int i = 0; i < I; ++i) ad[i] = nvfp4_value(ac, as, i, (double)g_h);
          for (int j = 0; j < H; ++j) {
            const uint8_t* dc = w2_codes[e] + (int64_t)j * (I / 2);
            const uint8_t* ds = w2_sf[e] + (int64_t)j * (I / 16);
            double acc = 0.0;
            for (int i = 0; i < I; ++i) acc += nvfp4_value(dc, ds, i, g_w2) * ad[i];
            ot[j] += weights[t * K + k] * acc;
          }
        }
      }
    }
    free(xf);
    free(xd);
    free(xc);
    free(xs);
    free(af);
    free(ad);
    free(ac);
    free(as);
  }
  return bad;
}
