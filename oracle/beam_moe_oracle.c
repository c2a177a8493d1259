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

int oracle_swiglu_expert(int32_t H, int32_t I, const double* x, const uint16_t* w13,
                         const uint16_t* w2, double* y) {
  if (H <= 0 || I <= 0 || !x || !w13 || !w2 || !y) return -1;
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  if (!a) return -2;
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
  for (int j = 0; j < H; ++j) {
    const uint16_t* wd = w2 + (int64_t)j * I;
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += bf16_to_double(wd[i]) * a[i];
    y[j] = acc;
  }
  free(a);
  return 0;
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
