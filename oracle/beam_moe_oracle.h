/*
 * beam_moe_oracle.h - plain, slow, fp64 CPU oracle of the Beam MoE block
 * forward. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg use it; the product path never does.
 *
 * What it computes is the block as the Hugging Face launch post "Welcome Beam"
 * describes it (sections "Mixture of Experts" and "Residual Stream"), restated
 * in the Russian-language summary (section "Экспертные блоки Mixture of
 * Experts") and the Miles "Beam 1.0" recipe page (section 1, "Key
 * highlights"): sigmoid scores over all experts, experts split into groups,
 * the groups ranked by the sum of their two best scores, the best groups
 * kept, the top experts taken inside them, SwiGLU experts, and a combine with
 * normalized router weights scaled by the routed scale. It shares no code with
 * the GPU library.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes of the repository):
 *  - ties break to the lower index, for groups and for experts;
 *  - the selected ids are listed by descending score;
 *  - "normalized router weights" means w_k = S * s_k / sum_j s_j over the
 *    selected experts (renormalize = 1); renormalize = 0 gives S * s_k;
 *  - bias_mode 0 adds the per-expert bias to the logits before the sigmoid;
 *    bias_mode 1 adds it to the scores for choosing only (weights from the
 *    unbiased scores), as in DeepSeek-V3, whose scheme the router follows;
 *  - no intermediate rounding: everything is fp64 after exact conversion of
 *    the bf16 / fp32 inputs.
 *
 * Arrays are row-major. bf16 values are passed as their 16-bit patterns.
 * Functions return 0 on success and a negative code on a bad argument.
 */
#ifndef BEAM_MOE_ORACLE_H
#define BEAM_MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t hidden;      /* H */
  int32_t inter;       /* I */
  int32_t n_experts;   /* E */
  int32_t n_group;     /* G, groups of E/G experts */
  int32_t topk_group;  /* Gk kept groups */
  int32_t top_k;       /* K experts per token */
  int32_t renormalize; /* 1: weights normalized over the K selected */
  int32_t bias_mode;   /* 0: bias on logits; 1: bias on choice only */
  double routed_scale; /* S */
} oracle_cfg;

/*
 * Routing of T tokens.
 *   x        [T][H] bf16 bits;  w_router [E][H] fp32;  bias [E] fp32 or NULL.
 * Outputs (any may be NULL):
 *   ids      [T][K]  selected experts, descending choice score
 *   weights  [T][K]  combine weights, routed scale included
 *   scores   [T][K]  sigmoid score of each selected expert
 *   kept     [T][Gk] kept groups, in the order they were chosen
 *   margins  [T][2]  (group margin, expert margin): the gap between the last
 *                    chosen and the best unchosen candidate, +inf if none
 *   all_s    [T][E]  every expert's sigmoid score
 */
int oracle_route(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const float* w_router,
                 const float* bias, int32_t* ids, double* weights, double* scores, int32_t* kept,
                 double* margins, double* all_s);

/*
 * One SwiGLU expert on one token (x in fp64, length H):
 *   g = Wg x, u = Wu x, a = silu(g) * u, y = Wd a       (y length H)
 * w13 [2I][H] (rows 0..I-1 gate, I..2I-1 up), w2 [H][I], bf16 bits.
 */
int oracle_swiglu_expert(int32_t H, int32_t I, const double* x, const uint16_t* w13,
                         const uint16_t* w2, double* y);

/*
 * The hidden activations of every routed (token, expert) pair, the quantity
 * the gate/up step produces before the down projection:
 *   a[t][k][i] = silu(Wg_e x_t)[i] * (Wu_e x_t)[i],   e = ids[t][k]    (fp64 [T][K][I])
 * w13[e] as for oracle_experts; w2 is not needed.
 */
int oracle_hidden(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                  const uint16_t* const* w13, double* a);

/*
 * Expert path and combine for T tokens given their routes:
 *   out[t] = sum_k weights[t][k] * expert_{ids[t][k]}(x[t])     (fp64 [T][H])
 * w13[e] / w2[e] point to expert e's weights; an expert no token selects may
 * be NULL (a selected NULL expert is an error).
 */
int oracle_experts(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                   const double* weights, const uint16_t* const* w13, const uint16_t* const* w2,
                   double* out);

/* ------------------------------------------------------------------ NVFP4
 * The 4-bit format the launch post names for Blackwell deployment ("Welcome
 * Beam", section "Mixture of Experts": the NVFP4 checkpoint stores most
 * parameters in 4-bit precision for NVIDIA Blackwell GPUs): E2M1 values
 * {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit, one FP8 E4M3 scale per 16
 * consecutive elements along the contraction dimension, one FP32 scale per
 * tensor. value = e2m1(code) * e4m3(scale) * tensor_scale. Codes are packed
 * two per byte, element 2j in the low nibble.
 */
double oracle_e2m1_value(uint8_t code);  /* low 4 bits used */
double oracle_e4m3_value(uint8_t byte);
/* Round to nearest, ties to even, saturating at 448 (v >= 0 finite). */
uint8_t oracle_e4m3_encode(float v);
/* Round to nearest, ties to even, saturating at +-6. */
uint8_t oracle_e2m1_encode(float v);

/* Quantise K values (K a multiple of 16), every step in fp32: per block,
 * amax = max |v|, scale = e4m3(amax / (6 g)), then each code =
 * e2m1(v / (scale * g)) (all zero when the scale is zero). codes[K/2],
 * sf[K/16]. */
int oracle_nvfp4_quantize(const float* v, int64_t K, float g, uint8_t* codes, uint8_t* sf);

/* Dequantised value of element i of a packed row. */
double oracle_nvfp4_value(const uint8_t* codes, const uint8_t* sf, int64_t i, double g);

/*
 * Expert path with NVFP4 experts and NVFP4 activations (the W4A4 scheme the
 * vLLM recipe's FlashInfer TRT-LLM backend uses): each token's x (bf16) is
 * quantised with tensor scale g_x; g = Wg xq, u = Wu xq exactly in fp64 on the
 * dequantised values; a = silu(g) * u in fp64, rounded to fp32 and quantised
 * with g_h; y = Wd aq; out[t] = sum_k weights[t][k] y.
 * w13_codes[e] [2I][H/2], w13_sf[e] [2I][H/16], w2_codes[e] [H][I/2],
 * w2_sf[e] [H][I/16] (scales row-major).
 */
int oracle_experts_nvfp4(const oracle_cfg* cfg, int64_t T, const uint16_t* x, const int32_t* ids,
                         const double* weights, const uint8_t* const* w13_codes,
                         const uint8_t* const* w13_sf, const uint8_t* const* w2_codes,
                         const uint8_t* const* w2_sf, double g_w13, double g_w2, float g_x,
                         float g_h, double* out);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_ORACLE_H */
