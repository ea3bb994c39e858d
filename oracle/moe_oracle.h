/*
 * moe_oracle.h -- CPU oracle for the MXFP4-weight / FP8-activation (W4A8)
 * mixture-of-experts decode step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
 * call this library: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do. It shares no code, header, table or constant with the
 * CUDA library under mxfp4_weight_streaming_fp8_b200/csrc.
 *
 * Every function is plain, slow and written to be checked by eye against the
 * passages it cites. Floating point is fp64 except where a step is defined in
 * fp32 (the activation quantiser, so FP8 codes can be compared bit for bit).
 *
 * Sources:
 *  [MX]   OCP Microscaling Formats (MX) Specification v1.0: element type E2M1
 *         and shared scale type E8M0, one scale per block of 32 elements.
 *  [OFP8] OCP 8-bit Floating Point Specification (OFP8): E4M3 (bias 7, no
 *         infinities, S.1111.111 is NaN, max finite 448).
 *  [MTP]  MarkTechPost, "NVIDIA Shows 3 Ways to Speed Up MoE Inference on DGX
 *         Spark" (aitujian.cn copy): sections "Why is MoE decoding on DGX Spark
 *         memory-bound?" (weight streaming, W4A8 recipe), "What are the 3
 *         optimizations?" (MXFP4 MoE kernels; up to 32 experts for a 4-token
 *         verify; the online FP8 LM head), "What is Ling 3.0 ..." (top-8
 *         routed experts plus one shared expert per token).
 *
 * Parity status: every function here is pinned by a CPU test (format tables,
 * a hand-derived 2-expert example, one-hot probes, brute-force dense
 * evaluation, invariants; the shared-expert step by reduction to the routed
 * step and to a single expert; the FP8-intermediate step by torch's float8
 * conversion, numpy's dequantised down projection and the E4M3 rounding
 * bound; the LM head by a hand row, torch's float8 conversion and one-hot
 * columns). None is "parity unpinned".
 *
 * Layouts (row-major, K contiguous):
 *   x        bf16 bit patterns [M][H]
 *   router_w fp32 [E][H]
 *   w13 codes  [2I][H/2] per expert: rows 0..I-1 gate, rows I..2I-1 up;
 *              byte j holds element 2j in bits 3:0 and element 2j+1 in 7:4
 *   w13 scales [2I][H/32] per expert: byte t scales elements [32t, 32t+32)
 *   w2 codes   [H][I/2] per expert, w2 scales [H][I/32]
 * Expert tensors are passed as arrays of E per-expert pointers so a caller can
 * supply only the experts a step touches (NULL for the rest).
 *
 * Return value of the int functions: 0 on success, negative on a bad argument
 * or a NaN E8M0 scale (0xFF) met on the way.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- element formats ---------------------------------------------------- */
double   oracle_e2m1_value(int code);          /* [MX] E2M1, code in 0..15        */
double   oracle_e8m0_value(int byte);          /* [MX] E8M0, NaN for 0xFF         */
double   oracle_e4m3_value(int code);          /* [OFP8] E4M3, NaN for S.1111.111 */
int      oracle_e4m3_encode(float v);          /* [OFP8] RNE, saturate to +-448   */
double   oracle_bf16_value(uint16_t bits);
uint16_t oracle_bf16_round(double v);          /* round to nearest even           */

/* ---- steps of the decode path ------------------------------------------- */
/* A1: per-token FP8 quantisation. q [M][H] E4M3 codes, s [M] fp32 scale. */
int oracle_quantize(int M, int H, const uint16_t* x, uint8_t* q, float* s);
/* A2: router logits in fp64 from the bf16 activations. logits [M][E]. */
int oracle_router_logits(int M, int H, int E, const uint16_t* x,
                         const float* router_w, double* logits);
/* A3: top-k ordered by (logit desc, index asc), softmax over the k kept. */
int oracle_topk(int M, int E, int k, const double* logits,
                int32_t* ids, double* weights);
/* A4: expert union. union_ids [<=M*k] ascending, returns U (>=0).
 * pair_off [U+1]; pair_tok / pair_slot [M*k] list the (token, slot) pairs of
 * union entry u at positions pair_off[u] .. pair_off[u+1]-1, in (token, slot)
 * order. */
int oracle_union(int M, int E, int k, const int32_t* ids, int32_t* union_ids,
                 int32_t* pair_off, int32_t* pair_tok, int32_t* pair_slot);
/* A5-A7 for one token through one expert: h [I] (optional) and d [H]. */
int oracle_expert(int H, int I, const uint8_t* q_m, float s_m,
                  const uint8_t* w13_codes, const uint8_t* w13_scales,
                  const uint8_t* w2_codes, const uint8_t* w2_scales,
                  double* h_out, double* d_out);
/* A1-A8: the whole step. Outputs (any may be NULL except y64):
 * q [M][H], s [M], logits [M][E], ids [M][k], weights [M][k], y64 [M][H],
 * y_bf16 [M][H]. */
int oracle_moe_decode(int H, int I, int E, int k, int M,
                      const uint16_t* x, const float* router_w,
                      const uint8_t* const* w13_codes,
                      const uint8_t* const* w13_scales,
                      const uint8_t* const* w2_codes,
                      const uint8_t* const* w2_scales,
                      uint8_t* q, float* s, double* logits, int32_t* ids,
                      double* weights, double* y64, uint16_t* y_bf16);
/* A1-A8 with one shared expert ("NVIDIA Shows 3 Ways to Speed Up MoE
 * Inference on DGX Spark", section "What is Ling 3.0, and why does it suit
 * DGX Spark?": each layer routes a token to 8 routed experts "along with 1
 * shared expert"). Readings: the shared expert has the routed experts' shape
 * and format and is always active with weight 1 (outside the router's
 * softmax); its output is added after the routed ones:
 *   y[m] = sum_j w[m][j] * expert_{ids[m][j]}(x_m) + expert_shared(x_m).
 * Outputs as oracle_moe_decode (q, s, logits may be NULL; ids and weights
 * cover the routed experts). */
int oracle_moe_decode_shared(int H, int I, int E, int k, int M,
                             const uint16_t* x, const float* router_w,
                             const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                             const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                             const uint8_t* sh_w13_codes, const uint8_t* sh_w13_scales,
                             const uint8_t* sh_w2_codes, const uint8_t* sh_w2_scales,
                             uint8_t* q, float* s, double* logits, int32_t* ids, double* weights,
                             double* y64);
/* The A1 rule on fp32 values (the FP8 intermediate below): amax = max|v|,
 * inv = fl32(448/amax), code = E4M3_RNE_sat(fl32(v*inv)), s = fl32(amax/448);
 * amax == 0 gives zero codes and s = 1. One vector of n values. */
int oracle_quantize_f32(int n, const float* v, uint8_t* q, float* s);

/* A5-A7 with an FP8 intermediate (a true A8 down projection: "W4A8",
 * section "Why is MoE decoding on DGX Spark memory-bound?" of the DGX Spark
 * MoE page). Reading: the SwiGLU output h of the pair, computed as in
 * oracle_expert and rounded to fp32, is quantised by oracle_quantize_f32
 * over its I elements; d = s_h * W2 . E4M3(hq) in fp64. hq_out [I] and
 * hs_out may be NULL. */
int oracle_expert_a8(int H, int I, const uint8_t* q_m, float s_m,
                     const uint8_t* w13_codes, const uint8_t* w13_scales,
                     const uint8_t* w2_codes, const uint8_t* w2_scales,
                     uint8_t* hq_out, float* hs_out, double* d_out);

/* A1-A8 with the FP8 intermediate for every expert, and optionally one
 * shared expert (sh_* all NULL for none; otherwise as in
 * oracle_moe_decode_shared). Outputs as oracle_moe_decode_shared. */
int oracle_moe_decode_a8(int H, int I, int E, int k, int M,
                         const uint16_t* x, const float* router_w,
                         const uint8_t* const* w13_codes, const uint8_t* const* w13_scales,
                         const uint8_t* const* w2_codes, const uint8_t* const* w2_scales,
                         const uint8_t* sh_w13_codes, const uint8_t* sh_w13_scales,
                         const uint8_t* sh_w2_codes, const uint8_t* sh_w2_scales,
                         uint8_t* q, float* s, double* logits, int32_t* ids, double* weights,
                         double* y64);
/* Brute force: every expert for every token, masked by a rank-count top-k
 * and weighted by a softmax renormalised over the kept experts. */
int oracle_moe_dense(int H, int I, int E, int k, int M,
                     const uint16_t* x, const float* router_w,
                     const uint8_t* const* w13_codes,
                     const uint8_t* const* w13_scales,
                     const uint8_t* const* w2_codes,
                     const uint8_t* const* w2_scales, double* y64);
/* A9: RMSNorm with unit weight between stacked layers:
 * out = bf16(y / sqrt(mean(y^2) + eps)), per token, fp64. */
int oracle_rmsnorm(int M, int H, const uint16_t* y, double eps, uint16_t* out);

/* FP8 LM head ("NVIDIA Shows 3 Ways to Speed Up MoE Inference on DGX Spark",
 * MarkTechPost, item 2 "Online FP8 LM head": the 157,184 x 2,560 BF16 output
 * matrix is quantised to FP8 once at load, halving the bytes each token
 * reads). The pages do not give the scale granularity; the reading here is
 * one fp32 scale per output row, set by the same rule as the activation
 * quantiser A1 applied to each row (amax, fp32 448/amax, E4M3
 * round-to-nearest-even with saturation, scale amax/448; an all-zero row
 * gives zero codes and scale 1). w [V][H] bf16 bits -> codes [V][H], scales
 * [V]. */
int oracle_lm_quantize(int V, int H, const uint16_t* w, uint8_t* codes, float* scales);
/* logits[m][v] = scales[v] * sum_h e4m3(codes[v][h]) * bf16(x[m][h]) in fp64
 * (weights FP8, activations kept in BF16). x [M][H], logits [M][V]. */
int oracle_lm_head(int V, int H, int M, const uint8_t* codes, const float* scales, const uint16_t* x,
                   double* logits);

#ifdef __cplusplus
}
#endif
#endif
