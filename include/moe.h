/*
 * moe.h -- C ABI of libmoe: the decode step of a mixture-of-experts layer with
 * MXFP4 expert weights and FP8 E4M3 activations (W4A8) on an NVIDIA B200
 * (sm_100a).
 *
 * What the step computes. Sources: MarkTechPost, "NVIDIA Shows 3 Ways to
 * Speed Up MoE Inference on DGX Spark" (aitujian.cn copy). The section "Why
 * is MoE decoding on DGX Spark memory-bound?" says batch-1 decode is bound by
 * reading weights, and that the recipe is W4A8 with MXFP4 MoE kernels. The
 * section "What are the 3 optimizations?" covers the MXFP4 MoE kernels for
 * the narrow 768-wide expert layer, and says a 4-token verify activates up
 * to 32 experts. The section "What is Ling 3.0 ..." says each token is routed
 * to 8 experts. The element formats follow OCP MX v1.0 (E2M1 codes with one
 * E8M0 scale per 32 elements) and OCP OFP8 (E4M3).
 *
 * Per token m (M tokens, hidden size H, expert width I, E experts, top_k):
 *   A1  q[m] = E4M3_rne_sat(x[m] * 448/amax_m), s_m = amax_m/448 (fp32)
 *   A2  logits[m][e] = sum_h x[m][h] * router_w[e][h]  (bf16 x, fp32 weights)
 *   A3  ids = top_k logits, highest first, ties to the lower expert index;
 *       w = softmax over the top_k kept logits (sums to 1)
 *   A4  union of the selected experts over the M tokens
 *   A5  g_n = s_m * <W13[e][n], q[m]>, up_n = s_m * <W13[e][I+n], q[m]>
 *   A6  h_n = silu(g_n) * up_n   (fp32, not requantised)
 *   A7  d_r = <W2[e][r], h>
 *   A8  y[m][r] = bf16( sum over the token's top_k slots of w * d_r )
 * where an MXFP4 weight is E2M1(code) * 2^(E8M0 - 127) per block of 32 along K.
 *
 * Weight layout (row-major, K contiguous; all device memory):
 *   w13_codes  uint8 [E][2I][H/2]  rows 0..I-1 gate, rows I..2I-1 up
 *   w13_scales uint8 [E][2I][H/32]
 *   w2_codes   uint8 [E][H][I/2]
 *   w2_scales  uint8 [E][H][I/32]
 *   Byte j of a code row holds element 2j in bits 3:0 and element 2j+1 in
 *   bits 7:4. Scale byte t of a row covers elements [32t, 32t+32).
 *   router_w   float [E][H]
 *
 * Threading and errors. A context serves one layer and one stream at a time.
 * Calls on one context must not overlap, because they share its workspace.
 * All argument checks are synchronous and happen before any GPU work. A
 * failed check returns an error code and enqueues nothing. Device-side
 * failures, such as a grid barrier that times out, set a status word in the
 * workspace. moe_sync_status() reads it. Nothing falls back silently: a shape
 * or device the kernels do not support returns MOE_ERR_UNSUPPORTED.
 */
#ifndef LIBMOE_MOE_H
#define LIBMOE_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer      */
  MOE_ERR_UNSUPPORTED = 2,  /* shape or device outside what the kernels cover  */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call failed                      */
  MOE_ERR_OOM = 4,          /* workspace allocation failed                     */
  MOE_ERR_NOT_LOADED = 5,   /* moe_decode before moe_load_experts              */
  MOE_ERR_TIMEOUT = 6,      /* a device-side wait gave up (see moe_sync_status) */
  MOE_ERR_BAD_WEIGHTS = 7   /* an E8M0 scale byte is 0xFF (NaN)                */
} moe_status;

/* moe_config.flags */
#define MOE_FLAG_SPLIT_KERNELS 0x1u /* run the step as three kernels (route, gate/up,
                                       down) instead of one persistent kernel */
#define MOE_FLAG_PRE_RMSNORM  0x2u  /* x <- bf16(x / sqrt(mean(x^2) + 1e-6)) per token
                                       before A1/A2 (unit-weight RMSNorm between
                                       stacked layers, fp32); persistent kernel
                                       only: with MOE_FLAG_SPLIT_KERNELS,
                                       moe_create returns MOE_ERR_UNSUPPORTED */
#define MOE_FLAG_SHARED_EXPERT 0x4u /* one shared expert besides the routed ones
                                       ("NVIDIA Shows 3 Ways to Speed Up MoE
                                       Inference on DGX Spark", section on
                                       Ling 3.0: each token goes to its 8
                                       routed experts and to one shared
                                       expert). The
                                       four expert arrays hold E + 1 experts;
                                       expert E (the last) is the shared one,
                                       same shape and format, never routed
                                       (router_w stays [E][H]). Every token
                                       passes it with weight 1, outside the
                                       softmax, and its output is added after
                                       the routed ones:
                                         y = sum_j w_j * FFN_{id_j}(x) + FFN_E(x)
                                       Persistent kernel only: with
                                       MOE_FLAG_SPLIT_KERNELS, moe_create
                                       returns MOE_ERR_UNSUPPORTED */
#define MOE_FLAG_SPLITK_DOWN 0x100u  /* down projection split over K (each CTA
                                       multiplies its own h slice by a K-major
                                       copy of W2 that moe_load_experts makes;
                                       partial outputs summed in a fixed
                                       order). A CUDA-core kernel option:
                                       max_tokens <= 4; not with
                                       MOE_FLAG_FP8_INTERMEDIATE,
                                       MOE_FLAG_SPLIT_KERNELS or
                                       MOE_FLAG_TENSOR_CORES */
#define MOE_FLAG_FP8_INTERMEDIATE 0x8u /* FP8 input to the down projection too
                                       (W4A8 on the same page, section "Why
                                       is MoE decoding on DGX Spark
                                       memory-bound?", read as 8-bit inputs
                                       for both projections): the SwiGLU
                                       output h of each (token, expert) pair
                                       is quantised like the activations,
                                       over its I elements: amax = max|h|,
                                       inv = fl32(448/amax), code =
                                       E4M3_RNE_sat(fl32(h*inv)), scale
                                       fl32(amax/448) (amax == 0: zero codes,
                                       scale 1); the down projection uses
                                       scale * E4M3(code). h itself is fp32
                                       SwiGLU of fp32 sums, so a code can
                                       differ from one computed from exact h
                                       where h*inv lies at a rounding
                                       boundary. Persistent kernel only, as
                                       MOE_FLAG_SHARED_EXPERT */
#define MOE_FLAG_CUDA_CORES 0x10u    /* run the persistent CUDA-core kernel
                                       (E2M1 decoded in registers for both
                                       projections) */
#define MOE_FLAG_TENSOR_CORES 0x20u  /* run the persistent tensor-core kernel
                                       (gate/up on tcgen05 block-scaled MMAs;
                                       down on them too from
                                       MOE_TC_DOWN_MMA_MIN_TOKENS tokens of
                                       max_tokens, else on CUDA cores; see
                                       MOE_FLAG_TC_DOWN_*); needs H and I to
                                       be multiples of 128 and its
                                       shared-memory plan to fit, else
                                       moe_create returns MOE_ERR_UNSUPPORTED.
                                       With neither flag (and without
                                       MOE_FLAG_SPLIT_KERNELS or
                                       MOE_FLAG_SPLITK_DOWN) moe_create
                                       picks the tensor-core kernel when the
                                       shape allows it and max_tokens is at
                                       least MOE_TC_MIN_TOKENS, else the
                                       CUDA-core kernel. Both compute the same
                                       step; moe_query names the one a context
                                       runs. Setting both flags, or this one
                                       with MOE_FLAG_SPLIT_KERNELS or
                                       MOE_FLAG_SPLITK_DOWN, is
                                       MOE_ERR_INVALID_ARG */
#define MOE_TC_MIN_TOKENS 4
#define MOE_FLAG_TC_DOWN_MMA 0x40u   /* tensor-core kernel: run the down
                                       projection on tcgen05 MMAs as well
                                       (tiles of 128 output rows x up to 16
                                       pairs of one expert; W2 decoded once
                                       per tile, not once per pair). h enters
                                       as per-pair-scaled E4M3 hi + lo/16
                                       (within 2^-8 of h; with
                                       MOE_FLAG_FP8_INTERMEDIATE, the FP8 h
                                       codes alone). Needs I <= 1024, else
                                       the tensor-core plan fails; also I <= H */
#define MOE_FLAG_TC_DOWN_CUDA 0x80u  /* tensor-core kernel: keep the down
                                       projection on CUDA cores. With neither
                                       TC_DOWN flag the tensor cores take the
                                       down projection from
                                       MOE_TC_DOWN_MMA_MIN_TOKENS tokens of
                                       max_tokens on. Both flags:
                                       MOE_ERR_INVALID_ARG */
#define MOE_TC_DOWN_MMA_MIN_TOKENS 2

typedef struct {
  int32_t hidden;      /* H: multiple of 32, 32..8192                        */
  int32_t inter;       /* I: multiple of 32, 32..4096                        */
  int32_t num_experts; /* E: 1..1024                                         */
  int32_t top_k;       /* 1..min(E, 32)                                      */
  int32_t max_tokens;  /* upper bound on M per call: 1..32                   */
  uint32_t flags;      /* MOE_FLAG_*                                         */
  int32_t device;      /* CUDA device ordinal the context lives on          */
  int32_t shard_index; /* intra-expert split: this context's part g, 0..G-1  */
  int32_t shard_count; /* G, the number of parts (0 or 1: the whole layer)   */
} moe_config;

/* Intra-expert split of one layer over G GPUs (shard_count = G > 1). Part g
 * holds rows [g*I/G, (g+1)*I/G) of every expert's gate and of its up
 * projection, and the same columns of its down projection: h_n depends on
 * row n of gate and up only, and the down product is a sum over n, so
 *   y[m][r] = bf16( sum over g of P_g[m][r] )
 * where P_g is A8's slot-order sum taken over part g's columns alone. Every
 * part reads 1/G of each active expert, so the parts stay balanced even for
 * one token. Routing (A1-A4, and the RMSNorm of MOE_FLAG_PRE_RMSNORM) is not
 * split: each part computes it from the same x and the whole router. Rules:
 * I must be a multiple of 32*G (each part keeps whole E8M0 blocks of W2);
 * G <= 128; 0 <= shard_index < G; MOE_FLAG_FP8_INTERMEDIATE is UNSUPPORTED
 * (its per-token scale of h spans all I columns, which would need a second
 * exchange). The context then plans its kernels for width I/G,
 * moe_load_experts takes the whole layer's arrays and keeps a copy of the
 * part (MOE_LOAD_COPY_REPACK is required), and moe_decode writes P_g as fp32
 * [M][H]. The caller adds the parts (one all-reduce over the G GPUs) and
 * rounds the sum with moe_round_bf16. */

typedef struct moe_ctx moe_ctx; /* opaque */

/* Create a context: validates cfg, checks the device is sm_100, allocates the
 * workspace (sized from max_tokens) on cfg->device. *out is set only on
 * MOE_OK. Returns INVALID_ARG / UNSUPPORTED / CUDA / OOM. */
moe_status moe_create(const moe_config* cfg, moe_ctx** out);

/* moe_load_experts load_flags */
#define MOE_LOAD_BORROW 0x0u        /* keep the caller's pointers (they must outlive the ctx) */
#define MOE_LOAD_SKIP_VALIDATE 0x1u /* do not scan scale bytes for 0xFF */
#define MOE_LOAD_COPY_REPACK 0x2u   /* copy the five arrays into memory the context
                                       owns, re-tiling the gate/up codes into the
                                       running kernel's private layout; the
                                       caller may free its arrays after the call */

/* Attach one layer's weights (device pointers, layouts above, each 16-byte
 * aligned; for a part of an intra-expert split, the whole layer's arrays).
 * Without MOE_LOAD_COPY_REPACK the context borrows them: nothing is copied,
 * and the caller keeps ownership; the arrays must outlive their use.
 * With MOE_LOAD_COPY_REPACK the context allocates one device buffer for a
 * copy of all five arrays (about the size of the inputs) and copies them,
 * synchronously. For the tensor-core kernel the gate/up codes are re-tiled
 * so that each 8-row unit (4 gate rows and the 4 up rows of the same
 * intermediate indices) and 128-element K-chunk is one contiguous 512-byte
 * block, [E][I/4][H/128][8][64 B]: each stage of the weight stream then reads
 * whole blocks instead of 64-byte pieces of 8 rows. The CUDA-core and split
 * kernels get a plain copy in the layout above. The buffer is freed by the
 * next moe_load_experts or by moe_destroy. OOM if the allocation fails.
 * Unless MOE_LOAD_SKIP_VALIDATE is set, the scale bytes are scanned on the
 * device for the NaN encoding 0xFF, synchronously on the legacy default
 * stream; MOE_ERR_BAD_WEIGHTS if any is found. May be called again to point
 * the context at other weights. A part of an intra-expert split
 * (shard_count > 1) copies its rows of W13 and its columns of W2 (and the
 * whole router), so the call needs MOE_LOAD_COPY_REPACK (INVALID_ARG
 * otherwise) and the copy is about 1/G of the layer. */
moe_status moe_load_experts(moe_ctx* ctx, const float* router_w,
                            const uint8_t* w13_codes, const uint8_t* w13_scales,
                            const uint8_t* w2_codes, const uint8_t* w2_scales,
                            uint32_t load_flags);

/* One decode step, enqueued on `stream` (a cudaStream_t; NULL = legacy
 * default stream), asynchronous, allocation-free and capturable into a CUDA
 * graph.
 *   x_bf16  [M][H] bf16 device, read only
 *   y_bf16  [M][H] bf16 device, written (must not alias x); for a part of
 *           an intra-expert split, [M][H] fp32: the part's P_g before the
 *           bf16 round
 *   M       0..max_tokens; M == 0 returns MOE_OK and enqueues nothing
 * Optional device outputs (NULL to skip):
 *   topk_ids [M][top_k] int32, highest logit first
 *   topk_w   [M][top_k] fp32 routing weights in the same order
 *   xq       [M][H] uint8 E4M3 activation codes
 *   xscale   [M] fp32 per-token activation scales
 *   xnorm    [M][H] bf16 normalised input (only with MOE_FLAG_PRE_RMSNORM)
 * Returns INVALID_ARG (null/misaligned/size), NOT_LOADED, CUDA (launch). */
moe_status moe_decode(moe_ctx* ctx, const void* x_bf16, int32_t M, void* y_bf16,
                      void* stream, int32_t* topk_ids, float* topk_w, uint8_t* xq,
                      float* xscale, void* xnorm_bf16);

/* y_bf16[i] = bf16(y_f32[i]), round to nearest even, for i < n: the last
 * step of an intra-expert split, after the parts' fp32 sums have been added
 * (an all-reduce, in place or not). Device pointers, y_f32 4-byte and y_bf16
 * 2-byte aligned, not overlapping; asynchronous on `stream` (NULL: the
 * legacy default stream) on the current device. n == 0 does nothing.
 * INVALID_ARG on a NULL or misaligned pointer, a negative n or overlap; CUDA
 * if the launch fails. */
moe_status moe_round_bf16(const float* y_f32, void* y_bf16, int64_t n, void* stream);

/* Synchronise `stream`, then read and clear the context's device status word.
 * Returns MOE_ERR_TIMEOUT if a device-side wait gave up since the last call,
 * and resets the barrier state so the context can be used again. */
moe_status moe_sync_status(moe_ctx* ctx, void* stream);

/* Write a JSON description of the context into buf (always NUL-terminated
 * when len > 0): device, sm, kernel variant, grid, threads, shared memory,
 * shapes. Lets a caller confirm at start-up which path runs. Returns
 * INVALID_ARG if buf is NULL or too small (the JSON is then truncated). */
moe_status moe_query(const moe_ctx* ctx, char* buf, size_t len);

/* Free the workspace and the context (NULL is a no-op). Borrowed weights are
 * not touched. */
void moe_destroy(moe_ctx* ctx);

/* Host-only: the launch plan the persistent kernel would get for cfg on a
 * device with sm_count SMs and smem_limit bytes of opt-in shared memory per
 * block (grid, shared-memory carving, ring slots), as JSON in buf. Makes no
 * CUDA call. Returns INVALID_ARG for a bad cfg or a NULL / too small buf,
 * UNSUPPORTED when the shape does not fit (buf still holds the plan). */
moe_status moe_plan_query(const moe_config* cfg, int32_t sm_count, size_t smem_limit,
                          char* buf, size_t len);

/* Test hook for the failure path of the persistent kernel (ignored by the
 * split path, which has no device-side waits). Sets the budget, in clock64
 * cycles, of every device-side wait; budget_cycles <= 0 restores the default
 * (about 0.5 s). With force_stall != 0 the logits wait looks for a tag no CTA
 * ever writes, so that wait runs out on purpose: the kernel sets the status
 * word, finishes with garbage output and returns, and moe_sync_status then
 * reports MOE_ERR_TIMEOUT. Returns INVALID_ARG for a NULL ctx. */
moe_status moe_debug_set_wait(moe_ctx* ctx, long long budget_cycles, int force_stall);

/* Test hook for timeline measurements of the persistent kernels (k_fused and
 * k_tc): with a non-NULL device pointer to grid x 64 uint64 words (8-byte
 * aligned; grid = the "grid" moe_query reports), every later moe_decode of
 * this context writes %globaltimer stamps of its phases, 64 slots per CTA
 * (lane 0 of the warp that reaches a phase writes it; the last writer wins).
 * Common slots: 0 kernel start, 1 after the programmatic-launch wait, 2 the
 * E4M3 codes written, 3 logit words gathered, 4 routing done, 8 top-k done,
 * 10/11 down work done and combine start, 12 kernel end; the other slots
 * mark kernel-specific points (stages landed, MMAs issued, epilogue, down
 * items or tiles). Slots not reached keep their value. NULL turns it off.
 * Ignored by the three-kernel form. Returns INVALID_ARG for a NULL ctx or a
 * misaligned pointer. */
moe_status moe_debug_set_trace(moe_ctx* ctx, unsigned long long* trace);

/* Size of the fixed device scratch array behind moe_decode_static. */
#define MOE_STATIC_SCRATCH_BYTES ((size_t)4 << 20)

/* One decode step that allocates nothing. The paper has no counterpart: this
 * is an interface for callers that cannot allocate device memory, such as a
 * plugin hosted by a runtime that owns all device memory, or a serving loop
 * that must never call cudaMalloc (the call can synchronise the device).
 *
 * It computes what moe_decode computes, with the three-kernel form of the
 * step (the MOE_FLAG_SPLIT_KERNELS path). There is no context. The layer's
 * shapes come from cfg (max_tokens and device are ignored; of the flags,
 * MOE_FLAG_SHARED_EXPERT, MOE_FLAG_PRE_RMSNORM and MOE_FLAG_FP8_INTERMEDIATE
 * return MOE_ERR_UNSUPPORTED, as does shard_count > 1
 * and MOE_FLAG_SPLIT_KERNELS is ignored), and the
 * weights, x and y are passed in directly with the layouts, alignment and
 * optional outputs of moe_load_experts and moe_decode. The scale bytes are not
 * scanned for 0xFF.
 *
 * Scratch is one file-scope device array of MOE_STATIC_SCRATCH_BYTES (4 MiB),
 * held by every GPU that loads the library until the process exits. A call
 * needs about M*(E*4 + H) + M*top_k*(4*I + 32) bytes of it. Larger shapes
 * return MOE_ERR_UNSUPPORTED, as do calls whose M*H*2 bytes of f16
 * activations exceed the gate/up kernel's shared memory. The first call on a
 * device, made with that device current, does that device's set-up (it finds
 * the array's device address and reads the device's limits). Make that first
 * call before any stream capture.
 *
 * Every call shares the array, which keeps what the last call left in it.
 * Each call clears the words that must start at zero. Calls that overlap on
 * the GPU (different streams or host threads) race on the array and corrupt
 * each other's results.
 *
 * No cudaMalloc, cudaFree or other allocating routine is called. Returns
 * INVALID_ARG (null/misaligned/bad size), UNSUPPORTED (device or shape),
 * CUDA (launch). */
moe_status moe_decode_static(const moe_config* cfg, const float* router_w,
                             const uint8_t* w13_codes, const uint8_t* w13_scales,
                             const uint8_t* w2_codes, const uint8_t* w2_scales,
                             const void* x_bf16, int32_t M, void* y_bf16, void* stream,
                             int32_t* topk_ids, float* topk_w, uint8_t* xq, float* xscale);

/* Static string naming a status code. */
const char* moe_status_string(moe_status s);

/* ------------------------------------------------------------ FP8 LM head
 * "NVIDIA Shows 3 Ways to Speed Up MoE Inference on DGX Spark"
 * (MarkTechPost), item 2 "Online FP8 LM head": the 157,184 x 2,560 output
 * matrix, stored in BF16, is quantised to FP8 once when it is loaded, which
 * halves the bytes every generated token reads. The pages do not give the
 * scale granularity; here each output row v gets one fp32 scale s_v and E4M3
 * codes by the activation quantiser's rule applied to the row (amax over the
 * row, fp32 448/amax, round to nearest even with saturation, s_v = amax/448;
 * an all-zero row gets zero codes and s_v = 1). A call computes
 *     logits[m][v] = s_v * sum_h e4m3(W[v][h]) * x[m][h]
 * for BF16 activations x, in fp32 (weights FP8, activations BF16).
 * The context owns the FP8 copy (V*H + 4*V bytes); it serves one matrix. */
typedef struct moe_lm moe_lm; /* opaque */

/* vocab >= 1; hidden a multiple of 64 in [64, 8192]; 1 <= max_tokens <= 16;
 * device an sm_100 GPU. Allocates the FP8 copy and a status word.
 * INVALID_ARG on bad arguments, UNSUPPORTED if the kernel does not fit the
 * device, OOM if an allocation fails. */
moe_status moe_lm_create(int32_t vocab, int32_t hidden, int32_t max_tokens, int32_t device, moe_lm** out);

/* Quantise the BF16 matrix w_bf16 [vocab][hidden] (device pointer, 16-byte
 * aligned, row-major) into the context. Synchronous; the caller may free w
 * afterwards. INVALID_ARG on a NULL or misaligned pointer, CUDA on a launch
 * failure. */
moe_status moe_lm_load(moe_lm* lm, const void* w_bf16);

/* logits [M][vocab] fp32 (device, 4-byte aligned) for x_bf16 [M][hidden]
 * (device, 16-byte aligned), 0 <= M <= max_tokens; M = 0 does nothing.
 * Asynchronous on `stream` (NULL: the legacy default stream); allocates
 * nothing. INVALID_ARG on bad sizes, misalignment or overlapping x and
 * logits; NOT_LOADED before moe_lm_load. A device-side wait that runs out of
 * budget sets the status word, read by moe_lm_sync_status. */
moe_status moe_lm_head(moe_lm* lm, const void* x_bf16, int32_t M, float* logits, void* stream);

/* Synchronise `stream` and report the status word: OK, or TIMEOUT (the word
 * is cleared). */
moe_status moe_lm_sync_status(moe_lm* lm, void* stream);

/* Copy the context's FP8 weights into caller buffers (device pointers):
 * codes [vocab][hidden] E4M3 and scales [vocab] fp32, asynchronously on
 * `stream`. NOT_LOADED before moe_lm_load; CUDA if a copy fails. */
moe_status moe_lm_read_weights(const moe_lm* lm, uint8_t* codes, float* scales, void* stream);

/* JSON description of the launch configuration (kernel, grid, shared memory,
 * ring slots) into buf; INVALID_ARG if it does not fit in len. */
moe_status moe_lm_query(const moe_lm* lm, char* buf, size_t len);

void moe_lm_destroy(moe_lm* lm);

#ifdef __cplusplus
}
#endif
#endif /* LIBMOE_MOE_H */
