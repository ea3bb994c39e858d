// moe_device.cuh -- device building blocks of the W4A8 MoE decode step for
// sm_100a: format conversions, warp/block reductions, and the per-step pieces
// (activation quantiser, router, top-k, union, MXFP4 dot products).
//
// Formats: OCP MX v1.0 (E2M1 element codes, E8M0 block scales, 32 elements per
// block) and OCP OFP8 (E4M3). The step itself is the MXFP4-expert / FP8-
// activation decode described in MarkTechPost, "NVIDIA Shows 3 Ways to Speed
// Up MoE Inference on DGX Spark", sections "Why is MoE decoding on DGX Spark
// memory-bound?" and "What are the 3 optimizations?".
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxTokens = 32;   // M bound per call
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kThreads = 256;    // threads per CTA in every kernel
constexpr int kWarps = kThreads / 32;

// Workspace carved out of one device allocation per context.
struct Workspace {
  unsigned* ctrl;     // [0] status, [1] barrier count, [2] barrier generation,
                      // [3] route ticket, [4] bad-scale counter
  float* logits;      // [maxM][E]
  uint8_t* xq;        // [maxM][H] E4M3 codes
  float* xscale;      // [maxM]
  int* ids;           // [maxM][k]
  float* wts;         // [maxM][k]
  int* meta;          // [0] U (union size), [1] number of (token, slot) pairs
  int* union_ids;     // [min(E, maxM*k)] ascending expert ids
  int* pair_off;      // [min(E, maxM*k) + 1]
  int* pair_tok;      // [maxM*k]
  int* pair_slot;     // [maxM*k]
  float* pair_w;      // [maxM*k]
  float* h;           // [maxM*k][I] SwiGLU output per (token, slot) pair
};

enum : unsigned { kStatusTimeout = 1u };

struct Params {
  int H, I, E, K, M;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  const float* wr;
  const uint8_t* w13c;
  const uint8_t* w13s;
  const uint8_t* w2c;
  const uint8_t* w2s;
  const uint8_t* w2kc;  // split-K down: W2 codes K-major [E][I][H/2] (low nibble = even output row)
  const uint8_t* w2ks;  // split-K down: W2 scales [E][I/32][H]
  Workspace ws;
  int* out_ids;
  float* out_w;
  uint8_t* out_xq;
  float* out_xscale;
  long long spin_limit;  // device-side wait budget in clock64 cycles
  int force_stall;       // test hook: the logits wait targets a tag nobody writes
  int pre_rmsnorm;       // x <- bf16(x * rsqrt(mean(x^2) + eps)) before A1/A2
  unsigned long long* trace;  // test hook: per-CTA phase timestamps (globaltimer), or null
  __nv_bfloat16* out_xn; // optional [M][H] normalised input
  float* y32;            // one part of an intra-expert split: fp32 [M][H] partial sums instead of y
};

// A8's store of output element i: bf16 y, or, for one part of an
// intra-expert split, the fp32 slot-order sum itself (the parts' sums are
// added before the one bf16 round).
__device__ __forceinline__ void store_y(const Params& p, size_t i, float v) {
  if (p.y32)
    p.y32[i] = v;
  else
    p.y[i] = __float2bfloat16_rn(v);
}

// Test hook: lane 0 of the calling warp stores the global timer into stamp
// `slot` of this CTA's row of the trace array (kTraceSlots stamps per CTA).
constexpr int kTraceSlots = 64;
__device__ __forceinline__ void trace_stamp(const Params& p, int slot) {
  if (p.trace && (threadIdx.x & 31) == 0 && slot < kTraceSlots) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    p.trace[(size_t)blockIdx.x * kTraceSlots + slot] = t;
  }
}

// ---------------------------------------------------------------- formats
// E8M0 scale byte -> fp32 2^(b-127) (exact; b = 0 is the subnormal 2^-127).
// 0xFF (NaN) is rejected when the weights are loaded.
__device__ __forceinline__ float e8m0_to_f32(uint32_t b) {
  return __uint_as_float(b ? (b << 23) : 0x00400000u);
}

// Two E2M1 codes in one byte -> f16x2 (bits 3:0 -> low half, 7:4 -> high).
// E2M1 values are exact in f16.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t r;
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;}"
      : "=r"(r) : "r"(byte_in_low8));
  return r;
}

// Four packed E2M1 pairs (one 32-bit word) -> four f16x2.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t out[4]) {
  asm("{.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3]) : "r"(w));
}

// Two E4M3 codes (16 bits, first element in the low byte) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t c2) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c2));
  return r;
}

// fp32 pair -> two E4M3 codes, round-to-nearest-even, saturating to +-448.
// `lo` lands in the low byte (the lower address).
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide max; `red` is shared scratch of >= kWarps floats. All threads get
// the result.
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) r = fmaxf(r, red[i]);
  return r;
}

// ---------------------------------------------------------------- MXFP4 dots
// Dot product of one 32-element MXFP4 block (16 code bytes) with 32 f16
// activations (16 f16x2, element order), without the block scale.
// Products E2M1 x E4M3 are exact in f16 (<= 6 significant bits, |p| <= 2688);
// each of the four f16 partial sums adds 8 products (|sum| <= 21504, no
// overflow); the partials are combined in fp32.
__device__ __forceinline__ float mxfp4_dot32_f16(const uint4 c, const uint4 a[4]) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  const uint32_t* aw = reinterpret_cast<const uint32_t*>(a);
  __half2 acc0 = __float2half2_rn(0.f), acc1 = __float2half2_rn(0.f);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
    e2m1x8_to_f16x2x4(cw[q], w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __half2 wv = *reinterpret_cast<__half2*>(&w[j]);
      __half2 av = *reinterpret_cast<const __half2*>(&aw[q * 4 + j]);
      if (q < 2) acc0 = __hfma2(wv, av, acc0); else acc1 = __hfma2(wv, av, acc1);
    }
  }
  float2 f0 = __half22float2(acc0), f1 = __half22float2(acc1);
  return (f0.x + f0.y) + (f1.x + f1.y);
}

// Dot product of one 32-element MXFP4 block with 32 fp32 values, fp32 FMA,
// without the block scale.
__device__ __forceinline__ float mxfp4_dot32_f32(const uint4 c, const float4* hv) {
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  float acc = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t w[4];
    e2m1x8_to_f16x2x4(cw[q], w);
    float4 h0 = hv[2 * q], h1 = hv[2 * q + 1];
    float2 f0 = __half22float2(*reinterpret_cast<__half2*>(&w[0]));
    float2 f1 = __half22float2(*reinterpret_cast<__half2*>(&w[1]));
    float2 f2 = __half22float2(*reinterpret_cast<__half2*>(&w[2]));
    float2 f3 = __half22float2(*reinterpret_cast<__half2*>(&w[3]));
    acc = fmaf(f0.x, h0.x, acc); acc = fmaf(f0.y, h0.y, acc);
    acc = fmaf(f1.x, h0.z, acc); acc = fmaf(f1.y, h0.w, acc);
    acc = fmaf(f2.x, h1.x, acc); acc = fmaf(f2.y, h1.y, acc);
    acc = fmaf(f3.x, h1.z, acc); acc = fmaf(f3.y, h1.w, acc);
  }
  return acc;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------- A1
// Per-token E4M3 quantisation, one CTA per token: amax = max|x|,
// inv = fl32(448/amax), code = E4M3_rne_sat(fl32(x*inv)), s = fl32(amax/448);
// amax == 0 gives all-zero codes and s = 1.
static __device__ void quantize_token(const Params& p, int m, float* red) {
  const __nv_bfloat16* xm = p.x + (size_t)m * p.H;
  float a = 0.f;
  for (int h = threadIdx.x; h < p.H; h += blockDim.x) a = fmaxf(a, fabsf(__bfloat162float(xm[h])));
  a = block_max(a, red);
  uint16_t* q2 = reinterpret_cast<uint16_t*>(p.ws.xq + (size_t)m * p.H);
  const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(xm);
  if (a == 0.f) {
    for (int i = threadIdx.x; i < p.H / 2; i += blockDim.x) q2[i] = 0;
  } else {
    const float inv = __fdiv_rn(448.f, a);
    for (int i = threadIdx.x; i < p.H / 2; i += blockDim.x) {
      float2 v = __bfloat1622float2(x2[i]);
      q2[i] = f32x2_to_e4m3x2(__fmul_rn(v.x, inv), __fmul_rn(v.y, inv));
    }
  }
  if (threadIdx.x == 0) p.ws.xscale[m] = (a == 0.f) ? 1.f : __fdiv_rn(a, 448.f);
}

// ---------------------------------------------------------------- A2
// One warp computes logits[m][e] for all M tokens of one router row e (fp32
// accumulation of bf16 x times fp32 weights), four tokens per pass.
static __device__ void router_row(const Params& p, int e) {
  const int lane = threadIdx.x & 31;
  const float4* w = reinterpret_cast<const float4*>(p.wr + (size_t)e * p.H);
  const int n4 = p.H / 4;
  for (int m0 = 0; m0 < p.M; m0 += 4) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = lane; i < n4; i += 32) {
      const float4 wv = __ldg(w + i);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (m0 + t < p.M) {
          const uint2 xv = __ldg(reinterpret_cast<const uint2*>(p.x + (size_t)(m0 + t) * p.H) + i);
          float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv.x));
          float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xv.y));
          acc[t] = fmaf(x01.x, wv.x, acc[t]);
          acc[t] = fmaf(x01.y, wv.y, acc[t]);
          acc[t] = fmaf(x23.x, wv.z, acc[t]);
          acc[t] = fmaf(x23.y, wv.w, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float s = warp_sum(acc[t]);
      if (lane == 0 && m0 + t < p.M) p.ws.logits[(size_t)(m0 + t) * p.E + e] = s;
    }
  }
}

// ---------------------------------------------------------------- A3
// One warp: top-k of token m's E logits (ranked by value, ties to the lower
// index) and the softmax over the kept logits. Lane e%32 holds logit e.
// Writes ws.ids/ws.wts (and the optional outputs).
static __device__ void topk_token(const Params& p, int m) {
  const int lane = threadIdx.x & 31;
  const float* l = p.ws.logits + (size_t)m * p.E;
  float v[kMaxExperts / 32];
#pragma unroll
  for (int j = 0; j < kMaxExperts / 32; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < p.E) ? __ldcg(l + e) : 0.f;
  }
  uint32_t taken = 0;
  float sel_v = 0.f, top = 0.f;
  int sel_i = 0;
  for (int r = 0; r < p.K; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane + 32 * j;
      if (e < p.E && !((taken >> j) & 1u) && (v[j] > bv || bi == 0x7fffffff)) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (r == 0) top = bv;
    if (lane == r) {
      sel_v = bv;
      sel_i = bi;
    }
  }
  const float ex = (lane < p.K) ? expf(sel_v - top) : 0.f;
  const float z = warp_sum(ex);
  if (lane < p.K) {
    const float w = ex / z;
    p.ws.ids[m * p.K + lane] = sel_i;
    p.ws.wts[m * p.K + lane] = w;
    if (p.out_ids) p.out_ids[m * p.K + lane] = sel_i;
    if (p.out_w) p.out_w[m * p.K + lane] = w;
  }
}

// ---------------------------------------------------------------- A4
// One CTA: the union of the selected experts (ascending ids) and the
// (token, slot) pairs of each union entry, in (token, slot) order. Reads
// ws.ids / ws.wts written earlier by this CTA (after __syncthreads).
// `cnt` is shared scratch of kMaxExperts ints.
static __device__ void build_union(const Params& p, int* cnt, int* s_u) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int np = p.M * p.K;
  for (int e = tid; e < p.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < np; i += blockDim.x) atomicAdd(&cnt[p.ws.ids[i]], 1);
  __syncthreads();
  if (tid < 32) {
    // each lane scans a contiguous range of experts
    const int per = (p.E + 31) / 32;
    const int e0 = min(p.E, lane * per), e1 = min(p.E, e0 + per);
    int nz = 0, cs = 0;
    for (int e = e0; e < e1; ++e) {
      nz += cnt[e] > 0;
      cs += cnt[e];
    }
    int nz_ex = nz, cs_ex = cs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, nz_ex, o);
      const int b = __shfl_up_sync(0xffffffffu, cs_ex, o);
      if (lane >= o) {
        nz_ex += a;
        cs_ex += b;
      }
    }
    nz_ex -= nz;
    cs_ex -= cs;
    for (int e = e0; e < e1; ++e) {
      const int c = cnt[e];
      if (c > 0) {
        p.ws.union_ids[nz_ex] = e;
        p.ws.pair_off[nz_ex] = cs_ex;
        ++nz_ex;
        cs_ex += c;
      }
      cnt[e] = cs_ex - c;  // start of expert e's pairs (valid where c > 0)
    }
    if (lane == 31) {
      p.ws.pair_off[nz_ex] = cs_ex;
      p.ws.meta[0] = nz_ex;
      p.ws.meta[1] = np;
      *s_u = nz_ex;
    }
  }
  __syncthreads();
  // pair i = (m, slot) goes after the earlier pairs that chose the same expert
  for (int i = tid; i < np; i += blockDim.x) {
    const int e = p.ws.ids[i];
    int before = 0;
    for (int j = 0; j < i; ++j) before += (p.ws.ids[j] == e);
    const int pos = cnt[e] + before;
    p.ws.pair_tok[pos] = i / p.K;
    p.ws.pair_slot[pos] = i % p.K;
    p.ws.pair_w[pos] = p.ws.wts[i];
  }
}

}  // namespace moe
