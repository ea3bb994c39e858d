// moe_split.cuh -- the decode step as three kernels (route, gate/up, down).
//
// This is the plain, launch-per-phase form of the step. It is kept beside the
// persistent kernel as a second path that the tests compare against, and it
// is selected with MOE_FLAG_SPLIT_KERNELS. The kernels have internal linkage:
// each translation unit that launches them gets its own copy.
//   k_route   quantise (A1), router logits (A2); the last CTA to finish does
//             top-k (A3) and the union (A4)
//   k_gateup  gate/up GEMV with in-register MXFP4 decode (A5) and SwiGLU (A6)
//   k_down    down GEMV (A7) and the routing-weighted combine (A8)
#pragma once

#include "moe_device.cuh"

namespace moe {

static __global__ void __launch_bounds__(kThreads) k_route(Params p) {
  __shared__ float red[kWarps];
  __shared__ int s_last, s_u;
  __shared__ int cnt[kMaxExperts];
  const int b = blockIdx.x, G = gridDim.x, warp = threadIdx.x >> 5;
  for (int m = b; m < p.M; m += G) quantize_token(p, m, red);
  const int e0 = (int)((long long)p.E * b / G), e1 = (int)((long long)p.E * (b + 1) / G);
  for (int e = e0 + warp; e < e1; e += kWarps) router_row(p, e);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&p.ws.ctrl[3], 1u) == (unsigned)(G - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int m = warp; m < p.M; m += kWarps) topk_token(p, m);
  __syncthreads();
  build_union(p, cnt, &s_u);
  if (p.out_xq || p.out_xscale) {
    for (int i = threadIdx.x; i < p.M * p.H; i += blockDim.x)
      if (p.out_xq) p.out_xq[i] = __ldcg(p.ws.xq + i);
    for (int m = threadIdx.x; m < p.M; m += blockDim.x)
      if (p.out_xscale) p.out_xscale[m] = __ldcg(p.ws.xscale + m);
  }
  if (threadIdx.x == 0) p.ws.ctrl[3] = 0;
}

// Gate/up: one warp per unit (union entry u, intermediate row n), reading the
// gate row n and the up row I+n of expert union_ids[u]; for each (token, slot)
// pair routed to the expert, h = silu(s*<gate,q>) * s*<up,q>.
// Activations are decoded once per CTA into shared memory as f16.
static __global__ void __launch_bounds__(kThreads) k_gateup(Params p) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t* act2 = reinterpret_cast<uint32_t*>(smem);  // [M][H/2] f16x2
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I;
  const uint16_t* xq2 = reinterpret_cast<const uint16_t*>(p.ws.xq);
  for (int i = tid; i < p.M * H / 2; i += blockDim.x) act2[i] = e4m3x2_to_f16x2(__ldcg(xq2 + i));
  __syncthreads();
  const int U = __ldcg(p.ws.meta);
  const long long T = (long long)U * I;
  const int gw = blockIdx.x * kWarps + warp, GW = gridDim.x * kWarps;
  const long long j0 = T * gw / GW, j1 = T * (gw + 1) / GW;
  const int nblk = H / 32;
  for (long long j = j0; j < j1; ++j) {
    const int u = (int)(j / I), n = (int)(j % I);
    const int e = __ldcg(p.ws.union_ids + u);
    const size_t grow = (size_t)e * 2 * I + n, urow = grow + I;
    const uint8_t* gc = p.w13c + grow * (H / 2);
    const uint8_t* uc = p.w13c + urow * (H / 2);
    const uint8_t* gs = p.w13s + grow * (H / 32);
    const uint8_t* us = p.w13s + urow * (H / 32);
    const int pb = __ldcg(p.ws.pair_off + u), pe = __ldcg(p.ws.pair_off + u + 1);
    for (int pp = pb; pp < pe; ++pp) {
      const int m = __ldcg(p.ws.pair_tok + pp);
      const uint4* am = reinterpret_cast<const uint4*>(act2 + (size_t)m * (H / 2));
      float ag = 0.f, au = 0.f;
      for (int blk = lane; blk < nblk; blk += 32) {
        const uint4 cg = ldg_stream(gc + (size_t)blk * 16);
        const uint4 cu = ldg_stream(uc + (size_t)blk * 16);
        const float sg = e8m0_to_f32(__ldg(gs + blk)), su = e8m0_to_f32(__ldg(us + blk));
        uint4 a[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) a[t] = am[blk * 4 + t];
        ag = fmaf(sg, mxfp4_dot32_f16(cg, a), ag);
        au = fmaf(su, mxfp4_dot32_f16(cu, a), au);
      }
      ag = warp_sum(ag);
      au = warp_sum(au);
      if (lane == 0) {
        const float s = __ldcg(p.ws.xscale + m);
        const float g = ag * s, up = au * s;
        p.ws.h[(size_t)pp * I + n] = g / (1.f + expf(-g)) * up;
      }
    }
  }
}

// Down + combine: one warp per output row r. For each union expert and each
// of its (token, slot) pairs, d = <W2[e][r], h_pair> is kept per (token,
// slot); then y[m][r] sums w * d over the token's slots in slot order (the
// order of the top-k, highest logit first), deterministic and without
// atomics, the same order the persistent kernel uses.
static __global__ void __launch_bounds__(kThreads) k_down(Params p) {
  __shared__ float dslot[kWarps][kMaxTokens * kMaxTopK];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I, K = p.K, nblk = I / 32;
  const int U = __ldcg(p.ws.meta);
  const int gw = blockIdx.x * kWarps + warp, GW = gridDim.x * kWarps;
  const int r0 = (int)((long long)H * gw / GW), r1 = (int)((long long)H * (gw + 1) / GW);
  for (int r = r0; r < r1; ++r) {
    for (int u = 0; u < U; ++u) {
      const int e = __ldcg(p.ws.union_ids + u);
      const size_t row = (size_t)e * H + r;
      const uint8_t* dc = p.w2c + row * (I / 2);
      const uint8_t* ds = p.w2s + row * (I / 32);
      const int pb = __ldcg(p.ws.pair_off + u), pe = __ldcg(p.ws.pair_off + u + 1);
      for (int pp = pb; pp < pe; ++pp) {
        const float4* hp = reinterpret_cast<const float4*>(p.ws.h + (size_t)pp * I);
        float acc = 0.f;
        for (int blk = lane; blk < nblk; blk += 32) {
          const uint4 c = ldg_stream(dc + (size_t)blk * 16);
          const float sc = e8m0_to_f32(__ldg(ds + blk));
          float4 hv[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) hv[t] = __ldcg(hp + blk * 8 + t);
          acc = fmaf(sc, mxfp4_dot32_f32(c, hv), acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) dslot[warp][__ldcg(p.ws.pair_tok + pp) * K + __ldcg(p.ws.pair_slot + pp)] = acc;
      }
    }
    __syncwarp();
    if (lane < p.M) {
      float y = 0.f;
      for (int s = 0; s < K; ++s) y = fmaf(__ldcg(p.ws.wts + lane * K + s), dslot[warp][lane * K + s], y);
      store_y(p, (size_t)lane * H + r, y);
    }
    __syncwarp();
  }
}

// Scan scale bytes for the E8M0 NaN encoding (0xFF); counts into *bad.
static __global__ void k_scan_scales(const uint8_t* s, size_t n, unsigned* bad) {
  unsigned c = 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    c += (s[i] == 0xFF);
  c = __reduce_add_sync(0xffffffffu, c);
  if ((threadIdx.x & 31) == 0 && c) atomicAdd(bad, c);
}

}  // namespace moe
