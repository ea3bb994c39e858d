// moe_lmhead.cuh -- FP8 LM head ("NVIDIA Shows 3 Ways to Speed Up MoE
// Inference on DGX Spark", MarkTechPost, item 2 "Online FP8 LM head": the
// 157,184 x 2,560 BF16 output matrix is quantised to FP8 once at load, which
// halves the bytes every generated token reads).
//
// k_lm_quantize (at load): one warp per output row v: amax = max |w|, then
// E4M3 codes of fl32(w * fl32(448 / amax)) (round to nearest even, saturating)
// and the fp32 row scale fl32(amax / 448); an all-zero row gives zero codes
// and scale 1 -- the activation quantiser's rule applied per row.
//
// k_lm_head (per decode call): logits[m][v] = s_v * sum_h e4m3(W[v][h]) * x[m][h].
// The matrix is read once per call (402 MB at the Ling shape), so the kernel
// streams it: one CTA per SM owns rows [V*b/G, V*(b+1)/G) and TMA-copies them
// in tiles of 16 rows through a shared-memory ring; warp 0, lane 0 issues the
// copies and the other 15 warps take tiles round-robin. A tile is one warp
// MMA chain (mma.sync m16n8k16, f16 in, fp32 accumulate): A = the 16 rows
// (E4M3 -> f16 is exact), B = up to 16 tokens of x in f16, each token scaled
// by a power of two so its largest element stays below 2^15 (exact unless a
// value falls into the f16 subnormal range, 2^-29 below the token's
// maximum). Within each 64-element K block, lane (g, t) supplies elements
// 16t .. 16t+15 of its rows, 4 per MMA step; B uses the same order, so each
// product pairs the same element. The row scale and the token's power of two
// multiply the fp32 sum once at the end.
//
// This file is its own translation unit, with its own few PTX wrappers, so
// that building it does not change how the MoE kernel's translation unit is
// compiled (that kernel runs at the register cap).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <new>

#include "../../include/moe.h"
#include "moe_device.cuh"
#include "moe_host.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t lm_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(lm_smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(lm_smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(lm_smem_u32(bar)) : "memory");
}
// try_wait with a suspend-time hint (the thread is parked until the phase
// completes or the hint expires)
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;}"
      : "=r"(ok) : "r"(lm_smem_u32(bar)), "r"(parity), "r"(20000u) : "memory");
  return ok != 0;
}
// 1-D TMA bulk copy global -> shared; dst, src 16-byte aligned, bytes a
// multiple of 16
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(lm_smem_u32(dst)), "l"(src), "r"(bytes), "r"(lm_smem_u32(bar))
               : "memory");
}
// Four E4M3 codes (one word, first element in the low byte) -> two f16x2
// (exact): elements 0, 1 in lo and 2, 3 in hi.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;}"
      : "=r"(lo), "=r"(hi) : "r"(w));
}
__device__ __forceinline__ unsigned atom_add_acqrel_cta(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(lm_smem_u32(p)), "r"(v) : "memory");
  return old;
}
// D = A(16x16, f16, row) * B(16x8, f16, col) + C, fp32 accumulate
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1,
                                              const float c[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

constexpr int kLmThreads = 512;
constexpr int kLmWarps = kLmThreads / 32;
constexpr int kLmTileRows = 16;
constexpr int kLmMaxSlots = 8;
constexpr int kLmMaxTokens = 16;
constexpr int kLmParts = 3;  // warps (K parts) per tile

struct LmParams {
  const uint8_t* codes;  // [V][H] E4M3
  const float* scales;   // [V]
  const __nv_bfloat16* x;  // [M][H]
  float* logits;         // [M][V]
  unsigned* status;      // status word (bit kStatusTimeout)
  long long spin_limit;  // wait budget in clock64 cycles
  int V, H, M;
  int ns;                // ring slots
  int o_bar, o_misc, o_x, o_part, o_ring;  // shared-memory offsets
};

// Bounded waits that report to a plain status word (the LM head has no
// MoE workspace): on timeout they set kStatusTimeout and return.
__device__ __forceinline__ void mbar_wait_status(uint64_t* bar, unsigned parity, long long limit, unsigned* status) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void smem_count_wait_status(const unsigned* c, unsigned target, long long limit,
                                                       unsigned* status) {
  const volatile unsigned* v = c;
  if (*v >= target) return;
  const long long t0 = clock64();
  while (*v < target) {
    __nanosleep(32);
    if (clock64() - t0 > limit) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

// ---------------------------------------------------------------- load time
__global__ void __launch_bounds__(256) k_lm_quantize(const __nv_bfloat16* __restrict__ w, int V, int H,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int v = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; v < V; v += warps) {
    const __nv_bfloat162* row = reinterpret_cast<const __nv_bfloat162*>(w + (size_t)v * H);
    float a = 0.f;
    for (int i = lane; i < H / 2; i += 32) {
      const float2 f = __bfloat1622float2(row[i]);
      a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    a = warp_max(a);
    uint16_t* out = reinterpret_cast<uint16_t*>(codes + (size_t)v * H);
    if (a == 0.f) {
      for (int i = lane; i < H / 2; i += 32) out[i] = 0;
      if (lane == 0) scales[v] = 1.f;
      continue;
    }
    const float inv = __fdiv_rn(448.f, a);
    for (int i = lane; i < H / 2; i += 32) {
      const float2 f = __bfloat1622float2(row[i]);
      out[i] = f32x2_to_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
    }
    if (lane == 0) scales[v] = __fdiv_rn(a, 448.f);
  }
}

// ---------------------------------------------------------------- decode
__global__ void __launch_bounds__(kLmThreads, 1) k_lm_head(LmParams q) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x, G = gridDim.x;
  const int H = q.H, M = q.M, ns = q.ns;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + q.o_bar);
  uint64_t* empty = full + kLmMaxSlots;
  unsigned* done = reinterpret_cast<unsigned*>(empty + kLmMaxSlots);  // tiles finished per slot (all uses)
  float* s_down = reinterpret_cast<float*>(smem + q.o_misc);          // [M] 2^-t per token
  int* s_exp = reinterpret_cast<int*>(s_down + kLmMaxTokens);          // [M] t per token
  __half* x16 = reinterpret_cast<__half*>(smem + q.o_x);               // [M][H]
  uint8_t* ring = smem + q.o_ring;
  const size_t tile_bytes = (size_t)kLmTileRows * H;

  const int v0 = (int)((long long)q.V * b / G), v1 = (int)((long long)q.V * (b + 1) / G);
  const int nt = (v1 - v0 + kLmTileRows - 1) / kLmTileRows;
  auto issue = [&](int i) {
    const int slot = i % ns;
    const int r0 = v0 + i * kLmTileRows, nr = min(kLmTileRows, v1 - r0);
    const unsigned bytes = (unsigned)(nr * H);
    mbar_expect_tx(full + slot, bytes);
    tma_load_1d(ring + slot * tile_bytes, q.codes + (size_t)r0 * H, bytes, full + slot);
  };
  if (tid < kLmMaxSlots) {
    mbar_init(full + tid, 1);
    mbar_init(empty + tid, 1);
    done[tid] = 0u;
    done[kLmMaxSlots + tid] = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  // start the stream before converting x, so the first copies overlap it
  if (tid == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    for (int i = 0; i < min(ns, nt); ++i) issue(i);
  }
  // per-token power of two: max |x| * 2^t below 2^15 (f16 range)
  for (int m = warp; m < M; m += kLmWarps) {
    const __nv_bfloat162* xr = reinterpret_cast<const __nv_bfloat162*>(q.x + (size_t)m * H);
    float a = 0.f;
    for (int i = lane; i < H / 2; i += 32) {
      const float2 f = __bfloat1622float2(xr[i]);
      a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    a = warp_max(a);
    if (lane == 0) {
      int e = 0;
      if (a > 0.f) frexpf(a, &e);  // a in [2^(e-1), 2^e)
      const int t = min(126, 15 - e);
      s_exp[m] = t;
      s_down[m] = ldexpf(1.f, -t);
    }
  }
  __syncthreads();
  for (int i = tid; i < M * H / 8; i += kLmThreads) {
    const int m = (i * 8) / H;
    const float up = ldexpf(1.f, s_exp[m]);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(q.x) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      const __half2 h = __floats2half2_rn(f.x * up, f.y * up);
      o[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(x16)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  __syncthreads();

  if (warp == 0) {
    // producer: refill each slot once its previous tile is consumed
    if (lane == 0) {
      for (int i = ns; i < nt; ++i) {
        const int slot = i % ns, use = i / ns;
        mbar_wait_status(empty + slot, (use - 1) & 1, q.spin_limit, q.status);
        issue(i);
      }
    }
    return;
  }

  const int g = lane >> 2, t = lane & 3;
  const int ntok = (M + 7) >> 3;
  const __half* xr0 = (g < M) ? x16 + (size_t)g * H + 16 * t : nullptr;
  const __half* xr1 = (g + 8 < M) ? x16 + (size_t)(g + 8) * H + 16 * t : nullptr;
  // items (tile i, K part p): kLmParts warps share a tile, each taking a
  // third of its K range, so every consumer warp has work while a slot fills
  const int nkb = H / 64;
  float4* part = reinterpret_cast<float4*>(smem + q.o_part);  // [ns][kLmParts][2][32]
  unsigned* pcnt = done + kLmMaxSlots;                          // parts finished per slot (all uses)
  for (int it = warp - 1; it < nt * kLmParts; it += kLmWarps - 1) {
    const int i = it / kLmParts, pk = it - i * kLmParts;
    const int slot = i % ns, use = i / ns;
    // every earlier use of the slot is finished, so the parity wait below
    // refers to this use (never to one two phases back)
    if (use > 0 && lane == 0) smem_count_wait_status(done + slot, (unsigned)use, q.spin_limit, q.status);
    __syncwarp();
    mbar_wait_status(full + slot, use & 1, q.spin_limit, q.status);
    const uint8_t* tile = ring + slot * tile_bytes;
    const uint8_t* ar0 = tile + (size_t)g * H + 16 * t;
    const uint8_t* ar1 = tile + (size_t)(g + 8) * H + 16 * t;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int kb0 = pk * nkb / kLmParts, kb1 = (pk + 1) * nkb / kLmParts;
#pragma unroll 2
    for (int kb = kb0; kb < kb1; ++kb) {
      const uint4 c0 = *reinterpret_cast<const uint4*>(ar0 + kb * 64);
      const uint4 c1 = *reinterpret_cast<const uint4*>(ar1 + kb * 64);
      const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w}, w1[4] = {c1.x, c1.y, c1.z, c1.w};
      uint32_t fa[8], fb[8];  // rows g, g+8: f16x2 of byte pairs 0..7
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        e4m3x4_to_f16x2x2(w0[k], fa[2 * k], fa[2 * k + 1]);
        e4m3x4_to_f16x2x2(w1[k], fb[2 * k], fb[2 * k + 1]);
      }
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        if (n >= ntok) break;
        const __half* xr = (n == 0) ? xr0 : xr1;
        uint4 bx0 = make_uint4(0u, 0u, 0u, 0u), bx1 = bx0;
        if (xr) {
          bx0 = *reinterpret_cast<const uint4*>(xr + kb * 64);
          bx1 = *reinterpret_cast<const uint4*>(xr + kb * 64 + 8);
        }
        const uint32_t bb[8] = {bx0.x, bx0.y, bx0.z, bx0.w, bx1.x, bx1.y, bx1.z, bx1.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t a[4] = {fa[2 * j], fb[2 * j], fa[2 * j + 1], fb[2 * j + 1]};
          mma_f16_16816(acc[n], a, bb[2 * j], bb[2 * j + 1], acc[n]);
        }
      }
    }
    // publish this part; the warp that finishes the tile's last part sums
    // the parts in order (deterministic) and writes the logits
    float4* pp = part + ((size_t)slot * kLmParts + pk) * 64;
#pragma unroll
    for (int n = 0; n < 2; ++n)
      if (n < ntok) pp[n * 32 + lane] = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
    __syncwarp();
    unsigned cnt = 0;
    if (lane == 0) cnt = atom_add_acqrel_cta(pcnt + slot, 1u) + 1u;
    cnt = __shfl_sync(0xffffffffu, cnt, 0);
    if (cnt != (unsigned)(kLmParts * (use + 1))) continue;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      if (n >= ntok) break;
      float4 sum = part[((size_t)slot * kLmParts) * 64 + n * 32 + lane];
      for (int k = 1; k < kLmParts; ++k) {
        const float4 v = part[((size_t)slot * kLmParts + k) * 64 + n * 32 + lane];
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      acc[n][0] = sum.x; acc[n][1] = sum.y; acc[n][2] = sum.z; acc[n][3] = sum.w;
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(empty + slot);
      atomicAdd(done + slot, 1u);
    }
    // lane (g, t) holds rows g and g+8 for tokens 8n + 2t, 8n + 2t + 1
    const int r0 = v0 + i * kLmTileRows, nr = min(kLmTileRows, v1 - r0);
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      if (n >= ntok) break;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = g + 8 * (k >> 1), m = 8 * n + 2 * t + (k & 1);
        if (row < nr && m < M)
          q.logits[(size_t)m * q.V + r0 + row] = acc[n][k] * q.scales[r0 + row] * s_down[m];
      }
    }
  }
}

}  // namespace
}  // namespace moe

using moe_host::aligned16;
using moe_host::align_up;
using moe_host::DeviceGuard;
using moe_host::kDefaultSpinLimit;

struct moe_lm {
  int dev = 0;
  int V = 0, H = 0, max_tokens = 0;
  int sm_count = 0;
  uint8_t* codes = nullptr;  // [V][H] E4M3 (owned)
  float* scales = nullptr;   // [V] (owned)
  unsigned* status = nullptr;
  bool loaded = false;
  int ns = 0;
  size_t smem = 0;
  int o_bar = 0, o_misc = 0, o_x = 0, o_part = 0, o_ring = 0;
  long long spin_limit = kDefaultSpinLimit;
};

namespace {

// Shared-memory plan of k_lm_head: barriers and done counts, per-token
// scales, the f16 activations, then as many 16-row tiles as fit (2..8).
bool lm_plan(int H, int max_tokens, size_t smem_limit, int* ns, size_t* smem, int* o_bar, int* o_misc, int* o_x,
             int* o_part, int* o_ring) {
  size_t off = 0;
  auto take = [&](size_t bytes, size_t a) { off = align_up(off, a); size_t o = off; off += bytes; return o; };
  *o_bar = (int)take(2 * moe::kLmMaxSlots * 8 + 2 * moe::kLmMaxSlots * 4, 16);
  *o_misc = (int)take(2 * moe::kLmMaxTokens * 4, 16);
  *o_x = (int)take((size_t)max_tokens * H * 2, 128);
  off = align_up(off, 128);
  // per slot: the tile, and the K parts' partial sums (2 token tiles x 32 lanes x float4)
  const size_t tile = (size_t)moe::kLmTileRows * H;
  const size_t parts = (size_t)moe::kLmParts * 2 * 32 * 16;
  if (off + 2 * (tile + parts) > smem_limit) return false;
  *ns = (int)std::min<size_t>(moe::kLmMaxSlots, (smem_limit - off) / (tile + parts));
  *o_part = (int)off;
  off = align_up(off + (size_t)*ns * parts, 128);
  *o_ring = (int)off;
  *smem = off + (size_t)*ns * tile;
  return *smem <= smem_limit;
}

}  // namespace

extern "C" {

moe_status moe_lm_create(int32_t vocab, int32_t hidden, int32_t max_tokens, int32_t device, moe_lm** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  if (vocab < 1 || hidden < 64 || hidden > 8192 || hidden % 64 || max_tokens < 1 ||
      max_tokens > moe::kLmMaxTokens || (long long)vocab * hidden > (1LL << 40))
    return MOE_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return MOE_ERR_CUDA;
  if (device < 0 || device >= ndev) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(device);
  if (!guard.ok) return MOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
  moe_lm* lm = new (std::nothrow) moe_lm();
  if (!lm) return MOE_ERR_OOM;
  lm->dev = device;
  lm->V = vocab;
  lm->H = hidden;
  lm->max_tokens = max_tokens;
  lm->sm_count = prop.multiProcessorCount;
  if (!lm_plan(hidden, max_tokens, prop.sharedMemPerBlockOptin, &lm->ns, &lm->smem, &lm->o_bar, &lm->o_misc,
               &lm->o_x, &lm->o_part, &lm->o_ring) ||
      // the limit is per device and process: raise it to the opt-in maximum,
      // never to this context's (possibly smaller) plan
      cudaFuncSetAttribute(moe::k_lm_head, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)prop.sharedMemPerBlockOptin) != cudaSuccess) {
    cudaGetLastError();
    delete lm;
    return MOE_ERR_UNSUPPORTED;
  }
  const size_t cb = (size_t)vocab * hidden;
  if (cudaMalloc(&lm->codes, cb) != cudaSuccess || cudaMalloc(&lm->scales, (size_t)vocab * 4) != cudaSuccess ||
      cudaMalloc(&lm->status, 64) != cudaSuccess || cudaMemset(lm->status, 0, 64) != cudaSuccess) {
    cudaGetLastError();
    if (lm->codes) cudaFree(lm->codes);
    if (lm->scales) cudaFree(lm->scales);
    if (lm->status) cudaFree(lm->status);
    delete lm;
    return MOE_ERR_OOM;
  }
  *out = lm;
  return MOE_OK;
}

void moe_lm_destroy(moe_lm* lm) {
  if (!lm) return;
  DeviceGuard guard(lm->dev);
  if (lm->codes) cudaFree(lm->codes);
  if (lm->scales) cudaFree(lm->scales);
  if (lm->status) cudaFree(lm->status);
  delete lm;
}

moe_status moe_lm_load(moe_lm* lm, const void* w_bf16) {
  if (!lm || !w_bf16 || !aligned16(w_bf16)) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(lm->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  lm->loaded = false;
  const int rows_per_block = 256 / 32;
  const int blocks = (int)std::min<long long>((lm->V + rows_per_block - 1) / rows_per_block, lm->sm_count * 16LL);
  moe::k_lm_quantize<<<blocks, 256>>>(static_cast<const __nv_bfloat16*>(w_bf16), lm->V, lm->H, lm->codes,
                                       lm->scales);
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  lm->loaded = true;
  return MOE_OK;
}

moe_status moe_lm_read_weights(const moe_lm* lm, uint8_t* codes, float* scales, void* stream) {
  if (!lm || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (!lm->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard guard(lm->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(codes, lm->codes, (size_t)lm->V * lm->H, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(scales, lm->scales, (size_t)lm->V * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status moe_lm_head(moe_lm* lm, const void* x_bf16, int32_t M, float* logits, void* stream) {
  if (!lm) return MOE_ERR_INVALID_ARG;
  if (M < 0 || M > lm->max_tokens) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  if (!x_bf16 || !logits || !aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(logits) & 3)) return MOE_ERR_INVALID_ARG;
  const char* xb = static_cast<const char*>(x_bf16);
  const char* lb = reinterpret_cast<const char*>(logits);
  const size_t xbytes = (size_t)M * lm->H * 2, lbytes = (size_t)M * lm->V * 4;
  if (xb < lb + lbytes && lb < xb + xbytes) return MOE_ERR_INVALID_ARG;  // aliasing
  if (!lm->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard guard(lm->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  moe::LmParams q{};
  q.codes = lm->codes;
  q.scales = lm->scales;
  q.x = static_cast<const __nv_bfloat16*>(x_bf16);
  q.logits = logits;
  q.status = lm->status;
  q.spin_limit = lm->spin_limit;
  q.V = lm->V;
  q.H = lm->H;
  q.M = M;
  q.ns = lm->ns;
  q.o_bar = lm->o_bar;
  q.o_misc = lm->o_misc;
  q.o_x = lm->o_x;
  q.o_part = lm->o_part;
  q.o_ring = lm->o_ring;
  moe::k_lm_head<<<lm->sm_count, moe::kLmThreads, lm->smem, static_cast<cudaStream_t>(stream)>>>(q);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_lm_sync_status(moe_lm* lm, void* stream) {
  if (!lm) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(lm->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned st = 0;
  if (cudaMemcpy(&st, lm->status, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (st == 0) return MOE_OK;
  if (cudaMemset(lm->status, 0, 64) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_ERR_TIMEOUT;
}

moe_status moe_lm_query(const moe_lm* lm, char* buf, size_t len) {
  if (!lm || !buf || len == 0) return MOE_ERR_INVALID_ARG;
  const int n = snprintf(buf, len,
                         "{\"arch\": \"sm_100a\", \"kernel\": \"k_lm_head\", \"vocab\": %d, \"hidden\": %d, "
                         "\"max_tokens\": %d, \"grid\": %d, \"threads\": %d, \"smem\": %zu, \"slots\": %d, "
                         "\"tile_rows\": %d, \"weights\": \"e4m3 + fp32 row scale\", \"loaded\": %s}",
                         lm->V, lm->H, lm->max_tokens, lm->sm_count, moe::kLmThreads, lm->smem, lm->ns,
                         moe::kLmTileRows, lm->loaded ? "true" : "false");
  if (n < 0 || (size_t)n >= len) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // extern "C"
