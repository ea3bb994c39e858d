// moe_tc.cuh -- the decode step as one persistent kernel whose gate/up and
// (from MOE_TC_DOWN_MMA_MIN_TOKENS tokens) down projections run on the
// tensor cores (tcgen05 block-scaled MMA).
//
// The step streams the active experts' MXFP4 weights from HBM once (MarkTechPost,
// "NVIDIA Shows 3 Ways to Speed Up MoE Inference on DGX Spark", section "Why is
// MoE decoding on DGX Spark memory-bound?"). Gate/up is two thirds of those
// bytes, and decoding E2M1 in registers caps CUDA cores near 40 weight
// elements per SM clock. The block-scaled MMA
// (tcgen05.mma.kind::mxf8f6f4.block_scale: E2M1 weights with E8M0 scales per
// 32 elements times E4M3 activations, fp32 accumulate in tensor memory) takes
// the weights as they are; one M=128 x K=32 MMA costs about 48 cycles for up
// to 32 tokens, about 85 weights per cycle per SM even at one token.
//
// One CTA per SM, 512 threads.
//  1. Before griddepcontrol.wait: tensor memory, barriers, and a TMA copy of
//     the CTA's router rows (the previous kernel never writes them).
//  2. Routing, all warps: x is staged, each CTA computes its router rows'
//     logits and stores each as one 64-bit word (launch epoch in the high half,
//     the fp32 value in the low half). Every CTA then reads all M*E words and
//     retries those whose epoch is stale: the data is its own flag, so no
//     barrier or fence round trip is needed. The E4M3 activation codes are
//     written straight into the MMA's B operand while the logits arrive. Top-k
//     (ties to the lower index), softmax, and the expert union follow.
//  3. Gate/up: the union's gate/up rows form one flat list of 8-row units
//     (4 gate rows and the 4 up rows of the same intermediate indices), entry
//     by entry. It is cut into tiles of at most 16 units (one M=128 MMA tile),
//     dealt round robin to the CTAs, so all CTAs stream about the same bytes.
//     Warp 0 loads each tile in stages of ks K-chunks (128 elements) with TMA
//     tensor copies that unpack the 4-bit codes to the MMA's padded layout
//     (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 128-byte swizzle), one copy per
//     run of units of the same expert, straight from the caller's row-major
//     [E][2I][H/2] array (a 5-D map whose strides select 4 gate rows, the 4 up
//     rows I rows further on, and the K-chunk). The tile's E8M0 scales come
//     first; warps 4..7 write them into tensor memory in the MMA's
//     scale-factor layout (tcgen05.st, once per tile). Warp 1 only issues the
//     MMAs (one thread, descriptors advanced by adds), B = the E4M3 codes of
//     every token. Warps 4..7 then read the accumulators
//     (tcgen05.ld), apply the per-token scale and SwiGLU, and store h of each
//     (token, slot) pair routed to the unit's expert to L2.
//     After its stores each epilogue warp adds one (release, GPU scope) to a
//     counter of every entry the tile touches; one gatekeeper thread per CTA
//     polls those counters in entry order and raises a shared-memory flag
//     per entry once its h is complete on every CTA.
//  4. Down on the tensor cores (the default from MOE_TC_DOWN_MMA_MIN_TOKENS
//     tokens of max_tokens): down tiles (entry, group of up to 16 pairs, 128
//     output rows) follow each CTA's gate/up tiles in the same pipeline. Warp
//     0 loads the tile's W2 codes (a 2-D tensor map, 128 rows x 128-element
//     K-chunks) and scales; warps 8..15 build the B operand once the entry's
//     flag is up: per pair an fp32 scale and the E4M3 codes of h/scale and of
//     16x its rounding residual, so the MMA sums hi + lo/16 (within 2^-8 of
//     h). The epilogue applies the pair scales and writes each pair's 128
//     outputs to L2; every CTA then arrives on a grid count (by launch
//     parity), waits for all CTAs, and combines its rows from the per-pair
//     outputs.
//     Down on CUDA cores (below that, or forced): each CTA owns output rows
//     [H*b/G, H*(b+1)/G) of every union expert, streamed by warp 2 into a
//     ring of 1-D TMA copies; consumer warps take down items in entry order,
//     each waiting for its entry's flag, and stage h once as f16 (rescaled by
//     a power of two per pair).
//  5. Each CTA combines its rows in slot order and writes bf16 y (fp32
//     partial sums for one part of an intra-expert split).
// Every wait is bounded: a wait that runs out sets the status word and the
// kernel finishes (with garbage output) instead of hanging.
#pragma once

#include <cuda.h>

#include "moe_fused.cuh"

namespace moe {

constexpr int kTcThreads = 512;
constexpr int kTcWarps = kTcThreads / 32;
constexpr int kTcMaxUnits = 16;   // 8-row units per gate/up tile: M = 128 MMA rows
constexpr int kTcMaxSlots = 16;   // gate/up ring slots
constexpr int kTcAccCols = 32;    // one gate/up accumulator: up to 32 tokens
constexpr int kTcSfCol = 64;      // first scale-factor column (two tile buffers of 4 columns per K-chunk)
// warp roles once routing is done
constexpr int kTcWarpProdGu = 0;  // gate/up TMA
constexpr int kTcWarpMma = 1;     // MMA issue
constexpr int kTcWarpProdD = 2;   // down TMA
constexpr int kTcWarpEpi = 4;     // warps 4..7: gate/up epilogue (tensor-memory lane quarters 0..3)

struct TcPlan {
  int G;
  int ks;        // K-chunks of 128 elements per gate/up stage
  int tu_max;    // units per gate/up tile
  int nb_max;    // MMA N: tokens rounded up to a multiple of 8
  int ns_gu, slot_gu;
  int ns_d, slot_d;
  int rpc_max, hslot, hpairs;
  int max_pairs, max_union;
  int wr_bytes_max;
  int x_staged;  // bf16 x fits in the down ring during routing
  int o_lg;      // gathered logits [maxM][E] fp32, then [E] union scratch (routing only)
  int o_hready;  // [max_union] entry's h complete on every CTA (set by the gatekeeper warp)
  int lg_own;    // o_lg is a region of its own (not in either ring)
  // shared-memory offsets from the 1024-aligned base
  int o_ring_gu, o_bx, o_sf, o_sc, o_ring_d, o_h, o_bar, o_misc, o_ids, o_w, o_pm, o_ppos, o_union, o_poff, o_dsm,
      o_sfb;
  int sc_bytes;  // one tile's scale buffer
  int tmem_cols; // tensor-memory columns allocated (power of two)
  int bx_bytes;
  int smem_bytes;  // including 1 KB of alignment slack
  // tensor-core down projection (mma_down): tiles of 128 output rows x up to
  // kTcDownPairs pairs of one entry; W2 stages share the gate/up ring (16 KB
  // slots), h of the pairs is the B operand (E4M3, two buffers)
  int mma_down;
  int dkch;      // K-chunks of the down projection (I / 128)
  int o_bd;      // [2][dkch][4][8][128 B] B operand buffers
  int bd_bytes;  // one buffer
  int o_dsc;     // [2][kTcDownPairs] per-pair h scales
  int o_dtoff;   // [max_union + 1] first down tile of each entry
};

constexpr int kTcXU2 = 20;     // 4-element groups of a token's x a lane holds when M >= 2 (H <= 2560: one read)
constexpr int kTcCntStride = 32;  // u32 words between per-entry counters (one 128-byte line each)
constexpr int kTcMaxTiles = 64;   // gate/up tiles per CTA
constexpr int kTcWarpGate = 3;    // polls the entry counters for the CTA
constexpr int kTcDownPairs = 16;  // pairs per tensor-core down tile: N = 2 x pairs (h = hi + lo/16)
constexpr int kTcWarpBuild = 8;   // warps 8..15 build the down tiles' B operands

// The gate/up code maps, passed by value as a __grid_constant__ kernel
// parameter (TMA reads its descriptor from parameter space).
struct TcMaps {
  CUtensorMap m[kTcMaxUnits];  // map n-1 loads n units x ks K-chunks
  CUtensorMap w2;              // down codes [Eall*H rows][I] 4-bit: 128 rows x one 128-element K-chunk
};

struct TcWs {
  int repacked;                // gate/up codes in the private [E][I/4][H/128][8][64 B] layout (4-D maps)
  unsigned long long* logits;  // [maxM][E]  epoch << 32 | fp32 bits
  float* h;                    // [pairs][I] SwiGLU output per (token, slot) pair
  unsigned* hcnt;              // [2][max_union * kTcCntStride] gate/up tiles done per entry, by launch parity
  unsigned* epoch;             // launch counter
  float* ypart;                // [pairs][H] tensor-core down: each pair's down output (fp32)
  unsigned* dcnt;              // [2][kTcCntStride] CTAs done with their down tiles, by launch parity
};

__device__ __forceinline__ void tc_trace(const Params& p, int slot) { trace_stamp(p, slot); }
// An 8-byte L2 load the compiler may not repeat (asm volatile): a row loaded
// once stays in registers instead of being re-read from L2.
__device__ __forceinline__ uint2 ld_cg_v2_once(const uint2* p) {
  uint2 v;
  asm volatile("ld.global.cg.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ unsigned ld_acquire_u32g(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u32(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// try_wait without a suspend-time hint: the hardware's own short limit, so a
// waiter on the stream's critical path resumes as soon as the phase completes.
__device__ __forceinline__ bool mbar_try_wait_fast(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase; false (and the status word set) if the
// wait ran out.
__device__ __forceinline__ bool mbar_wait_ok(uint64_t* bar, unsigned parity, const Params& p) {
  if (mbar_try_wait_fast(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_fast(bar, parity)) {
    if (clock64() - t0 > p.spin_limit) {
      atomicOr(p.ws.ctrl, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// Warp-uniform form: lane 0 waits, every lane gets the outcome (warps that
// run .sync.aligned instructions after the wait must not diverge on it).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, unsigned parity, const Params& p) {
  bool r = true;
  if ((threadIdx.x & 31) == 0) r = mbar_wait_ok(bar, parity, p);
  return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
}

// ---------------------------------------------------------------- tcgen05 / TMA wrappers
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major with 128-byte swizzle: 8-row x
// 128-byte atoms (1024 bytes, 1024-aligned), `sbo` bytes between the atoms of
// consecutive 8-row groups; the start moves 32 bytes per 32-element K block
// inside an atom. Version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;  // leading byte offset: unused for swizzled K-major
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}
// Descriptor of a 512-byte scale-factor block for tcgen05.cp.32x128b.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((128u >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}
// Instruction descriptor, kind::mxf8f6f4 block-scaled: A = E2M1 (weights), B
// = E4M3 (tokens), both K-major, fp32 accumulate, M = 128, E8M0 scales;
// sf_id selects the scale byte (K block 0..3 of a 4-block scale word).
__device__ __forceinline__ uint32_t umma_idesc_mx(int n, int sf_id) {
  return ((uint32_t)(sf_id & 3) << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) |
         ((uint32_t)(128 >> 4) << 24) | ((uint32_t)(sf_id & 3) << 29);
}
__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc,
                                        uint32_t sfa_tmem, uint32_t sfb_tmem) {
  asm volatile(
      "{.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa_tmem), "r"(sfb_tmem));
}
__device__ __forceinline__ void tc_cp_sf(uint32_t tmem, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(sdesc));
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// One warp reads 32 tensor-memory lanes (its quarter) x 32 columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t v[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3, int c4,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
      "%6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_v2(const unsigned long long* p, unsigned long long* b) {
  unsigned long long a;
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(*b) : "l"(p) : "memory");
  return a;
}
__device__ __forceinline__ void st_relaxed_v2(unsigned long long* p, unsigned long long a, unsigned long long b) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

// Byte offset of K element k of row r in a K-major 128-byte-swizzled operand
// laid out as [K-chunk][8-row group][8][128 B] with `groups` row groups.
__device__ __forceinline__ uint32_t sw128_offset(int r, int k, int groups) {
  const int kc = k >> 7, col = k & 127, rr = r & 7;
  return (uint32_t)(kc * groups * 1024 + (r >> 3) * 1024 + rr * 128 + ((((col >> 4) ^ rr) & 7) << 4) + (col & 15));
}

// Wait (one lane, acquire at CTA scope) until a shared-memory flag is set;
// the warp gets one outcome.
// Down item: rows [a, a+cnt) of one entry's chunk for each of its pairs. Lane
// l takes 32-element block l of the pair's h, read once from L2 (I <= 1024:
// one block per lane); the pair's power-of-two rescale (kFp8H: its E4M3
// quantisation) comes from the warp maximum of those values.
template <bool kFp8H>
__device__ __forceinline__ void tc_d_item(const Params& p, const TcWs& tw, const DChunk& ch, int a, int cnt, int pb,
                                          int pe, float* dsm, int rpc, int trace_base = -1) {
  const int lane = threadIdx.x & 31;
  const int I = p.I, nblk = I / 32;
  for (int pp = pb; pp < pe; ++pp) {
    const float* hp = tw.h + (size_t)pp * I;
    if (nblk <= 32) {
      float hv[32];
      float mx = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float4 v = (lane < nblk) ? __ldcg(reinterpret_cast<const float4*>(hp + lane * 32) + t)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
        hv[4 * t] = v.x; hv[4 * t + 1] = v.y; hv[4 * t + 2] = v.z; hv[4 * t + 3] = v.w;
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
      mx = warp_max(mx);
      if (trace_base >= 0) tc_trace(p, trace_base);
      uint32_t h2[16];
      float down;
      if constexpr (kFp8H) {
        const float inv = h_fp8_inv(mx);
        down = h_fp8_scale(mx);
#pragma unroll
        for (int q = 0; q < 16; ++q) h2[q] = h_fp8x2(hv[2 * q], hv[2 * q + 1], inv);
      } else {
        const int t = h_rescale_exp(mx);
        const float up = ldexpf(1.f, t);
        down = ldexpf(1.f, -t);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          __half2 hh = __floats2half2_rn(hv[2 * q] * up, hv[2 * q + 1] * up);
          h2[q] = *reinterpret_cast<uint32_t*>(&hh);
        }
      }
      if (trace_base >= 0) tc_trace(p, trace_base + 1);
      d_rows(p, ch, a, cnt, lane, h2, down, dsm + (size_t)pp * rpc, true);
      __syncwarp();
      if (trace_base >= 0) tc_trace(p, trace_base + 2);
    } else {
      // wide intermediate: the maximum first, then block by block
      float mx = 0.f;
      for (int q = lane; q < I; q += 32) mx = fmaxf(mx, fabsf(__ldcg(hp + q)));
      mx = warp_max(mx);
      int t_exp = 0;
      float inv = 0.f, down;
      if constexpr (kFp8H) {
        inv = h_fp8_inv(mx);
        down = h_fp8_scale(mx);
      } else {
        t_exp = h_rescale_exp(mx);
        down = ldexpf(1.f, -t_exp);
      }
      const float up = ldexpf(1.f, t_exp);
      for (int b0 = 0; b0 < nblk; b0 += 32) {
        const int blk = b0 + lane;
        uint32_t h2[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float v0 = 0.f, v1 = 0.f;
          if (blk < nblk) {
            v0 = __ldcg(hp + blk * 32 + 2 * q);
            v1 = __ldcg(hp + blk * 32 + 2 * q + 1);
          }
          if constexpr (kFp8H) {
            h2[q] = h_fp8x2(v0, v1, inv);
          } else {
            __half2 hh = __floats2half2_rn(v0 * up, v1 * up);
            h2[q] = *reinterpret_cast<uint32_t*>(&hh);
          }
        }
        d_rows(p, ch, a, cnt, blk, h2, down, dsm + (size_t)pp * rpc, b0 == 0);
        __syncwarp();
      }
    }
  }
}


// Re-tiles gate/up codes [Eall][2I][H/2] into [Eall][I/4][H/128][8][64 B]:
// block (e, j, c) holds rows 4j..4j+3 (gate) and I+4j..I+4j+3 (up) of
// expert e, 64 bytes (128 codes) of K-chunk c each. 16 bytes per thread.
__global__ void k_repack_w13(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int Eall, int H, int I) {
  const size_t KCH = H / 128, upe = I / 4;
  const size_t total = (size_t)Eall * upe * KCH * 32;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    const size_t piece = idx & 31, blk = idx >> 5;
    const size_t c = blk % KCH, u = blk / KCH, e = u / upe, j = u % upe;
    const size_t i = piece >> 2, qq = piece & 3;
    const size_t row = e * 2 * I + (i < 4 ? 4 * j + i : I + 4 * j + (i - 4));
    const uint4 v = *reinterpret_cast<const uint4*>(src + row * (H / 2) + c * 64 + qq * 16);
    *reinterpret_cast<uint4*>(dst + blk * 512 + i * 64 + qq * 16) = v;
  }
}

// ---------------------------------------------------------------- the kernel
// kShared: expert E of E + 1 is a shared expert every token passes with
// weight 1 ("NVIDIA Shows 3 Ways to Speed Up MoE Inference on DGX Spark",
// section on Ling 3.0: one shared expert beside the 8 routed ones); it is
// union entry 0 with pairs 0..M-1. kFp8H: the SwiGLU output is quantised to
// E4M3 per pair before the down projection.
template <bool kShared, bool kFp8H>
__global__ void __launch_bounds__(kTcThreads, 1) k_tc(Params p, TcWs tw, TcPlan pl, const __grid_constant__ TcMaps maps) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x, G = gridDim.x;
  const int H = p.H, I = p.I, E = p.E, K = p.K, M = p.M;
  const int KCH = H / 128;

  uint64_t* full_gu = reinterpret_cast<uint64_t*>(smem + pl.o_bar);
  uint64_t* empty_gu = full_gu + kTcMaxSlots;
  uint64_t* acc_full = empty_gu + kTcMaxSlots;  // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2]
  uint64_t* full_d = acc_empty + 2;             // [kMaxSlots]
  uint64_t* empty_d = full_d + kMaxSlots;
  uint64_t* h_bar = empty_d + kMaxSlots;
  uint64_t* wr_bar = h_bar + kMaxSlots;
  uint64_t* sc_full = wr_bar + 1;   // [2] a tile's scale bytes landed
  uint64_t* sc_empty = sc_full + 2;  // [2] its scale factors are in tensor memory (4 warps)
  uint64_t* sf_ready = sc_empty + 2; // [2] same, for the MMA warp
  uint64_t* b_full = sf_ready + 2;   // [2] a down tile's B operand built (builder warps)
  uint64_t* b_empty = b_full + 2;    // [2] its MMAs are done with it
  uint64_t* dsc_full = b_empty + 2;  // [4] a down tile's pair scales written (builder warps)
  unsigned* done_d = reinterpret_cast<unsigned*>(dsc_full + 4);  // [kMaxSlots]
  float* s_amax = reinterpret_cast<float*>(smem + pl.o_misc);  // [32]
  float* s_xs = s_amax + kMaxTokens;                           // [32]
  float* s_rn = s_xs + kMaxTokens;                             // [32]
  float* s_red = s_rn + kMaxTokens;                            // [kTcWarps][kMaxRowsPerCta * 4]
  int* s_int = reinterpret_cast<int*>(s_red + kTcWarps * kMaxRowsPerCta * 4);  // [0] U [1] epoch [2] queue [3] tmem
  unsigned* s_tdone = reinterpret_cast<unsigned*>(s_int + 8);                  // [kTcMaxTiles] epilogue warps done
  unsigned* s_hready = reinterpret_cast<unsigned*>(smem + pl.o_hready);         // [max_union]
  int* s_ids = reinterpret_cast<int*>(smem + pl.o_ids);
  float* s_w = reinterpret_cast<float*>(smem + pl.o_w);
  int* s_pm = reinterpret_cast<int*>(smem + pl.o_pm);
  int* s_ppos = reinterpret_cast<int*>(smem + pl.o_ppos);
  int* s_union = reinterpret_cast<int*>(smem + pl.o_union);
  int* s_poff = reinterpret_cast<int*>(smem + pl.o_poff);
  float* dsm = reinterpret_cast<float*>(smem + pl.o_dsm);
  uint8_t* bd = smem + pl.o_bd;                                   // mma_down: [2] B operand buffers
  float* s_dsc = reinterpret_cast<float*>(smem + pl.o_dsc);       // mma_down: [4][kTcDownPairs] pair h scales
  int* s_dtoff = reinterpret_cast<int*>(smem + pl.o_dtoff);       // mma_down: [max_union + 1]
  uint8_t* ring_gu = smem + pl.o_ring_gu;
  uint8_t* bx = smem + pl.o_bx;
  uint8_t* scbuf = smem + pl.o_sc;
  uint8_t* ring_d = smem + pl.o_ring_d;
  // routing scratch, dead before the first weight copy lands
  float* wr_s = reinterpret_cast<float*>(ring_gu);                             // router rows
  float* s_logit = reinterpret_cast<float*>(smem + pl.o_lg);                    // [M][E]
  int* s_ec = reinterpret_cast<int*>(smem + pl.o_lg + M * E * 4);              // [E] union scratch
  uint4* x_s = reinterpret_cast<uint4*>(ring_d);                               // staged bf16 x (x_staged)
  const int ub = kShared ? 1 : 0;

  const int e0 = (int)((long long)E * b / G), e1 = (int)((long long)E * (b + 1) / G), ne = e1 - e0;
  const int r0 = (int)((long long)H * b / G), nrd = (int)((long long)H * (b + 1) / G) - r0;
  const int d_items = (nrd > 0) ? (nrd + kDownRowsPerItem - 1) / kDownRowsPerItem : 0;
  bool ok = true;  // this thread's waits all finished

  // ---------------- set-up that does not depend on the previous kernel
  tc_trace(p, 0);
  if (warp == kTcWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_int + 3)),
                 "r"((uint32_t)pl.tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid < kMaxSlots) {
    if (tid < kTcMaxSlots) {
      mbar_init(full_gu + tid, 1);
      mbar_init(empty_gu + tid, 1);
    }
    if (tid < 2) {
      mbar_init(acc_full + tid, 1);
      mbar_init(acc_empty + tid, 4);
    }
    mbar_init(full_d + tid, 1);
    mbar_init(empty_d + tid, max(1, d_items));
    mbar_init(h_bar + tid, 1);
    done_d[tid] = 0u;
    fence_mbar_init();
  }
  if (tid == 32 * kTcWarpProdGu) {
    for (int n = 0; n < kTcMaxUnits; ++n) prefetch_tensormap(&maps.m[n]);
    if (pl.mma_down) prefetch_tensormap(&maps.w2);
  }
  if (tid == 0) {
    mbar_init(wr_bar, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(sc_full + i, 1);
      mbar_init(sc_empty + i, 4);
      mbar_init(sf_ready + i, 4);
      mbar_init(b_full + i, kTcWarps - kTcWarpBuild);
      mbar_init(b_empty + i, 1);
      mbar_init(dsc_full + 2 * i, kTcWarps - kTcWarpBuild);
      mbar_init(dsc_full + 2 * i + 1, kTcWarps - kTcWarpBuild);
    }
    fence_mbar_init();
    if (ne > 0) {
      mbar_expect_tx(wr_bar, (unsigned)(ne * H * 4));
      tma_load_1d(wr_s, p.wr + (size_t)e0 * H, (unsigned)(ne * H * 4), wr_bar);
    }
  }
  pdl_wait();
  if (tid == 0) {
    s_int[1] = (int)(ld_relaxed_u32(tw.epoch) + 1u);
    s_int[2] = 0;
    s_int[5] = 0;  // epilogue warps done with their down tiles
    if constexpr (kShared) {
      s_union[0] = E;
      s_poff[0] = 0;
      s_poff[1] = M;
    }
  }
  if constexpr (kShared) {
    if (tid < M) s_pm[tid] = tid;
  }
  unsigned* s_amax_u = reinterpret_cast<unsigned*>(s_amax);
  if (tid < M) s_amax_u[tid] = 0u;
  if (tid < kTcMaxTiles) s_tdone[tid] = 0u;
  for (int i = tid; i < pl.max_union; i += kTcThreads) s_hready[i] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned epoch = (unsigned)s_int[1];
  const uint32_t tmem = (uint32_t)s_int[3];
  tc_trace(p, 1);
  // per-entry completion counters: this launch counts in array epoch & 1 and
  // clears the other one, which the previous launch used and the next will
  const int cstride = pl.max_union * kTcCntStride;
  unsigned* hcnt = tw.hcnt + (size_t)(epoch & 1) * cstride;
  if (b == 0) {
    unsigned* other = tw.hcnt + (size_t)((epoch + 1) & 1) * cstride;
    for (int i = tid; i < pl.max_union; i += kTcThreads) other[i * kTcCntStride] = 0u;
    if (tid == 0) tw.dcnt[(size_t)((epoch + 1) & 1) * kTcCntStride] = 0u;
  }

  // 8 bf16 of x (group i of M*H/8), normalised when the layer normalises
  // its input and x is not staged (a staged copy is normalised in place)
  auto ld_x8 = [&](int i) -> uint4 {
    if (pl.x_staged) return x_s[i];
    uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.x) + i);
    if (p.pre_rmsnorm) {
      const float r = s_rn[(i * 8) / H];
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        const __nv_bfloat162 o = __floats2bfloat162_rn(__fmul_rn(f.x, r), __fmul_rn(f.y, r));
        w[t] = *reinterpret_cast<const uint32_t*>(&o);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return v;
  };
  const int nbg = pl.nb_max / 8;
  if (M >= 2) {
    // ---- A9 + A1 + A2 for several tokens: one warp per token. Lane l holds
    //      the 4-element groups l + 32j of the row (a single L2 read when the
    //      row fits kTcXU2 groups per lane; else chunks, read twice). Pass 1:
    //      the RMSNorm sum of squares (fixed order) and amax (the normalised
    //      amax is bf16(fl32(amax * r)): rounding is monotonic and symmetric),
    //      and without RMSNorm the router logits; pass 2: the logits of the
    //      normalised row (with RMSNorm) and the E4M3 codes straight into the
    //      MMA's B operand (K-major, 128-byte swizzle; rows >= M never read).
    //      A lane's router values are one float4 per row and group, so the
    //      warp reads each router row contiguously.
    if (ne > 0 && !mbar_wait_ok(wr_bar, 0, p)) ok = false;
    tc_trace(p, 14);
    const int n2 = H / 4;
    const bool one = n2 <= 32 * kTcXU2;
    if (tid < kMaxTokens) s_xs[tid] = 1.f;
    __syncwarp();
    for (int m = warp; m < M; m += kTcWarps) {
      const uint2* xg = reinterpret_cast<const uint2*>(p.x) + (size_t)m * n2;
      uint2 xr[kTcXU2];
      auto load_chunk = [&](int c0) {
#pragma unroll
        for (int j = 0; j < kTcXU2; ++j) {
          const int i = c0 + lane + 32 * j;
          xr[j] = (i < n2) ? ld_cg_v2_once(xg + i) : make_uint2(0u, 0u);
        }
      };
      float ss = 0.f, a = 0.f;
      for (int c0 = 0; c0 < n2; c0 += 32 * kTcXU2) {
        load_chunk(c0);
#pragma unroll
        for (int j = 0; j < kTcXU2; ++j) {
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].y));
          ss = __fmaf_rn(f0.x, f0.x, ss);
          ss = __fmaf_rn(f0.y, f0.y, ss);
          ss = __fmaf_rn(f1.x, f1.x, ss);
          ss = __fmaf_rn(f1.y, f1.y, ss);
          a = fmaxf(a, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
        }
      }
      a = warp_max(a);
      if (m == warp) tc_trace(p, 36);
      float r = 1.f;
      if (p.pre_rmsnorm) {
        ss = warp_sum(ss);
        r = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)H), 1e-6f)));
        a = __bfloat162float(__float2bfloat16_rn(__fmul_rn(a, r)));
      }
      const float inv = (a != 0.f) ? __fdiv_rn(448.f, a) : 0.f;
      // (reloaded) chunk, normalised in place with RMSNorm
      auto norm_chunk = [&](int c0) {
        if (!p.pre_rmsnorm) return;
#pragma unroll
        for (int j = 0; j < kTcXU2; ++j) {
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].y));
          const __nv_bfloat162 o0 = __floats2bfloat162_rn(__fmul_rn(f0.x, r), __fmul_rn(f0.y, r));
          const __nv_bfloat162 o1 = __floats2bfloat162_rn(__fmul_rn(f1.x, r), __fmul_rn(f1.y, r));
          xr[j] = make_uint2(*reinterpret_cast<const uint32_t*>(&o0), *reinterpret_cast<const uint32_t*>(&o1));
        }
      };
      for (int c0 = 0; c0 < n2; c0 += 32 * kTcXU2) {
        if (!one) load_chunk(c0);
        norm_chunk(c0);
#pragma unroll
        for (int j = 0; j < kTcXU2; ++j) {
          const int i = c0 + lane + 32 * j;
          if (i < n2) {
            if (p.pre_rmsnorm && b == 0 && p.out_xn) reinterpret_cast<uint2*>(p.out_xn)[(size_t)m * n2 + i] = xr[j];
            uint32_t out = 0u;
            if (a != 0.f) {
              const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].x));
              const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].y));
              const uint32_t c0v = f32x2_to_e4m3x2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv));
              const uint32_t c1v = f32x2_to_e4m3x2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv));
              out = c0v | (c1v << 16);
            }
            *reinterpret_cast<uint32_t*>(bx + sw128_offset(m, 4 * i, nbg)) = out;
            if (b == 0 && p.out_xq) *reinterpret_cast<uint32_t*>(p.out_xq + (size_t)m * H + 4 * i) = out;
          }
        }
      }
      if (m == warp) tc_trace(p, 37);
      // logits of the CTA's router rows, two at a time
      for (int el0 = 0; el0 < ne; el0 += 2) {
        float acc0 = 0.f, acc1 = 0.f;
        const bool two = el0 + 1 < ne;
        const float4* w0 = reinterpret_cast<const float4*>(wr_s + (size_t)el0 * H);
        const float4* w1 = reinterpret_cast<const float4*>(wr_s + (size_t)(el0 + (two ? 1 : 0)) * H);
        for (int c0 = 0; c0 < n2; c0 += 32 * kTcXU2) {
          if (!one) {
            load_chunk(c0);
            norm_chunk(c0);
          }
#pragma unroll
          for (int j = 0; j < kTcXU2; ++j) {
            const int i = c0 + lane + 32 * j;
            if (i < n2) {
              const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].x));
              const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xr[j].y));
              const float4 u = w0[i], v = w1[i];
              acc0 = fmaf(x01.x, u.x, acc0); acc0 = fmaf(x01.y, u.y, acc0);
              acc0 = fmaf(x23.x, u.z, acc0); acc0 = fmaf(x23.y, u.w, acc0);
              acc1 = fmaf(x01.x, v.x, acc1); acc1 = fmaf(x01.y, v.y, acc1);
              acc1 = fmaf(x23.x, v.z, acc1); acc1 = fmaf(x23.y, v.w, acc1);
            }
          }
        }
        acc0 = warp_sum(acc0);
        acc1 = warp_sum(acc1);
        if (lane == 0) st_relaxed_u64(tw.logits + (size_t)m * E + e0 + el0, tag_word(epoch, acc0));
        if (lane == 0 && two) st_relaxed_u64(tw.logits + (size_t)m * E + e0 + el0 + 1, tag_word(epoch, acc1));
      }
      if (lane == 0) {
        s_amax[m] = a;
        s_xs[m] = (a == 0.f) ? 1.f : __fdiv_rn(a, 448.f);
        if (b == 0 && p.out_xscale) p.out_xscale[m] = s_xs[m];
      }
      if (m == warp) tc_trace(p, 38);
    }
    tc_trace(p, 15);
    // the B operand is read by the tensor cores (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  } else {
  // ---- A1 (first half): stage x (when it fits), per-token amax
  const int nx8 = M * H / 8, rot8 = (int)((b * 8u) % (unsigned)nx8);  // CTA-rotated start
  for (int i0 = tid; i0 < nx8; i0 += kTcThreads) {
    const int i = (i0 + rot8 >= nx8) ? i0 + rot8 - nx8 : i0 + rot8;
    const int m = (i * 8) / H;
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.x) + i);
    if (pl.x_staged) x_s[i] = v;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
      a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    atomicMax(&s_amax_u[m], __float_as_uint(a));
  }
  __syncthreads();
  tc_trace(p, 13);
  // ---- A9 (stacked layers): x <- bf16(x / sqrt(mean(x^2) + 1e-6)) per token,
  //      one warp per token, fixed summation order (every CTA derives the
  //      same factor); the new amax is bf16(fl32(amax * r)).
  if (p.pre_rmsnorm) {
    for (int m = warp; m < M; m += kTcWarps) {
      float ss = 0.f;
      for (int i = lane; i < H / 8; i += 32) {
        const uint4 v = pl.x_staged ? x_s[(size_t)m * (H / 8) + i]
                                    : __ldcg(reinterpret_cast<const uint4*>(p.x) + (size_t)m * (H / 8) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
          ss = __fmaf_rn(f.x, f.x, ss);
          ss = __fmaf_rn(f.y, f.y, ss);
        }
      }
      ss = warp_sum(ss);
      if (lane == 0) {
        const float r = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)H), 1e-6f)));
        s_rn[m] = r;
        s_amax[m] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_amax[m], r)));
      }
    }
    __syncthreads();
    for (int i = tid; i < M * H / 8; i += kTcThreads) {
      const int m = (i * 8) / H;
      const float r = s_rn[m];
      uint4 v = pl.x_staged ? x_s[i] : __ldcg(reinterpret_cast<const uint4*>(p.x) + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        const __nv_bfloat162 o = __floats2bfloat162_rn(__fmul_rn(f.x, r), __fmul_rn(f.y, r));
        w[t] = *reinterpret_cast<const uint32_t*>(&o);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
      if (pl.x_staged) x_s[i] = v;
      if (b == 0 && p.out_xn) reinterpret_cast<uint4*>(p.out_xn)[i] = v;
    }
    __syncthreads();
  }
  // ---- A2: logits of the CTA's router rows
  if (ne > 0 && !mbar_wait_ok(wr_bar, 0, p)) ok = false;
  tc_trace(p, 14);
  if (M == 1 && ne > 0 && ne <= 2)
    router_logits_m1(ld_x8, wr_s, H, ne, epoch, tw.logits + e0, s_red);
  for (int m0 = 0; m0 < M && ne > 0 && !(M == 1 && ne <= 2); m0 += 4) {
    const int mt = min(4, M - m0);
    for (int el = 0; el < ne; ++el) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float4* wrow = reinterpret_cast<const float4*>(wr_s + (size_t)el * H);
      for (int i = tid; i < H / 4; i += kTcThreads) {
        const float4 wv = wrow[i];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (t < mt) {
            const uint4 x8 = ld_x8((int)(((size_t)(m0 + t) * H) / 8 + i / 2));
            const uint2 q = (i & 1) ? make_uint2(x8.z, x8.w) : make_uint2(x8.x, x8.y);
            const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
            const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
            acc[t] = fmaf(x01.x, wv.x, acc[t]);
            acc[t] = fmaf(x01.y, wv.y, acc[t]);
            acc[t] = fmaf(x23.x, wv.z, acc[t]);
            acc[t] = fmaf(x23.y, wv.w, acc[t]);
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (t < mt) s_red[warp * (kMaxRowsPerCta * 4) + el * 4 + t] = acc[t];
      }
    }
    __syncthreads();
    if (tid < ne * 4) {
      const int el = tid >> 2, t = tid & 3;
      if (t < mt) {
        float sum = 0.f;
        for (int w = 0; w < kTcWarps; ++w) sum += s_red[w * (kMaxRowsPerCta * 4) + el * 4 + t];
        // the value and this launch's epoch in one 64-bit word
        st_relaxed_u64(tw.logits + (size_t)(m0 + t) * E + e0 + el, tag_word(epoch, sum));
      }
    }
    __syncthreads();
  }
  tc_trace(p, 15);
  // ---- A1 (second half): E4M3 codes straight into the MMA's B operand
  //      (K-major, 128-byte swizzle, nb_max token rows; rows >= M are zero)
  if (tid < kMaxTokens) {
    const float a = (tid < M) ? s_amax[tid] : 0.f;
    s_xs[tid] = (a == 0.f) ? 1.f : __fdiv_rn(a, 448.f);
  }
  // (rows M..nb_max-1 are left as they are: the accumulator columns they
  // feed are never read)
  for (int i = tid; i < M * H / 16; i += kTcThreads) {
    const int m = i / (H / 16), k = (i % (H / 16)) * 16;
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    {
      const float a = s_amax[m];
      if (a != 0.f) {
        const float inv = __fdiv_rn(448.f, a);
        uint32_t q[4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 v = ld_x8((int)(((size_t)m * H + k) / 8 + hh));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int t = 0; t < 4; t += 2) {
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
            const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t + 1]));
            const uint32_t c0 = f32x2_to_e4m3x2(__fmul_rn(f0.x, inv), __fmul_rn(f0.y, inv));
            const uint32_t c1 = f32x2_to_e4m3x2(__fmul_rn(f1.x, inv), __fmul_rn(f1.y, inv));
            q[2 * hh + (t >> 1)] = c0 | (c1 << 16);
          }
        }
        out = make_uint4(q[0], q[1], q[2], q[3]);
      }
      if (b == 0 && p.out_xq) *reinterpret_cast<uint4*>(p.out_xq + (size_t)m * H + k) = out;
    }
    *reinterpret_cast<uint4*>(bx + sw128_offset(m, k, nbg)) = out;
  }
  if (b == 0 && p.out_xscale && tid < M) p.out_xscale[tid] = s_xs[tid];
  // the B operand is read by the tensor cores (async proxy)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  tc_trace(p, 2);

  // ---- A2 exchange: read every logit word until all carry this epoch
  if (!poll_tagged_logits(p, tw.logits, M * E, p.force_stall ? epoch + 0x40000000u : epoch, s_logit)) ok = false;
  pdl_launch_dependents();
  __syncthreads();
  tc_trace(p, 3);

  // ---- A3: top-k and softmax: every warp on the one token when M == 1,
  //      else one warp per token
  if (M == 1 && E <= 32 * kTcWarps && K <= 8) {
    topk_cta_small(s_logit, E, K, s_ids, s_w, reinterpret_cast<unsigned*>(s_red),
                   reinterpret_cast<int*>(s_red) + 136, p);
    if (b == 0 && tid < K) {
      if (p.out_ids) p.out_ids[tid] = s_ids[tid];
      if (p.out_w) p.out_w[tid] = s_w[tid];
    }
  }
  if (M >= 2 && E <= 512 && K <= 8) {
    // two tokens per warp, one per half
    for (int m = 2 * warp + (lane >> 4); m < M; m += 2 * kTcWarps) {
      const float* lrow = s_logit + (size_t)m * E;
      int* ids = s_ids + m * K;
      float* ws = s_w + m * K;
      if (E <= 16) topk_half<1>(lrow, E, K, ids, ws);
      else if (E <= 32) topk_half<2>(lrow, E, K, ids, ws);
      else if (E <= 64) topk_half<4>(lrow, E, K, ids, ws);
      else if (E <= 128) topk_half<8>(lrow, E, K, ids, ws);
      else if (E <= 256) topk_half<16>(lrow, E, K, ids, ws);
      else topk_half<32>(lrow, E, K, ids, ws);
      if (b == 0 && (lane & 15) < K) {
        if (p.out_ids) p.out_ids[m * K + (lane & 15)] = ids[lane & 15];
        if (p.out_w) p.out_w[m * K + (lane & 15)] = ws[lane & 15];
      }
      if (m == 2 * warp) tc_trace(p, 39);
    }
    tc_trace(p, 40);
  }
  for (int m = warp; m < M && !(M == 1 && E <= 32 * kTcWarps && K <= 8) && !(M >= 2 && E <= 512 && K <= 8);
       m += kTcWarps) {
    const float* lrow = s_logit + (size_t)m * E;
    int* ids = s_ids + m * K;
    float* ws = s_w + m * K;
    if (E <= 32) topk_warp<1>(lrow, E, K, ids, ws);
    else if (E <= 64) topk_warp<2>(lrow, E, K, ids, ws);
    else if (E <= 128) topk_warp<4>(lrow, E, K, ids, ws);
    else if (E <= 256) topk_warp<8>(lrow, E, K, ids, ws);
    else if (E <= 512) topk_warp<16>(lrow, E, K, ids, ws);
    else topk_warp<32>(lrow, E, K, ids, ws);
    __syncwarp();
    if (b == 0 && lane < K) {
      if (p.out_ids) p.out_ids[m * K + lane] = ids[lane];
      if (p.out_w) p.out_w[m * K + lane] = ws[lane];
    }
  }
  __syncthreads();
  tc_trace(p, 8);

  // ---- A4: union (ascending ids) and the pairs of each entry in (token, slot) order
  const int np = M * K, pbase = kShared ? M : 0;
  if (M == 1) {
    union_m1(s_ids, K, ub, pbase, s_union, s_poff, s_pm, s_ppos, &s_int[0]);
  } else if (np <= 32) {
    if (warp == 0) {
      const int Us = union_small(s_ids, np, K, s_union + ub, s_poff + ub, s_pm, s_ppos, pbase);
      if (lane == 0) s_int[0] = ub + Us;
    }
  } else {
    // many pairs: the whole CTA. Counts per expert, a block-wide exclusive
    // scan over the experts (ascending: the union and each entry's first
    // pair position), then each pair's place among the earlier pairs of its
    // expert (token, slot order)
    int* s_ws = reinterpret_cast<int*>(s_red);  // [kTcWarps][2] warp totals
    for (int e = tid; e < E; e += kTcThreads) s_ec[e] = 0;
    __syncthreads();
    tc_trace(p, 41);
    for (int i = tid; i < np; i += kTcThreads) atomicAdd(&s_ec[s_ids[i]], 1);
    __syncthreads();
    const int per = (E + kTcThreads - 1) / kTcThreads;
    const int ea = min(E, tid * per), eb = min(E, ea + per);
    int nz = 0, cs = 0;
    for (int e = ea; e < eb; ++e) { nz += s_ec[e] > 0; cs += s_ec[e]; }
    int nz_in = nz, cs_in = cs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x1 = __shfl_up_sync(0xffffffffu, nz_in, o);
      const int x2 = __shfl_up_sync(0xffffffffu, cs_in, o);
      if (lane >= o) { nz_in += x1; cs_in += x2; }
    }
    if (lane == 31) {
      s_ws[2 * warp] = nz_in;
      s_ws[2 * warp + 1] = cs_in;
    }
    __syncthreads();
    int nz_ex = nz_in - nz, cs_ex = cs_in - cs;
    for (int w = 0; w < warp; ++w) {
      nz_ex += s_ws[2 * w];
      cs_ex += s_ws[2 * w + 1];
    }
    for (int e = ea; e < eb; ++e) {
      const int c = s_ec[e];
      if (c > 0) {
        s_union[ub + nz_ex] = e;
        s_poff[ub + nz_ex] = pbase + cs_ex;
        ++nz_ex;
        cs_ex += c;
      }
      s_ec[e] = pbase + cs_ex - c;  // first pair position of expert e
    }
    if (tid == kTcThreads - 1) {
      s_poff[ub + nz_ex] = pbase + cs_ex;
      s_int[0] = ub + nz_ex;
    }
    __syncthreads();
    tc_trace(p, 34);
    for (int i = tid; i < np; i += kTcThreads) {
      const int e = s_ids[i];
      // earlier pairs of the same expert: whole int4 blocks (16-byte aligned
      // s_ids), then the rest
      int rank = 0, j2 = 0;
      const int4* ids4 = reinterpret_cast<const int4*>(s_ids);
      for (; j2 + 4 <= i; j2 += 4) {
        const int4 v = ids4[j2 >> 2];
        rank += (v.x == e) + (v.y == e) + (v.z == e) + (v.w == e);
      }
      for (; j2 < i; ++j2) rank += s_ids[j2] == e;
      const int pos = s_ec[e] + rank;
      s_pm[pos] = i / K;
      s_ppos[i] = pos;
    }
  }
  // ring_gu and ring_d held routing scratch (generic proxy): order that
  // before the TMA writes into them (not needed when the only generic
  // accesses to them were the router-row and staged-x reads before the
  // activation codes' fence)
  if (!pl.lg_own) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  // one outcome for the CTA: after a routing wait ran out, no role starts
  ok = __syncthreads_and(ok ? 1 : 0) != 0;
  const int U = s_int[0];
  // tensor-core down tiles, entry-major: entry u has ceil(pairs / kTcDownPairs)
  // pair groups x H/128 row blocks; s_dtoff[u] = first tile of entry u
  const int RB = H / 128;
  if (pl.mma_down) {
    if (warp == 0) {
      const int per = (U + 31) / 32, ua = min(U, lane * per), ubd = min(U, ua + per);
      int cnt = 0;
      for (int u = ua; u < ubd; ++u) cnt += (s_poff[u + 1] - s_poff[u] + kTcDownPairs - 1) / kTcDownPairs * RB;
      int ex = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ex, o);
        if (lane >= o) ex += y;
      }
      ex -= cnt;
      for (int u = ua; u < ubd; ++u) {
        s_dtoff[u] = ex;
        ex += (s_poff[u + 1] - s_poff[u] + kTcDownPairs - 1) / kTcDownPairs * RB;
      }
      if (lane == 31) s_dtoff[U] = ex + 0;  // lane 31 holds the total (its range may be empty)
    }
    __syncthreads();
  }
  const int D = pl.mma_down ? s_dtoff[U] : 0;
  const int my_dtiles = (b < D) ? (D - b + G - 1) / G : 0;
  // down tile d -> entry u (hint: advances monotonically), pair group g, row block R
  auto dtile_of = [&](int d, int& u, int& g, int& R) {
    while (s_dtoff[u + 1] <= d) ++u;
    const int rem = d - s_dtoff[u];
    g = rem / RB;
    R = rem - g * RB;
  };
  tc_trace(p, 4);

  // ---------------- gate/up schedule: flat units, tiles dealt round robin
  const int upe = I / 4;                     // units per entry
  const int T = U * upe;                     // units of the step
  const int rounds = max(1, (T + G * pl.tu_max - 1) / (G * pl.tu_max));
  const int tu = (T + G * rounds - 1) / (G * rounds);
  const int ntile = (T + tu - 1) / tu;
  const int my_tiles = (b < ntile) ? (ntile - b + G - 1) / G : 0;
  const int ks = pl.ks, nstage = KCH / ks;
  const int scb = pl.sc_bytes;  // one tile's scale buffer: [gate rows 4*tu_max][up rows 4*tu_max] x H/32 bytes
  // tensor memory: accumulators in columns [0, 64), the scale factors of tile
  // buffer t at kTcSfCol + 4*KCH*t (4 columns per K-chunk), the tokens' unit
  // scale factors after them
  const uint32_t sfb_col = tmem + (uint32_t)(kTcSfCol + 8 * KCH);

  if (warp == kTcWarpProdGu) {
    // ---------------- gate/up producer (one thread): per tile its E8M0
    //   scales (own barrier), then the code stages
    if (lane == 0) {
      int stage = 0, slot = 0;
      unsigned ph = 0;
      bool reuse = false;  // the slot held an earlier stage
      for (int it = 0; it < my_tiles && ok; ++it) {
        const int t = b + it * G;
        const int f0 = t * tu, f1 = min(T, f0 + tu), nu = f1 - f0;
        const int sb = it & 1;
        uint8_t* sc = scbuf + (size_t)sb * scb;
        // the tile's runs of units of one expert: at most 2 (a tile has at
        // most 16 units and an entry I/4 >= 32)
        int rcoord[2], runit[2], rn[2], rg[2], nrun = 0;
        for (int f = f0; f < f1 && nrun < 2;) {
          const int u = f / upe, j = f % upe, n = min(f1 - f, upe - j);
          const int e = s_union[u];
          rcoord[nrun] = e * (I / 2) + j;  // 5-D map: quad of gate rows 4j.. of expert e
          runit[nrun] = e * upe + j;       // 4-D map over the re-tiled copy: unit j of expert e
          rn[nrun] = n;
          rg[nrun] = f - f0;
          ++nrun;
          f += n;
        }
        if (it >= 2 && !mbar_wait_ok(sc_empty + sb, ((it >> 1) - 1) & 1, p)) { ok = false; break; }
        mbar_expect_tx(sc_full + sb, (unsigned)(8 * nu * (H / 32)));
        for (int r = 0; r < nrun; ++r) {
          const size_t grow = (size_t)4 * rcoord[r];  // gate row 4j of expert e: 4 * (e*I/2 + j)
          tma_load_1d(sc + (size_t)4 * rg[r] * (H / 32), p.w13s + grow * (H / 32), (unsigned)(4 * rn[r] * (H / 32)),
                      sc_full + sb);
          tma_load_1d(sc + (size_t)(4 * pl.tu_max + 4 * rg[r]) * (H / 32), p.w13s + (grow + I) * (H / 32),
                      (unsigned)(4 * rn[r] * (H / 32)), sc_full + sb);
        }
        const unsigned bytes = (unsigned)(nu * ks * 512);
        for (int k = 0; k < nstage; ++k, ++stage) {
          if (reuse && !mbar_wait_ok(empty_gu + slot, ph ^ 1u, p)) { ok = false; break; }
          if (stage >= pl.ns_gu && stage < pl.ns_gu + 4) tc_trace(p, 42 + stage - pl.ns_gu);
          mbar_expect_tx(full_gu + slot, bytes);
          if (stage < 2) tc_trace(p, 32 + stage);
          uint8_t* dst = ring_gu + (size_t)slot * pl.slot_gu;
          for (int r = 0; r < nrun; ++r) {
            if (tw.repacked)
              tma_load_4d(dst + (size_t)rg[r] * ks * 1024, &maps.m[rn[r] - 1], 0, 0, k * ks, runit[r], full_gu + slot);
            else
              tma_load_5d(dst + (size_t)rg[r] * ks * 1024, &maps.m[rn[r] - 1], 0, 0, 0, k * ks, rcoord[r],
                          full_gu + slot);
          }
          if (++slot == pl.ns_gu) { slot = 0; ph ^= 1u; reuse = true; }
        }
      }
      // tensor-core down tiles: the 128 rows' E8M0 scales (one copy, 128 x
      // I/32 bytes), then one stage per K-chunk of 128: a 128 x 128 box of
      // W2 codes (16 KB unpacked, the same slot shape as a 16-unit gate/up
      // stage)
      int du = 0;
      for (int k = 0; k < my_dtiles && ok; ++k) {
        int g, R;
        dtile_of(b + k * G, du, g, R);
        const int it = my_tiles + k, sb = it & 1;
        const int row0 = s_union[du] * H + R * 128;
        if (it >= 2 && !mbar_wait_ok(sc_empty + sb, ((it >> 1) - 1) & 1, p)) { ok = false; break; }
        mbar_expect_tx(sc_full + sb, (unsigned)(128 * (I / 32)));
        tma_load_1d(scbuf + (size_t)sb * scb, p.w2s + (size_t)row0 * (I / 32), (unsigned)(128 * (I / 32)),
                    sc_full + sb);
        for (int kc = 0; kc < pl.dkch; ++kc, ++stage) {
          if (reuse && !mbar_wait_ok(empty_gu + slot, ph ^ 1u, p)) { ok = false; break; }
          mbar_expect_tx(full_gu + slot, 128u * 64u);
          tma_load_2d(ring_gu + (size_t)slot * pl.slot_gu, &maps.w2, kc * 128, row0, full_gu + slot);
          if (++slot == pl.ns_gu) { slot = 0; ph ^= 1u; reuse = true; }
        }
      }
      if (my_dtiles > 0) tc_trace(p, 59);
    }
  } else if (warp == kTcWarpMma) {
    // ---------------- MMA issue (one thread); descriptors move by adding the
    //   byte offset / 16 to the start-address field
    const uint64_t ad0 = umma_desc_sw128(smem_u32(ring_gu), (uint32_t)(ks * 1024));
    const uint64_t bd0 = umma_desc_sw128(smem_u32(bx), 1024u);
    uint32_t idk[4];
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) idk[kb] = umma_idesc_mx(pl.nb_max, kb);
    const uint64_t slot_step = (uint64_t)(pl.slot_gu >> 4), kc_step = (uint64_t)(nbg * 64);
    int stage = 0, slot = 0;
    unsigned ph = 0;
    for (int it = 0; it < my_tiles && ok; ++it) {
      const int buf = it & 1;
      const uint32_t acc_col = tmem + (uint32_t)(buf * kTcAccCols);
      const uint32_t sf_base = tmem + (uint32_t)(kTcSfCol + 4 * KCH * buf);
      if (it >= 2 && !mbar_wait_warp(acc_empty + buf, ((it >> 1) - 1) & 1, p)) { ok = false; break; }
      if (!mbar_wait_warp(sf_ready + buf, (it >> 1) & 1, p)) { ok = false; break; }
      tc_fence_after();
      for (int k = 0; k < nstage; ++k, ++stage) {
        if (!mbar_wait_warp(full_gu + slot, ph, p)) { ok = false; break; }
        if (stage < 8) tc_trace(p, 16 + stage);
        if (lane == 0) {
          tc_fence_after();
          const uint64_t ads = ad0 + (uint64_t)slot * slot_step;
          for (int c = 0; c < ks; ++c) {
            const int kc = k * ks + c;
            const uint64_t adc = ads + (uint64_t)(c * 64);
            const uint64_t bdc = bd0 + (uint64_t)kc * kc_step;
            const uint32_t sfa = sf_base + 4u * (uint32_t)kc;
            const uint32_t acc0 = (k > 0 || c > 0) ? 1u : 0u;
            umma_mx(acc_col, adc, bdc, idk[0], acc0, sfa, sfb_col);
            umma_mx(acc_col, adc + 2, bdc + 2, idk[1], 1u, sfa, sfb_col);
            umma_mx(acc_col, adc + 4, bdc + 4, idk[2], 1u, sfa, sfb_col);
            umma_mx(acc_col, adc + 6, bdc + 6, idk[3], 1u, sfa, sfb_col);
          }
          tc_commit(empty_gu + slot);
          if (k == nstage - 1) tc_commit(acc_full + buf);
          if (stage < 4) tc_trace(p, 26 + stage);
        }
        __syncwarp();
        if (++slot == pl.ns_gu) { slot = 0; ph ^= 1u; }
      }
    }
    // tensor-core down tiles: A = 128 W2 rows (slot, SBO 1 KB), B = the
    // tile's h codes (buffer k & 1: K-chunk kc at kc * 4 KB, N <= 32 rows),
    // scale factors of A in the tile buffer's columns, B's all 1.0
    const uint64_t bdd0 = umma_desc_sw128(smem_u32(bd), 1024u);
    int du = 0;
    for (int k = 0; k < my_dtiles && ok; ++k) {
      int g, R;
      dtile_of(b + k * G, du, g, R);
      const int np_t = min(kTcDownPairs, s_poff[du + 1] - s_poff[du] - kTcDownPairs * g);
      const int nn = kFp8H ? np_t : 2 * np_t;
      uint32_t idd[4];
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) idd[kb] = umma_idesc_mx(max(8, (nn + 7) / 8 * 8), kb);
      const int it = my_tiles + k, buf = it & 1, bb = k & 1;
      const uint32_t acc_col = tmem + (uint32_t)(buf * kTcAccCols);
      const uint32_t sf_base = tmem + (uint32_t)(kTcSfCol + 4 * KCH * buf);
      if (it >= 2 && !mbar_wait_warp(acc_empty + buf, ((it >> 1) - 1) & 1, p)) { ok = false; break; }
      if (!mbar_wait_warp(sf_ready + buf, (it >> 1) & 1, p)) { ok = false; break; }
      if (!mbar_wait_warp(b_full + bb, (k >> 1) & 1, p)) { ok = false; break; }
      tc_fence_after();
      const uint64_t bdb = bdd0 + (uint64_t)((bb * pl.bd_bytes) >> 4);
      for (int kc = 0; kc < pl.dkch; ++kc, ++stage) {
        if (!mbar_wait_warp(full_gu + slot, ph, p)) { ok = false; break; }
        if (lane == 0) {
          tc_fence_after();
          const uint64_t adc = ad0 + (uint64_t)slot * slot_step;
          const uint64_t bdc = bdb + (uint64_t)kc * 256u;  // 4 KB per K-chunk
          const uint32_t sfa = sf_base + 4u * (uint32_t)kc;
          umma_mx(acc_col, adc, bdc, idd[0], kc > 0 ? 1u : 0u, sfa, sfb_col);
          umma_mx(acc_col, adc + 2, bdc + 2, idd[1], 1u, sfa, sfb_col);
          umma_mx(acc_col, adc + 4, bdc + 4, idd[2], 1u, sfa, sfb_col);
          umma_mx(acc_col, adc + 6, bdc + 6, idd[3], 1u, sfa, sfb_col);
          tc_commit(empty_gu + slot);
          if (kc == pl.dkch - 1) {
            tc_commit(acc_full + buf);
            tc_commit(b_empty + bb);
          }
        }
        __syncwarp();
        if (++slot == pl.ns_gu) { slot = 0; ph ^= 1u; }
      }
    }
    tc_trace(p, 6);
  } else if (warp == kTcWarpProdD) {
    // ---------------- down producer: rows [r0, r0+nrd) of every entry, in order
    if (lane == 0 && nrd > 0 && !pl.mma_down) {
      // the gate/up stream goes first: wait for its first stage to land
      if (my_tiles > 0 && !mbar_wait_ok(full_gu, 0, p)) ok = false;
      int slot = 0;
      unsigned ph = 0;
      bool reuse = false;
      for (int u = 0; u < U && ok; ++u) {
        if (reuse && !mbar_wait_ok(empty_d + slot, ph ^ 1u, p)) { ok = false; break; }
        const int e = s_union[u];
        uint8_t* sp = ring_d + (size_t)slot * pl.slot_d;
        DChunk ch;
        size_t sa0;
        unsigned sn;
        const unsigned bytes = d_layout(p, e, r0, nrd, sp, &ch, &sa0, &sn);
        mbar_expect_tx(full_d + slot, bytes);
        const unsigned codes = (unsigned)(nrd * I / 2);
        tma_load_1d(sp, p.w2c + ((size_t)e * H + r0) * (I / 2), codes, full_d + slot);
        tma_load_1d(sp + codes, p.w2s + sa0, sn, full_d + slot);
        if (u == 0) tc_trace(p, 59);
        if (++slot == pl.ns_d) { slot = 0; ph ^= 1u; reuse = true; }
      }
      tc_trace(p, 60);
    }
  }

  if (warp >= kTcWarpEpi && warp < kTcWarpEpi + 4) {
    // ---------------- scale factors into tensor memory, and the gate/up
    //   epilogue. Warp quarter q owns tensor-memory lanes 32q..32q+31.
    const int q = warp - kTcWarpEpi;
    // Scale factors of tile `ti` into buffer ti & 1: lane L of every quarter
    // holds, in column 4*kc + j, the scale word (4 E8M0 bytes, K blocks
    // 4kc..4kc+3) of tile row L + 32j (unit (L+32j)/8; its rows 0..3 gate,
    // 4..7 up). The first call also writes the tokens' unit scales.
    // A down tile (ti >= my_tiles): row r is W2 row row0 + r, whose scale
    // bytes sit at r * I/32 in the buffer; dkch K-chunks.
    auto write_sf = [&](int ti) -> bool {
      const int sb = ti & 1;
      if (!mbar_wait_warp(sc_full + sb, (ti >> 1) & 1, p)) return false;
      const uint8_t* sc = scbuf + (size_t)sb * scb;
      const uint32_t lane_base = (uint32_t)(32 * q) << 16;
      const uint32_t col = tmem + (uint32_t)(kTcSfCol + 4 * KCH * sb) + lane_base;
      int rowoff[4], nkc = KCH;
      if (ti < my_tiles) {
        const int t = b + ti * G;
        const int f0 = t * tu, nu = min(T, f0 + tu) - f0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j, g = r >> 3, i8 = r & 7;
          rowoff[j] = (g < nu) ? ((i8 < 4) ? 4 * g + i8 : 4 * pl.tu_max + 4 * g + (i8 - 4)) * (H / 32) : -1;
        }
      } else {
        nkc = pl.dkch;
#pragma unroll
        for (int j = 0; j < 4; ++j) rowoff[j] = (lane + 32 * j) * (I / 32);
      }
      for (int kc = 0; kc < nkc; ++kc) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w[j] = rowoff[j] >= 0 ? *reinterpret_cast<const uint32_t*>(sc + rowoff[j] + 4 * kc) : 0x7F7F7F7Fu;
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(col + 4u * kc),
                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]));
      }
      if (ti == 0)
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sfb_col + lane_base),
                     "r"(0x7F7F7F7Fu));
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sf_ready + sb);
        mbar_arrive(sc_empty + sb);
      }
      return true;
    };
    const int all_tiles = my_tiles + my_dtiles;
    if (ok && all_tiles > 0 && !write_sf(0)) ok = false;
    if (ok && all_tiles > 1 && !write_sf(1)) ok = false;
    int du = 0;
    for (int it = 0; it < all_tiles && ok; ++it) {
      if (it >= my_tiles) {
        // ---- tensor-core down tile: y of each pair of the group for the
        //      tile's 128 output rows (lane = row), h = scale * (hi + lo/16)
        const int k = it - my_tiles, buf = it & 1;
        int g, R;
        dtile_of(b + k * G, du, g, R);
        const int pb0 = s_poff[du] + kTcDownPairs * g, np_t = min(kTcDownPairs, s_poff[du + 1] - pb0);
        if (!mbar_wait_warp(acc_full + buf, (it >> 1) & 1, p)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t)(buf * kTcAccCols) + ((uint32_t)(32 * q) << 16), v);
        // the pair scales of tile k (ring of 4: the builders reuse this entry
        // for tile k + 4 only after tile k + 2's MMAs, which wait for this
        // epilogue to release the accumulator below)
        if (!mbar_wait_warp(dsc_full + (k & 3), (k >> 2) & 1, p)) { ok = false; break; }
        float dsc[kTcDownPairs];
#pragma unroll
        for (int qq = 0; qq < kTcDownPairs; ++qq) dsc[qq] = s_dsc[(k & 3) * kTcDownPairs + qq];
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty + buf);
        if (it + 2 < all_tiles && !write_sf(it + 2)) { ok = false; break; }
        const int row = R * 128 + 32 * q + lane;
#pragma unroll
        for (int qq = 0; qq < kTcDownPairs; ++qq) {
          if (qq < np_t) {
            const float val = kFp8H ? __uint_as_float(v[qq]) * dsc[qq]
                                    : (__uint_as_float(v[2 * qq]) + __uint_as_float(v[2 * qq + 1]) * 0.0625f) * dsc[qq];
            tw.ypart[(size_t)(pb0 + qq) * H + row] = val;
          }
        }
        if (q == 0 && k == 0) tc_trace(p, 24);
        if (q == 0 && k == my_dtiles - 1) tc_trace(p, 25);
        continue;
      }
      const int t = b + it * G;
      const int f0 = t * tu, f1 = min(T, f0 + tu), nu = f1 - f0;
      const int buf = it & 1;
      if (!mbar_wait_warp(acc_full + buf, (it >> 1) & 1, p)) { ok = false; break; }
      if (q == 0 && it == my_tiles - 1) tc_trace(p, 48);
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + (uint32_t)(buf * kTcAccCols) + ((uint32_t)(32 * q) << 16), v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + buf);
      const int r = 32 * q + lane, g = r >> 3, i8 = r & 7;
      float upv[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) upv[c] = __shfl_down_sync(0xffffffffu, __uint_as_float(v[c]), 4);
      if (g < nu && i8 < 4) {
        const int f = f0 + g, u = f / upe, j = f % upe, n = 4 * j + i8;
        const int pb = s_poff[u], pe = s_poff[u + 1];
        for (int pp = pb; pp < pe; ++pp) {
          const int m = s_pm[pp];
          float gv = 0.f, uv = 0.f;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c == m) { gv = __uint_as_float(v[c]); uv = upv[c]; }
          gv *= s_xs[m];
          uv *= s_xs[m];
          tw.h[(size_t)pp * I + n] = gv / (1.f + expf(-gv)) * uv;
        }
      }
      // publish: the last of the four warps to finish the tile (CTA-scope
      // acq_rel counter, so it sees the others' stores) adds one to the
      // counter of every entry the tile touches, with release at GPU scope
      __syncwarp();
      if (q == 0 && it == my_tiles - 1) tc_trace(p, 49);
      if (lane == 0 && atom_add_acqrel_cta_smem(s_tdone + it, 1u) == 3u)
        for (int u = f0 / upe; u <= (f1 - 1) / upe; ++u) red_release_add_u32(hcnt + u * kTcCntStride, 1u);
      if (q == 0 && it == my_tiles - 1) tc_trace(p, 50);
      // the MMAs of tile it are complete: its scale-factor buffer takes tile
      // it+2. Only after the publish: tile it+2 may be a down tile, whose
      // scales the producer issues behind down stages that wait (through the
      // B operand) for every CTA's h, this one's included.
      if (it + 2 < all_tiles && !write_sf(it + 2)) { ok = false; break; }
    }
    if (pl.mma_down && ok) {
      // this CTA's down tiles are all in ypart: the last of the four warps
      // (CTA-scope acq_rel, so it sees the others' stores) counts the CTA in,
      // with release at GPU scope
      __syncwarp();
      if (lane == 0 && atom_add_acqrel_cta_smem(reinterpret_cast<unsigned*>(s_int + 5), 1u) == 3u)
        red_release_add_u32(tw.dcnt + (size_t)(epoch & 1) * kTcCntStride, 1u);
    }
    tc_trace(p, 7);
  }

  // ---------------- gatekeeper: one thread polls the entry counters in
  //   order (acquire, GPU scope) and raises each entry's flag in shared
  //   memory (release, CTA scope) once every tile covering it has published
  //   its h; the down items wait on the flags. One poller per CTA keeps the
  //   counters' L2 lines cool.
  if (warp == kTcWarpGate && lane == 0) {
    const long long t0 = clock64();
    for (int u = 0; u < U && ok; ++u) {
      const unsigned tiles = (unsigned)(((u + 1) * upe - 1) / tu - (u * upe) / tu + 1);
      const unsigned* c = hcnt + u * kTcCntStride;
      while (ld_acquire_u32g(c) < tiles) {
        __nanosleep(128);
        if (clock64() - t0 > p.spin_limit) {
          atomicOr(p.ws.ctrl, kStatusTimeout);
          ok = false;
          break;
        }
      }
      asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(s_hready + u)), "r"(1u) : "memory");
      if (u == 0) tc_trace(p, 30);
    }
    tc_trace(p, 31);
  }
  if (warp == kTcWarpGate) {
    __syncwarp();
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  }

  if (pl.mma_down) {
    // ---------------- tensor-core down: the builder warps turn each tile's
    //   pairs' h (read from L2 once the entry is complete on every CTA) into
    //   the B operand: per pair an fp32 scale amax/448 and E4M3 codes of
    //   h/scale (row 2q), plus (unless kFp8H) the codes of 16x the rounding
    //   residual (row 2q+1), so the MMA sums hi + lo/16, within 2^-8 of h.
    //   Then every CTA waits for all CTAs' tiles and combines its rows.
    if (warp >= kTcWarpBuild && ok) {
      const int wb = warp - kTcWarpBuild, nwb = kTcWarps - kTcWarpBuild;
      const int nf4 = I / 128;  // float4 of h per lane (I <= 1024)
      int du = 0;
      for (int k = 0; k < my_dtiles; ++k) {
        int g, R;
        dtile_of(b + k * G, du, g, R);
        const int pb0 = s_poff[du] + kTcDownPairs * g, np_t = min(kTcDownPairs, s_poff[du + 1] - pb0);
        const int bb = k & 1;
        if (!wait_flag_warp(p, s_hready + du)) { ok = false; break; }
        if (k >= 2 && !mbar_wait_warp(b_empty + bb, ((k >> 1) - 1) & 1, p)) { ok = false; break; }
        uint8_t* bdb = bd + (size_t)bb * pl.bd_bytes;
        for (int qq = wb; qq < np_t; qq += nwb) {
          const float4* hp = reinterpret_cast<const float4*>(tw.h + (size_t)(pb0 + qq) * I) + lane * nf4;
          float4 hv[8];
          float mx = 0.f;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            hv[t] = (t < nf4) ? __ldcg(hp + t) : make_float4(0.f, 0.f, 0.f, 0.f);
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(hv[t].x), fabsf(hv[t].y)), fmaxf(fabsf(hv[t].z), fabsf(hv[t].w))));
          }
          const float amax = warp_max(mx), inv = h_fp8_inv(amax);
          const int nhi = kFp8H ? qq : 2 * qq;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            if (t < nf4) {
              const int kk = (lane * nf4 + t) * 4;
              const float y0 = __fmul_rn(hv[t].x, inv), y1 = __fmul_rn(hv[t].y, inv);
              const float y2 = __fmul_rn(hv[t].z, inv), y3 = __fmul_rn(hv[t].w, inv);
              const uint32_t c01 = f32x2_to_e4m3x2(y0, y1), c23 = f32x2_to_e4m3x2(y2, y3);
              *reinterpret_cast<uint32_t*>(bdb + sw128_offset(nhi, kk, 4)) = c01 | (c23 << 16);
              if constexpr (!kFp8H) {
                const uint32_t h01 = e4m3x2_to_f16x2((uint16_t)c01), h23 = e4m3x2_to_f16x2((uint16_t)c23);
                const float2 q01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                const float2 q23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                const uint32_t l01 = f32x2_to_e4m3x2((y0 - q01.x) * 16.f, (y1 - q01.y) * 16.f);
                const uint32_t l23 = f32x2_to_e4m3x2((y2 - q23.x) * 16.f, (y3 - q23.y) * 16.f);
                *reinterpret_cast<uint32_t*>(bdb + sw128_offset(nhi + 1, kk, 4)) = l01 | (l23 << 16);
              }
            }
          }
          if (lane == 0) s_dsc[(k & 3) * kTcDownPairs + qq] = h_fp8_scale(amax);
        }
        // the codes are read by the tensor cores (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(b_full + bb);
          mbar_arrive(dsc_full + (k & 3));
        }
        if (k == 0) tc_trace(p, 51);
      }
      tc_trace(p, 52);
    }
    tc_trace(p, 10);
    // grid-wide: every CTA's down tiles are in ypart once the count reaches G
    if (tid == 0 && ok) {
      const unsigned* c = tw.dcnt + (size_t)(epoch & 1) * kTcCntStride;
      const long long t0 = clock64();
      while (ld_acquire_u32g(c) < (unsigned)G) {
        __nanosleep(128);
        if (clock64() - t0 > p.spin_limit) {
          atomicOr(p.ws.ctrl, kStatusTimeout);
          ok = false;
          break;
        }
      }
    }
    const bool all_ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_trace(p, 11);
    // ---- A8: combine in slot order, bf16 out (fp32 for one part of a split)
    for (int i = tid; i < M * nrd && all_ok; i += kTcThreads) {
      const int m = i / nrd, r = r0 + i % nrd;
      float acc = 0.f;
      for (int s = 0; s < K; ++s)
        acc = fmaf(s_w[m * K + s], __ldcg(tw.ypart + (size_t)s_ppos[m * K + s] * H + r), acc);
      if constexpr (kShared) acc += __ldcg(tw.ypart + (size_t)m * H + r);
      store_y(p, (size_t)m * H + r, acc);
    }
  } else {
    // ---------------- down (CUDA cores): every warp once its role is done.
    //   Items (entry, 9 output rows) in entry order; each waits for its
    //   entry's flag (h complete on every CTA) and its chunk.
    {
      const int per = d_items;
      const int total = U * per;
      for (;;) {
        if (!ok) break;  // a wait of this warp ran out: the step's output is lost anyway
        int it = 0;
        if (lane == 0) it = atomicAdd(&s_int[2], 1);
        it = __shfl_sync(0xffffffffu, it, 0);
        if (it >= total) break;
        const int u = it / per, gd = it - u * per;
        const int slot = u % pl.ns_d, use = u / pl.ns_d;
        const int pb = s_poff[u], pe = s_poff[u + 1];
        // the slot's previous use is fully consumed, so the parity waits
        // below cannot see an earlier phase
        if (use > 0 && lane == 0) smem_count_wait(done_d + slot, (unsigned)(use * per), p);
        __syncwarp();
        if (it == 0) tc_trace(p, 51);
        if (it == total - 1) tc_trace(p, 54);
        if (!wait_flag_warp(p, s_hready + u)) ok = false;
        if (u == U - 1 && gd == 0) tc_trace(p, 9);
        if (it == 0) tc_trace(p, 52);
        if (it == total - 1) tc_trace(p, 55);
        if (!mbar_wait_warp(full_d + slot, use & 1, p)) ok = false;
        if (it == 0) tc_trace(p, 53);
        if (it == total - 1) tc_trace(p, 56);
        DChunk ch;
        size_t sa0;
        unsigned sn;
        d_layout(p, s_union[u], r0, nrd, ring_d + (size_t)slot * pl.slot_d, &ch, &sa0, &sn);
        const int a = gd * kDownRowsPerItem, cnt = min(kDownRowsPerItem, nrd - a);
        tc_d_item<kFp8H>(p, tw, ch, a, cnt, pb, pe, dsm, pl.rpc_max, it == 0 ? 61 : -1);
        if (it == 0) tc_trace(p, 57);
        if (it == total - 1) tc_trace(p, 58);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(empty_d + slot);
          atomicAdd(done_d + slot, 1u);
        }
      }
      tc_trace(p, 10);
      __syncthreads();
      tc_trace(p, 11);
      // ---- A8: combine in slot order, bf16 out (fp32 for one part of a split)
      for (int i = tid; i < M * nrd; i += kTcThreads) {
        const int m = i / nrd, rl = i % nrd;
        float acc = 0.f;
        for (int s = 0; s < K; ++s) acc = fmaf(s_w[m * K + s], dsm[(size_t)s_ppos[m * K + s] * pl.rpc_max + rl], acc);
        if constexpr (kShared) acc += dsm[(size_t)m * pl.rpc_max + rl];
        store_y(p, (size_t)m * H + r0 + rl, acc);
      }
    }
  
  }

  // ---------------- teardown
  if (!ok) {
    // a wait ran out: copies may still be landing in shared memory
    const long long t1 = clock64();
    while (clock64() - t1 < 20000000ll) {}
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)pl.tmem_cols));
  }
  if (b == 0 && tid == 0) st_relaxed_u32(tw.epoch, epoch);
  tc_trace(p, 12);
}

}  // namespace moe
