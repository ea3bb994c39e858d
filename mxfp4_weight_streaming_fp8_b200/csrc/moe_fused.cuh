// moe_fused.cuh -- the whole decode step as one persistent kernel per layer.
//
// One CTA per SM (grid = SM count, 512 threads). A step is a chain of
// dependent phases (routing -> expert gate/up -> expert down). At batch 1 the
// time goes into streaming the weights from memory (MarkTechPost, "NVIDIA
// Shows 3 Ways to Speed Up MoE Inference on DGX Spark", section "Why is MoE
// decoding on DGX Spark memory-bound?"). So the
// kernel is built to start the weight stream as early as possible, and to
// leave only a short tail once the last byte arrives.
//
//  1. Before griddepcontrol.wait (programmatic dependent launch), each CTA
//     starts a TMA bulk copy of its slice of the router weights into shared
//     memory. Router weights never depend on the previous kernel.
//  2. Each CTA quantises all M tokens to E4M3 into shared memory (A1) and
//     computes the logits of its router rows (A2). Each logit goes to L2 as
//     one 64-bit word holding the launch epoch next to the fp32 value, so
//     the data is its own flag: there is no arrival counter.
//  3. Every CTA reads all M x E logit words until each carries this launch's
//     epoch (bounded, CTA-rotated order), and, redundantly, computes top-k,
//     softmax and the expert union (A3, A4) in shared memory.
//  4. The CTA streams its share of every union expert into two
//     shared-memory rings with TMA bulk copies:
//       - gate/up: intermediate rows [I*b/G, I*(b+1)/G) of each expert, i.e.
//         gate rows, up rows and their E8M0 scale bytes
//       - down: output rows [H*b/G, H*(b+1)/G) of each expert, with scales
//     Each active weight byte is read from HBM once, by one CTA. A bulk copy
//     costs its issuing thread about a hundred nanoseconds, so the first use
//     of every slot is issued by all 16 warps at once; refills of drained
//     slots come from one thread of warp 0 that polls both rings.
//  5. Warps 1..15 first drain an in-order queue of gate/up items (A5, A6):
//     for an expert with one or two (token, slot) pairs they decode E2M1 in
//     registers, run f16x2 FMAs on exact products per pair, apply
//     the E8M0 scale in fp32, then SwiGLU, and write h to L2. An expert
//     with three or more pairs splits K over its items instead: each runs
//     warp MMAs (m16n8k16, f16) over all rows and pairs, so a weight is
//     decoded once, and the last item sums the partials. When a CTA has
//     finished entry u, it arrives on that entry's grid counter. Then they
//     drain an in-order queue of down items (A7). The first down item of u
//     waits on the counter and stages h once into shared memory for the CTA;
//     the other items of u wait for that.
//  6. Each CTA combines its output rows in slot order (A8) and writes bf16 y
//     (fp32 partial sums for one part of an intra-expert split).
//
// Every wait is bounded: on timeout the kernel sets the status word and goes
// on (with garbage results) instead of hanging. moe_sync_status reports it.
#pragma once

#include "moe_device.cuh"

namespace moe {

constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kConsumers = kFusedWarps - 1;  // warp 0 produces
constexpr int kDownLag = 8;                 // down items of entry k follow the gate/up items of entry k + kDownLag
constexpr int kGuRowsPerItem = 2;           // intermediate rows per gate/up item
constexpr int kDownRowsPerItem = 9;         // output rows per down item (two items per expert at 17-18 rows per CTA)
constexpr int kHPairs = 4;                  // (token, slot) pairs of one expert whose h is staged in smem
constexpr int kMaxRowsPerCta = 8;           // router rows a CTA may own (E <= 8 * G)
constexpr int kMaxSlots = 64;
constexpr int kMaxPairTiles = 4;            // 8-pair MMA column tiles per entry (32 pairs)
constexpr int kMmaMinPairs = 3;             // entries with at least this many pairs take the MMA gate/up path
constexpr int kCounterStride = 16;          // u64 words between per-entry counters (one 128-byte line)
constexpr int kSkMaxTokens = 4;             // split-K down: tokens per call (partial y of a CTA in smem)
constexpr int kSkRowsPerLane = 8;           // split-K down: output rows per lane of a chunk (one code word)
constexpr int kSkChunk = 32 * kSkRowsPerLane;  // output rows per down chunk

// Launch-invariant plan computed on the host at moe_create.
struct FusedPlan {
  int G;                // grid size (CTAs)
  int max_tokens, max_pairs, max_union;
  int slot_gu, slot_d;  // bytes per ring slot
  int ns_gu, ns_d;      // slots per ring
  int rpc_max;          // max output rows per CTA
  int hslot;            // bytes of staged h per down slot
  int hpairs;           // pairs staged per down slot (min(kHPairs, max_tokens))
  // shared memory offsets (bytes)
  int o_bar, o_misc, o_ids, o_w, o_pm, o_ppos, o_union, o_poff, o_cnt, o_act, o_dsm, o_h, o_part, o_ring_gu, o_ring_d;
  int part_slot;        // bytes of MMA partials per gate/up slot (0: one token, never used)
  int part_ct;          // 8-pair column tiles a slot's partials hold (min(kMaxPairTiles, max_tokens / 8 rounded up))
  int smem_bytes;
  int wr_bytes_max;     // router rows staged per CTA (alias ring_gu)
  int x_staged;         // bf16 x fits in ring_d and is staged there during routing
  // split-K down (kSplitK): CTA-local h [max_union][max_tokens][nr_max],
  // partial y [max_tokens][H], per-chunk entry progress, pair weights
  int nr_max, dchunks, o_hsm, o_ycta, o_chunk, o_pw;
};

// Workspace pieces only the persistent kernel uses.
struct FusedWs {
  unsigned long long* logits;     // [maxM][E] tagged router logits (epoch, fp32)
  unsigned long long* gu_cnt;     // [max_union][kCounterStride] gate/up arrivals per entry; += G per launch
  unsigned* epoch;                // launch counter
  float* ypart;                   // split-K: [G][max_tokens][H] partial y of every CTA
  unsigned long long* fin_cnt;    // split-K: partial-y arrivals; += G per launch
};

// Counter of union entry u, alone on its L2 line.
__host__ __device__ __forceinline__ unsigned long long* gu_counter(const FusedWs& fw, int u) {
  return fw.gu_cnt + (size_t)u * kCounterStride;
}

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// try_wait with a suspend-time hint: a waiting thread is parked (up to the
// hint) until the phase completes instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(20000u) : "memory");
  return ok != 0;
}

// Non-blocking test of an mbarrier phase (no suspension).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase; on timeout sets the status word.
__device__ __forceinline__ void mbar_wait(uint64_t* bar, unsigned parity, const Params& p) {
  if (mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > p.spin_limit) {
      atomicOr(p.ws.ctrl, kStatusTimeout);
      return;
    }
  }
}

// 1-D TMA bulk copy global -> shared, completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16. (No L2 eviction hint: an
// evict-first policy measured slower on this stream.)
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u32(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long atom_add_acqrel_u64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acqrel_cta_smem(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
  return old;
}

// CTA-scope release/acquire on a shared-memory word (a ready flag).
__device__ __forceinline__ void st_release_cta_smem(unsigned* p, unsigned v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_cta_smem(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
// Wait (one thread) until a shared-memory word written with a CTA-scope
// release reaches `target`; acquire, so the writer's earlier stores are
// visible after it returns.
__device__ __forceinline__ void smem_acquire_wait(const unsigned* c, unsigned target, const Params& p) {
  if (ld_acquire_cta_smem(c) >= target) return;
  const long long t0 = clock64();
  while (ld_acquire_cta_smem(c) < target) {
    __nanosleep(32);
    if (clock64() - t0 > p.spin_limit) {
      atomicOr(p.ws.ctrl, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Grid-wide completion points are monotonic 64-bit counters that gain G per
// launch: a CTA arrives with a fire-and-forget release add, and a waiter
// polls the counter with acquire loads until it reaches epoch * G. (Measured
// on B200 with 148 CTAs: about 1.35 us per barrier. A returning acq_rel
// atomic with a last-arriver flag took about 4.7 us; per-CTA flag words
// polled by a warp took about 2.4 us.)
__device__ __forceinline__ void grid_arrive(unsigned long long* cnt) { red_release_add_u64(cnt, 1ull); }

// One thread waits until *cnt >= target, with a short sleep between polls;
// bounded by the wait budget.
__device__ __forceinline__ void grid_wait(const unsigned long long* cnt, unsigned long long target, const Params& p) {
  if (ld_acquire_u64(cnt) >= target) return;
  const long long t0 = clock64();
  while (ld_acquire_u64(cnt) < target) {
    __nanosleep(32);
    if (clock64() - t0 > p.spin_limit) {
      atomicOr(p.ws.ctrl, kStatusTimeout);
      return;
    }
  }
}

// Whole warp: wait (lane 0 polls, bounded) until a shared-memory flag is set;
// false, with the status bit set, when the wait ran out.
__device__ __forceinline__ bool wait_flag_warp(const Params& p, const unsigned* flag) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0 && ld_acquire_cta_smem(flag) == 0u) {
    const long long t0 = clock64();
    while (ld_acquire_cta_smem(flag) == 0u) {
      __nanosleep(32);
      if (clock64() - t0 > p.spin_limit) {
        atomicOr(p.ws.ctrl, kStatusTimeout);
        ok = false;
        break;
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Wait (one thread) until a shared-memory count reaches `target`.
__device__ __forceinline__ void smem_count_wait(const unsigned* c, unsigned target, const Params& p) {
  const volatile unsigned* v = c;
  if (*v >= target) return;
  const long long t0 = clock64();
  while (*v < target) {
    __nanosleep(32);
    if (clock64() - t0 > p.spin_limit) {
      atomicOr(p.ws.ctrl, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers * 32) : "memory");
}

__device__ __forceinline__ uint4 ld_cg_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// ---------------------------------------------------------------- geometry
// Bytes of the 16-aligned superset copied for scale bytes [a, b).
__device__ __forceinline__ void round16(size_t a, size_t b, size_t* a0, unsigned* n) {
  *a0 = a & ~size_t(15);
  *n = (unsigned)(((b + 15) & ~size_t(15)) - *a0);
}

struct GuChunk {  // gate/up slice of one union expert in smem
  const uint8_t* gc;  // gate codes  [nr][H/2]
  const uint8_t* uc;  // up codes    [nr][H/2]
  const uint8_t* gs;  // gate scales [nr][H/32]
  const uint8_t* us;  // up scales
};

// Layout of gate/up chunk `e` (rows n0..n0+nr-1) inside a slot, mirrored by
// the producer and the consumers.
__device__ __forceinline__ unsigned gu_layout(const Params& p, int e, int n0, int nr, uint8_t* slot,
                                              GuChunk* c, size_t* gsa0, unsigned* gsn, size_t* usa0,
                                              unsigned* usn) {
  const size_t H = p.H, I = p.I;
  const size_t grow = (size_t)e * 2 * I + n0, urow = grow + I;
  const size_t gsa = grow * (H / 32), gsb = gsa + nr * (H / 32);
  const size_t usa = urow * (H / 32), usb = usa + nr * (H / 32);
  round16(gsa, gsb, gsa0, gsn);
  round16(usa, usb, usa0, usn);
  const unsigned codes = (unsigned)(nr * H / 2);
  c->gc = slot;
  c->uc = slot + codes;
  c->gs = slot + 2 * codes + (gsa - *gsa0);
  c->us = slot + 2 * codes + *gsn + (usa - *usa0);
  return 2 * codes + *gsn + *usn;
}

struct DChunk {
  const uint8_t* c;  // down codes  [nr][I/2]
  const uint8_t* s;  // down scales [nr][I/32]
};

__device__ __forceinline__ unsigned d_layout(const Params& p, int e, int r0, int nr, uint8_t* slot,
                                             DChunk* c, size_t* sa0, unsigned* sn) {
  const size_t H = p.H, I = p.I;
  const size_t row = (size_t)e * H + r0;
  const size_t sa = row * (I / 32), sb = sa + nr * (I / 32);
  round16(sa, sb, sa0, sn);
  const unsigned codes = (unsigned)(nr * I / 2);
  c->c = slot;
  c->s = slot + codes + (sa - *sa0);
  return codes + *sn;
}

// ---------------------------------------------------------------- compute items
// Gate/up item: rows [a, a+cnt) of the chunk (local index), every pair of the
// expert. Lane owns half-blocks hb = lane + 32j (16 elements, 8 code bytes).
// Products E2M1 x E4M3 are exact in f16; each f16x2 half sums 8 of them
// (|sum| <= 8*6*448 = 21504) before the fp32 block-scale FMA.
__device__ __forceinline__ void gu_item(const Params& p, const GuChunk& ch, int a, int cnt, float* hout,
                                        size_t hstride, int pb, int pe, const int* s_pm, const uint8_t* act,
                                        const float* s_xs) {
  const int lane = threadIdx.x & 31;
  const int H = p.H, nhb = H / 16;
  for (int pp = pb; pp < pe; ++pp) {
    const int m = s_pm[pp];
    const uint8_t* am = act + (size_t)m * H;
    float ag[kGuRowsPerItem], au[kGuRowsPerItem];
#pragma unroll
    for (int r = 0; r < kGuRowsPerItem; ++r) ag[r] = au[r] = 0.f;
#pragma unroll 2
    for (int hb = lane; hb < nhb; hb += 32) {
      const uint4 aq = *reinterpret_cast<const uint4*>(am + hb * 16);  // 16 E4M3 codes
      uint32_t a2[8];
      const uint32_t aw[4] = {aq.x, aq.y, aq.z, aq.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a2[2 * t] = e4m3x2_to_f16x2((uint16_t)(aw[t] & 0xFFFFu));
        a2[2 * t + 1] = e4m3x2_to_f16x2((uint16_t)(aw[t] >> 16));
      }
#pragma unroll
      for (int r = 0; r < kGuRowsPerItem; ++r) {
        if (r < cnt) {
          const int row = a + r;
          const uint2 cg = *reinterpret_cast<const uint2*>(ch.gc + (size_t)row * (H / 2) + hb * 8);
          const uint2 cu = *reinterpret_cast<const uint2*>(ch.uc + (size_t)row * (H / 2) + hb * 8);
          const float sg = e8m0_to_f32(ch.gs[(size_t)row * (H / 32) + (hb >> 1)]);
          const float su = e8m0_to_f32(ch.us[(size_t)row * (H / 32) + (hb >> 1)]);
          uint32_t wg[8], wu[8];
          e2m1x8_to_f16x2x4(cg.x, wg);
          e2m1x8_to_f16x2x4(cg.y, wg + 4);
          e2m1x8_to_f16x2x4(cu.x, wu);
          e2m1x8_to_f16x2x4(cu.y, wu + 4);
          __half2 hg0 = __float2half2_rn(0.f), hu0 = hg0, hg1 = hg0, hu1 = hg0;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const __half2 av0 = *reinterpret_cast<const __half2*>(&a2[t]);
            const __half2 av1 = *reinterpret_cast<const __half2*>(&a2[t + 4]);
            hg0 = __hfma2(*reinterpret_cast<const __half2*>(&wg[t]), av0, hg0);
            hu0 = __hfma2(*reinterpret_cast<const __half2*>(&wu[t]), av0, hu0);
            hg1 = __hfma2(*reinterpret_cast<const __half2*>(&wg[t + 4]), av1, hg1);
            hu1 = __hfma2(*reinterpret_cast<const __half2*>(&wu[t + 4]), av1, hu1);
          }
          const float2 fg0 = __half22float2(hg0), fu0 = __half22float2(hu0);
          const float2 fg1 = __half22float2(hg1), fu1 = __half22float2(hu1);
          ag[r] = fmaf(sg, (fg0.x + fg0.y) + (fg1.x + fg1.y), ag[r]);
          au[r] = fmaf(su, (fu0.x + fu0.y) + (fu1.x + fu1.y), au[r]);
        }
      }
    }
    const float s = s_xs[m];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
#pragma unroll
      for (int r = 0; r < kGuRowsPerItem; ++r) {
        ag[r] += __shfl_xor_sync(0xffffffffu, ag[r], o);
        au[r] += __shfl_xor_sync(0xffffffffu, au[r], o);
      }
    }
#pragma unroll
    for (int r = 0; r < kGuRowsPerItem; ++r) {
      const float g = ag[r] * s, u = au[r] * s;
      if (lane == 0 && r < cnt) hout[(size_t)(pp - pb) * hstride + a + r] = g / (1.f + expf(-g)) * u;
    }
  }
}

// D = A(16x16, f16, row) * B(16x8, f16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1,
                                              const float c[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
        "f"(c[3]));
}

// Gate/up of an expert with several (token, slot) pairs: warp MMAs
// (m16n8k16, f16 x f16 -> fp32) decode each weight once for all pairs. The
// A tile's rows 0..7 are gate rows r0g.. of the chunk and rows 8..15 the up
// rows with the same index (nrg <= 8 valid); the B tile's 8 columns are
// pairs pb + 8*ct.. (up to kMaxPairTiles tiles). Within each 32-element
// scale block lane (g, t) supplies elements 8t..8t+7: 8t+4s+{0,1} as the K
// positions 2t, 2t+1 of step s and 8t+4s+{2,3} as 2t+8, 2t+9, for A and B
// alike, so each product pairs the same element; E2M1 and E4M3 are exact in
// f16. Each scale block is a fresh two-step MMA scaled in fp32 by the E8M0
// scales of gate row g and up row g. acc[4*ct + i]: gate (i = 0, 1) and up
// (i = 2, 3) of row g for pairs pb + 8*ct + 2t + (i & 1).
__device__ __forceinline__ void gu_mma_slice(const Params& p, const GuChunk& ch, int r0g, int nrg, int kb0, int kb1,
                                             int pb, int pe, const int* s_pm, const uint8_t* act,
                                             float acc[4 * kMaxPairTiles]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int H = p.H, hs = H / 32;
  const int np = pe - pb, nct = min(kMaxPairTiles, (np + 7) >> 3);
  const bool rv = g < nrg;
  const uint8_t* gc = ch.gc + (size_t)(r0g + g) * (H / 2) + 4 * t;
  const uint8_t* uc = ch.uc + (size_t)(r0g + g) * (H / 2) + 4 * t;
  const uint8_t* gs = ch.gs + (size_t)(r0g + g) * hs;
  const uint8_t* us = ch.us + (size_t)(r0g + g) * hs;
  const uint8_t* br[kMaxPairTiles];
#pragma unroll
  for (int ct = 0; ct < kMaxPairTiles; ++ct) {
    const int q = 8 * ct + g;
    br[ct] = (q < np) ? act + (size_t)s_pm[pb + q] * H + 8 * t : nullptr;
  }
#pragma unroll
  for (int i = 0; i < 4 * kMaxPairTiles; ++i) acc[i] = 0.f;
  const float z[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kb = kb0; kb < kb1; ++kb) {
    uint32_t fg[4] = {0u, 0u, 0u, 0u}, fu[4] = {0u, 0u, 0u, 0u};
    float sg = 0.f, su = 0.f;
    if (rv) {
      e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(gc + kb * 16), fg);
      e2m1x8_to_f16x2x4(*reinterpret_cast<const uint32_t*>(uc + kb * 16), fu);
      sg = e8m0_to_f32(gs[kb]);
      su = e8m0_to_f32(us[kb]);
    }
    const uint32_t a0[4] = {fg[0], fu[0], fg[1], fu[1]};
    const uint32_t a1[4] = {fg[2], fu[2], fg[3], fu[3]};
#pragma unroll
    for (int ct = 0; ct < kMaxPairTiles; ++ct) {
      if (ct >= nct) break;
      uint4 bv = make_uint4(0u, 0u, 0u, 0u);
      if (br[ct]) {
        const uint2 c = *reinterpret_cast<const uint2*>(br[ct] + kb * 32);
        bv = make_uint4(e4m3x2_to_f16x2((uint16_t)(c.x & 0xFFFFu)), e4m3x2_to_f16x2((uint16_t)(c.x >> 16)),
                        e4m3x2_to_f16x2((uint16_t)(c.y & 0xFFFFu)), e4m3x2_to_f16x2((uint16_t)(c.y >> 16)));
      }
      float d[4];
      mma_f16_16816(d, a0, bv.x, bv.y, z);
      mma_f16_16816(d, a1, bv.z, bv.w, d);
      acc[4 * ct + 0] = fmaf(d[0], sg, acc[4 * ct + 0]);
      acc[4 * ct + 1] = fmaf(d[1], sg, acc[4 * ct + 1]);
      acc[4 * ct + 2] = fmaf(d[2], su, acc[4 * ct + 2]);
      acc[4 * ct + 3] = fmaf(d[3], su, acc[4 * ct + 3]);
    }
  }
}

// Power-of-two rescale that maps max|h| of one pair vector below 2^9, so
// f16 partial sums of 8 E2M1 x h' products stay below 8*6*2^9 = 24576.
__device__ __forceinline__ int h_rescale_exp(float mx) {
  int ex = 0;
  if (mx > 0.f) frexpf(mx, &ex);  // mx in [2^(ex-1), 2^ex)
  return min(126, 9 - ex);
}

// FP8 intermediate (kFp8H): h of a pair is quantised like the activations
// before the down projection (the W4A8 recipe on "NVIDIA Shows 3 Ways to
// Speed Up MoE Inference on DGX Spark", section "Why is MoE decoding on DGX
// Spark memory-bound?", read as 8-bit inputs for both projections): over the
// pair's I elements, amax = max|h|, inv = fl32(448/amax), code =
// E4M3_RNE_sat(fl32(h*inv)), scale fl32(amax/448) (amax == 0: zero codes,
// scale 1). The codes' values are exact in f16, so the down path's f16
// products stay exact.
__device__ __forceinline__ uint32_t h_fp8x2(float a, float b, float inv) {
  return e4m3x2_to_f16x2(f32x2_to_e4m3x2(__fmul_rn(a, inv), __fmul_rn(b, inv)));
}
__device__ __forceinline__ float h_fp8_inv(float amax) { return amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f; }
__device__ __forceinline__ float h_fp8_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }

// Stage h of the pairs [pb, pe) of one expert (pe - pb <= kHPairs) into
// shared memory as f16, each pair vector rescaled by 2^t, with 2^-t kept in
// hscale (kFp8H: as E4M3 values, with the pair's FP8 scale in hscale). One
// warp; h is read from L2 (written by other CTAs).
template <bool kFp8H>
__device__ __forceinline__ void stage_h(const Params& p, int pb, int pe, __half2* hbuf, float* hscale) {
  const int lane = threadIdx.x & 31;
  const int I = p.I;
  constexpr int kQ = 8;  // uint4 per lane kept in registers: one L2 pass when I <= 1024
  for (int pp = pb; pp < pe; ++pp) {
    const int j = pp - pb;
    const uint4* hp = reinterpret_cast<const uint4*>(p.ws.h + (size_t)pp * I);
    __half2* dst = hbuf + (size_t)j * (I / 2);
    if (I / 4 <= 32 * kQ) {
      // lane's groups q = (lane + 32k + rot) mod I/4: the start rotates with
      // the CTA, so the 148 CTAs that stage an expert's h together spread
      // their first reads over its L2 lines instead of all asking for the
      // same line at once
      const int nq = I / 4, rot = (int)((blockIdx.x * 8u) % (unsigned)nq);
      uint4 v[kQ];
      float mx = 0.f;
#pragma unroll
      for (int k = 0; k < kQ; ++k) {
        const int q0 = lane + 32 * k, q = (q0 + rot >= nq) ? q0 + rot - nq : q0 + rot;
        v[k] = (q0 < nq) ? ld_cg_u4(hp + q) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < kQ; ++k)
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(__uint_as_float(v[k].x)), fabsf(__uint_as_float(v[k].y))),
                             fmaxf(fabsf(__uint_as_float(v[k].z)), fabsf(__uint_as_float(v[k].w)))));
      if constexpr (kFp8H) {
        const float amax = warp_max(mx), inv = h_fp8_inv(amax);
#pragma unroll
        for (int k = 0; k < kQ; ++k) {
          const int q0 = lane + 32 * k, q = (q0 + rot >= nq) ? q0 + rot - nq : q0 + rot;
          if (q0 < nq) {
            uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + 2 * q);
            d32[0] = h_fp8x2(__uint_as_float(v[k].x), __uint_as_float(v[k].y), inv);
            d32[1] = h_fp8x2(__uint_as_float(v[k].z), __uint_as_float(v[k].w), inv);
          }
        }
        if (lane == 0) hscale[j] = h_fp8_scale(amax);
      } else {
        const int t = h_rescale_exp(warp_max(mx));
        const float up = ldexpf(1.f, t);
#pragma unroll
        for (int k = 0; k < kQ; ++k) {
          const int q0 = lane + 32 * k, q = (q0 + rot >= nq) ? q0 + rot - nq : q0 + rot;
          if (q0 < nq) {
            dst[2 * q] = __floats2half2_rn(__uint_as_float(v[k].x) * up, __uint_as_float(v[k].y) * up);
            dst[2 * q + 1] = __floats2half2_rn(__uint_as_float(v[k].z) * up, __uint_as_float(v[k].w) * up);
          }
        }
        if (lane == 0) hscale[j] = ldexpf(1.f, -t);
      }
    } else {
      // wide intermediate: one pass for the max, one to convert
      float mx = 0.f;
      for (int q = lane; q < I / 4; q += 32) {
        const uint4 v = ld_cg_u4(hp + q);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                             fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
      }
      if constexpr (kFp8H) {
        const float amax = warp_max(mx), inv = h_fp8_inv(amax);
        for (int q = lane; q < I / 4; q += 32) {
          const uint4 v = ld_cg_u4(hp + q);
          uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + 2 * q);
          d32[0] = h_fp8x2(__uint_as_float(v.x), __uint_as_float(v.y), inv);
          d32[1] = h_fp8x2(__uint_as_float(v.z), __uint_as_float(v.w), inv);
        }
        if (lane == 0) hscale[j] = h_fp8_scale(amax);
      } else {
        const int t = h_rescale_exp(warp_max(mx));
        const float up = ldexpf(1.f, t);
        for (int q = lane; q < I / 4; q += 32) {
          const uint4 v = ld_cg_u4(hp + q);
          dst[2 * q] = __floats2half2_rn(__uint_as_float(v.x) * up, __uint_as_float(v.y) * up);
          dst[2 * q + 1] = __floats2half2_rn(__uint_as_float(v.z) * up, __uint_as_float(v.w) * up);
        }
        if (lane == 0) hscale[j] = ldexpf(1.f, -t);
      }
    }
  }
}

// Down rows [a, a+cnt) of one chunk for one pair, given the lane's block of
// the pair's rescaled h (h2, 16 f16x2) and its inverse scale; accumulates
// into dsm[pp][row] (fresh when `first`).
__device__ __forceinline__ void d_rows(const Params& p, const DChunk& ch, int a, int cnt, int blk, const uint32_t* h2,
                                       float down, float* dsm_pp, bool first) {
  const int lane = threadIdx.x & 31;
  const int I = p.I, nblk = I / 32;
  float part[kDownRowsPerItem];
#pragma unroll
  for (int r = 0; r < kDownRowsPerItem; ++r) {
    part[r] = 0.f;
    if (r < cnt && blk < nblk) {
      const int row = a + r;
      const uint4 c = *reinterpret_cast<const uint4*>(ch.c + (size_t)row * (I / 2) + blk * 16);
      const float sc = e8m0_to_f32(ch.s[(size_t)row * (I / 32) + blk]);
      const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
      __half2 acc0 = __float2half2_rn(0.f), acc1 = acc0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
        e2m1x8_to_f16x2x4(cw[q], w);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 wv = *reinterpret_cast<const __half2*>(&w[j]);
          const __half2 hv = *reinterpret_cast<const __half2*>(&h2[q * 4 + j]);
          if (q < 2) acc0 = __hfma2(wv, hv, acc0); else acc1 = __hfma2(wv, hv, acc1);
        }
      }
      const float2 f0 = __half22float2(acc0), f1 = __half22float2(acc1);
      part[r] = sc * ((f0.x + f0.y) + (f1.x + f1.y));
    }
  }
  // the rows' reductions are independent: interleave their shuffle rounds
#pragma unroll
  for (int o = 16; o; o >>= 1) {
#pragma unroll
    for (int r = 0; r < kDownRowsPerItem; ++r) part[r] += __shfl_xor_sync(0xffffffffu, part[r], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < kDownRowsPerItem; ++r)
      if (r < cnt) dsm_pp[a + r] = (first ? 0.f : dsm_pp[a + r]) + part[r] * down;
  }
}

// Down item: rows [a, a+cnt) for every pair of the expert; h from the staged
// shared-memory copy when the expert has at most `hpairs` pairs, else read
// and rescaled (kFp8H: quantised) here from L2.
template <bool kFp8H>
__device__ __forceinline__ void d_item(const Params& p, const DChunk& ch, int a, int cnt, int pb, int pe,
                                       const __half2* hbuf, const float* hscale, int hpairs, float* dsm, int rpc) {
  const int lane = threadIdx.x & 31;
  const int I = p.I, nblk = I / 32;
  const bool staged = (pe - pb) <= hpairs;
  for (int pp = pb; pp < pe; ++pp) {
    for (int b0 = 0; b0 < nblk; b0 += 32) {
      const int blk = b0 + lane;
      uint32_t h2[16];
      float down;
      if (staged) {
        const uint4* src = reinterpret_cast<const uint4*>(hbuf + (size_t)(pp - pb) * (I / 2)) + blk * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = (blk < nblk) ? src[q] : make_uint4(0u, 0u, 0u, 0u);
          h2[4 * q] = v.x; h2[4 * q + 1] = v.y; h2[4 * q + 2] = v.z; h2[4 * q + 3] = v.w;
        }
        down = hscale[pp - pb];
      } else {
        const float* hp = p.ws.h + (size_t)pp * I;
        float hv[32];
        float mx = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const uint4 q = (blk < nblk) ? ld_cg_u4(hp + blk * 32 + t * 4) : make_uint4(0u, 0u, 0u, 0u);
          hv[4 * t] = __uint_as_float(q.x); hv[4 * t + 1] = __uint_as_float(q.y);
          hv[4 * t + 2] = __uint_as_float(q.z); hv[4 * t + 3] = __uint_as_float(q.w);
        }
        if (nblk <= 32) {
#pragma unroll
          for (int t = 0; t < 32; ++t) mx = fmaxf(mx, fabsf(hv[t]));
        } else {
          // the rescale must cover the whole vector: reduce over all passes
          for (int b1 = 0; b1 < nblk; b1 += 32) {
            const int bk = b1 + lane;
            if (bk < nblk)
              for (int t = 0; t < 32; ++t) mx = fmaxf(mx, fabsf(__ldcg(hp + bk * 32 + t)));
          }
        }
        if constexpr (kFp8H) {
          const float amax = warp_max(mx), inv = h_fp8_inv(amax);
          down = h_fp8_scale(amax);
#pragma unroll
          for (int q = 0; q < 16; ++q) h2[q] = h_fp8x2(hv[2 * q], hv[2 * q + 1], inv);
        } else {
          const int t = h_rescale_exp(warp_max(mx));
          const float up = ldexpf(1.f, t);
          down = ldexpf(1.f, -t);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            __half2 v = __floats2half2_rn(hv[2 * q] * up, hv[2 * q + 1] * up);
            h2[q] = *reinterpret_cast<uint32_t*>(&v);
          }
        }
      }
      d_rows(p, ch, a, cnt, blk, h2, down, dsm + (size_t)pp * rpc, b0 == 0);
      __syncwarp();
    }
  }
}

// Split-K down chunk: output rows [c*kSkChunk, (c+1)*kSkChunk) of one entry
// over this CTA's K slice [n0, n0+nr): lane owns rows r..r+7 (one code word
// per K row). slot: codes [nr][H/2] (K-major, byte j = rows 2j, 2j+1), then
// scale rows [nskb][H] of the 32-blocks from skb0. hu[q * hstride + j] is
// h of pair pb + q at K row n0 + j. Adds w * partial into the CTA's
// partial y of each pair's token.
__device__ __forceinline__ void sk_down_chunk(const Params& p, const uint8_t* slot, int n0, int nr, int skb0, int c,
                                              int pb, int pe, const float* hu, int hstride, const int* s_pm,
                                              const float* s_pw, float* ycta) {
  const int lane = threadIdx.x & 31, H = p.H;
  const int r = c * kSkChunk + lane * kSkRowsPerLane;
  if (r >= H) return;  // H % 8 == 0: a lane's rows are all in range or all out
  const uint8_t* codes = slot;
  const uint8_t* scl = slot + (size_t)nr * (H / 2);
  const int np = pe - pb;
  float acc[kSkMaxTokens][kSkRowsPerLane];
#pragma unroll
  for (int q = 0; q < kSkMaxTokens; ++q)
#pragma unroll
    for (int i = 0; i < kSkRowsPerLane; ++i) acc[q][i] = 0.f;
  for (int j = 0; j < nr; ++j) {
    const uint32_t cw = *reinterpret_cast<const uint32_t*>(codes + (size_t)j * (H / 2) + r / 2);
    const uint2 sw = *reinterpret_cast<const uint2*>(scl + (size_t)((n0 + j) / 32 - skb0) * H + r);
    uint32_t f[4];
    e2m1x8_to_f16x2x4(cw, f);
    const uint32_t sb[2] = {sw.x, sw.y};
    float wv[kSkRowsPerLane];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&f[t]));
      wv[2 * t] = v.x * e8m0_to_f32((sb[t >> 1] >> (16 * (t & 1))) & 0xFFu);
      wv[2 * t + 1] = v.y * e8m0_to_f32((sb[t >> 1] >> (16 * (t & 1) + 8)) & 0xFFu);
    }
#pragma unroll
    for (int q = 0; q < kSkMaxTokens; ++q) {
      if (q < np) {
        const float hv = hu[(size_t)q * hstride + j];
#pragma unroll
        for (int i = 0; i < kSkRowsPerLane; ++i) acc[q][i] = fmaf(wv[i], hv, acc[q][i]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kSkMaxTokens; ++q) {
    if (q < np) {
      const float w = s_pw[pb + q];
      float4* yr = reinterpret_cast<float4*>(ycta + (size_t)s_pm[pb + q] * H + r);
      float4 y0 = yr[0], y1 = yr[1];
      y0.x = fmaf(w, acc[q][0], y0.x); y0.y = fmaf(w, acc[q][1], y0.y);
      y0.z = fmaf(w, acc[q][2], y0.z); y0.w = fmaf(w, acc[q][3], y0.w);
      y1.x = fmaf(w, acc[q][4], y1.x); y1.y = fmaf(w, acc[q][5], y1.y);
      y1.z = fmaf(w, acc[q][6], y1.z); y1.w = fmaf(w, acc[q][7], y1.w);
      yr[0] = y0;
      yr[1] = y1;
    }
  }
}

// ---------------------------------------------------------------- routing
// One warp: top-k of E logits (shared memory), ranked by value with ties to
// the lower index, and the softmax over the k kept. Lane l holds experts
// l + 32j, j < NJ (NJ = ceil(E/32) rounded up to a power of two).
template <int NJ>
__device__ __forceinline__ void topk_warp(const float* l, int E, int K, int* ids, float* w) {
  const int lane = threadIdx.x & 31;
  float v[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? l[e] : -INFINITY;
  }
  uint32_t taken = 0;
  float sel_v = 0.f, top = 0.f;
  int sel_i = 0;
  for (int r = 0; r < K; ++r) {
    // lane-local best among the lane's untaken experts (ascending index, so
    // a strictly greater value is needed to replace)
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      const bool ok = e < E && !((taken >> j) & 1u);
      if (ok && (v[j] > bv || bi == 0x7fffffff)) {
        bv = v[j];
        bi = e;
      }
    }
    // warp-wide: largest value (order-preserving integer image of the
    // float), then the lowest expert index holding it
    const unsigned u = __float_as_uint(bv);
    const unsigned key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    const unsigned kmax = __reduce_max_sync(0xffffffffu, key);
    const int win = (int)__reduce_min_sync(0xffffffffu, (unsigned)((key == kmax) ? bi : 0x7fffffff));
    const unsigned ub = (kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax;
    const float wv = __uint_as_float(ub);
    if ((win & 31) == lane) taken |= 1u << (win >> 5);
    if (r == 0) top = wv;
    if (lane == r) {
      sel_v = wv;
      sel_i = win;
    }
  }
  const float ex = (lane < K) ? expf(sel_v - top) : 0.f;
  const float z = warp_sum(ex);
  if (lane < K) {
    ids[lane] = sel_i;
    w[lane] = ex / z;
  }
}

// Router logit exchange word: the launch's epoch in the high half, the fp32
// logit in the low half. A reader that sees its own epoch has the value of
// this launch (one 64-bit store is single-copy atomic), so the word is its
// own ready flag.
__device__ __forceinline__ unsigned long long tag_word(unsigned epoch, float v) {
  return ((unsigned long long)epoch << 32) | __float_as_uint(v);
}

// Order-preserving 32-bit image of a float, and back.
__device__ __forceinline__ unsigned fkey(float v) {
  const unsigned u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_value(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k (K <= 8) of one token's E <= 512 logits with every warp of the CTA.
// Order: larger logit first, ties to the lower expert. Warp w ranks experts
// 32w..32w+31 among themselves (each lane counts the keys ahead of its own
// over the warp's shuffles) and keeps its K best; then every kept candidate
// counts the candidates ahead of it over all warps (several threads per
// candidate), and the K of rank < K are the result in order; warp 0 forms
// the softmax over them. Same result as topk_warp; all threads must call it.
// s_ck, s_ce: 136 words each (W*8 <= 128 candidates, then the K results).
__device__ void topk_cta_small(const float* l, int E, int K, int* ids, float* wts, unsigned* s_ck, int* s_ce,
                               const Params& p_trace) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = (E + 31) / 32;
  if (warp < W) {
    const int e = 32 * warp + lane;
    const unsigned key = (e < E) ? fkey(l[e]) : 0u;  // 0 is below every float's key
    int rank = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const unsigned kj = __shfl_sync(0xffffffffu, key, j);
      rank += (kj > key) || (kj == key && j < lane);
    }
    if (rank < 8) {
      const bool keep = rank < K && key != 0u;
      s_ck[warp * 8 + rank] = keep ? key : 0u;
      s_ce[warp * 8 + rank] = keep ? e : 0x7fffffff;
    }
  }
  trace_stamp(p_trace, 46);
  __syncthreads();
  {
    const int nc = W * 8, tpc = (nc <= 64) ? 8 : 4;  // threads per candidate
    const int c = threadIdx.x / tpc, part = threadIdx.x % tpc;
    int rank = 0;
    unsigned kc = 0u;
    int ec = 0x7fffffff;
    if (c < nc) {
      kc = s_ck[c];
      ec = s_ce[c];
      for (int d = part; d < nc; d += tpc) {
        const unsigned kd = s_ck[d];
        const int ed = s_ce[d];
        rank += (kd > kc) || (kd == kc && ed < ec);
      }
    }
    for (int o = 1; o < tpc; o <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    __syncthreads();
    if (c < nc && part == 0 && kc != 0u && rank < K) {
      s_ck[128 + rank] = kc;
      s_ce[128 + rank] = ec;
    }
    __syncthreads();
  }
  trace_stamp(p_trace, 47);
  if (warp == 0) {
    const float top = fkey_value(s_ck[128]);
    const float v = (lane < K) ? fkey_value(s_ck[128 + lane]) : 0.f;
    const float ex = (lane < K) ? expf(v - top) : 0.f;
    const float z = warp_sum(ex);
    if (lane < K) {
      ids[lane] = s_ce[128 + lane];
      wts[lane] = ex / z;
    }
  }
}

// Top-k (K <= 8) of one token's E <= 512 logits with half a warp (lanes
// 16h..16h+15, so a warp takes two tokens): lane l holds experts l + 16j;
// K rounds of (lane's best untaken, the half's largest key, the lowest expert
// holding it; shuffle butterflies within the half), ties to the lower expert;
// softmax over the K kept as in topk_warp. Same result as topk_warp.
template <int NJ2>
__device__ __forceinline__ void topk_half(const float* l, int E, int K, int* ids, float* w) {
  const int lane = threadIdx.x & 31, hl = lane & 15;
  const unsigned hm = 0xFFFFu << (lane & 16);
  unsigned key[NJ2];
#pragma unroll
  for (int j = 0; j < NJ2; ++j) {
    const int e = hl + 16 * j;
    key[j] = (e < E) ? fkey(l[e]) : 0u;  // 0: absent or taken (below every float's key)
  }
  unsigned sel = 0u;
  int sel_e = 0;
  for (int r = 0; r < K; ++r) {
    unsigned bk = 0u;
    int bj = 0;
#pragma unroll
    for (int j = 0; j < NJ2; ++j)
      if (key[j] > bk) {
        bk = key[j];
        bj = j;
      }
    // the half's largest key, then the lowest expert holding it (butterflies
    // within the half)
    unsigned kmax = bk;
#pragma unroll
    for (int o = 8; o; o >>= 1) kmax = max(kmax, __shfl_xor_sync(hm, kmax, o));
    int win = (bk == kmax && bk != 0u) ? hl + 16 * bj : 0x7fffffff;
#pragma unroll
    for (int o = 8; o; o >>= 1) win = min(win, __shfl_xor_sync(hm, win, o));
#pragma unroll
    for (int j = 0; j < NJ2; ++j)
      if (hl + 16 * j == win) key[j] = 0u;
    if (hl == r) {
      sel = kmax;
      sel_e = win;
    }
  }
  const float top = fkey_value(__shfl_sync(hm, sel, lane & 16));
  float ex = (hl < K) ? expf(fkey_value(sel) - top) : 0.f;
  float z = ex;
#pragma unroll
  for (int o = 8; o; o >>= 1) z += __shfl_xor_sync(hm, z, o);
  if (hl < K) {
    ids[hl] = sel_e;
    w[hl] = ex / z;
  }
}

// Logits of this CTA's ne <= 2 router rows (wr_s, fp32, row-major) for one
// token: every thread takes a strided share of both rows; warp sums, then
// warp 0 sums the warps' partials in warp order and stores the tagged words
// out[0], out[1]. ld_x8(i) returns bf16 elements 8i..8i+7 of the token.
// s_red: 2 * (blockDim.x / 32) floats. All threads must call it.
template <class LdX8>
__device__ __forceinline__ void router_logits_m1(LdX8 ld_x8, const float* wr_s, int H, int ne, unsigned epoch,
                                                 unsigned long long* out, float* s_red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  float acc0 = 0.f, acc1 = 0.f;
  for (int i = tid; i < H / 8; i += blockDim.x) {
    const uint4 x8 = ld_x8(i);
    const uint32_t xw[4] = {x8.x, x8.y, x8.z, x8.w};
    const float4* w0 = reinterpret_cast<const float4*>(wr_s) + 2 * i;
    const float4 a0 = w0[0], a1 = w0[1];
    const float4 b0 = (ne > 1) ? w0[H / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 b1 = (ne > 1) ? w0[H / 4 + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float2 x0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[0]));
    const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[1]));
    const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[2]));
    const float2 x3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[3]));
    acc0 = fmaf(x0.x, a0.x, acc0); acc0 = fmaf(x0.y, a0.y, acc0); acc0 = fmaf(x1.x, a0.z, acc0);
    acc0 = fmaf(x1.y, a0.w, acc0); acc0 = fmaf(x2.x, a1.x, acc0); acc0 = fmaf(x2.y, a1.y, acc0);
    acc0 = fmaf(x3.x, a1.z, acc0); acc0 = fmaf(x3.y, a1.w, acc0);
    acc1 = fmaf(x0.x, b0.x, acc1); acc1 = fmaf(x0.y, b0.y, acc1); acc1 = fmaf(x1.x, b0.z, acc1);
    acc1 = fmaf(x1.y, b0.w, acc1); acc1 = fmaf(x2.x, b1.x, acc1); acc1 = fmaf(x2.y, b1.y, acc1);
    acc1 = fmaf(x3.x, b1.z, acc1); acc1 = fmaf(x3.y, b1.w, acc1);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
    acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
  }
  if (lane == 0) {
    s_red[warp] = acc0;
    s_red[nw + warp] = acc1;
  }
  __syncthreads();
  if (warp == 0) {
    float v0 = (lane < nw) ? s_red[lane] : 0.f;
    float v1 = (lane < nw) ? s_red[nw + lane] : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      v0 += __shfl_xor_sync(0xffffffffu, v0, o);
      v1 += __shfl_xor_sync(0xffffffffu, v1, o);
    }
    if (lane == 0) st_relaxed_u64(out, tag_word(epoch, v0));
    if (lane == 1 && ne > 1) st_relaxed_u64(out + 1, tag_word(epoch, v1));
  }
}

// Read n tagged logit words into s_logit until every one carries `want`
// (eight independent loads in flight per thread, re-polling the stale ones).
// Returns false, with the status bit set, when the wait runs out.
__device__ __forceinline__ bool poll_tagged_logits(const Params& p, const unsigned long long* words, int n,
                                                   unsigned want, float* s_logit) {
  constexpr int kB = 8;
  const long long t0 = clock64();
  // word order rotated by CTA, so the CTAs do not all ask for the same
  // L2 line at once
  const int rot = (int)((blockIdx.x * 16u) % (unsigned)n);
  bool ok = true;
  for (int i0 = threadIdx.x; i0 < n; i0 += kB * blockDim.x) {
    unsigned long long w[kB];
    int idx[kB];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int i = i0 + j * blockDim.x;
      idx[j] = (i + rot >= n) ? i + rot - n : i + rot;
      w[j] = (i < n) ? ld_relaxed_u64(words + idx[j]) : ((unsigned long long)want << 32);
    }
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int i = i0 + j * blockDim.x;
      while ((unsigned)(w[j] >> 32) != want && ok) {
        __nanosleep(32);
        if (clock64() - t0 > p.spin_limit) {
          atomicOr(p.ws.ctrl, kStatusTimeout);
          ok = false;
        }
        w[j] = ld_relaxed_u64(words + idx[j]);
      }
      if (i < n) s_logit[idx[j]] = __uint_as_float((unsigned)w[j]);
    }
  }
  return ok;
}

// One token: the union is its K distinct experts in ascending order, one
// pair each (threads 0..K-1; pair positions from pbase, entries from ub).
__device__ __forceinline__ void union_m1(const int* s_ids, int K, int ub, int pbase, int* s_union, int* s_poff,
                                         int* s_pm, int* s_ppos, int* s_U) {
  const int tid = threadIdx.x;
  if (tid < K) {
    const int id = s_ids[tid];
    int rank = 0;
    for (int j = 0; j < K; ++j) rank += s_ids[j] < id;
    s_union[ub + rank] = id;
    s_poff[ub + rank] = pbase + rank;
    s_pm[pbase + rank] = 0;
    s_ppos[tid] = pbase + rank;
    if (rank == K - 1) {
      s_poff[ub + K] = pbase + K;
      *s_U = ub + K;
    }
  }
}

// One warp, M*K <= 32 pairs: the expert union (ascending ids) and the pairs
// grouped by expert in (token, slot) order, from ranks computed with
// shuffles (no shared-memory scratch). Pair i = (i / K, i % K); pair
// positions start at pbase.
__device__ __forceinline__ int union_small(const int* s_ids, int np, int K, int* s_union, int* s_poff, int* s_pm,
                                           int* s_ppos, int pbase) {
  const int lane = threadIdx.x & 31;
  const int id = (lane < np) ? s_ids[lane] : 0x7fffffff;
  int rank = 0, urank = 0;
  const unsigned same = __match_any_sync(0xffffffffu, id);
  const bool leader = (lane < np) && (__ffs(same) - 1 == lane);
  for (int j = 0; j < np; ++j) {
    const int oj = __shfl_sync(0xffffffffu, id, j);
    const bool lj = __shfl_sync(0xffffffffu, leader, j);
    rank += (oj < id) || (oj == id && j < lane);
    urank += lj && (oj < id);
  }
  const int U = __popc(__ballot_sync(0xffffffffu, leader));
  if (lane < np) {
    s_pm[pbase + rank] = lane / K;
    s_ppos[lane] = pbase + rank;
    if (leader) {
      s_union[urank] = id;
      s_poff[urank] = pbase + rank;
    }
  }
  if (lane == 0) s_poff[U] = pbase + np;
  return U;
}

// ---------------------------------------------------------------- the kernel
// kShared: the weight arrays hold E + 1 experts and expert E is a shared
// expert that every token passes with weight 1 ("NVIDIA Shows 3 Ways to Speed
// Up MoE Inference on DGX Spark", section on Ling 3.0: one shared expert
// beside the 8 routed ones).
// It is union entry 0, with pairs 0 .. M-1 (token order); the routed entries
// follow. It needs no routing, so its chunks are requested before routing
// starts (by two warps that have no activation rows to scan at M=1), and the
// routing scratch sits one slot into each ring, clear of slot 0. Its gate/up
// items are the head of the work queue. (Running them while the router
// logits arrive measured slower: the wait for the router is shorter than an
// item, so they lengthened routing.)
// kFp8H: the FP8 intermediate (see h_fp8x2) for every expert.
// kSplitK: the down projection is split over K instead of output rows (see
// the split-K block below); needs max_tokens <= kSkMaxTokens and the
// K-major W2 copy (w2kc, w2ks).
template <bool kShared, bool kFp8H, bool kSplitK>
__global__ void __launch_bounds__(kFusedThreads, 1) k_fused(Params p, FusedWs fw, FusedPlan pl) {
  static_assert(!(kSplitK && kFp8H), "the FP8 intermediate needs the whole h of a pair");
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x, G = gridDim.x;
  const int H = p.H, I = p.I, E = p.E, K = p.K, M = p.M;

  uint64_t* full_gu = reinterpret_cast<uint64_t*>(smem + pl.o_bar);
  uint64_t* empty_gu = full_gu + kMaxSlots;
  uint64_t* full_d = empty_gu + kMaxSlots;
  uint64_t* empty_d = full_d + kMaxSlots;
  uint64_t* h_bar = empty_d + kMaxSlots;
  uint64_t* wr_bar = h_bar + kMaxSlots;
  // items finished per ring slot (all uses): an item of use k waits until use
  // k-1 of its slot is fully consumed before any parity wait, so a parity
  // wait can never see a barrier two phases behind and pass early
  unsigned* done_gu = reinterpret_cast<unsigned*>(wr_bar + 1);
  unsigned* done_d = done_gu + kMaxSlots;
  float* s_amax = reinterpret_cast<float*>(smem + pl.o_misc);  // [32]
  float* s_xs = s_amax + kMaxTokens;                           // [32] per-token scales
  float* s_red = s_xs + kMaxTokens;                            // [kFusedWarps][kMaxRowsPerCta * 4]
  int* s_int = reinterpret_cast<int*>(s_red + kFusedWarps * kMaxRowsPerCta * 4);  // [0] U, [1] epoch, [2..3] queue heads
  int* s_ids = reinterpret_cast<int*>(smem + pl.o_ids);
  float* s_w = reinterpret_cast<float*>(smem + pl.o_w);
  int* s_pm = reinterpret_cast<int*>(smem + pl.o_pm);
  int* s_ppos = reinterpret_cast<int*>(smem + pl.o_ppos);
  int* s_union = reinterpret_cast<int*>(smem + pl.o_union);
  int* s_poff = reinterpret_cast<int*>(smem + pl.o_poff);
  int* s_cnt = reinterpret_cast<int*>(smem + pl.o_cnt);  // [E] union scratch, then per-entry item counters
  uint8_t* act = smem + pl.o_act;
  float* dsm = reinterpret_cast<float*>(smem + pl.o_dsm);
  uint8_t* hstage = smem + pl.o_h;
  uint8_t* ring_gu = smem + pl.o_ring_gu;
  // split-K down: CTA-local h, partial y, chunk progress, per-entry h ready
  float* hsm = reinterpret_cast<float*>(smem + pl.o_hsm);     // [max_union][max_tokens][nr_max]
  float* ycta = reinterpret_cast<float*>(smem + pl.o_ycta);   // [max_tokens][H]
  unsigned* s_chunk = reinterpret_cast<unsigned*>(smem + pl.o_chunk);  // [dchunks] entries done
  unsigned* s_hrdy = s_chunk + pl.dchunks;                              // [max_union] h of the entry complete
  float* s_pw = reinterpret_cast<float*>(smem + pl.o_pw);    // [pairs] routing weight per pair position
  uint8_t* ring_d = smem + pl.o_ring_d;
  float* wr_s = reinterpret_cast<float*>(ring_gu + (kShared ? pl.slot_gu : 0));  // router rows (routing phase only)
  float* s_logit = wr_s;                                                          // gathered logits (after them)
  uint4* x_s = reinterpret_cast<uint4*>(ring_d + (kShared ? pl.slot_d : 0));      // staged bf16 x (routing only)
  const int ub = kShared ? 1 : 0;  // first routed union entry

  const int e0 = (int)((long long)E * b / G), e1 = (int)((long long)E * (b + 1) / G), ne = e1 - e0;
  // this CTA's share of every union expert (independent of the routing)
  const int n0 = (int)((long long)I * b / G), nr = (int)((long long)I * (b + 1) / G) - n0;
  const int r0 = (int)((long long)H * b / G), nrd = (int)((long long)H * (b + 1) / G) - r0;
  const int gu_items = (nr > 0) ? (nr + kGuRowsPerItem - 1) / kGuRowsPerItem : 0;  // per expert
  // down items per entry: output-row items, or (split-K) output chunks of the
  // CTA's K slice
  const int d_items = kSplitK ? ((nr > 0) ? pl.dchunks : 0)
                              : ((nrd > 0) ? (nrd + kDownRowsPerItem - 1) / kDownRowsPerItem : 0);
  // split-K: scale-block rows of W2 the CTA's K slice touches
  const int skb0 = n0 / 32, nskb = (nr > 0) ? (n0 + nr - 1) / 32 - skb0 + 1 : 0;

  // ---------------- weight stream. Each bulk copy costs its issuing thread
  //   about a hundred nanoseconds, so the first use of every ring slot is
  //   issued by all warps in parallel (lane 0 of warp w takes entries w, w+16,
  //   ...; gate/up chunks first, then down chunks); later uses wait for their
  //   slot to drain and are issued by lane 0 of warp 0.
  auto issue_gu = [&](int u) {
    const int e = s_union[u];
    const int slot = u % pl.ns_gu;
    uint8_t* sp = ring_gu + (size_t)slot * pl.slot_gu;
    GuChunk ch;
    size_t ga0, ua0;
    unsigned gn, un;
    const unsigned bytes = gu_layout(p, e, n0, nr, sp, &ch, &ga0, &gn, &ua0, &un);
    mbar_expect_tx(full_gu + slot, bytes);
    const size_t grow = (size_t)e * 2 * I + n0, urow = grow + I;
    const unsigned codes = (unsigned)(nr * H / 2);
    tma_load_1d(sp, p.w13c + grow * (H / 2), codes, full_gu + slot);
    tma_load_1d(sp + codes, p.w13c + urow * (H / 2), codes, full_gu + slot);
    tma_load_1d(sp + 2 * codes, p.w13s + ga0, gn, full_gu + slot);
    tma_load_1d(sp + 2 * codes + gn, p.w13s + ua0, un, full_gu + slot);
  };
  auto issue_d = [&](int u) {
    const int e = s_union[u];
    const int slot = u % pl.ns_d;
    uint8_t* sp = ring_d + (size_t)slot * pl.slot_d;
    if constexpr (kSplitK) {
      // codes of W2 columns [n0, n0+nr) for every output row (K-major rows
      // n, each H/2 bytes), then the scale rows of their 32-blocks
      const unsigned codes = (unsigned)(nr * H / 2), sb = (unsigned)(nskb * H);
      mbar_expect_tx(full_d + slot, codes + sb);
      tma_load_1d(sp, p.w2kc + ((size_t)e * I + n0) * (H / 2), codes, full_d + slot);
      tma_load_1d(sp + codes, p.w2ks + ((size_t)e * (I / 32) + skb0) * H, sb, full_d + slot);
      return;
    }
    DChunk ch;
    size_t sa0;
    unsigned sn;
    const unsigned bytes = d_layout(p, e, r0, nrd, sp, &ch, &sa0, &sn);
    mbar_expect_tx(full_d + slot, bytes);
    const unsigned codes = (unsigned)(nrd * I / 2);
    tma_load_1d(sp, p.w2c + ((size_t)e * H + r0) * (I / 2), codes, full_d + slot);
    tma_load_1d(sp + codes, p.w2s + sa0, sn, full_d + slot);
  };
  // one gate/up item: rows of item g of this CTA's chunk of entry u, every
  // pair of the entry; the last item of the entry publishes it GPU-wide
  auto gu_work = [&](int u, int g) {
    const int slot = u % pl.ns_gu, use = u / pl.ns_gu;
    if (use > 0 && lane == 0) smem_count_wait(done_gu + slot, (unsigned)(use * gu_items), p);
    __syncwarp();
    mbar_wait(full_gu + slot, use & 1, p);
    if (u == 0 && g == 0) trace_stamp(p, 5);
    if (u == s_int[0] - 1 && g == gu_items - 1) trace_stamp(p, 16);
    GuChunk ch;
    size_t ga0, ua0;
    unsigned gn, un;
    gu_layout(p, s_union[u], n0, nr, ring_gu + (size_t)slot * pl.slot_gu, &ch, &ga0, &gn, &ua0, &un);
    const int pb = s_poff[u], pe = s_poff[u + 1];
    // h of pair pb + q, local row j: hout[q * hstride + j] (global h, or the
    // CTA-local copy for the split-K down)
    float* hout = kSplitK ? hsm + (size_t)u * pl.max_tokens * pl.nr_max : p.ws.h + (size_t)pb * I + n0;
    const size_t hstride = kSplitK ? (size_t)pl.nr_max : (size_t)I;
    if (pe - pb >= kMmaMinPairs && pl.part_slot > 0) {
      // several pairs: the entry's items split K; each runs warp MMAs over
      // all rows and pairs, and the last one to finish sums the partials
      // in chunk order (deterministic), applies SwiGLU and writes h
      const int nkb = H / 32, nrg = (nr + 7) >> 3, nct = min(pl.part_ct, (pe - pb + 7) >> 3);
      const int kb0 = g * nkb / gu_items, kb1 = (g + 1) * nkb / gu_items;
      float4* part = reinterpret_cast<float4*>(smem + pl.o_part + (size_t)slot * pl.part_slot);
      for (int rg = 0; rg < nrg; ++rg) {
        float acc[4 * kMaxPairTiles];
        gu_mma_slice(p, ch, 8 * rg, min(8, nr - 8 * rg), kb0, kb1, pb, pe, s_pm, act, acc);
#pragma unroll
        for (int ct = 0; ct < kMaxPairTiles; ++ct)
          if (ct < nct)
            part[((g * nrg + rg) * pl.part_ct + ct) * 32 + lane] =
                make_float4(acc[4 * ct], acc[4 * ct + 1], acc[4 * ct + 2], acc[4 * ct + 3]);
      }
      __syncwarp();
      unsigned done = 0;
      if (lane == 0) done = atom_add_acqrel_cta_smem(reinterpret_cast<unsigned*>(s_cnt + u), 1u) + 1u;
      done = __shfl_sync(0xffffffffu, done, 0);
      if ((int)done == gu_items) {
        const int gq = lane >> 2, tq = lane & 3;
        for (int rg = 0; rg < nrg; ++rg) {
          const int row = 8 * rg + gq;
          for (int ct = 0; ct < nct; ++ct) {
            float4 v = part[(rg * pl.part_ct + ct) * 32 + lane];
            for (int c = 1; c < gu_items; ++c) {
              const float4 w = part[((c * nrg + rg) * pl.part_ct + ct) * 32 + lane];
              v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
            }
            const float gg[2] = {v.x, v.y}, uu[2] = {v.z, v.w};
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int q = 8 * ct + 2 * tq + i;
              if (q < pe - pb && row < nr) {
                const float sx = s_xs[s_pm[pb + q]];
                const float gv = gg[i] * sx, uv = uu[i] * sx;
                hout[(size_t)q * hstride + row] = gv / (1.f + expf(-gv)) * uv;
              }
            }
          }
        }
        __syncwarp();
        // orders the warp's h stores (through the warp barrier) before the
        // GPU-wide arrival for the entry (split-K: the CTA-local ready flag)
        if (lane == 0) {
          if constexpr (kSplitK) st_release_cta_smem(s_hrdy + u, 1u);
          else grid_arrive(gu_counter(fw, u));
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(empty_gu + slot);
        atomicAdd(done_gu + slot, 1u);
      }
      __syncwarp();
      return;
    }
    const int a = g * kGuRowsPerItem, cnt = min(kGuRowsPerItem, nr - a);
    gu_item(p, ch, a, cnt, hout, hstride, pb, pe, s_pm, act, s_xs);
    if (u == 0 && g == 0) trace_stamp(p, 17);
    if (u == s_int[0] - 1 && g == gu_items - 1) trace_stamp(p, 6);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(empty_gu + slot);
      atomicAdd(done_gu + slot, 1u);
      // acq_rel at CTA scope: the warp completing the entry sees every
      // other warp's h stores, then releases them GPU-wide
      const unsigned done = atom_add_acqrel_cta_smem(reinterpret_cast<unsigned*>(s_cnt + u), 1u) + 1u;
      if ((int)done == gu_items) {
        if constexpr (kSplitK) st_release_cta_smem(s_hrdy + u, 1u);
        else grid_arrive(gu_counter(fw, u));
      }
    }
    __syncwarp();
  };
  if (tid < kMaxSlots) {
    if (tid < pl.ns_gu) { mbar_init(full_gu + tid, 1); mbar_init(empty_gu + tid, max(1, gu_items)); }
    if (tid < pl.ns_d) {
      mbar_init(full_d + tid, 1);
      mbar_init(empty_d + tid, max(1, d_items));
      mbar_init(h_bar + tid, 1);
    }
    done_gu[tid] = done_d[tid] = 0u;
    fence_mbar_init();
  }
  if constexpr (kSplitK) {
    for (int i = tid; i < M * H; i += kFusedThreads) ycta[i] = 0.f;
    for (int i = tid; i < pl.dchunks + pl.max_union; i += kFusedThreads) s_chunk[i] = 0u;  // and s_hrdy
  }
  if (tid == 0) {
    mbar_init(wr_bar, 1);
    fence_mbar_init();
    if (ne > 0) {
      mbar_expect_tx(wr_bar, (unsigned)(ne * H * 4));
      tma_load_1d(wr_s, p.wr + (size_t)e0 * H, (unsigned)(ne * H * 4), wr_bar);
    }
  }
  trace_stamp(p, 0);
  // Everything above is independent of the previous kernel on the stream.
  pdl_wait();
  trace_stamp(p, 1);
  if (tid == 0) {
    s_int[1] = (int)(ld_relaxed_u32(fw.epoch) + 1u);
    s_int[2] = 0;  // gate/up queue head
    s_int[3] = 0;  // down queue head
  }
  if (tid == 0) {
    if constexpr (kShared) {
      s_union[0] = E;
      s_poff[0] = 0;
      s_poff[1] = M;
      s_cnt[0] = 0;
    }
  }
  if constexpr (kShared) {
    if (tid < M) s_pm[tid] = tid;
    if constexpr (kSplitK) {
      if (tid < M) s_pw[tid] = 1.f;  // the shared expert's weight
    }
  }
  unsigned* s_amax_u = reinterpret_cast<unsigned*>(s_amax);
  if (tid < M) s_amax_u[tid] = 0u;
  __syncthreads();
  const unsigned epoch = (unsigned)s_int[1];
  if constexpr (kShared) {
    // the shared entry's chunks, into slot 0 of each ring (its barriers were
    // initialised before the block barrier above)
    if (lane == 0 && warp == kFusedWarps - 1 && nr > 0) issue_gu(0);
    if (lane == 0 && warp == kFusedWarps - 2 && (kSplitK ? nr > 0 : nrd > 0)) issue_d(0);
  }

  // ---- A1: per-token amax (unsigned max of |x| bit patterns) and, when it
  //          fits, a shared-memory copy of x for the router
  {
    const uint4* x16 = reinterpret_cast<const uint4*>(p.x);
    int mcur = -1;
    float a = 0.f;
    // start rotated by CTA: the CTAs spread their first reads over x's lines
    const int nx8 = M * H / 8, rot8 = (int)((b * 8u) % (unsigned)nx8);
    for (int i0 = tid; i0 < nx8; i0 += kFusedThreads) {
      const int i = (i0 + rot8 >= nx8) ? i0 + rot8 - nx8 : i0 + rot8;
      const int m = (i * 8) / H;
      if (m != mcur) {
        if (mcur >= 0) atomicMax(&s_amax_u[mcur], __float_as_uint(a));
        mcur = m;
        a = 0.f;
      }
      const uint4 v = __ldcg(x16 + i);
      if (pl.x_staged) x_s[i] = v;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    if (mcur >= 0) atomicMax(&s_amax_u[mcur], __float_as_uint(a));
  }
  __syncthreads();
  trace_stamp(p, 13);
  const uint4* xsrc = pl.x_staged ? x_s : reinterpret_cast<const uint4*>(p.x);
  // ---- A9 (stacked layers): x <- bf16(x / sqrt(mean(x^2) + 1e-6)) per token.
  //      One warp per token sums x^2 in a fixed order with IEEE fp32 ops, so
  //      every CTA derives the same factor. Rounding is monotonic and
  //      symmetric, so the new amax is bf16(fl32(amax * r)).
  float* s_rn = reinterpret_cast<float*>(s_int + 8);  // [32] per-token RMSNorm factors
  if (p.pre_rmsnorm) {
    for (int m = warp; m < M; m += kFusedWarps) {
      float ss = 0.f;
      for (int i = lane; i < H / 8; i += 32) {
        const uint4 v = pl.x_staged ? xsrc[(size_t)m * (H / 8) + i] : __ldcg(xsrc + (size_t)m * (H / 8) + i);
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
    // normalise the staged copy in place (bf16); unstaged reads apply it on use
    for (int i = tid; i < M * H / 8; i += kFusedThreads) {
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
  // normalised value of one bf16 pair read from global x (unstaged case)
  auto xn2 = [&](uint32_t raw, int m) -> uint32_t {
    if (!p.pre_rmsnorm || pl.x_staged) return raw;
    const float r = s_rn[m];
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
    const __nv_bfloat162 o = __floats2bfloat162_rn(__fmul_rn(f.x, r), __fmul_rn(f.y, r));
    return *reinterpret_cast<const uint32_t*>(&o);
  };
  // ---- A2: logits of this CTA's router rows (ne <= kMaxRowsPerCta), four
  //          tokens per pass; warp partials go to shared memory and one block
  //          barrier per pass ends it
  if (ne > 0) mbar_wait(wr_bar, 0, p);
  trace_stamp(p, 14);
  const bool lg_m1 = (M == 1 && ne > 0 && ne <= 2);
  if (lg_m1) {
    auto ld_x8 = [&](int i) -> uint4 {
      uint4 v = pl.x_staged ? xsrc[i] : __ldcg(xsrc + i);
      v.x = xn2(v.x, 0); v.y = xn2(v.y, 0); v.z = xn2(v.z, 0); v.w = xn2(v.w, 0);
      return v;
    };
    router_logits_m1(ld_x8, wr_s, H, ne, epoch, fw.logits + e0, s_red);
  }
  for (int m0 = 0; m0 < M && ne > 0 && !lg_m1; m0 += 4) {
    const int mt = min(4, M - m0);
    for (int el = 0; el < ne; ++el) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float4* wrow = reinterpret_cast<const float4*>(wr_s + (size_t)el * H);
      for (int i = tid; i < H / 4; i += kFusedThreads) {
        const float4 wv = wrow[i];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (t < mt) {
            const uint2* xrow = reinterpret_cast<const uint2*>(xsrc) + (size_t)(m0 + t) * (H / 4);
            uint2 q = pl.x_staged ? xrow[i] : __ldcg(xrow + i);
            q.x = xn2(q.x, m0 + t);
            q.y = xn2(q.y, m0 + t);
            const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
            const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
            acc[t] = fmaf(x01.x, wv.x, acc[t]);
            acc[t] = fmaf(x01.y, wv.y, acc[t]);
            acc[t] = fmaf(x23.x, wv.z, acc[t]);
            acc[t] = fmaf(x23.y, wv.w, acc[t]);
          }
        }
      }
      if (mt == 1) {
        acc[0] = warp_sum(acc[0]);
      } else {
#pragma unroll
        for (int o = 16; o; o >>= 1) {
#pragma unroll
          for (int t = 0; t < 4; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        }
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
        for (int w = 0; w < kFusedWarps; ++w) sum += s_red[w * (kMaxRowsPerCta * 4) + el * 4 + t];
        st_relaxed_u64(fw.logits + (size_t)(m0 + t) * E + e0 + el, tag_word(epoch, sum));
      }
    }
    __syncthreads();
  }
  trace_stamp(p, 15);
  // ---- A1 (second half): E4M3 codes and scales, done while the other CTAs'
  //      logits arrive (the router works on the bf16 x, not on the codes)
  if (tid < M) {
    const float a = s_amax[tid];
    s_xs[tid] = (a == 0.f) ? 1.f : __fdiv_rn(a, 448.f);
  }
  for (int i = tid; i < M * H / 8; i += kFusedThreads) {
    const int m = (i * 8) / H;
    const float a = s_amax[m];
    uint2 out = make_uint2(0u, 0u);
    if (a != 0.f) {
      const float inv = __fdiv_rn(448.f, a);
      const uint4 v = pl.x_staged ? xsrc[i] : __ldcg(xsrc + i);
      const uint32_t w[4] = {xn2(v.x, m), xn2(v.y, m), xn2(v.z, m), xn2(v.w, m)};
      uint32_t q[2] = {0u, 0u};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        const uint32_t c2 = f32x2_to_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
        q[t >> 1] |= c2 << (16 * (t & 1));
      }
      out = make_uint2(q[0], q[1]);
    }
    *reinterpret_cast<uint2*>(act + (size_t)i * 8) = out;
    if (b == 0 && p.out_xq) *reinterpret_cast<uint2*>(p.out_xq + (size_t)i * 8) = out;
  }
  if (b == 0 && p.out_xscale && tid < M) p.out_xscale[tid] = s_xs[tid];
  trace_stamp(p, 2);

  // ---- A2 exchange: every logit word of this launch (the tag is the flag)
  poll_tagged_logits(p, fw.logits, M * E, p.force_stall ? epoch + 0x40000000u : epoch, s_logit);
  trace_stamp(p, 3);
  pdl_launch_dependents();
  __syncthreads();
  trace_stamp(p, 20);

  // ---- A3: top-k (ties to the lower index) and its softmax: every warp on
  //          the one token when M == 1, else one warp per token
  const bool tk_m1 = (M == 1 && E <= 32 * kFusedWarps && K <= 8);
  if (tk_m1) {
    topk_cta_small(s_logit, E, K, s_ids, s_w, reinterpret_cast<unsigned*>(s_red),
                   reinterpret_cast<int*>(s_red) + 136, p);
    if (b == 0 && tid < K) {
      if (p.out_ids) p.out_ids[tid] = s_ids[tid];
      if (p.out_w) p.out_w[tid] = s_w[tid];
    }
  }
  for (int m = warp; m < M && !tk_m1; m += kFusedWarps) {
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
  trace_stamp(p, 8);

  // ---- A4: expert union (ascending ids) and the (token, slot) pairs of each
  //          entry in (token, slot) order; one warp, no block barriers
  // (with a shared expert, routed entries start at 1 and their pairs at M)
  const int np = M * K, pbase = kShared ? M : 0;
  if (M == 1) {
    union_m1(s_ids, K, ub, pbase, s_union, s_poff, s_pm, s_ppos, &s_int[0]);
    if (tid < K) s_cnt[ub + tid] = 0;  // per-entry gate/up item counters
  } else if (warp == 0 && np <= 32) {
    const int Us = union_small(s_ids, np, K, s_union + ub, s_poff + ub, s_pm, s_ppos, pbase);
    if (lane == 0) s_int[0] = ub + Us;
    for (int u = lane; u < Us; u += 32) s_cnt[ub + u] = 0;  // per-entry gate/up item counters
  } else if (warp == 0) {
    int* s_ec = s_cnt + ub;  // [E] per-expert scratch, clear of the shared entry's counter
    for (int e = lane; e < E; e += 32) s_ec[e] = 0;
    __syncwarp();
    for (int i = lane; i < np; i += 32) atomicAdd(&s_ec[s_ids[i]], 1);
    __syncwarp();
    const int per = (E + 31) / 32;
    const int ea = min(E, lane * per), eb = min(E, ea + per);
    int nz = 0, cs = 0;
    for (int e = ea; e < eb; ++e) { nz += s_ec[e] > 0; cs += s_ec[e]; }
    int nz_ex = nz, cs_ex = cs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x1 = __shfl_up_sync(0xffffffffu, nz_ex, o);
      const int x2 = __shfl_up_sync(0xffffffffu, cs_ex, o);
      if (lane >= o) { nz_ex += x1; cs_ex += x2; }
    }
    nz_ex -= nz;
    cs_ex -= cs;
    __syncwarp();
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
    if (lane == 31) {
      s_poff[ub + nz_ex] = pbase + cs_ex;
      s_int[0] = ub + nz_ex;
    }
    __syncwarp();
    // stable placement: rank within each 32-pair batch by matching experts
    for (int base = 0; base < np; base += 32) {
      const int i = base + lane;
      const int e = (i < np) ? s_ids[i] : -1 - lane;
      const unsigned same = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(same & ((1u << lane) - 1u));
      int pos = 0;
      if (i < np) {
        pos = s_ec[e] + rank;
        s_pm[pos] = i / K;
        s_ppos[i] = pos;
      }
      __syncwarp();
      if (i < np && rank == 0) s_ec[e] += __popc(same);
      __syncwarp();
    }
    const int U = s_int[0];
    __syncwarp();
    for (int u = ub + lane; u < U; u += 32) s_cnt[u] = 0;  // per-entry gate/up item counters
  }
  if constexpr (kSplitK) {
    // routing weight of every routed pair position
    if (warp == 0) {
      __syncwarp();
      for (int i = lane; i < np; i += 32) s_pw[s_ppos[i]] = s_w[i];
    }
  }
  __syncthreads();
  const int U = s_int[0];
  trace_stamp(p, 4);

  const int n_gu0 = (nr > 0) ? min(U, pl.ns_gu) : 0;
  const bool has_d = kSplitK ? (nr > 0) : (nrd > 0);  // this CTA streams down chunks
  const int n_d0 = has_d ? min(U, pl.ns_d) : 0;
  if (lane == 0 && (ub + warp < n_gu0 || ub + warp < n_d0)) {
    // ring_gu and ring_d were read and written through the generic proxy
    // during routing; order that before the async-proxy (TMA) writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    for (int u = ub + warp; u < n_gu0; u += kFusedWarps) issue_gu(u);
    for (int u = ub + warp; u < n_d0; u += kFusedWarps) issue_d(u);
  }
  if (warp == 0) trace_stamp(p, 59);
  if (warp == 0) trace_stamp(p, 59);
  if (warp == 0) {
    // refills of drained slots (more union entries than slots): one thread
    // polls both rings without suspending and issues whichever slot drains
    // first, in entry order per ring, so neither ring waits behind the other
    if (lane == 0) {
      int ug = (nr > 0) ? n_gu0 : U, ud = has_d ? n_d0 : U;
      if (ug < U || ud < U) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        long long t0 = clock64();
        while (ug < U || ud < U) {
          bool moved = false;
          if (ug < U && mbar_test(empty_gu + ug % pl.ns_gu, (ug / pl.ns_gu - 1) & 1)) {
            issue_gu(ug++);
            moved = true;
          }
          if (ud < U && mbar_test(empty_d + ud % pl.ns_d, (ud / pl.ns_d - 1) & 1)) {
            issue_d(ud++);
            moved = true;
          }
          if (moved) {
            t0 = clock64();
          } else {
            __nanosleep(64);
            if (clock64() - t0 > p.spin_limit) {
              atomicOr(p.ws.ctrl, kStatusTimeout);
              break;
            }
          }
        }
      }
    }
    return;
  }

  // ---------------- consumers. Two in-order queues: every consumer warp
  //   first takes gate/up items (entry-major) until that queue is empty, then
  //   down items (entry-major). Gate/up items depend only on their chunk, so
  //   the first queue always drains; down items depend on their chunk and on
  //   gate/up of the entry on every CTA, which never waits on down work, so
  //   the second cannot deadlock either.
  const unsigned long long tgt = (unsigned long long)epoch * G;
  if (!kSplitK && gu_items == 0 && warp == 1 && lane == 0) {
    // no gate/up rows here: this CTA's part of every entry is trivially done
    for (int u = 0; u < U; ++u) grid_arrive(gu_counter(fw, u));
  }
  // One in-order queue: round k holds the gate/up items of entry k, then the
  // down items of entry k - kDownLag, so down work on early entries overlaps
  // gate/up work on later ones. Gate/up items wait only for their chunk, and
  // a down item is handed out only after every gate/up item of its entry,
  // here and (by the same order) on every CTA, so the queue cannot deadlock.
  const int DL = min(kDownLag, U);
  const int n1 = DL * gu_items, per2 = gu_items + d_items, n2 = (U - DL) * per2;
  const int total = U * (gu_items + d_items);
  for (;;) {
    int it = 0;
    if (lane == 0) it = atomicAdd(&s_int[2], 1);
    it = __shfl_sync(0xffffffffu, it, 0);
    if (it >= total) break;
    bool is_down;
    int u, sub;
    if (it < n1) {
      is_down = false;
      u = it / gu_items;
      sub = it - u * gu_items;
    } else if (it < n1 + n2) {
      const int r = (it - n1) / per2, w = (it - n1) - r * per2;
      is_down = w >= gu_items;
      u = is_down ? r : DL + r;
      sub = is_down ? w - gu_items : w;
    } else {
      const int q = it - n1 - n2;
      is_down = true;
      u = U - DL + q / d_items;
      sub = q % d_items;
    }
    if (!is_down) {
      gu_work(u, sub);
    } else if constexpr (kSplitK) {
      // split-K down chunk `sub` of entry u over this CTA's K slice; chunk c
      // of entry u accumulates after chunk c of entry u - 1 (fixed order)
      const int c = sub;
      const int slot = u % pl.ns_d, use = u / pl.ns_d;
      const int pb = s_poff[u], pe = s_poff[u + 1];
      if (lane == 0) {
        if (use > 0) smem_count_wait(done_d + slot, (unsigned)(use * d_items), p);
        smem_acquire_wait(s_hrdy + u, 1u, p);
        smem_acquire_wait(s_chunk + c, (unsigned)u, p);
      }
      __syncwarp();
      mbar_wait(full_d + slot, use & 1, p);
      sk_down_chunk(p, ring_d + (size_t)slot * pl.slot_d, n0, nr, skb0, c, pb, pe,
                    hsm + (size_t)u * pl.max_tokens * pl.nr_max, pl.nr_max, s_pm, s_pw, ycta);
      __syncwarp();
      if (lane == 0) {
        st_release_cta_smem(s_chunk + c, (unsigned)(u + 1));
        mbar_arrive(empty_d + slot);
        atomicAdd(done_d + slot, 1u);
      }
    } else {
      const int gd = sub;
      const int slot = u % pl.ns_d, use = u / pl.ns_d;
      const int pb = s_poff[u], pe = s_poff[u + 1];
      __half2* hbuf = reinterpret_cast<__half2*>(hstage + (size_t)slot * pl.hslot);
      float* hscale = reinterpret_cast<float*>(hstage + (size_t)slot * pl.hslot + (size_t)pl.hpairs * I * 2);
      // every down item of the slot's previous use is finished (so its
      // staged h and data may be replaced, and parity waits are unambiguous)
      if (use > 0 && lane == 0) smem_count_wait(done_d + slot, (unsigned)(use * d_items), p);
      __syncwarp();
      if (gd == 0) {
        // first down item of the entry: wait for gate/up of the entry on all
        // CTAs, then stage h once for the CTA
        if (lane == 0) grid_wait(gu_counter(fw, u), tgt, p);
        __syncwarp();
        if (pe - pb <= pl.hpairs) stage_h<kFp8H>(p, pb, pe, hbuf, hscale);
        __syncwarp();
        if (lane == 0) mbar_arrive(h_bar + slot);
      } else {
        mbar_wait(h_bar + slot, use & 1, p);
      }
      mbar_wait(full_d + slot, use & 1, p);
      DChunk ch;
      size_t sa0;
      unsigned sn;
      d_layout(p, s_union[u], r0, nrd, ring_d + (size_t)slot * pl.slot_d, &ch, &sa0, &sn);
      const int a = gd * kDownRowsPerItem, cnt = min(kDownRowsPerItem, nrd - a);
      d_item<kFp8H>(p, ch, a, cnt, pb, pe, hbuf, hscale, pl.hpairs, dsm, pl.rpc_max);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(empty_d + slot);
        atomicAdd(done_d + slot, 1u);
      }
    }
  }
  trace_stamp(p, 10);
  consumers_sync();
  trace_stamp(p, 11);
  const int ct = tid - 32;
  if constexpr (kSplitK) {
    // ---- A8 (split-K): publish this CTA's partial y, one grid barrier, then
    //      rows [r0, r0+nrd) of every token summed over the G partials: thread
    //      (o, j) adds partials [j*G/T, (j+1)*G/T) of output o, and the T sums
    //      of an output are added in j order (deterministic)
    float4* dst = reinterpret_cast<float4*>(fw.ypart + (size_t)b * pl.max_tokens * H);
    const float4* src = reinterpret_cast<const float4*>(ycta);
    for (int i = ct; i < M * H / 4; i += kConsumers * 32) dst[i] = src[i];
    consumers_sync();
    if (ct == 0) {
      __threadfence();
      grid_arrive(fw.fin_cnt);
      grid_wait(fw.fin_cnt, (unsigned long long)epoch * G, p);
    }
    consumers_sync();
    const int nout = M * nrd;
    if (nout > 0) {
      const int tpo = max(1, (kConsumers * 32) / nout);
      float* red = ycta;  // [nout][tpo], free once published
      const int o = ct / tpo, j = ct % tpo;
      if (o < nout) {
        const int m = o / nrd, rl = o % nrd;
        const int c0 = j * G / tpo, c1 = (j + 1) * G / tpo;
        float acc = 0.f;
        for (int c = c0; c < c1; ++c) acc += __ldcg(fw.ypart + ((size_t)c * pl.max_tokens + m) * H + r0 + rl);
        red[o * tpo + j] = acc;
      }
      consumers_sync();
      if (ct < nout) {
        float acc = 0.f;
        for (int j2 = 0; j2 < tpo; ++j2) acc += red[ct * tpo + j2];
        store_y(p, (size_t)(ct / nrd) * H + r0 + ct % nrd, acc);
      }
    }
    if (b == 0 && ct == 0) st_relaxed_u32(fw.epoch, epoch);
  } else {
  // ---- A8: combine in slot order, bf16 out (fp32 for one part of a split)
  for (int i = ct; i < M * nrd; i += kConsumers * 32) {
    const int m = i / nrd, rl = i % nrd;
    float acc = 0.f;
    for (int s = 0; s < K; ++s) acc = fmaf(s_w[m * K + s], dsm[(size_t)s_ppos[m * K + s] * pl.rpc_max + rl], acc);
    if constexpr (kShared) acc += dsm[(size_t)m * pl.rpc_max + rl];  // shared expert, weight 1
    store_y(p, (size_t)m * H + r0 + rl, acc);
  }
  if (b == 0 && ct == 0) {
    // keep every entry's counter at epoch * G for the next launch
    for (int u = U; u < pl.max_union; ++u) red_release_add_u64(gu_counter(fw, u), (unsigned long long)G);
    st_relaxed_u32(fw.epoch, epoch);
  }
  }
  trace_stamp(p, 12);
}

}  // namespace moe
