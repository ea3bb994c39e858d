// moe_api.cu -- the C ABI of libmoe (declared in include/moe.h): argument
// validation, the per-context workspace, and kernel launches on the caller's
// stream. moe_decode allocates nothing; moe_load_experts allocates only the
// context's own weight copies (MOE_LOAD_COPY_REPACK, a part of an
// intra-expert split, the split-K down projection's K-major W2). Nothing
// falls back to the CPU.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/moe.h"
#include "moe_device.cuh"
#include "moe_host.h"
#include "moe_fused.cuh"
#include "moe_split.cuh"
#include "moe_tc.cuh"

using moe_host::aligned16;
using moe_host::align_up;
using moe_host::DeviceGuard;
using moe_host::kDefaultSpinLimit;

namespace {

enum Variant { kFused = 0, kSplit = 1, kTc = 2 };



moe_status validate_config(const moe_config& c) {
  if (c.hidden < 32 || c.hidden > 8192 || c.hidden % 32) return MOE_ERR_INVALID_ARG;
  if (c.inter < 32 || c.inter > 4096 || c.inter % 32) return MOE_ERR_INVALID_ARG;
  if (c.num_experts < 1 || c.num_experts > moe::kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > c.num_experts || c.top_k > moe::kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (c.max_tokens < 1 || c.max_tokens > moe::kMaxTokens) return MOE_ERR_INVALID_ARG;
  const uint32_t fused_only =
      MOE_FLAG_PRE_RMSNORM | MOE_FLAG_SHARED_EXPERT | MOE_FLAG_FP8_INTERMEDIATE | MOE_FLAG_SPLITK_DOWN;
  if (c.flags & ~(MOE_FLAG_SPLIT_KERNELS | MOE_FLAG_CUDA_CORES | MOE_FLAG_TENSOR_CORES | MOE_FLAG_TC_DOWN_MMA |
                  MOE_FLAG_TC_DOWN_CUDA | fused_only))
    return MOE_ERR_INVALID_ARG;
  if ((c.flags & MOE_FLAG_TC_DOWN_MMA) && (c.flags & MOE_FLAG_TC_DOWN_CUDA)) return MOE_ERR_INVALID_ARG;
  if ((c.flags & MOE_FLAG_CUDA_CORES) && (c.flags & MOE_FLAG_TENSOR_CORES)) return MOE_ERR_INVALID_ARG;
  if ((c.flags & MOE_FLAG_TENSOR_CORES) && (c.flags & (MOE_FLAG_SPLIT_KERNELS | MOE_FLAG_SPLITK_DOWN)))
    return MOE_ERR_INVALID_ARG;
  if ((c.flags & fused_only) && (c.flags & MOE_FLAG_SPLIT_KERNELS)) return MOE_ERR_UNSUPPORTED;
  if ((c.flags & MOE_FLAG_SPLITK_DOWN) &&
      ((c.flags & MOE_FLAG_FP8_INTERMEDIATE) || c.max_tokens > moe::kSkMaxTokens))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Intra-expert split (shard_count = G > 1): part g computes gate/up rows
// [g*I/G, (g+1)*I/G) and the same columns of the down projection, i.e. the
// step of a layer of width I/G whose A8 sum stays in fp32. Gives the part's
// config (inter = I/G, shard_count normalised to >= 1) after checking the
// split's own rules; the whole layer's config is checked by validate_config.
moe_status shard_config(const moe_config& c, moe_config* part) {
  const int G = c.shard_count == 0 ? 1 : c.shard_count;
  if (G < 1 || G > 128 || c.shard_index < 0 || c.shard_index >= G) return MOE_ERR_INVALID_ARG;
  if (c.inter % (32 * G)) return MOE_ERR_INVALID_ARG;  // whole E8M0 blocks of W2 per part
  if (G > 1 && (c.flags & MOE_FLAG_FP8_INTERMEDIATE)) return MOE_ERR_UNSUPPORTED;
  *part = c;
  part->inter = c.inter / G;
  part->shard_count = G;
  return MOE_OK;
}

// Union entries and (token, slot) pairs a call can have; a shared expert adds
// one entry holding one pair per token.
void union_bounds(const moe_config& c, size_t* np, size_t* umax) {
  const size_t E = c.num_experts, NP = (size_t)c.max_tokens * c.top_k;
  const size_t sh = (c.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0;
  *np = NP + sh * c.max_tokens;
  *umax = (E < NP ? E : NP) + sh;
}

// Shared-memory plan of the persistent kernel (mirrors k_fused's carving).
bool make_plan(const moe_config& c, int sm_count, size_t smem_limit, moe::FusedPlan* pl) {
  const size_t H = c.hidden, I = c.inter, E = c.num_experts, MM = c.max_tokens;
  const size_t G = sm_count;
  size_t NP, UMAX;
  union_bounds(c, &NP, &UMAX);
  const bool shared = (c.flags & MOE_FLAG_SHARED_EXPERT) != 0;
  const bool splitk = (c.flags & MOE_FLAG_SPLITK_DOWN) != 0;
  const size_t n_cnt = shared ? E + 1 : E;
  const size_t nr_max = (I + G - 1) / G, nrd_max = (H + G - 1) / G;
  *pl = moe::FusedPlan{};
  pl->G = (int)G;
  pl->max_tokens = (int)MM;
  pl->max_pairs = (int)NP;
  pl->max_union = (int)UMAX;
  pl->rpc_max = (int)nrd_max;
  pl->slot_gu = (int)align_up(nr_max * H + 2 * (nr_max * H / 32 + 32), 128);
  pl->slot_d = (int)align_up(nrd_max * (I / 2) + nrd_max * (I / 32) + 32, 128);
  pl->nr_max = (int)nr_max;
  pl->dchunks = (int)((H + moe::kSkChunk - 1) / moe::kSkChunk);
  if (splitk) pl->slot_d = (int)align_up(nr_max * (H / 2) + 2 * H, 128);  // K rows + <= 2 scale rows
  // MMA partials of entries with several pairs: per gate/up slot, one float4
  // per lane for each (K chunk = item, 8-row group, 8-pair tile)
  const size_t gu_items_max = (nr_max + moe::kGuRowsPerItem - 1) / moe::kGuRowsPerItem;
  pl->part_ct = (int)std::min<size_t>(moe::kMaxPairTiles, (MM + 7) / 8);
  pl->part_slot = (MM >= (size_t)moe::kMmaMinPairs) ? (int)(gu_items_max * ((nr_max + 7) / 8) * pl->part_ct * 32 * 16) : 0;
  pl->hpairs = (int)std::min<size_t>(moe::kHPairs, MM);
  pl->hslot = splitk ? 0 : (int)align_up((size_t)pl->hpairs * I * 2 + moe::kHPairs * 4, 16);
  const size_t kMaxSlots = moe::kMaxSlots;
  size_t off = 0;
  auto take = [&](size_t bytes, size_t a) { off = align_up(off, a); size_t o = off; off += bytes; return o; };
  pl->o_bar = (int)take((5 * kMaxSlots + 1) * 8 + 2 * kMaxSlots * 4, 16);
  pl->o_misc = (int)take((3 * moe::kMaxTokens + moe::kFusedWarps * moe::kMaxRowsPerCta * 4 + 8) * 4, 16);
  pl->o_ids = (int)take(NP * 4, 16);
  pl->o_w = (int)take(NP * 4, 16);
  pl->o_pm = (int)take(NP * 4, 16);
  pl->o_ppos = (int)take(NP * 4, 16);
  pl->o_union = (int)take(UMAX * 4, 16);
  pl->o_poff = (int)take((UMAX + 1) * 4, 16);
  pl->o_cnt = (int)take(n_cnt * 4, 16);
  pl->o_act = (int)take(MM * H, 16);
  pl->o_dsm = (int)take(splitk ? 0 : NP * nrd_max * 4, 16);
  if (splitk) {
    pl->o_hsm = (int)take(UMAX * MM * nr_max * 4, 16);
    pl->o_ycta = (int)take(std::max<size_t>(MM * H, moe::kConsumers * 32) * 4, 16);
    pl->o_chunk = (int)take((pl->dchunks + UMAX) * 4, 16);
    pl->o_pw = (int)take(NP * 4, 16);
  }
  off = align_up(off, 128);
  if (off >= smem_limit) return false;
  // each down slot carries its staged h
  const size_t room = smem_limit - off;
  const size_t per = pl->slot_gu + pl->part_slot + pl->slot_d + pl->hslot;
  size_t n_both = room / per;
  if (n_both < 2) return false;
  size_t ns_gu, ns_d;
  if (n_both >= UMAX) {
    ns_gu = ns_d = UMAX;
  } else {
    ns_gu = ns_d = n_both;
    ns_gu += (room - n_both * per) / (pl->slot_gu + pl->part_slot);
    if (ns_gu > UMAX) ns_gu = UMAX;
  }
  if (ns_gu > kMaxSlots) ns_gu = kMaxSlots;
  if (ns_d > kMaxSlots) ns_d = kMaxSlots;
  pl->ns_gu = (int)ns_gu;
  pl->ns_d = (int)ns_d;
  pl->o_h = (int)off;
  off = align_up(off + ns_d * pl->hslot, 128);
  pl->o_part = (int)off;
  off = align_up(off + ns_gu * (size_t)pl->part_slot, 128);
  // ring_gu also holds the router rows of the CTA and then the gathered
  // logits [M][E] fp32 between routing and the first weight chunk; with a
  // shared expert they start one slot in (slot 0 fills during routing)
  pl->wr_bytes_max = (int)(((E + G - 1) / G) * H * 4);
  if ((E + G - 1) / G > (size_t)moe::kMaxRowsPerCta) return false;  // router rows per CTA
  const size_t staged = std::max((size_t)pl->wr_bytes_max, MM * E * 4) + (shared ? pl->slot_gu : 0);
  const size_t ring_gu_bytes = align_up(std::max(ns_gu * (size_t)pl->slot_gu, staged), 128);
  pl->o_ring_gu = (int)off;
  pl->o_ring_d = (int)(off + ring_gu_bytes);
  pl->smem_bytes = (int)(pl->o_ring_d + ns_d * pl->slot_d);
  // ring_d holds the bf16 activations during routing when they fit (after
  // slot 0 with a shared expert)
  pl->x_staged = (MM * H * 2 + (shared ? pl->slot_d : 0) <= ns_d * (size_t)pl->slot_d) ? 1 : 0;
  return (size_t)pl->smem_bytes <= smem_limit;
}

// Shared-memory plan of the tensor-core kernel (mirrors k_tc's carving).
// Returns false when the shape is outside what k_tc covers or does not fit.
bool make_tc_plan(const moe_config& c, int sm_count, size_t smem_limit, moe::TcPlan* pl) {
  const size_t H = c.hidden, I = c.inter, E = c.num_experts, MM = c.max_tokens;
  const size_t G = sm_count;
  if (H % 128 || I % 128) return false;  // K-chunks of 128 elements
  size_t NP, UMAX;
  union_bounds(c, &NP, &UMAX);
  const size_t KCH = H / 128;
  *pl = moe::TcPlan{};
  pl->G = (int)G;
  pl->max_pairs = (int)NP;
  pl->max_union = (int)UMAX;
  const size_t units_max = UMAX * (I / 4);
  // down projection on tensor cores: forced by a flag, else from
  // MOE_TC_DOWN_MMA_MIN_TOKENS tokens on; its W2 stages (128 rows x 128
  // elements) take 16-unit gate/up slots of one K-chunk, a lane holds I/32
  // values of h (I <= 1024), and I <= H
  const bool mma_down = !(c.flags & MOE_FLAG_TC_DOWN_CUDA) &&
                        ((c.flags & MOE_FLAG_TC_DOWN_MMA) || MM >= MOE_TC_DOWN_MMA_MIN_TOKENS) && I <= 1024 &&
                        I <= H;  // a down tile's scale factors fit a gate/up tile's tensor-memory columns
  if ((c.flags & MOE_FLAG_TC_DOWN_MMA) && !mma_down) return false;
  const size_t tu_max =
      mma_down ? moe::kTcMaxUnits : std::min<size_t>(moe::kTcMaxUnits, (units_max + G - 1) / G);
  pl->tu_max = (int)tu_max;
  pl->ks = (!mma_down && tu_max <= 12 && KCH % 2 == 0) ? 2 : 1;
  pl->mma_down = mma_down ? 1 : 0;
  pl->dkch = (int)(I / 128);
  pl->bd_bytes = (int)(I / 128 * 4 * 1024);
  const size_t ks = pl->ks, nstage = KCH / ks;
  pl->nb_max = (int)std::max<size_t>(8, (MM + 7) / 8 * 8);
  pl->slot_gu = (int)(tu_max * ks * 1024);
  pl->bx_bytes = (int)(KCH * (pl->nb_max / 8) * 1024);
  const size_t overread = (moe::kTcMaxUnits - tu_max) * ks * 1024;  // junk MMA rows past the last slot
  pl->sc_bytes = (int)align_up(std::max<size_t>(8 * tu_max * (H / 32), mma_down ? 128 * (I / 32) : 0), 128);
  const size_t nrd_max = (H + G - 1) / G;
  pl->rpc_max = (int)nrd_max;
  pl->slot_d = (int)align_up(nrd_max * (I / 2) + nrd_max * (I / 32) + 32, 128);
  pl->hpairs = 0;  // h is read from L2 by each down item (no staged copy)
  pl->hslot = 0;
  if ((E + G - 1) / G > (size_t)moe::kMaxRowsPerCta) return false;
  pl->wr_bytes_max = (int)align_up(((E + G - 1) / G) * H * 4, 128);
  const size_t lg_bytes = align_up(MM * E * 4 + E * 4, 128);  // gathered logits + union scratch
  // fixed regions
  size_t fixed = align_up(std::max<size_t>(pl->bx_bytes, overread), 1024) + 2 * pl->sc_bytes;
  const size_t bar_bytes = (2 * moe::kTcMaxSlots + 4 + 3 * moe::kMaxSlots + 1 + 14) * 8 + moe::kMaxSlots * 4;
  // tensor memory: 2 accumulators of 32 columns, 2 tiles' scale factors (4
  // columns per K-chunk), 4 columns of token scale factors
  const size_t cols = 64 + 8 * KCH + 4;
  if (cols > 512) return false;
  pl->tmem_cols = 32;
  while ((size_t)pl->tmem_cols < cols) pl->tmem_cols *= 2;
  const size_t misc_bytes = (3 * moe::kMaxTokens + moe::kTcWarps * moe::kMaxRowsPerCta * 4 + 8 + moe::kTcMaxTiles) * 4;
  // tiles a CTA may get: at most one more than the rounds of tu_max-unit tiles
  if ((units_max + G * tu_max - 1) / (G * tu_max) + 1 > (size_t)moe::kTcMaxTiles) return false;
  const size_t dsm_bytes = mma_down ? 0 : NP * nrd_max * 4;  // per-pair down rows (CUDA-core down)
  const size_t small = align_up(bar_bytes, 16) + align_up(misc_bytes, 16) + align_up(UMAX * 4, 16) + 4 * align_up(NP * 4, 16) +
                       align_up(UMAX * 4, 16) + align_up((UMAX + 1) * 4, 16) + align_up(dsm_bytes, 16);
  fixed += small + 1024 /* alignment slack */ + 4 * 128;
  if (mma_down) fixed += 2 * (size_t)pl->bd_bytes + 1024 + 4 * moe::kTcDownPairs * 4 + align_up((UMAX + 1) * 4, 16);
  if (fixed >= smem_limit) return false;
  size_t room = smem_limit - fixed;
  // down ring (CUDA-core down): up to 8 entries in flight, at least 2
  size_t ns_d = mma_down ? 0 : std::min<size_t>(UMAX, 8), per_d = pl->slot_d + pl->hslot;
  while (ns_d > 2 && room < ns_d * per_d + 2 * (size_t)pl->slot_gu) --ns_d;
  if (room < ns_d * per_d) return false;
  room -= ns_d * per_d;
  // the deepest gate/up ring whose exact layout fits (the estimate above
  // is conservative)
  const size_t ns_min = (nstage >= 2) ? 2 : 1;
  if (room / pl->slot_gu < ns_min) return false;
  for (size_t ns_gu = std::min<size_t>({(size_t)moe::kTcMaxSlots, nstage, room / pl->slot_gu + 2}); ns_gu >= ns_min;
       --ns_gu) {
  pl->ns_gu = (int)ns_gu;
  pl->ns_d = (int)ns_d;
  // layout
  // routing scratch: the router rows at the start of the gate/up ring; the
  // gathered logits after them when they fit there, else in the down ring
  // after the staged x (both rings are idle until routing ends)
  const size_t ring_gu_bytes = ns_gu * (size_t)pl->slot_gu;
  const size_t ring_d_bytes = ns_d * (size_t)pl->slot_d + ns_d * (size_t)pl->hslot;
  const bool x_fits = MM * H * 2 <= ring_d_bytes;
  // a region of its own when there is room (then no second proxy fence);
  // with the tensor-core down, the B operand buffers (idle until routing ends)
  const bool lg_in_bd = mma_down && lg_bytes <= 2 * (size_t)pl->bd_bytes;
  const bool lg_own = lg_in_bd || (fixed + ns_gu * (size_t)pl->slot_gu + ns_d * per_d + lg_bytes + 128 <= smem_limit &&
                                   lg_bytes <= 16384);
  const bool lg_in_gu = !lg_own && pl->wr_bytes_max + lg_bytes <= ring_gu_bytes;
  const bool lg_in_d = !lg_own && !lg_in_gu && (x_fits ? align_up(MM * H * 2, 128) : 0) + lg_bytes <= ring_d_bytes;
  size_t off = 0;
  auto take = [&](size_t bytes, size_t a) { off = align_up(off, a); size_t o = off; off += bytes; return o; };
  pl->o_ring_gu = (int)take(
      std::max(ring_gu_bytes, (size_t)pl->wr_bytes_max + ((lg_own || lg_in_gu || lg_in_d) ? 0 : lg_bytes)), 1024);
  pl->o_bx = (int)take(std::max<size_t>(pl->bx_bytes, overread), 1024);
  pl->o_sf = (int)off;  // (no shared-memory scale-factor staging)
  pl->o_sc = (int)take(2 * (size_t)pl->sc_bytes, 128);
  pl->o_sfb = (int)off;
  pl->o_bd = mma_down ? (int)take(2 * (size_t)pl->bd_bytes, 1024) : 0;
  pl->o_dsc = mma_down ? (int)take(4 * moe::kTcDownPairs * 4, 16) : 0;
  pl->o_dtoff = mma_down ? (int)take((UMAX + 1) * 4, 16) : 0;
  pl->o_ring_d = (int)take(ns_d * (size_t)pl->slot_d, 128);
  pl->o_h = (int)take(ns_d * (size_t)pl->hslot, 16);
  pl->x_staged = x_fits ? 1 : 0;
  pl->lg_own = lg_own ? 1 : 0;
  pl->o_lg = lg_in_bd ? pl->o_bd
             : lg_own ? (int)take(lg_bytes, 128)
             : lg_in_d ? pl->o_ring_d + (int)(x_fits ? align_up(MM * H * 2, 128) : 0)
                       : pl->o_ring_gu + pl->wr_bytes_max;
  pl->o_bar = (int)take(bar_bytes, 16);
  pl->o_misc = (int)take(misc_bytes, 16);
  pl->o_hready = (int)take(UMAX * 4, 16);
  pl->o_ids = (int)take(NP * 4, 16);
  pl->o_w = (int)take(NP * 4, 16);
  pl->o_pm = (int)take(NP * 4, 16);
  pl->o_ppos = (int)take(NP * 4, 16);
  pl->o_union = (int)take(UMAX * 4, 16);
  pl->o_poff = (int)take((UMAX + 1) * 4, 16);
  pl->o_dsm = (int)take(dsm_bytes, 16);
  pl->smem_bytes = (int)(off + 1024);
  if ((size_t)pl->smem_bytes <= smem_limit) return true;
  }
  return false;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

// The gate/up code maps of k_tc over the caller's w13_codes [Eall][2I][H/2]
// (4-bit elements): dimensions (128 elements of a K-chunk | 4 rows, H/2 bytes
// apart | gate/up, I rows apart | K-chunk, 64 bytes apart | 4-row quad,
// 4 rows apart), unpacked to 16 bytes per 16 codes with a 128-byte swizzle.
// Map n-1 copies n units (quads, coordinate e*I/2 + j for gate rows 4j..4j+3
// of expert e) x ks K-chunks. The coordinates k_tc issues keep j < I/4, so a
// copy never reaches past expert e's up rows.
bool encode_w13_maps(const void* w13c, size_t Eall, size_t H, size_t I, int ks, CUtensorMap* maps) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(w13c) & 31) return false;  // 16U4_ALIGN16B wants 32-byte alignment
  const cuuint64_t dims[5] = {128, 4, 2, (cuuint64_t)(H / 128), (cuuint64_t)(Eall * (I / 2))};
  const cuuint64_t strides[4] = {(cuuint64_t)(H / 2), (cuuint64_t)(I * (H / 2)), 64, (cuuint64_t)(4 * (H / 2))};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  for (int n = 1; n <= moe::kTcMaxUnits; ++n) {
    const cuuint32_t box[5] = {128, 4, 2, (cuuint32_t)ks, (cuuint32_t)n};
    if (enc(maps + n - 1, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 5, const_cast<void*>(w13c), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// The same maps over the re-tiled copy [Eall][I/4][H/128][8][64 B]:
// dimensions (128 elements | 8 rows, 64 bytes apart | K-chunk, 512 bytes
// apart | unit e*I/4 + j, H/128 * 512 bytes apart).
bool encode_w13_maps_repacked(const void* w13r, size_t Eall, size_t H, size_t I, int ks, CUtensorMap* maps) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(w13r) & 31) return false;
  const cuuint64_t dims[4] = {128, 8, (cuuint64_t)(H / 128), (cuuint64_t)(Eall * (I / 4))};
  const cuuint64_t strides[3] = {64, 512, (cuuint64_t)((H / 128) * 512)};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  for (int n = 1; n <= moe::kTcMaxUnits; ++n) {
    const cuuint32_t box[4] = {128, 8, (cuuint32_t)ks, (cuuint32_t)n};
    if (enc(maps + n - 1, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<void*>(w13r), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// The down code map of k_tc's tensor-core down over w2_codes [Eall*H][I]
// (4-bit elements, I/2 bytes a row): a box is one 128-element K-chunk of 128
// rows, unpacked to 16 bytes per 16 codes with a 128-byte swizzle.
bool encode_w2_map(const void* w2c, size_t Eall, size_t H, size_t I, CUtensorMap* map) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  if (reinterpret_cast<uintptr_t>(w2c) & 31) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)I, (cuuint64_t)(Eall * H)};
  const cuuint64_t strides[1] = {(cuuint64_t)(I / 2)};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(w2c), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major copy of W2 for the split-K down projection:
//   kc[e][n][j] = code of W2[e][2j][n] | code of W2[e][2j+1][n] << 4
//   ks[e][nb][r] = scale byte of W2[e][r][32nb .. 32nb+31]
__global__ void k_repack_w2(const uint8_t* w2c, const uint8_t* w2s, int E, int H, int I, uint8_t* kc, uint8_t* ks) {
  const size_t step = (size_t)gridDim.x * blockDim.x;
  const size_t nc = (size_t)E * I * (H / 2);
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < nc; idx += step) {
    const size_t j = idx % (H / 2), n = (idx / (H / 2)) % I, e = idx / ((size_t)(H / 2) * I);
    const uint8_t b0 = w2c[(e * H + 2 * j) * (I / 2) + n / 2], b1 = w2c[(e * H + 2 * j + 1) * (I / 2) + n / 2];
    const uint8_t v0 = (n & 1) ? (b0 >> 4) : (b0 & 0xF), v1 = (n & 1) ? (b1 >> 4) : (b1 & 0xF);
    kc[idx] = (uint8_t)(v0 | (v1 << 4));
  }
  const size_t ns = (size_t)E * (I / 32) * H;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < ns; idx += step) {
    const size_t r = idx % H, nb = (idx / H) % (I / 32), e = idx / ((size_t)H * (I / 32));
    ks[idx] = w2s[(e * H + r) * (I / 32) + nb];
  }
}

// dst[r * dp + j] = src[r * sp + j] for j < width, r < rows (bytes).
__global__ void k_copy_rows(const uint8_t* src, size_t sp, uint8_t* dst, size_t dp, size_t width, size_t rows) {
  const size_t n = width * rows, stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += stride) {
    const size_t r = i / width, j = i - r * width;
    dst[r * dp + j] = src[r * sp + j];
  }
}

bool copy_rows(const uint8_t* src, size_t sp, uint8_t* dst, size_t dp, size_t width, size_t rows) {
  if (width == 0 || rows == 0) return true;
  const size_t blocks = (width * rows + 255) / 256;
  k_copy_rows<<<(unsigned)(blocks < 8192 ? blocks : 8192), 256>>>(src, sp, dst, dp, width, rows);
  return cudaGetLastError() == cudaSuccess;
}

// The one bf16 round of an intra-expert split, after the parts are added.
__global__ void k_round_bf16(const float* y32, __nv_bfloat16* y, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = __float2bfloat16_rn(y32[i]);
}

}  // namespace

struct moe_ctx {
  moe_config cfg{};
  int dev = 0;
  int sm_count = 0;
  int variant = kFused;
  void* ws_base = nullptr;
  size_t ws_bytes = 0;
  moe::Workspace ws{};
  const float* wr = nullptr;
  const uint8_t* w13c = nullptr;
  const uint8_t* w13s = nullptr;
  const uint8_t* w2c = nullptr;
  const uint8_t* w2s = nullptr;
  bool loaded = false;
  // launch shapes
  int grid_route = 0, grid_gateup = 0, grid_down = 0, grid_fused = 0;
  size_t smem_gateup = 0, smem_fused = 0;
  long long spin_limit = 0;
  int force_stall = 0;
  unsigned long long* trace = nullptr;
  void (*fused)(moe::Params, moe::FusedWs, moe::FusedPlan) = nullptr;  // k_fused instantiation
  uint8_t* w2k = nullptr;  // split-K: context-owned K-major W2 (codes, then scales)
  size_t w2k_codes = 0, w2k_bytes = 0;
  moe::FusedPlan plan{};
  moe::FusedWs fws{};
  void (*tc)(moe::Params, moe::TcWs, moe::TcPlan, const moe::TcMaps) = nullptr;  // k_tc instantiation
  moe::TcPlan tplan{};
  moe::TcWs tws{};
  moe::TcMaps maps{};  // encoded at load, passed by value at every launch
  void* owned = nullptr;  // MOE_LOAD_COPY_REPACK: the context's copy of the weights
  int inter_full = 0;     // I of the whole layer (cfg.inter is this part's I/G)
};

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_OOM: return "MOE_ERR_OOM";
    case MOE_ERR_NOT_LOADED: return "MOE_ERR_NOT_LOADED";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_BAD_WEIGHTS: return "MOE_ERR_BAD_WEIGHTS";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status moe_create(const moe_config* cfg, moe_ctx** out) {
  if (!cfg || !out) return MOE_ERR_INVALID_ARG;
  moe_status v = validate_config(*cfg);
  if (v != MOE_OK) return v;
  moe_config part{};
  v = shard_config(*cfg, &part);
  if (v != MOE_OK) return v;
  const moe_config c = part;  // from here on, the layer this context computes
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) return MOE_ERR_CUDA;
  if (c.device < 0 || c.device >= ndev) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(c.device);
  if (!guard.ok) return MOE_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, c.device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;  // built for sm_100a only

  moe_ctx* ctx = new (std::nothrow) moe_ctx();
  if (!ctx) return MOE_ERR_OOM;
  ctx->cfg = c;
  ctx->inter_full = cfg->inter;
  ctx->dev = c.device;
  ctx->sm_count = prop.multiProcessorCount;
  ctx->variant = (c.flags & MOE_FLAG_SPLIT_KERNELS) ? kSplit : kFused;
  ctx->spin_limit = kDefaultSpinLimit;
  {
    const bool sh = (c.flags & MOE_FLAG_SHARED_EXPERT) != 0, f8 = (c.flags & MOE_FLAG_FP8_INTERMEDIATE) != 0;
    const bool sk = (c.flags & MOE_FLAG_SPLITK_DOWN) != 0;
    if (sk)
      ctx->fused = sh ? moe::k_fused<true, false, true> : moe::k_fused<false, false, true>;
    else
      ctx->fused = sh ? (f8 ? moe::k_fused<true, true, false> : moe::k_fused<true, false, false>)
                      : (f8 ? moe::k_fused<false, true, false> : moe::k_fused<false, false, false>);
    ctx->tc = sh ? (f8 ? moe::k_tc<true, true> : moe::k_tc<true, false>)
                 : (f8 ? moe::k_tc<false, true> : moe::k_tc<false, false>);
  }
  // the tensor-core kernel when asked for, or by default from
  // MOE_TC_MIN_TOKENS tokens on, wherever its shape rules hold (the split-K
  // down projection is a CUDA-core kernel option)
  {
    const bool want_tc = (c.flags & MOE_FLAG_TENSOR_CORES) ||
                         (!(c.flags & (MOE_FLAG_CUDA_CORES | MOE_FLAG_SPLITK_DOWN)) && c.max_tokens >= MOE_TC_MIN_TOKENS);
    const bool tc_ok = make_tc_plan(c, prop.multiProcessorCount, (size_t)prop.sharedMemPerBlockOptin, &ctx->tplan) &&
                       encode_tiled() != nullptr;
    if ((c.flags & MOE_FLAG_TENSOR_CORES) && !tc_ok) {
      delete ctx;
      return MOE_ERR_UNSUPPORTED;
    }
    if (ctx->variant == kFused && want_tc && tc_ok) ctx->variant = kTc;
  }

  // workspace layout
  const size_t H = c.hidden, I = c.inter, E = c.num_experts, K = c.top_k, MM = c.max_tokens;
  const size_t NP = MM * K, UMAX = (E < NP ? E : NP);
  size_t NPF, UMAXF;  // pairs and entries of the persistent kernel
  union_bounds(c, &NPF, &UMAXF);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  const size_t o_ctrl = take(64 * sizeof(unsigned));
  const size_t o_logits = take(MM * E * sizeof(float));
  const size_t o_xq = take(MM * H);
  const size_t o_xscale = take(MM * sizeof(float));
  const size_t o_ids = take(NP * sizeof(int));
  const size_t o_wts = take(NP * sizeof(float));
  const size_t o_meta = take(16 * sizeof(int));
  const size_t o_union = take(UMAX * sizeof(int));
  const size_t o_poff = take((UMAX + 1) * sizeof(int));
  const size_t o_ptok = take(NP * sizeof(int));
  const size_t o_pslot = take(NP * sizeof(int));
  const size_t o_pw = take(NP * sizeof(float));
  const size_t o_h = take(NPF * I * sizeof(float));
  const size_t o_flog = take(MM * E * sizeof(unsigned long long));
  const size_t o_gcnt = take(UMAXF * moe::kCounterStride * sizeof(unsigned long long));
  const size_t o_tlog = take(MM * E * sizeof(unsigned long long));
  const size_t o_th = take(NPF * I * sizeof(float));
  const size_t o_tcnt = take(2 * UMAXF * moe::kTcCntStride * sizeof(unsigned));
  const size_t o_typ = take(NPF * H * sizeof(float));
  const size_t o_tdc = take(2 * moe::kTcCntStride * sizeof(unsigned));
  const bool splitk = (c.flags & MOE_FLAG_SPLITK_DOWN) != 0;
  const size_t o_ypart = take(splitk ? (size_t)ctx->sm_count * MM * H * sizeof(float) : 0);
  const size_t o_fcnt = take(sizeof(unsigned long long));
  ctx->ws_bytes = off;
  if (cudaMalloc(&ctx->ws_base, ctx->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete ctx;
    return MOE_ERR_OOM;
  }
  if (cudaMemset(ctx->ws_base, 0, ctx->ws_bytes) != cudaSuccess) {
    cudaFree(ctx->ws_base);
    delete ctx;
    return MOE_ERR_CUDA;
  }
  char* b = static_cast<char*>(ctx->ws_base);
  moe::Workspace& w = ctx->ws;
  w.ctrl = reinterpret_cast<unsigned*>(b + o_ctrl);
  w.logits = reinterpret_cast<float*>(b + o_logits);
  w.xq = reinterpret_cast<uint8_t*>(b + o_xq);
  w.xscale = reinterpret_cast<float*>(b + o_xscale);
  w.ids = reinterpret_cast<int*>(b + o_ids);
  w.wts = reinterpret_cast<float*>(b + o_wts);
  w.meta = reinterpret_cast<int*>(b + o_meta);
  w.union_ids = reinterpret_cast<int*>(b + o_union);
  w.pair_off = reinterpret_cast<int*>(b + o_poff);
  w.pair_tok = reinterpret_cast<int*>(b + o_ptok);
  w.pair_slot = reinterpret_cast<int*>(b + o_pslot);
  w.pair_w = reinterpret_cast<float*>(b + o_pw);
  w.h = reinterpret_cast<float*>(b + o_h);
  ctx->fws.logits = reinterpret_cast<unsigned long long*>(b + o_flog);
  ctx->fws.gu_cnt = reinterpret_cast<unsigned long long*>(b + o_gcnt);
  ctx->fws.epoch = w.ctrl + 5;
  ctx->tws.logits = reinterpret_cast<unsigned long long*>(b + o_tlog);
  ctx->tws.h = reinterpret_cast<float*>(b + o_th);
  ctx->tws.hcnt = reinterpret_cast<unsigned*>(b + o_tcnt);
  ctx->tws.ypart = reinterpret_cast<float*>(b + o_typ);
  ctx->tws.dcnt = reinterpret_cast<unsigned*>(b + o_tdc);
  ctx->tws.epoch = w.ctrl + 6;
  ctx->fws.ypart = reinterpret_cast<float*>(b + o_ypart);
  ctx->fws.fin_cnt = reinterpret_cast<unsigned long long*>(b + o_fcnt);

  // launch shapes
  ctx->grid_route = (int)(E < (size_t)ctx->sm_count ? E : (size_t)ctx->sm_count);
  ctx->smem_gateup = MM * H * 2;
  // The dynamic shared-memory limit of a kernel is per device and process,
  // not per context: every context raises it to the device's opt-in maximum
  // (the same value each time), so creating a context with a smaller plan
  // never lowers the limit another context's launches rely on.
  const int smem_optin = (int)prop.sharedMemPerBlockOptin;
  cudaError_t err = cudaFuncSetAttribute(moe::k_gateup, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
  int occ_g = 0, occ_d = 0;
  if (err == cudaSuccess)
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_g, moe::k_gateup, moe::kThreads, ctx->smem_gateup);
  if (err == cudaSuccess)
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_d, moe::k_down, moe::kThreads, 0);
  const bool plan_ok = make_plan(c, ctx->sm_count, (size_t)prop.sharedMemPerBlockOptin, &ctx->plan);
  if (err == cudaSuccess && plan_ok)
    err = cudaFuncSetAttribute(ctx->fused, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
  int occ_f = 0;
  if (err == cudaSuccess && plan_ok)
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_f, ctx->fused, moe::kFusedThreads,
                                                        ctx->plan.smem_bytes);
  if (err == cudaSuccess && ctx->variant == kTc) {
    err = cudaFuncSetAttribute(ctx->tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_optin);
    int occ_t = 0;
    if (err == cudaSuccess)
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_t, ctx->tc, moe::kTcThreads, ctx->tplan.smem_bytes);
    if (err == cudaSuccess && occ_t < 1) ctx->variant = kFused;
  }
  if (err != cudaSuccess || occ_g < 1 || occ_d < 1 || !plan_ok || occ_f < 1) {
    cudaGetLastError();
    cudaFree(ctx->ws_base);
    delete ctx;
    return MOE_ERR_UNSUPPORTED;
  }
  ctx->grid_gateup = occ_g * ctx->sm_count;
  ctx->grid_down = occ_d * ctx->sm_count;
  ctx->grid_fused = ctx->plan.G;
  ctx->smem_fused = ctx->plan.smem_bytes;
  *out = ctx;
  return MOE_OK;
}

void moe_destroy(moe_ctx* ctx) {
  if (!ctx) return;
  DeviceGuard guard(ctx->dev);
  if (ctx->ws_base) cudaFree(ctx->ws_base);
  if (ctx->owned) cudaFree(ctx->owned);
  if (ctx->w2k) cudaFree(ctx->w2k);
  delete ctx;
}

moe_status moe_load_experts(moe_ctx* ctx, const float* router_w, const uint8_t* w13_codes,
                            const uint8_t* w13_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                            uint32_t load_flags) {
  if (!ctx || !router_w || !w13_codes || !w13_scales || !w2_codes || !w2_scales) return MOE_ERR_INVALID_ARG;
  if (load_flags & ~(MOE_LOAD_SKIP_VALIDATE | MOE_LOAD_COPY_REPACK)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(router_w) || !aligned16(w13_codes) || !aligned16(w13_scales) || !aligned16(w2_codes) ||
      !aligned16(w2_scales))
    return MOE_ERR_INVALID_ARG;
  const moe_config& c = ctx->cfg;
  const bool part = c.shard_count > 1;
  if (part && !(load_flags & MOE_LOAD_COPY_REPACK)) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  if (!(load_flags & MOE_LOAD_SKIP_VALIDATE)) {
    // the caller's arrays: the whole layer's, also for a part of a split
    const size_t E = c.num_experts + ((c.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0), H = c.hidden,
                 I = ctx->inter_full;
    unsigned* bad = ctx->ws.ctrl + 4;
    if (cudaMemset(bad, 0, sizeof(unsigned)) != cudaSuccess) return MOE_ERR_CUDA;
    moe::k_scan_scales<<<ctx->sm_count * 4, 256>>>(w13_scales, E * 2 * I * (H / 32), bad);
    moe::k_scan_scales<<<ctx->sm_count * 4, 256>>>(w2_scales, E * H * (I / 32), bad);
    unsigned nbad = 0;
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(&nbad, bad, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (nbad) {
      ctx->loaded = false;
      return MOE_ERR_BAD_WEIGHTS;
    }
  }
  const size_t Eall = c.num_experts + ((c.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0);
  const size_t H = c.hidden, I = c.inter;
  if (ctx->owned) {  // a previous copy
    cudaFree(ctx->owned);
    ctx->owned = nullptr;
  }
  ctx->loaded = false;
  ctx->tws.repacked = 0;
  if (load_flags & MOE_LOAD_COPY_REPACK) {
    const size_t b_wr = align_up((size_t)c.num_experts * H * 4, 256), b_13 = align_up(Eall * 2 * I * (H / 2), 256),
                 b_13s = align_up(Eall * 2 * I * (H / 32), 256), b_2 = align_up(Eall * H * (I / 2), 256),
                 b_2s = align_up(Eall * H * (I / 32), 256);
    if (cudaMalloc(&ctx->owned, b_wr + b_13 + b_13s + b_2 + b_2s) != cudaSuccess) {
      cudaGetLastError();
      ctx->owned = nullptr;
      return MOE_ERR_OOM;
    }
    char* o = static_cast<char*>(ctx->owned);
    float* wr = reinterpret_cast<float*>(o);
    uint8_t* w13 = reinterpret_cast<uint8_t*>(o + b_wr);
    uint8_t* w13s = w13 + b_13;
    uint8_t* w2 = w13s + b_13s;
    uint8_t* w2s = w2 + b_2;
    bool okc = cudaMemcpy(wr, router_w, (size_t)c.num_experts * H * 4, cudaMemcpyDeviceToDevice) == cudaSuccess;
    void* w13_part = nullptr;  // a part's gate/up codes before the tensor-core re-tiling
    if (okc && part) {
      // this part's rows of W13 (gate rows g*I.., up rows I_full + g*I..) and
      // columns of W2, from the whole layer's arrays
      const size_t IF = ctx->inter_full, g = c.shard_index;
      uint8_t* d13 = w13;
      if (ctx->variant == kTc) {
        okc = cudaMalloc(&w13_part, b_13) == cudaSuccess;
        d13 = static_cast<uint8_t*>(w13_part);
      }
      const size_t rc = H / 2, rs = H / 32;  // bytes per W13 row: codes, scales
      for (int half = 0; half < 2 && okc; ++half) {
        const size_t src_row = half * IF + g * I, dst_row = half * I;
        okc = copy_rows(w13_codes + src_row * rc, 2 * IF * rc, d13 + dst_row * rc, 2 * I * rc, I * rc, Eall) &&
              copy_rows(w13_scales + src_row * rs, 2 * IF * rs, w13s + dst_row * rs, 2 * I * rs, I * rs, Eall);
      }
      okc = okc && copy_rows(w2_codes + g * (I / 2), IF / 2, w2, I / 2, I / 2, Eall * H) &&
            copy_rows(w2_scales + g * (I / 32), IF / 32, w2s, I / 32, I / 32, Eall * H) &&
            cudaDeviceSynchronize() == cudaSuccess;
      if (okc && ctx->variant == kTc) w13_codes = static_cast<const uint8_t*>(w13_part);
    } else if (okc) {
      okc = cudaMemcpy(w13s, w13_scales, Eall * 2 * I * (H / 32), cudaMemcpyDeviceToDevice) == cudaSuccess &&
            cudaMemcpy(w2, w2_codes, Eall * H * (I / 2), cudaMemcpyDeviceToDevice) == cudaSuccess &&
            cudaMemcpy(w2s, w2_scales, Eall * H * (I / 32), cudaMemcpyDeviceToDevice) == cudaSuccess;
    }
    if (okc && ctx->variant == kTc) {
      moe::k_repack_w13<<<ctx->sm_count * 8, 256>>>(w13_codes, w13, (int)Eall, (int)H, (int)I);
      okc = cudaGetLastError() == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
      ctx->tws.repacked = 1;
    } else if (okc && !part) {
      okc = cudaMemcpy(w13, w13_codes, Eall * 2 * I * (H / 2), cudaMemcpyDeviceToDevice) == cudaSuccess &&
            cudaDeviceSynchronize() == cudaSuccess;
    }
    if (w13_part) cudaFree(w13_part);
    if (!okc) {
      cudaGetLastError();
      cudaFree(ctx->owned);
      ctx->owned = nullptr;
      ctx->tws.repacked = 0;
      return MOE_ERR_CUDA;
    }
    router_w = wr;
    w13_codes = w13;
    w13_scales = w13s;
    w2_codes = w2;
    w2_scales = w2s;
  }
  if (ctx->variant == kTc) {
    const bool enc_ok = ctx->tws.repacked
                            ? encode_w13_maps_repacked(w13_codes, Eall, H, I, ctx->tplan.ks, ctx->maps.m)
                            : encode_w13_maps(w13_codes, Eall, H, I, ctx->tplan.ks, ctx->maps.m);
    if (!enc_ok) return MOE_ERR_INVALID_ARG;
    if (ctx->tplan.mma_down && (!encode_w2_map(w2_codes, Eall, H, I, &ctx->maps.w2) || !aligned16(w2_scales)))
      return MOE_ERR_INVALID_ARG;
  }
  if (c.flags & MOE_FLAG_SPLITK_DOWN) {
    // the K-major W2 copy the split-K down projection streams
    const size_t E = c.num_experts + ((c.flags & MOE_FLAG_SHARED_EXPERT) ? 1 : 0), H = c.hidden, I = c.inter;
    const size_t nc = E * I * (H / 2), ns = E * (I / 32) * H;
    if (!ctx->w2k) {
      if (cudaMalloc(&ctx->w2k, nc + ns) != cudaSuccess) {
        cudaGetLastError();
        ctx->w2k = nullptr;
        ctx->loaded = false;
        return MOE_ERR_OOM;
      }
      ctx->w2k_codes = nc;
      ctx->w2k_bytes = nc + ns;
    }
    k_repack_w2<<<ctx->sm_count * 8, 256>>>(w2_codes, w2_scales, (int)E, (int)H, (int)I, ctx->w2k, ctx->w2k + nc);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      ctx->loaded = false;
      return MOE_ERR_CUDA;
    }
  }
  ctx->wr = router_w;
  ctx->w13c = w13_codes;
  ctx->w13s = w13_scales;
  ctx->w2c = w2_codes;
  ctx->w2s = w2_scales;
  ctx->loaded = true;
  return MOE_OK;
}

moe_status moe_decode(moe_ctx* ctx, const void* x_bf16, int32_t M, void* y_bf16, void* stream,
                      int32_t* topk_ids, float* topk_w, uint8_t* xq, float* xscale, void* xnorm_bf16) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  const moe_config& c = ctx->cfg;
  if (M < 0 || M > c.max_tokens) return MOE_ERR_INVALID_ARG;
  if (M == 0) return MOE_OK;
  if (!x_bf16 || !y_bf16 || !aligned16(x_bf16) || !aligned16(y_bf16)) return MOE_ERR_INVALID_ARG;
  const bool part = c.shard_count > 1;  // y is the part's fp32 sum
  const size_t xbytes = (size_t)M * c.hidden * 2, ybytes = xbytes * (part ? 2 : 1);
  const char* xb = static_cast<const char*>(x_bf16);
  const char* yb = static_cast<const char*>(y_bf16);
  if (xb < yb + ybytes && yb < xb + xbytes) return MOE_ERR_INVALID_ARG;  // aliasing
  if ((xq && !aligned16(xq)) || (topk_ids && (reinterpret_cast<uintptr_t>(topk_ids) & 3)) ||
      (topk_w && (reinterpret_cast<uintptr_t>(topk_w) & 3)) ||
      (xscale && (reinterpret_cast<uintptr_t>(xscale) & 3)) || (xnorm_bf16 && !aligned16(xnorm_bf16)))
    return MOE_ERR_INVALID_ARG;
  if (xnorm_bf16 && !(c.flags & MOE_FLAG_PRE_RMSNORM)) return MOE_ERR_INVALID_ARG;
  if (!ctx->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard guard(ctx->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  moe::Params p{};
  p.H = c.hidden;
  p.I = c.inter;
  p.E = c.num_experts;
  p.K = c.top_k;
  p.M = M;
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.y = part ? nullptr : static_cast<__nv_bfloat16*>(y_bf16);
  p.y32 = part ? static_cast<float*>(y_bf16) : nullptr;
  p.wr = ctx->wr;
  p.w13c = ctx->w13c;
  p.w13s = ctx->w13s;
  p.w2c = ctx->w2c;
  p.w2s = ctx->w2s;
  p.w2kc = ctx->w2k;
  p.w2ks = ctx->w2k ? ctx->w2k + ctx->w2k_codes : nullptr;
  p.ws = ctx->ws;
  p.out_ids = topk_ids;
  p.out_w = topk_w;
  p.out_xq = xq;
  p.out_xscale = xscale;
  p.spin_limit = ctx->spin_limit;
  p.force_stall = ctx->force_stall;
  p.trace = ctx->trace;
  p.pre_rmsnorm = (c.flags & MOE_FLAG_PRE_RMSNORM) ? 1 : 0;
  p.out_xn = static_cast<__nv_bfloat16*>(xnorm_bf16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ctx->variant == kSplit) {
    moe::k_route<<<ctx->grid_route, moe::kThreads, 0, st>>>(p);
    moe::k_gateup<<<ctx->grid_gateup, moe::kThreads, (size_t)M * c.hidden * 2, st>>>(p);
    moe::k_down<<<ctx->grid_down, moe::kThreads, 0, st>>>(p);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctx->variant == kTc ? ctx->tplan.G : ctx->grid_fused);
    cfg.blockDim = dim3(ctx->variant == kTc ? moe::kTcThreads : moe::kFusedThreads);
    cfg.dynamicSmemBytes = ctx->variant == kTc ? ctx->tplan.smem_bytes : ctx->smem_fused;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t le = ctx->variant == kTc ? cudaLaunchKernelEx(&cfg, ctx->tc, p, ctx->tws, ctx->tplan, ctx->maps)
                                               : cudaLaunchKernelEx(&cfg, ctx->fused, p, ctx->fws, ctx->plan);
    if (le != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
  }
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_sync_status(moe_ctx* ctx, void* stream) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(ctx->dev);
  if (!guard.ok) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  unsigned status = 0;
  if (cudaMemcpy(&status, ctx->ws.ctrl, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (status == 0) return MOE_OK;
  // a wait gave up: clear the whole workspace (status, barrier state, epoch
  // and every epoch-tagged word) on the context's stream, so the next call
  // starts clean; only that stream is waited for
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ctx->ws_base, 0, ctx->ws_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_ERR_TIMEOUT;
}

moe_status moe_plan_query(const moe_config* cfg, int32_t sm_count, size_t smem_limit, char* buf, size_t len) {
  if (!cfg || !buf || len == 0 || sm_count < 1) return MOE_ERR_INVALID_ARG;
  moe_status v = validate_config(*cfg);
  if (v != MOE_OK) return v;
  moe_config part{};
  v = shard_config(*cfg, &part);
  if (v != MOE_OK) return v;
  cfg = &part;  // the plan of this part's layer (the whole layer when unsplit)
  moe::FusedPlan pl{};
  const bool ok = make_plan(*cfg, sm_count, smem_limit, &pl);
  moe::TcPlan tp{};
  const bool tok = make_tc_plan(*cfg, sm_count, smem_limit, &tp);
  const bool tc = tok && !(cfg->flags & (MOE_FLAG_SPLIT_KERNELS | MOE_FLAG_CUDA_CORES | MOE_FLAG_SPLITK_DOWN)) &&
                  ((cfg->flags & MOE_FLAG_TENSOR_CORES) || cfg->max_tokens >= MOE_TC_MIN_TOKENS);
  const int n = snprintf(buf, len,
                         "{\"ok\": %s, \"variant\": \"%s\", \"grid\": %d, \"threads\": %d, \"smem\": %d, "
                         "\"slot_gu\": %d, "
                         "\"ns_gu\": %d, \"slot_d\": %d, \"ns_d\": %d, \"rows_per_cta_down\": %d, "
                         "\"router_bytes_per_cta\": %d, \"o_act\": %d, \"o_dsm\": %d, \"o_ring_gu\": %d, "
                         "\"o_ring_d\": %d, \"o_h\": %d, \"hslot\": %d, \"hpairs\": %d, \"x_staged\": %d, "
                         "\"tc\": {\"ok\": %s, \"grid\": %d, \"threads\": %d, \"smem\": %d, \"ks\": %d, "
                         "\"tu_max\": %d, \"nb_max\": %d, \"ns_gu\": %d, \"slot_gu\": %d, \"ns_d\": %d, "
                         "\"slot_d\": %d, \"rpc_max\": %d, \"hslot\": %d, \"hpairs\": %d, \"wr_bytes_max\": %d, "
                         "\"x_staged\": %d, \"o_ring_gu\": %d, \"o_bx\": %d, \"o_sf\": %d, \"o_sc\": %d, "
                         "\"o_sfb\": %d, \"o_ring_d\": %d, \"o_h\": %d, \"o_bar\": %d, \"o_misc\": %d, "
                         "\"o_ids\": %d, \"o_w\": %d, \"o_pm\": %d, \"o_ppos\": %d, \"o_union\": %d, "
                         "\"o_poff\": %d, \"o_dsm\": %d, \"sc_bytes\": %d, \"bx_bytes\": %d, "
                         "\"max_pairs\": %d, \"max_union\": %d, \"o_lg\": %d, \"tmem_cols\": %d, \"lg_own\": %d, "
                         "\"mma_down\": %d, \"dkch\": %d, \"o_bd\": %d, \"bd_bytes\": %d, \"o_dsc\": %d, "
                         "\"o_dtoff\": %d}}",
                         (tc || ok) ? "true" : "false", tc ? "tc" : "fused", pl.G, moe::kFusedThreads, pl.smem_bytes,
                         pl.slot_gu, pl.ns_gu, pl.slot_d, pl.ns_d, pl.rpc_max, pl.wr_bytes_max, pl.o_act, pl.o_dsm,
                         pl.o_ring_gu, pl.o_ring_d, pl.o_h, pl.hslot, pl.hpairs, pl.x_staged, tok ? "true" : "false",
                         tp.G, moe::kTcThreads, tp.smem_bytes, tp.ks, tp.tu_max, tp.nb_max, tp.ns_gu, tp.slot_gu,
                         tp.ns_d, tp.slot_d, tp.rpc_max, tp.hslot, tp.hpairs, tp.wr_bytes_max, tp.x_staged,
                         tp.o_ring_gu, tp.o_bx, tp.o_sf, tp.o_sc, tp.o_sfb, tp.o_ring_d, tp.o_h, tp.o_bar, tp.o_misc,
                         tp.o_ids, tp.o_w, tp.o_pm, tp.o_ppos, tp.o_union, tp.o_poff, tp.o_dsm, tp.sc_bytes,
                         tp.bx_bytes, tp.max_pairs, tp.max_union, tp.o_lg, tp.tmem_cols, tp.lg_own, tp.mma_down, tp.dkch,
                         tp.o_bd, tp.bd_bytes, tp.o_dsc, tp.o_dtoff);
  if (n < 0 || (size_t)n >= len) return MOE_ERR_INVALID_ARG;
  return (tc || ok) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

moe_status moe_debug_set_wait(moe_ctx* ctx, long long budget_cycles, int force_stall) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  ctx->spin_limit = budget_cycles > 0 ? budget_cycles : kDefaultSpinLimit;
  ctx->force_stall = force_stall ? 1 : 0;
  return MOE_OK;
}

moe_status moe_debug_set_trace(moe_ctx* ctx, unsigned long long* trace) {
  if (!ctx) return MOE_ERR_INVALID_ARG;
  if (trace && (reinterpret_cast<uintptr_t>(trace) & 7)) return MOE_ERR_INVALID_ARG;
  ctx->trace = trace;
  return MOE_OK;
}

moe_status moe_query(const moe_ctx* ctx, char* buf, size_t len) {
  if (!ctx || !buf || len == 0) return MOE_ERR_INVALID_ARG;
  const moe_config& c = ctx->cfg;
  const moe::FusedPlan& pl = ctx->plan;
  int n;
  if (ctx->variant == kSplit) {
    n = snprintf(buf, len,
                 "{\"lib\": \"libmoe\", \"arch\": \"sm_100a\", \"device\": %d, \"sm_count\": %d, "
                 "\"variant\": \"split\", \"kernels\": [\"k_route\", \"k_gateup\", \"k_down\"], "
                 "\"grid\": [%d, %d, %d], \"threads\": %d, \"smem_gateup\": %zu, "
                 "\"hidden\": %d, \"inter\": %d, \"num_experts\": %d, \"top_k\": %d, \"max_tokens\": %d}",
                 ctx->dev, ctx->sm_count, ctx->grid_route, ctx->grid_gateup, ctx->grid_down, moe::kThreads,
                 ctx->smem_gateup, c.hidden, c.inter, c.num_experts, c.top_k, c.max_tokens);
  } else if (ctx->variant == kTc) {
    const moe::TcPlan& tp = ctx->tplan;
    n = snprintf(buf, len,
                 "{\"lib\": \"libmoe\", \"arch\": \"sm_100a\", \"device\": %d, \"sm_count\": %d, "
                 "\"variant\": \"tc\", \"kernels\": [\"k_tc\"], \"grid\": [%d], \"threads\": %d, "
                 "\"smem\": %d, \"gate_up\": \"tcgen05.mma kind::mxf8f6f4 block_scale M=128 N=%d\", "
                 "\"units_per_tile\": %d, \"kchunks_per_stage\": %d, \"ring_gu\": [%d, %d], \"ring_d\": [%d, %d], "
                 "\"x_staged\": %d, \"down\": \"%s\", \"pdl\": true, \"pre_rmsnorm\": %s, \"shared_expert\": %s, "
                 "\"fp8_intermediate\": %s, \"hidden\": %d, \"inter\": %d, \"num_experts\": %d, \"top_k\": %d, "
                 "\"max_tokens\": %d}",
                 ctx->dev, ctx->sm_count, tp.G, moe::kTcThreads, tp.smem_bytes, tp.nb_max, tp.tu_max, tp.ks, tp.ns_gu,
                 tp.slot_gu, tp.ns_d, tp.slot_d, tp.x_staged, tp.mma_down ? "tensor_cores" : "cuda_cores", (c.flags & MOE_FLAG_PRE_RMSNORM) ? "true" : "false",
                 (c.flags & MOE_FLAG_SHARED_EXPERT) ? "true" : "false",
                 (c.flags & MOE_FLAG_FP8_INTERMEDIATE) ? "true" : "false", c.hidden, c.inter, c.num_experts, c.top_k,
                 c.max_tokens);
  } else {
    n = snprintf(buf, len,
                 "{\"lib\": \"libmoe\", \"arch\": \"sm_100a\", \"device\": %d, \"sm_count\": %d, "
                 "\"variant\": \"fused\", \"kernels\": [\"k_fused\"], \"grid\": [%d], \"threads\": %d, "
                 "\"smem\": %d, \"ring_gu\": [%d, %d], \"ring_d\": [%d, %d], \"pdl\": true, \"pre_rmsnorm\": %s, "
                 "\"shared_expert\": %s, \"fp8_intermediate\": %s, "
                 "\"hidden\": %d, \"inter\": %d, \"num_experts\": %d, \"top_k\": %d, \"max_tokens\": %d}",
                 ctx->dev, ctx->sm_count, pl.G, moe::kFusedThreads, pl.smem_bytes, pl.ns_gu, pl.slot_gu, pl.ns_d,
                 pl.slot_d, (c.flags & MOE_FLAG_PRE_RMSNORM) ? "true" : "false",
                 (c.flags & MOE_FLAG_SHARED_EXPERT) ? "true" : "false",
                 (c.flags & MOE_FLAG_FP8_INTERMEDIATE) ? "true" : "false", c.hidden, c.inter, c.num_experts,
                 c.top_k, c.max_tokens);
  }
  if (n < 0 || (size_t)n >= len) return MOE_ERR_INVALID_ARG;
  // the split: "inter" above is this part's width
  const int m = snprintf(buf + n - 1, len - (n - 1), ", \"shard\": [%d, %d], \"inter_full\": %d, \"y\": \"%s\"}",
                         c.shard_index, c.shard_count, ctx->inter_full, c.shard_count > 1 ? "f32" : "bf16");
  if (m < 0 || (size_t)m >= len - (n - 1)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status moe_round_bf16(const float* y_f32, void* y_bf16, int64_t n, void* stream) {
  if (n < 0 || !y_f32 || !y_bf16 || (reinterpret_cast<uintptr_t>(y_f32) & 3) ||
      (reinterpret_cast<uintptr_t>(y_bf16) & 1))
    return MOE_ERR_INVALID_ARG;
  const char* a = reinterpret_cast<const char*>(y_f32);
  const char* b = static_cast<const char*>(y_bf16);
  if (a < b + 2 * n && b < a + 4 * n) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  const int64_t blocks = (n + 255) / 256;
  k_round_bf16<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      y_f32, static_cast<__nv_bfloat16*>(y_bf16), n);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
