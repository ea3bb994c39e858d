// moe_static.cu -- moe_decode_static: one decode step that allocates nothing.
//
// Some callers cannot allocate device memory at all. Examples are a plugin
// inside a host runtime that owns every byte of device memory, and a serving
// loop that must never call cudaMalloc (the call can synchronise the
// device). Such a caller cannot use moe_create, which allocates the context's
// workspace. moe_decode_static runs the three-kernel form of the step (route,
// gate/up, down). Its scratch comes from the fixed device array g_scratch
// below, which every GPU that loads this library holds until the process
// exits.
//
// Set-up happens once per device, on the first call made with that device
// current. That call looks up the device address of g_scratch with
// cudaGetSymbolAddress, reads the SM count and raises the gate/up kernel's
// dynamic shared-memory limit. Make that first call before any stream
// capture. All calls share the one array and it keeps whatever the last call
// left there, so each call clears the words that must start at zero. Calls
// that overlap on the GPU (different streams, or different host threads)
// race on the array and corrupt each other's results.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_device.cuh"
#include "moe_split.cuh"

namespace {

// Scratch of the allocation-free entry point (MOE_STATIC_SCRATCH_BYTES).
constexpr size_t kStaticScratchBytes = MOE_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
struct DeviceSetup {
  bool done = false;
  unsigned char* scratch = nullptr;  // device address of g_scratch on this device
  int sm_count = 0;
  size_t smem_optin = 0;
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mutex;

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// Carve the workspace for one call out of the scratch array; returns the
// bytes needed (also when they exceed the array, so the caller can reject).
size_t carve(unsigned char* base, size_t H, size_t I, size_t E, size_t K, size_t M, moe::Workspace* w) {
  const size_t NP = M * K, UMAX = (E < NP ? E : NP);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return base + o; };
  w->ctrl = reinterpret_cast<unsigned*>(take(64 * sizeof(unsigned)));
  w->logits = reinterpret_cast<float*>(take(M * E * sizeof(float)));
  w->xq = take(M * H);
  w->xscale = reinterpret_cast<float*>(take(M * sizeof(float)));
  w->ids = reinterpret_cast<int*>(take(NP * sizeof(int)));
  w->wts = reinterpret_cast<float*>(take(NP * sizeof(float)));
  w->meta = reinterpret_cast<int*>(take(16 * sizeof(int)));
  w->union_ids = reinterpret_cast<int*>(take(UMAX * sizeof(int)));
  w->pair_off = reinterpret_cast<int*>(take((UMAX + 1) * sizeof(int)));
  w->pair_tok = reinterpret_cast<int*>(take(NP * sizeof(int)));
  w->pair_slot = reinterpret_cast<int*>(take(NP * sizeof(int)));
  w->pair_w = reinterpret_cast<float*>(take(NP * sizeof(float)));
  w->h = reinterpret_cast<float*>(take(NP * I * sizeof(float)));
  return off;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status setup_device(int dev, DeviceSetup** out) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceSetup& s = g_setup[dev];
  if (!s.done) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(moe::k_gateup, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)prop.sharedMemPerBlockOptin) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    s.scratch = static_cast<unsigned char*>(ptr);
    s.sm_count = prop.multiProcessorCount;
    s.smem_optin = prop.sharedMemPerBlockOptin;
    s.done = true;
  }
  *out = &s;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_decode_static(const moe_config* cfg, const float* router_w, const uint8_t* w13_codes,
                             const uint8_t* w13_scales, const uint8_t* w2_codes, const uint8_t* w2_scales,
                             const void* x_bf16, int32_t M, void* y_bf16, void* stream, int32_t* topk_ids,
                             float* topk_w, uint8_t* xq, float* xscale) {
  if (!cfg) return MOE_ERR_INVALID_ARG;
  const moe_config c = *cfg;
  if (c.hidden < 32 || c.hidden > 8192 || c.hidden % 32) return MOE_ERR_INVALID_ARG;
  if (c.inter < 32 || c.inter > 4096 || c.inter % 32) return MOE_ERR_INVALID_ARG;
  if (c.num_experts < 1 || c.num_experts > moe::kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > c.num_experts || c.top_k > moe::kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (M < 0 || M > moe::kMaxTokens) return MOE_ERR_INVALID_ARG;
  if (c.flags & (MOE_FLAG_SHARED_EXPERT | MOE_FLAG_PRE_RMSNORM | MOE_FLAG_FP8_INTERMEDIATE | MOE_FLAG_SPLITK_DOWN))
    return MOE_ERR_UNSUPPORTED;
  if (c.shard_count > 1) return MOE_ERR_UNSUPPORTED;  // no context to hold a part's copy
  if (M == 0) return MOE_OK;
  if (!router_w || !w13_codes || !w13_scales || !w2_codes || !w2_scales || !x_bf16 || !y_bf16)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(router_w) || !aligned16(w13_codes) || !aligned16(w13_scales) || !aligned16(w2_codes) ||
      !aligned16(w2_scales) || !aligned16(x_bf16) || !aligned16(y_bf16))
    return MOE_ERR_INVALID_ARG;
  const size_t xbytes = (size_t)M * c.hidden * 2;
  const char* xb = static_cast<const char*>(x_bf16);
  const char* yb = static_cast<const char*>(y_bf16);
  if (xb < yb + xbytes && yb < xb + xbytes) return MOE_ERR_INVALID_ARG;
  if ((xq && !aligned16(xq)) || (topk_ids && (reinterpret_cast<uintptr_t>(topk_ids) & 3)) ||
      (topk_w && (reinterpret_cast<uintptr_t>(topk_w) & 3)) ||
      (xscale && (reinterpret_cast<uintptr_t>(xscale) & 3)))
    return MOE_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  DeviceSetup* ds = nullptr;
  const moe_status st = setup_device(dev, &ds);
  if (st != MOE_OK) return st;
  const size_t gate_smem = (size_t)M * c.hidden * 2;  // f16 activations of the gate/up kernel
  if (gate_smem > ds->smem_optin) return MOE_ERR_UNSUPPORTED;

  moe::Params p{};
  const size_t need = carve(ds->scratch, c.hidden, c.inter, c.num_experts, c.top_k, M, &p.ws);
  if (need > kStaticScratchBytes) return MOE_ERR_UNSUPPORTED;
  p.H = c.hidden;
  p.I = c.inter;
  p.E = c.num_experts;
  p.K = c.top_k;
  p.M = M;
  p.x = static_cast<const __nv_bfloat16*>(x_bf16);
  p.y = static_cast<__nv_bfloat16*>(y_bf16);
  p.wr = router_w;
  p.w13c = w13_codes;
  p.w13s = w13_scales;
  p.w2c = w2_codes;
  p.w2s = w2_scales;
  p.out_ids = topk_ids;
  p.out_w = topk_w;
  p.out_xq = xq;
  p.out_xscale = xscale;
  p.spin_limit = 0;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the route kernel's last-CTA ticket (ctrl[3]) must start at zero
  if (cudaMemsetAsync(p.ws.ctrl, 0, 64 * sizeof(unsigned), s) != cudaSuccess) return MOE_ERR_CUDA;
  int occ_g = 0, occ_d = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_g, moe::k_gateup, moe::kThreads, gate_smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_d, moe::k_down, moe::kThreads, 0) != cudaSuccess ||
      occ_g < 1 || occ_d < 1) {
    cudaGetLastError();
    return MOE_ERR_UNSUPPORTED;
  }
  const int grid_route = c.num_experts < ds->sm_count ? c.num_experts : ds->sm_count;
  moe::k_route<<<grid_route, moe::kThreads, 0, s>>>(p);
  moe::k_gateup<<<occ_g * ds->sm_count, moe::kThreads, gate_smem, s>>>(p);
  moe::k_down<<<occ_d * ds->sm_count, moe::kThreads, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"
