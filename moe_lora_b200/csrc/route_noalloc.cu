// moe_lora_route_noalloc: the routing entry point for callers that cannot allocate
// device memory.
//
// Some callers get only their input and output buffers from the framework that hosts
// them (for example a plugin or custom-op interface that hands over tensors but no
// workspace) and must not call cudaMalloc themselves: an allocation can synchronise
// the device, is not allowed while a stream is being captured, and can break a memory
// budget planned ahead of time.  This entry point runs the same routing kernels as
// moe_lora_route, with their scratch (status word, per-key pair counts, per-token sort
// keys and, when logits_out is NULL, the logits) in a fixed-size array that the
// library defines at file scope.  Every GPU that loads the library holds that array
// (about 1.07 MiB) until the process exits.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace mlb {
void set_error_message(const char* msg);
}

namespace {

constexpr int kNoAllocMaxM = 1024;
constexpr int kNoAllocMaxE = 256;
constexpr int kNoAllocMaxL = 64;

constexpr size_t round256(size_t v) { return (v + 255) & ~size_t(255); }
constexpr size_t kCountBytes = round256(sizeof(int32_t) * kNoAllocMaxE * (kNoAllocMaxL + 1));
constexpr size_t kKeyBytes = round256(sizeof(int32_t) * kNoAllocMaxM);
constexpr size_t kLogitBytes = round256(sizeof(float) * kNoAllocMaxM * kNoAllocMaxE);
constexpr size_t kScratchBytes = mlb::kStatusBytes + kCountBytes + kKeyBytes + kLogitBytes;

// The scratch itself.  In host code `g_route_scratch` is only a host-side stand-in for
// the symbol: its device address comes from cudaGetSymbolAddress (below).
__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

using mlb::kMaxDevices;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;


// Device address of the scratch on the current device; looked up once per device.
cudaError_t scratch_for_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_ptr[dev]);
  return cudaSuccess;
}

moe_lora_status noalloc_fail(moe_lora_status st, const char* msg) {
  char buf[256];
  snprintf(buf, sizeof(buf), "moe_lora_route_noalloc: %s", msg);
  mlb::set_error_message(buf);
  return st;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" MOE_LORA_API moe_lora_status moe_lora_route_noalloc(
    const void* x, const void* w_router, const float* bias, const float* logits_in,
    const int32_t* adapter_ids, int M, int H, int E, int k, int L, float* logits_out,
    int32_t* topk_ids, float* topk_w, int32_t* sorted_pairs, int32_t* seg_offsets,
    moe_lora_stream stream) {
  if (M < 0 || E < 1 || k < 1 || L < 0) return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "need M >= 0, E >= 1, k >= 1, L >= 0");
  if (M > kNoAllocMaxM || E > kNoAllocMaxE || L > kNoAllocMaxL || k > E)
    return noalloc_fail(MOE_LORA_ERR_UNSUPPORTED,
                        "sizes beyond the fixed scratch: need M <= 1024, k <= E <= 256, L <= 64");
  if (seg_offsets == nullptr || !al16(seg_offsets))
    return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "seg_offsets must be a 16-byte aligned device pointer");
  if (M > 0) {
    const void* need[] = {adapter_ids, topk_ids, topk_w, sorted_pairs};
    for (const void* p : need)
      if (p == nullptr || !al16(p)) return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "output/input pointer NULL or misaligned");
    if (logits_in == nullptr) {
      if (x == nullptr || w_router == nullptr || !al16(x) || !al16(w_router) || H <= 0 || H % 8 != 0)
        return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "x and w_router (H a positive multiple of 8) are required");
      if (bias != nullptr && !al16(bias)) return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "bias misaligned");
    } else if (!al16(logits_in)) {
      return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "logits_in misaligned");
    }
    if (logits_out != nullptr && !al16(logits_out)) return noalloc_fail(MOE_LORA_ERR_INVALID_ARG, "logits_out misaligned");
  }
  // the same answer as moe_lora_route on a device that is not sm_100a (or no device)
  const moe_lora_status dst = mlb::check_current_device();
  if (dst != MOE_LORA_OK) return dst;
  unsigned char* base = nullptr;
  if (scratch_for_current_device(&base) != cudaSuccess)
    return noalloc_fail(MOE_LORA_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the status word must start at zero; the key counts are zeroed by launch_route
  if (cudaMemsetAsync(base, 0, 8, cs) != cudaSuccess) return noalloc_fail(MOE_LORA_ERR_CUDA, "status clear failed");
  mlb::RouteArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.w_router = static_cast<const __nv_bfloat16*>(w_router);
  a.bias = bias;
  a.logits_in = logits_in;
  a.adapter_ids = adapter_ids;
  a.M = M;
  a.H = H;
  a.E = E;
  a.k = k;
  a.L = L;
  a.status = reinterpret_cast<int*>(base);
  int nsm = 0;
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, cur) != cudaSuccess || nsm <= 0)
    nsm = 148;
  a.num_sms = nsm;
  a.key_count = reinterpret_cast<int32_t*>(base + mlb::kStatusBytes);
  a.a_key = reinterpret_cast<int32_t*>(base + mlb::kStatusBytes + kCountBytes);
  a.logits = logits_out ? logits_out : reinterpret_cast<float*>(base + mlb::kStatusBytes + kCountBytes + kKeyBytes);
  a.logits_out = logits_out;
  a.topk_ids = topk_ids;
  a.topk_w = topk_w;
  a.sorted_pairs = sorted_pairs;
  a.seg_offsets = seg_offsets;
  if (mlb::launch_route(a, cs) != cudaSuccess) return noalloc_fail(MOE_LORA_ERR_CUDA, "kernel launch failed");
  return MOE_LORA_OK;
}
