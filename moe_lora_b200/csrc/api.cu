// C ABI of libmoe_lora.so: argument validation, workspace layout and the launch
// sequence of each call.  No allocation, no synchronisation, no host read-back
// (moe_lora_check_status excepted).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "prof.h"

#include <atomic>
#include <vector>

using namespace mlb;

namespace mlb {

namespace {
struct ProfState {
  bool on = false;
  std::vector<cudaEvent_t> ev;
  size_t next = 0;
  std::vector<std::pair<int, int>> pairs[K_COUNT];
  int open[K_COUNT];
};
ProfState g_prof;
std::atomic<long long> g_launches{0};
}  // namespace

// Under stream capture an event record becomes a graph node only with the external
// flag; each replay of the graph then re-records the event.
static void prof_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}

void prof_begin(int id, cudaStream_t st) {
  if (!g_prof.on || id < 0 || id >= K_COUNT) return;
  if (g_prof.next >= g_prof.ev.size()) return;
  g_prof.open[id] = static_cast<int>(g_prof.next);
  prof_record(g_prof.ev[g_prof.next++], st);
}

void prof_end(int id, cudaStream_t st) {
  if (!g_prof.on || id < 0 || id >= K_COUNT || g_prof.open[id] < 0) return;
  if (g_prof.next >= g_prof.ev.size()) {
    g_prof.open[id] = -1;
    return;
  }
  prof_record(g_prof.ev[g_prof.next], st);
  g_prof.pairs[id].push_back({g_prof.open[id], static_cast<int>(g_prof.next)});
  ++g_prof.next;
  g_prof.open[id] = -1;
}

void count_launch(int n) { g_launches += n; }

}  // namespace mlb

namespace {

thread_local char g_err[512] = "";

moe_lora_status fail(moe_lora_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

}  // namespace

namespace mlb {
// Lets other entry points of the library report through moe_lora_last_error().
void set_error_message(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
}  // namespace mlb

namespace {

moe_lora_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_LORA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool rank_ok(int r) { return r == 8 || r == 16 || r == 32 || r == 64 || r == 128; }

}  // namespace

namespace mlb {
int current_device_index() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

moe_lora_status check_current_device() {
  // 0 = not looked up yet, 1 = sm_100a, 2 = another architecture
  static std::atomic<int> state[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return fail(MOE_LORA_ERR_CUDA, "no CUDA device available");
  int s = state[dev].load(std::memory_order_acquire);
  if (s == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return fail(MOE_LORA_ERR_CUDA, "cannot query device %d", dev);
    s = (major == 10 && minor == 0) ? 1 : 2;
    state[dev].store(s, std::memory_order_release);
  }
  if (s == 2) return fail(MOE_LORA_ERR_UNSUPPORTED, "libmoe_lora is built for sm_100a (B200) only");
  return MOE_LORA_OK;
}
}  // namespace mlb

namespace {

// SM count of the current device (cached per device; 148 if it cannot be read).
int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

moe_lora_status check_device() { return check_current_device(); }

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  return v ? std::atoi(v) : dflt;
}

// N tile for the grouped GEMM from the mean number of rows per group.
int choose_bn(long long rows, int groups) {
  const int forced = env_int("MOE_LORA_FORCE_BN", 0);
  if (forced == 16 || forced == 32 || forced == 64 || forced == 128 || forced == 256) return forced;
  const double avg = groups > 0 ? static_cast<double>(rows) / groups : rows;
  if (avg <= 12) return 16;
  if (avg <= 24) return 32;
  if (avg <= 64) return 64;
  if (avg <= 96) return 128;
  return 256;
}

// Where the LoRA work of the grouped GEMMs runs.
//   LORA_DELTA  short groups (decode, <= 64 rows per group): the SIMT segmented LoRA
//               kernel writes an fp32 delta that the GEMM epilogue prefetches and adds,
//               so the GEMM's weight stream stays unbroken.
//   LORA_TC     long groups (prefill): the tensor-core LoRA kernel (shrink and expand on
//               tcgen05, z on chip) writes a bf16 delta that the GEMM epilogue adds.
// MOE_LORA_EXPAND=delta|tc overrides (used by the tests and the measurements).
enum LoraPlace { LORA_DELTA = 0, LORA_TC = 1 };

LoraPlace lora_place(long long rows, int groups) {
  const char* v = std::getenv("MOE_LORA_EXPAND");
  if (v != nullptr && std::strcmp(v, "delta") == 0) return LORA_DELTA;
  if (v != nullptr && std::strcmp(v, "tc") == 0) return LORA_TC;
  return rows > 64LL * (groups > 0 ? groups : 1) ? LORA_TC : LORA_DELTA;
}

int shrink_rows_per_cta(long long rows) {
  long long rb = rows / (2LL * num_sms());
  if (rb < 1) rb = 1;
  if (rb > 8) rb = 8;
  return static_cast<int>(rb);
}

struct ForwardWs {
  int* status;
  __nv_bfloat16* x_sorted;
  __nv_bfloat16* act;
  float* delta_gu;     // expand in the LoRA kernel: deltas the GEMM epilogues add
  float* delta_d;
  __nv_bfloat16* dgu;  // tensor-core LoRA: bf16 deltas [M*k][2I] and [M*k][H]
  __nv_bfloat16* dd;
  float* z_part;       // split LoRA shrink: fp32 partials [ceil(max(H, I) / 1024)][M*k][r]
  long long z_part_cap;
  int2* items;         // LoRA work list and its length
  int* item_count;
  int2* items_tc;      // tensor-core LoRA kernel: chunks of <= 128 rows of each segment
  int* item_count_tc;
  __nv_bfloat16* o;   // per-pair weighted outputs [M*k][H], summed by the combine
  uint8_t* q_hi;      // e4m3 weights: activation planes [M*k][max(H, I)]
  uint8_t* q_lo;
  float* q_scales;    // [M*k][2]
  size_t bytes;
};

ForwardWs forward_layout(void* base, int M, int H, int I, int k, int r, bool fp8, LoraPlace place, int nkeys) {
  const size_t mk = static_cast<size_t>(M) * k;
  const bool dl = r && place == LORA_DELTA, tc = r && place == LORA_TC;
  size_t off = kStatusBytes;
  ForwardWs w{};
  uint8_t* b = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) {
    uint8_t* p = b ? b + off : nullptr;
    off += align256(bytes);
    return p;
  };
  w.status = reinterpret_cast<int*>(b);
  w.x_sorted = reinterpret_cast<__nv_bfloat16*>(take(mk * H * 2));
  w.act = reinterpret_cast<__nv_bfloat16*>(take(mk * I * 2));
  w.delta_gu = reinterpret_cast<float*>(take(dl ? mk * 2 * I * 4 : 0));
  w.delta_d = reinterpret_cast<float*>(take(dl ? mk * H * 4 : 0));
  w.dgu = reinterpret_cast<__nv_bfloat16*>(take(tc ? mk * 2 * I * 2 : 0));
  w.dd = reinterpret_cast<__nv_bfloat16*>(take(tc ? mk * H * 2 : 0));
  // split LoRA shrink partials: rank r, or 2 r for separate gate and up adapters (r <= 64)
  w.z_part_cap = dl ? static_cast<long long>((std::max(H, I) + 1023) / 1024) * mk * (r <= 64 ? 2 * r : r) : 0;
  w.z_part = reinterpret_cast<float*>(take(static_cast<size_t>(w.z_part_cap) * 4));
  w.items = reinterpret_cast<int2*>(take(static_cast<size_t>(lora_items_bound(static_cast<int>(mk), nkeys, 4)) * 8));
  w.item_count = reinterpret_cast<int*>(take(mk > 0 ? 4 : 0));
  w.items_tc = reinterpret_cast<int2*>(
      take(tc ? static_cast<size_t>(lora_items_bound(static_cast<int>(mk), nkeys, kLtN)) * 8 : 0));
  w.item_count_tc = reinterpret_cast<int*>(take(tc ? 4 : 0));
  w.o = reinterpret_cast<__nv_bfloat16*>(take(mk * H * 2));
  const size_t kmax = H > I ? H : I;
  w.q_hi = reinterpret_cast<uint8_t*>(take(fp8 ? mk * kmax : 0));
  w.q_lo = reinterpret_cast<uint8_t*>(take(fp8 ? mk * kmax : 0));
  w.q_scales = reinterpret_cast<float*>(take(fp8 ? mk * 2 * 4 : 0));
  w.bytes = off;
  return w;
}

struct RouteWs {
  int* status;
  int32_t* key_count;
  int32_t* a_key;
  float* logits;
  size_t bytes;
};

RouteWs route_layout(void* base, int M, int E, int L) {
  size_t off = kStatusBytes;
  RouteWs w{};
  uint8_t* b = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) {
    uint8_t* p = b ? b + off : nullptr;
    off += align256(bytes);
    return p;
  };
  w.status = reinterpret_cast<int*>(b);
  // adapter key per token; tickets of the one-launch routing (ceil(M / 8) + 1), right
  // behind the status block so that one memset clears both
  w.a_key = reinterpret_cast<int32_t*>(take(static_cast<size_t>(M > (M + 7) / 8 + 1 ? M : (M + 7) / 8 + 1) * 4));
  w.key_count = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E) * (L + 1) * 4));
  w.logits = reinterpret_cast<float*>(take(static_cast<size_t>(M) * E * 4));
  w.bytes = off;
  return w;
}

struct DenseWs {
  int* status;
  float* z;             // fp32 path: shrink output
  int32_t* row_adapter; // fp32 path
  float* delta;         // bf16 path, expand in the LoRA kernel: delta the GEMM adds
  __nv_bfloat16* dbf;   // bf16 path, tensor-core LoRA: bf16 delta [T][h_out]
  float* z_part;        // bf16 path, split LoRA shrink partials
  long long z_part_cap;
  int2* items;          // bf16 path: LoRA work list and its length
  int* item_count;
  int2* items_tc;       // bf16 path, tensor-core LoRA kernel: its work list
  int* item_count_tc;
  size_t bytes;
};

DenseWs dense_layout(void* base, int T, int h_in, int h_out, int r, bool f32, LoraPlace place) {
  const bool dl = r && place == LORA_DELTA, tc = r && place == LORA_TC;
  size_t off = kStatusBytes;
  DenseWs w{};
  uint8_t* b = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) {
    uint8_t* p = b ? b + off : nullptr;
    off += align256(bytes);
    return p;
  };
  w.status = reinterpret_cast<int*>(b);
  if (f32) {
    w.z = reinterpret_cast<float*>(take(static_cast<size_t>(T) * r * 4));
    w.row_adapter = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * 4));
  } else {
    w.delta = reinterpret_cast<float*>(take(dl ? static_cast<size_t>(T) * h_out * 4 : 0));
    w.dbf = reinterpret_cast<__nv_bfloat16*>(take(tc ? static_cast<size_t>(T) * h_out * 2 : 0));
    w.z_part_cap = dl ? static_cast<long long>((h_in + 1023) / 1024) * T * r : 0;
    w.z_part = reinterpret_cast<float*>(take(static_cast<size_t>(w.z_part_cap) * 4));
    w.items = reinterpret_cast<int2*>(take(static_cast<size_t>(lora_items_bound(T, T, 4)) * 8));
    w.item_count = reinterpret_cast<int*>(take(T > 0 ? 4 : 0));
    w.items_tc = reinterpret_cast<int2*>(take(tc ? static_cast<size_t>(lora_items_bound(T, T, kLtN)) * 8 : 0));
    w.item_count_tc = reinterpret_cast<int*>(take(tc ? 4 : 0));
  }
  w.bytes = off;
  return w;
}

moe_lora_status check_ws(void* ws, size_t have, size_t need) {
  if (ws == nullptr) return fail(MOE_LORA_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned16(ws)) return fail(MOE_LORA_ERR_INVALID_ARG, "workspace not 16-byte aligned");
  if (have < need)
    return fail(MOE_LORA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", have, need);
  return MOE_LORA_OK;
}

#define ML_REQUIRE(cond, code, ...)              \
  do {                                           \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

#define ML_PTR(p) ML_REQUIRE((p) != nullptr && aligned16(p), MOE_LORA_ERR_INVALID_ARG, \
                             "%s must be a non-NULL 16-byte aligned device pointer", #p)

#define ML_CUDA(expr, where)                     \
  do {                                           \
    cudaError_t _e = (expr);                     \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

}  // namespace

extern "C" {

const char* moe_lora_last_error(void) { return g_err; }

long long moe_lora_launch_count(void) { return g_launches.load(); }

moe_lora_status moe_lora_profile_enable(int max_launches) {
  ML_REQUIRE(max_launches >= 0 && max_launches <= (1 << 20), MOE_LORA_ERR_INVALID_ARG,
             "max_launches must be in [0, 2^20]");
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.next = 0;
  for (int i = 0; i < K_COUNT; ++i) {
    g_prof.pairs[i].clear();
    g_prof.open[i] = -1;
  }
  g_prof.on = false;
  if (max_launches == 0) return MOE_LORA_OK;
  g_prof.ev.resize(2 * static_cast<size_t>(max_launches));
  for (auto& e : g_prof.ev) ML_CUDA(cudaEventCreate(&e), "cudaEventCreate");
  g_prof.on = true;
  return MOE_LORA_OK;
}

moe_lora_status moe_lora_profile_read(int kernel_id, double* total_ms, int* launches) {
  ML_REQUIRE(kernel_id >= 0 && kernel_id < K_COUNT && total_ms && launches, MOE_LORA_ERR_INVALID_ARG,
             "bad kernel id or output pointer");
  *total_ms = 0.0;
  *launches = 0;
  const auto& v = g_prof.pairs[kernel_id];
  if (v.empty()) return MOE_LORA_OK;
  ML_CUDA(cudaEventSynchronize(g_prof.ev[v.back().second]), "cudaEventSynchronize");
  double tot = 0.0;
  for (const auto& pr : v) {
    float ms = 0.f;
    ML_CUDA(cudaEventElapsedTime(&ms, g_prof.ev[pr.first], g_prof.ev[pr.second]), "cudaEventElapsedTime");
    tot += ms;
  }
  *total_ms = tot;
  *launches = static_cast<int>(v.size());
  return MOE_LORA_OK;
}

const char* moe_lora_version(void) { return "moe_lora_b200 0.1 sm_100a"; }

size_t moe_lora_workspace_size(int op, int M, int H, int I, int E, int k, int L, int r) {
  if (M < 0 || H < 0 || I < 0 || E < 0 || k < 0 || L < 0 || r < 0) return 0;
  switch (op) {
    case MOE_LORA_OP_ROUTE: return route_layout(nullptr, M, E, L).bytes;
    case MOE_LORA_OP_FORWARD:
    case MOE_LORA_OP_FORWARD_E4M3:
      return forward_layout(nullptr, M, H, I, k, L > 0 ? r : 0, true, lora_place(1LL * M * k, E), E * (L + 1))
          .bytes;
    case MOE_LORA_OP_FORWARD_BF16:
      return forward_layout(nullptr, M, H, I, k, L > 0 ? r : 0, false, lora_place(1LL * M * k, E), E * (L + 1))
          .bytes;
    case MOE_LORA_OP_SGMV_SHRINK:
    case MOE_LORA_OP_SGMV_EXPAND: return kStatusBytes;
    case MOE_LORA_OP_DENSE: {
      const size_t a = dense_layout(nullptr, M, H, I, L > 0 ? r : 0, true, LORA_DELTA).bytes;
      const size_t b = dense_layout(nullptr, M, H, I, L > 0 ? r : 0, false, lora_place(M, 1)).bytes;
      return a > b ? a : b;
    }
    default: return 0;
  }
}

moe_lora_status moe_lora_check_status(void* workspace, moe_lora_stream stream) {
  if (workspace == nullptr) return fail(MOE_LORA_ERR_INVALID_ARG, "workspace is NULL");
  int h[2] = {0, 0};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ML_CUDA(cudaStreamSynchronize(st), "cudaStreamSynchronize");
  ML_CUDA(cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost), "status read");
  ML_CUDA(cudaMemset(workspace, 0, sizeof(h)), "status clear");
  if (h[0] == MOE_LORA_OK) return MOE_LORA_OK;
  return fail(static_cast<moe_lora_status>(h[0]), "device-side check failed (code %d, detail %d)", h[0], h[1]);
}

}  // extern "C"


extern "C" {

moe_lora_status moe_lora_route(const void* x, const void* w_router, const float* bias,
                               const float* logits_in, const int32_t* adapter_ids, int M, int H, int E,
                               int k, int L, float* logits_out, int32_t* topk_ids, float* topk_w,
                               int32_t* sorted_pairs, int32_t* seg_offsets, void* workspace,
                               size_t workspace_bytes, moe_lora_stream stream) {
  ML_REQUIRE(M >= 0 && E >= 1 && k >= 1 && L >= 0, MOE_LORA_ERR_INVALID_ARG,
             "need M >= 0, E >= 1, k >= 1, L >= 0 (got M=%d E=%d k=%d L=%d)", M, E, k, L);
  ML_REQUIRE(k <= E && E <= 256 && L <= 64, MOE_LORA_ERR_UNSUPPORTED,
             "supported: k <= E <= 256, L <= 64 (got k=%d E=%d L=%d)", k, E, L);
  ML_REQUIRE(static_cast<long long>(M) * k <= (1 << 20), MOE_LORA_ERR_UNSUPPORTED, "M*k > 2^20");
  ML_PTR(seg_offsets);
  const RouteWs need = route_layout(nullptr, M, E, L);
  moe_lora_status st = check_ws(workspace, workspace_bytes, need.bytes);
  if (st != MOE_LORA_OK) return st;
  if (M > 0) {
    ML_PTR(adapter_ids);
    ML_PTR(topk_ids);
    ML_PTR(topk_w);
    ML_PTR(sorted_pairs);
    if (logits_in == nullptr) {
      ML_PTR(x);
      ML_PTR(w_router);
      ML_REQUIRE(H > 0 && H % 8 == 0, MOE_LORA_ERR_UNSUPPORTED, "H must be a positive multiple of 8");
      if (bias) ML_PTR(bias);
    } else {
      ML_PTR(logits_in);
    }
    if (logits_out) ML_PTR(logits_out);
  }
  st = check_device();
  if (st != MOE_LORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const RouteWs w = route_layout(workspace, M, E, L);
  // one memset for the status word and, for the one-launch routing, its tickets
  const int tickets = route_fused_tickets(M, k);
  ML_CUDA(cudaMemsetAsync(workspace, 0, tickets > 0 ? kStatusBytes + 4 * static_cast<size_t>(tickets) : 8, cs),
          "status clear");
  RouteArgs a{};
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
  a.logits = logits_out ? logits_out : w.logits;
  a.logits_out = logits_out;
  a.topk_ids = topk_ids;
  a.topk_w = topk_w;
  a.sorted_pairs = sorted_pairs;
  a.seg_offsets = seg_offsets;
  a.key_count = w.key_count;
  a.a_key = w.a_key;
  a.status = w.status;
  a.num_sms = num_sms();
  a.tickets_zeroed = tickets > 0 ? 1 : 0;
  ML_CUDA(launch_route(a, cs), "moe_lora_route launch");
  return MOE_LORA_OK;
}

moe_lora_status moe_lora_forward(const void* x, int M, int H, int I, int E, int k, int L, int r,
                                 const float* topk_w, const int32_t* sorted_pairs,
                                 const int32_t* seg_offsets, const void* w_gateup, const void* w_down,
                                 ml_dtype w_dtype, const float* w_scales, const void* lora_a_gu,
                                 const void* lora_b_gu, const void* lora_a_d, const void* lora_b_d,
                                 const moe_lora_adapter_format* format, void* y, void* workspace,
                                 size_t workspace_bytes, moe_lora_stream stream) {
  ML_REQUIRE(M >= 0 && H > 0 && I > 0 && E >= 1 && k >= 1 && L >= 0, MOE_LORA_ERR_INVALID_ARG,
             "need M >= 0, H > 0, I > 0, E >= 1, k >= 1, L >= 0");
  ML_REQUIRE(w_dtype == ML_BF16 || w_dtype == ML_E4M3, MOE_LORA_ERR_INVALID_ARG,
             "w_dtype must be ML_BF16 or ML_E4M3");
  ML_REQUIRE(k <= E && E <= 256 && L <= 64, MOE_LORA_ERR_UNSUPPORTED, "supported: k <= E <= 256, L <= 64");
  ML_REQUIRE(H % 8 == 0 && I % 8 == 0, MOE_LORA_ERR_UNSUPPORTED, "H and I must be multiples of 8");
  ML_REQUIRE(static_cast<long long>(M) * k <= (1 << 20), MOE_LORA_ERR_UNSUPPORTED, "M*k > 2^20");
  if (L > 0) ML_REQUIRE(rank_ok(r), MOE_LORA_ERR_UNSUPPORTED, "r must be one of 8, 16, 32, 64, 128");
  const int rr = L > 0 ? r : 0;
  const bool fp8 = w_dtype == ML_E4M3;
  const moe_lora_adapter_format fmt = format ? *format : moe_lora_adapter_format{0, 1.0f, 1.0f};
  ML_REQUIRE(fmt.gate_up_split == 0 || fmt.gate_up_split == 1, MOE_LORA_ERR_INVALID_ARG,
             "format->gate_up_split must be 0 or 1");
  const bool split = fmt.gate_up_split == 1 && rr > 0;
  if (split) ML_REQUIRE(r <= 64, MOE_LORA_ERR_UNSUPPORTED, "separate gate and up adapters need r <= 64");
  const LoraPlace place = lora_place(1LL * M * k, E);
  // the tensor-core LoRA kernel takes separate gate and up adapters at whole 64-feature boxes
  if (split && place == LORA_TC)
    ML_REQUIRE(I % 64 == 0, MOE_LORA_ERR_UNSUPPORTED,
               "separate gate and up adapters with more than 64 rows per expert need I a multiple of 64");
  const ForwardWs need = forward_layout(nullptr, M, H, I, k, rr, fp8, place, E * (L + 1));
  moe_lora_status st = check_ws(workspace, workspace_bytes, need.bytes);
  if (st != MOE_LORA_OK) return st;
  if (w_dtype == ML_E4M3) {
    ML_REQUIRE(H % 16 == 0 && I % 16 == 0, MOE_LORA_ERR_UNSUPPORTED,
               "ML_E4M3 expert weights need H and I multiples of 16 (16-byte rows)");
  }
  if (M == 0) return MOE_LORA_OK;
  ML_PTR(x);
  ML_PTR(topk_w);
  ML_PTR(sorted_pairs);
  ML_PTR(seg_offsets);
  ML_PTR(w_gateup);
  ML_PTR(w_down);
  ML_PTR(y);
  if (w_dtype == ML_E4M3) ML_PTR(w_scales);
  if (L > 0) {
    ML_PTR(lora_a_gu);
    ML_PTR(lora_b_gu);
    ML_PTR(lora_a_d);
    ML_PTR(lora_b_d);
  }
  st = check_device();
  if (st != MOE_LORA_OK) return st;
  if (!tensor_map_encode_available())
    return fail(MOE_LORA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const ForwardWs w = forward_layout(workspace, M, H, I, k, rr, fp8, place, E * (L + 1));
  const bool tcl = rr && place == LORA_TC;  // tensor-core LoRA kernel, bf16 deltas
  const int mk = M * k;
  const int nkeys = E * (L + 1);
  // the status block (status word, work counters) is zeroed by the call's first kernel,
  // the row gather below, which writes no status itself; every later kernel of the call
  // starts after it has finished

  // 1. gather x rows into (expert, adapter) order, and the gate_up LoRA:
  //    LORA_DELTA: one SIMT kernel gathers, shrinks z = x A_gu per (adapter, expert)
  //                segment chunk and expands z B_gu into an fp32 delta;
  //    LORA_TC:    a row gather, then the tensor-core LoRA kernel (bf16 delta);
  LoraDeltaArgs l1{};
  l1.src = static_cast<const __nv_bfloat16*>(x);
  l1.gather = sorted_pairs;
  l1.gather_div = k;
  l1.nsrc = M;
  l1.gather_dst = w.x_sorted;
  l1.nrows = mk;
  l1.K = H;
  l1.r = rr;
  l1.NB = 2 * I;
  l1.seg_offsets = seg_offsets;
  l1.nseg = nkeys;
  l1.seg_adapter = nullptr;
  l1.L = L;
  l1.E = E;
  l1.lora_a = static_cast<const __nv_bfloat16*>(lora_a_gu);
  l1.lora_b = static_cast<const __nv_bfloat16*>(lora_b_gu);
  l1.r_exp = rr;
  l1.split_I = split ? I : 0;
  l1.scale = fmt.scale_gu;
  if (split) l1.r = 2 * rr;  // the shrink covers both adapters' rows
  l1.delta = rr && place == LORA_DELTA ? w.delta_gu : nullptr;  // otherwise this launch only gathers
  l1.z_part = w.z_part;
  l1.z_part_cap = w.z_part_cap;
  l1.status = w.status;
  l1.num_sms = num_sms();
  l1.rb = lora_rows_per_chunk(mk, nkeys);
  l1.items_bound = lora_items_bound(mk, nkeys, l1.rb);
  l1.items = w.items;
  l1.item_count = w.item_count;
  LoraTcArgs t1{};
  if (tcl) {
    if (fp8)  // one pass over x: the gathered bf16 rows (the LoRA kernel's operand) and their planes
      ML_CUDA(launch_gather_quant(static_cast<const __nv_bfloat16*>(x), M, sorted_pairs, k, mk, H, w.q_hi, w.q_lo,
                                  w.q_scales, w.x_sorted, cs, w.status),
              "gather and activation planes launch");
    else
      ML_CUDA(launch_gather_rows(static_cast<const __nv_bfloat16*>(x), M, sorted_pairs, k, mk, H, w.x_sorted, cs,
                                 w.status),
              "row gather launch");
    const int bound = lora_items_bound(mk, nkeys, kLtN);
    ML_CUDA(launch_lora_plan_all(seg_offsets, nullptr, nkeys, L, mk, kLtN, w.items_tc, w.item_count_tc, bound,
                                 w.status, cs),
            "LoRA work list launch");
    t1.src = w.x_sorted;
    t1.nrows = mk;
    t1.K = H;
    t1.r = rr;
    t1.F = 2 * I;
    t1.seg_offsets = seg_offsets;
    t1.nseg = nkeys;
    t1.seg_adapter = nullptr;
    t1.L = L;
    t1.E = E;
    t1.lora_a = static_cast<const __nv_bfloat16*>(lora_a_gu);
    t1.lora_b = static_cast<const __nv_bfloat16*>(lora_b_gu);
    t1.r = split ? 2 * rr : rr;
    t1.r_exp = rr;
    t1.split_I = split ? I : 0;
    t1.scale = fmt.scale_gu;
    t1.items = w.items_tc;
    t1.item_count = w.item_count_tc;
    t1.items_bound = bound;
    t1.delta = w.dgu;
    t1.status = w.status;
    t1.work_counter = w.status + 2;  // inside the status block: cleared with it by every call
    t1.pdl_trigger = 1;  // the gate_up GEMM takes each SM this kernel leaves
    t1.num_sms = num_sms();
    ML_CUDA(launch_lora_tc(t1, cs), "gate_up tensor-core LoRA launch");
  } else {
    // the GEMM's operand first (gathered x rows, or their e4m3 planes), then the LoRA
    // kernel, which lets the GEMM start at once: the GEMM streams its weights while the
    // LoRA kernel runs, and only its epilogue loader waits for the delta
    if (fp8)
      ML_CUDA(launch_gather_quant(static_cast<const __nv_bfloat16*>(x), M, sorted_pairs, k, mk, H, w.q_hi, w.q_lo,
                                  w.q_scales, nullptr, cs, w.status),
              "activation planes launch");
    else
      ML_CUDA(launch_gather_rows(static_cast<const __nv_bfloat16*>(x), M, sorted_pairs, k, mk, H, w.x_sorted, cs,
                                 w.status),
              "row gather launch");
    if (rr) {
      l1.gather_dst = nullptr;
      l1.pdl_trigger = 1;
      l1.pdl_after_plan = 1;
      ML_CUDA(launch_lora_plan(l1, cs), "LoRA plan launch");
      ML_CUDA(launch_lora_delta(l1, cs), "gate_up LoRA launch");
    }
  }

  // 2. gate_up grouped GEMM; epilogue adds delta_gu and applies SiLU-and-mul -> act
  GemmArgs g{};
  g.epi = EPI_GATEUP;
  g.w_fp8 = w_dtype == ML_E4M3;
  g.K = H;
  g.E = E;
  g.group_offsets = seg_offsets;
  g.group_stride = L + 1;
  g.rows_per_group = 2 * I;
  g.n_out = I;
  g.I = I;
  g.total_rows = mk;
  g.delta_cols = 2 * I;
  g.delta = rr && place == LORA_DELTA ? w.delta_gu : nullptr;
  g.delta_bf16 = tcl ? w.dgu : nullptr;
  // behind the LoRA kernel (PDL): the GEMM streams its weights while that kernel ends, and
  // only what reads the delta waits for it
  g.pdl_secondary = (rr && place == LORA_DELTA) || tcl ? 1 : 0;
  g.pdl_full_smem = tcl ? 1 : 0;
  g.out_bf16 = w.act;
  g.w_scales = w_dtype == ML_E4M3 ? w_scales : nullptr;
  g.scale_idx = 0;
  g.status = w.status;
  g.w = w_gateup;
  g.b = w.x_sorted;
  g.bn = choose_bn(mk, E);
  if (fp8) {
    if (g.bn > 128) g.bn = 128;  // e4m3: the hi and lo planes make the MMA's N = 2 BN <= 256
    g.b_hi = w.q_hi;
    g.b_lo = w.q_lo;
    g.b_scales = w.q_scales;
  }
  g.num_sms = num_sms();
  // tests only: the gate_up GEMM's first stage in CTA 0 never arrives and every bounded
  // wait is shortened to MOE_LORA_TEST_STALL milliseconds (exercises the abort path)
  g.test_stall_ms = env_int("MOE_LORA_TEST_STALL", 0);
  ML_CUDA(launch_gemm_tc(g, cs), "gate_up GEMM launch");
  g.test_stall_ms = 0;

  g.pdl_secondary = 0;
  g.pdl_full_smem = 0;

  // 3. down LoRA shrink + expand on act: delta_d = (act A_d) B_d (LORA_DELTA: after the
  //    down GEMM's launch, overlapped with it, into a pair-order delta the combine adds)
  if (tcl) {
    LoraTcArgs t2 = t1;
    t2.src = w.act;
    t2.K = I;
    t2.F = H;
    t2.lora_a = static_cast<const __nv_bfloat16*>(lora_a_d);
    t2.lora_b = static_cast<const __nv_bfloat16*>(lora_b_d);
    t2.r = rr;
    t2.r_exp = rr;
    t2.split_I = 0;
    t2.scale = fmt.scale_d;
    t2.prof_id = K_LORA_DOWN;
    t2.delta = w.dd;
    t2.scatter = sorted_pairs;  // pair order: the combine adds it
    t2.work_counter = w.status + 3;
    t2.pdl_trigger = 1;  // the down GEMM (which does not read this delta) starts as SMs free up
    ML_CUDA(launch_lora_tc(t2, cs), "down tensor-core LoRA launch");
  }

  // 4. down grouped GEMM; the epilogue applies the routing weight -> o (per pair, bf16);
  //    the combine adds the weighted down LoRA delta
  GemmArgs d = g;
  d.epi = EPI_DOWN;
  d.K = I;
  d.rows_per_group = H;
  d.n_out = H;
  d.delta_cols = H;
  d.delta = nullptr;
  d.delta_bf16 = nullptr;  // the down LoRA delta (delta and tc placements) goes to the combine
  d.pdl_trigger = rr && place == LORA_DELTA ? 1 : 0;
  d.pdl_end_wait = tcl ? 1 : 0;  // behind the tensor-core down LoRA: waits for it only to finish
  d.pdl_full_smem = tcl ? 1 : 0;
  d.out_bf16 = w.o;
  d.out_f32 = nullptr;
  d.sorted_pairs = sorted_pairs;
  d.topk_w = topk_w;
  d.scale_idx = 1;
  d.w = w_down;
  d.b = w.act;
  if (fp8) ML_CUDA(launch_quant_planes(w.act, mk, I, w.q_hi, w.q_lo, w.q_scales, cs), "activation planes launch");
  ML_CUDA(launch_gemm_tc(d, cs), "down GEMM launch");
  if (rr && place == LORA_DELTA) {
    LoraDeltaArgs l2 = l1;
    l2.src = w.act;
    l2.gather = nullptr;
    l2.gather_dst = nullptr;
    l2.q_hi = nullptr;
    l2.K = I;
    l2.NB = H;
    l2.lora_a = static_cast<const __nv_bfloat16*>(lora_a_d);
    l2.lora_b = static_cast<const __nv_bfloat16*>(lora_b_d);
    l2.r = rr;
    l2.r_exp = rr;
    l2.split_I = 0;
    l2.scale = fmt.scale_d;
    l2.prof_id = K_LORA_DOWN;
    l2.delta = w.delta_d;
    l2.scatter = sorted_pairs;  // pair order, for the combine
    l2.pdl_trigger = 0;
    l2.pdl_secondary = 1;
    l2.pdl_after_plan = 0;  // behind the down GEMM, not the work-list kernel
    ML_CUDA(launch_lora_delta(l2, cs), "down LoRA launch");
  }

  // 5. fixed-order combine over the k slots (+ the weighted down LoRA delta)
  ML_CUDA(launch_combine(w.o, M, k, H, rr && place == LORA_DELTA ? w.delta_d : nullptr, tcl ? w.dd : nullptr,
                         topk_w, static_cast<__nv_bfloat16*>(y), cs),
          "combine launch");
  return MOE_LORA_OK;
}

moe_lora_status sgmv_shrink(const void* x, const void* lora_a, const int32_t* seg_offsets,
                            const int32_t* seg_adapter, int S, int T, int h_in, int r, int L, ml_dtype dt,
                            float* z, void* workspace, size_t workspace_bytes, moe_lora_stream stream) {
  ML_REQUIRE(S >= 0 && T >= 0 && L >= 0 && h_in > 0, MOE_LORA_ERR_INVALID_ARG, "need S, T, L >= 0, h_in > 0");
  ML_REQUIRE(dt == ML_F32 || dt == ML_BF16, MOE_LORA_ERR_INVALID_ARG, "dt must be ML_F32 or ML_BF16");
  ML_REQUIRE(rank_ok(r), MOE_LORA_ERR_UNSUPPORTED, "r must be one of 8, 16, 32, 64, 128");
  ML_REQUIRE(h_in % 8 == 0 && L <= 64, MOE_LORA_ERR_UNSUPPORTED, "h_in must be a multiple of 8, L <= 64");
  ML_REQUIRE(S >= 1 || T == 0, MOE_LORA_ERR_INVALID_ARG, "segments must cover the T tokens");
  moe_lora_status st = check_ws(workspace, workspace_bytes, kStatusBytes);
  if (st != MOE_LORA_OK) return st;
  if (T == 0) return MOE_LORA_OK;
  ML_PTR(x);
  ML_PTR(seg_offsets);
  ML_PTR(seg_adapter);
  ML_PTR(z);
  if (L > 0) ML_PTR(lora_a);
  st = check_device();
  if (st != MOE_LORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  ML_CUDA(cudaMemsetAsync(workspace, 0, 8, cs), "status clear");
  ShrinkArgs a{};
  a.src = x;
  a.src_f32 = dt == ML_F32;
  a.gather = nullptr;
  a.gather_div = 1;
  a.gather_dst = nullptr;
  a.nrows = T;
  a.K = h_in;
  a.r = r;
  a.seg_offsets = seg_offsets;
  a.nseg = S;
  a.seg_adapter = seg_adapter;
  a.L = L;
  a.E = 1;
  a.lora_a = lora_a;
  a.z = z;
  a.row_adapter = nullptr;
  a.rows_per_cta = shrink_rows_per_cta(T);
  a.status = static_cast<int*>(workspace);
  ML_CUDA(launch_shrink(a, cs), "sgmv_shrink launch");
  return MOE_LORA_OK;
}

moe_lora_status sgmv_expand(const float* z, const void* lora_b, const int32_t* seg_offsets,
                            const int32_t* seg_adapter, int S, int T, int h_out, int r, int L, ml_dtype dt,
                            void* y, void* workspace, size_t workspace_bytes, moe_lora_stream stream) {
  ML_REQUIRE(S >= 0 && T >= 0 && L >= 0 && h_out > 0, MOE_LORA_ERR_INVALID_ARG, "need S, T, L >= 0, h_out > 0");
  ML_REQUIRE(dt == ML_F32 || dt == ML_BF16, MOE_LORA_ERR_INVALID_ARG, "dt must be ML_F32 or ML_BF16");
  ML_REQUIRE(rank_ok(r), MOE_LORA_ERR_UNSUPPORTED, "r must be one of 8, 16, 32, 64, 128");
  ML_REQUIRE(h_out % 8 == 0 && L <= 64, MOE_LORA_ERR_UNSUPPORTED, "h_out must be a multiple of 8, L <= 64");
  ML_REQUIRE(S >= 1 || T == 0, MOE_LORA_ERR_INVALID_ARG, "segments must cover the T tokens");
  moe_lora_status st = check_ws(workspace, workspace_bytes, kStatusBytes);
  if (st != MOE_LORA_OK) return st;
  if (T == 0) return MOE_LORA_OK;
  ML_PTR(z);
  ML_PTR(seg_offsets);
  ML_PTR(seg_adapter);
  ML_PTR(y);
  if (L > 0) ML_PTR(lora_b);
  st = check_device();
  if (st != MOE_LORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  ML_CUDA(cudaMemsetAsync(workspace, 0, 8, cs), "status clear");
  ExpandArgs a{};
  a.z = z;
  a.lora_b = lora_b;
  a.f32 = dt == ML_F32;
  a.seg_offsets = seg_offsets;
  a.nseg = S;
  a.seg_adapter = seg_adapter;
  a.L = L;
  a.T = T;
  a.h_out = h_out;
  a.r = r;
  a.y = y;
  a.status = static_cast<int*>(workspace);
  ML_CUDA(launch_expand(a, cs), "sgmv_expand launch");
  return MOE_LORA_OK;
}

moe_lora_status dense_lora_forward(const void* x, const void* w, const void* lora_a, const void* lora_b,
                                   const int32_t* seg_offsets, const int32_t* seg_adapter, int S, int T,
                                   int h_in, int h_out, int r, int L, ml_dtype dt, void* y, void* workspace,
                                   size_t workspace_bytes, moe_lora_stream stream) {
  ML_REQUIRE(S >= 0 && T >= 0 && L >= 0 && h_in > 0 && h_out > 0, MOE_LORA_ERR_INVALID_ARG,
             "need S, T, L >= 0 and h_in, h_out > 0");
  ML_REQUIRE(dt == ML_F32 || dt == ML_BF16, MOE_LORA_ERR_INVALID_ARG, "dt must be ML_F32 or ML_BF16");
  ML_REQUIRE(h_in % 8 == 0 && h_out % 8 == 0 && L <= 64, MOE_LORA_ERR_UNSUPPORTED,
             "h_in, h_out must be multiples of 8, L <= 64");
  if (L > 0) ML_REQUIRE(rank_ok(r), MOE_LORA_ERR_UNSUPPORTED, "r must be one of 8, 16, 32, 64, 128");
  ML_REQUIRE(S >= 1 || T == 0, MOE_LORA_ERR_INVALID_ARG, "segments must cover the T tokens");
  const int rr = L > 0 ? r : 0;
  const bool f32 = dt == ML_F32;
  const LoraPlace place = f32 ? LORA_DELTA : lora_place(T, 1);
  const DenseWs need = dense_layout(nullptr, T, h_in, h_out, rr, f32, place);
  moe_lora_status st = check_ws(workspace, workspace_bytes, need.bytes);
  if (st != MOE_LORA_OK) return st;
  if (T == 0) return MOE_LORA_OK;
  ML_PTR(x);
  ML_PTR(w);
  ML_PTR(seg_offsets);
  ML_PTR(seg_adapter);
  ML_PTR(y);
  if (L > 0) {
    ML_PTR(lora_a);
    ML_PTR(lora_b);
  }
  st = check_device();
  if (st != MOE_LORA_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const DenseWs ws = dense_layout(workspace, T, h_in, h_out, rr, f32, place);
  const bool tcl = rr && place == LORA_TC;  // tensor-core LoRA kernel, bf16 delta
  // with adapters (bf16) the LoRA work-list kernel comes first and zeroes the status block
  // itself; the kernels behind it write status only after they have waited for it
  const bool plan_clears = !f32 && rr > 0;
  if (!plan_clears) ML_CUDA(cudaMemsetAsync(workspace, 0, f32 ? 8 : kStatusBytes, cs), "status clear");

  if (f32) {
    ShrinkArgs a{};
    a.src = x;
    a.src_f32 = true;
    a.gather_div = 1;
    a.nrows = T;
    a.K = h_in;
    a.r = rr;
    a.seg_offsets = seg_offsets;
    a.nseg = S;
    a.seg_adapter = seg_adapter;
    a.L = L;
    a.E = 1;
    a.lora_a = lora_a;
    a.z = ws.z;
    a.row_adapter = ws.row_adapter;
    a.rows_per_cta = shrink_rows_per_cta(T);
    a.status = ws.status;
    ML_CUDA(launch_shrink(a, cs), "dense shrink launch");
    DenseF32Args d{};
    d.x = static_cast<const float*>(x);
    d.w = static_cast<const float*>(w);
    d.lora_b = static_cast<const float*>(lora_b);
    d.z = rr ? ws.z : nullptr;
    d.row_adapter = ws.row_adapter;
    d.T = T;
    d.h_in = h_in;
    d.h_out = h_out;
    d.r = rr;
    d.L = L;
    d.y = static_cast<float*>(y);
    ML_CUDA(launch_dense_f32(d, cs), "dense fp32 GEMM launch");
    return MOE_LORA_OK;
  }
  if (!tensor_map_encode_available())
    return fail(MOE_LORA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (rr) {
    LoraDeltaArgs l{};
    l.src = static_cast<const __nv_bfloat16*>(x);
    l.gather_div = 1;
    l.nrows = T;
    l.K = h_in;
    l.r = rr;
    l.NB = h_out;
    l.seg_offsets = seg_offsets;
    l.nseg = S;
    l.seg_adapter = seg_adapter;
    l.L = L;
    l.E = 1;
    l.lora_a = static_cast<const __nv_bfloat16*>(lora_a);
    l.lora_b = static_cast<const __nv_bfloat16*>(lora_b);
    l.delta = place == LORA_DELTA ? ws.delta : nullptr;
    l.z_part = ws.z_part;
    l.z_part_cap = ws.z_part_cap;
    l.status = ws.status;
    l.num_sms = num_sms();
    l.rb = lora_rows_per_chunk(T, S);
    l.items_bound = lora_items_bound(T, S, l.rb);
    l.items = ws.items;
    l.item_count = ws.item_count;
    l.r_exp = rr;
    l.scale = 1.f;  // the dense adapters carry their scale in B
    if (tcl) {  // shrink and expand on the tensor cores, bf16 delta for the epilogue
      const int bound = lora_items_bound(T, S, kLtN);
      ML_CUDA(launch_lora_plan_all(seg_offsets, seg_adapter, S, L, T, kLtN, ws.items_tc, ws.item_count_tc, bound,
                                   ws.status, cs, true),
              "LoRA work list launch");
      LoraTcArgs t{};
      t.src = static_cast<const __nv_bfloat16*>(x);
      t.nrows = T;
      t.K = h_in;
      t.r = rr;
      t.F = h_out;
      t.seg_offsets = seg_offsets;
      t.nseg = S;
      t.seg_adapter = seg_adapter;
      t.L = L;
      t.E = 1;
      t.lora_a = static_cast<const __nv_bfloat16*>(lora_a);
      t.lora_b = static_cast<const __nv_bfloat16*>(lora_b);
      t.items = ws.items_tc;
      t.item_count = ws.item_count_tc;
      t.items_bound = bound;
      t.delta = ws.dbf;
      t.status = ws.status;
      t.work_counter = ws.status + 2;  // inside the status block: cleared with it by every call
      t.num_sms = num_sms();
      t.r_exp = rr;
      t.scale = 1.f;
      ML_CUDA(launch_lora_tc(t, cs), "dense tensor-core LoRA launch");
    } else {
      // the LoRA kernel lets the GEMM start at once: the GEMM streams W while it runs,
      // and only the GEMM's epilogue loader waits for the delta
      l.pdl_trigger = 1;
      l.pdl_after_plan = 1;
      l.clear_status = 1;
      ML_CUDA(launch_lora_plan(l, cs), "LoRA plan launch");
      l.clear_status = 0;
      ML_CUDA(launch_lora_delta(l, cs), "dense LoRA launch");
    }
  }
  GemmArgs g{};
  g.epi = EPI_DENSE;
  g.K = h_in;
  g.E = 1;
  g.group_offsets = seg_offsets;  // [0] = 0 and [S] = T bound the single group
  g.group_stride = S;
  g.rows_per_group = h_out;
  g.n_out = h_out;
  g.I = 0;
  g.total_rows = T;
  g.delta_cols = h_out;
  g.delta = rr && place == LORA_DELTA ? ws.delta : nullptr;
  g.delta_bf16 = tcl ? ws.dbf : nullptr;
  g.out_bf16 = static_cast<__nv_bfloat16*>(y);
  g.status = ws.status;
  g.w = w;
  g.b = static_cast<const __nv_bfloat16*>(x);
  g.bn = choose_bn(T, 1);
  g.pdl_secondary = rr && place == LORA_DELTA ? 1 : 0;

  g.num_sms = num_sms();
  ML_CUDA(launch_gemm_tc(g, cs), "dense GEMM launch");
  return MOE_LORA_OK;
}

}  // extern "C"
