// Optional per-kernel timing (CUDA events recorded around each launch on its own
// stream) and a launch counter.  Off by default; enabled through the C ABI
// (moe_lora_profile_enable) by measurement code.
#pragma once

#include <cuda_runtime.h>

namespace mlb {

enum KernelId : int {
  K_ROUTE_LOGITS = 0,
  K_TOPK = 1,
  K_SORT = 2,
  K_SHRINK = 3,
  K_GEMM_GATEUP = 4,
  K_GEMM_DOWN = 5,
  K_COMBINE = 6,
  K_EXPAND = 7,
  K_DENSE_F32 = 8,
  K_GEMM_DENSE = 9,
  K_QUANT = 10,
  K_LORA = 11,
  K_ROUTE = 12,
  K_LORA_DOWN = 13,  // the down projection's LoRA kernel (K_LORA: gate_up's and the work lists)
  K_GATHER = 14,     // token rows gathered into (expert, adapter) order
  K_COUNT = 15
};

void prof_begin(int id, cudaStream_t st);
void prof_end(int id, cudaStream_t st);
void count_launch(int n = 1);

struct ProfScope {
  int id;
  cudaStream_t st;
  ProfScope(int i, cudaStream_t s) : id(i), st(s) { prof_begin(id, st); }
  ~ProfScope() { prof_end(id, st); }
};

}  // namespace mlb
