// Routing: router logits, softmax top-k with renormalised weights, and the stable
// (expert, adapter) counting sort of the routing pairs.
//
// A router sends each token to its most relevant experts ([vLLM MoE-LoRA page],
// "Entendendo os Modelos MoE"), k = 8 of them ([SageMaker MoE kernels page], first
// item); expert routing and adapter selection are combined into one sort key
// ([vLLM MoE-LoRA page], "Implementação Técnica no vLLM") so that every
// (expert, adapter) pair owns one contiguous segment, as in SGMV ([Punica review
// page], "提案手法").
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

namespace mlb {

// ---------------------------------------------------------------- router logits
// l[t, e] = sum_h x[t, h] * Wr[e, h] + bias[e], fp32 accumulation.
// Block: 8 warps, one expert per warp; RT_TB tokens per block share each Wr row load.
constexpr int RT_TB = 8;
constexpr int RT_EB = 8;

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const float* __restrict__ bias, int M,
                                                            int H, int E, float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * RT_TB;
  const int e = blockIdx.y * RT_EB + warp;
  if (e >= E) return;
  const int nt = min(RT_TB, M - t0);
  float acc[RT_TB];
#pragma unroll
  for (int i = 0; i < RT_TB; ++i) acc[i] = 0.f;
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e) * H);
  const int h8n = H >> 3;
  for (int h8 = lane; h8 < h8n; h8 += 32) {
    const uint4 w8 = __ldg(wrow + h8);
#pragma unroll
    for (int i = 0; i < RT_TB; ++i) {
      if (i < nt) {
        const uint4 x8 = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + i) * H) + h8);
        acc[i] += dot8_bf16(w8, x8);
      }
    }
  }
  const float b = bias ? bias[e] : 0.f;
#pragma unroll
  for (int i = 0; i < RT_TB; ++i) {
    const float s = warp_sum(acc[i]);
    if (lane == 0 && i < nt) logits[static_cast<size_t>(t0 + i) * E + e] = s + b;
  }
}

// Small batches: one CTA per (expert, block of RS_TB tokens); the 256 threads split H
// (128-bit loads, all independent), then a shuffle + shared-memory reduction.  Every
// CTA reads its W_r row once; the grid has E * ceil(M / RS_TB) CTAs.
constexpr int RS_TB = 16;

__global__ void __launch_bounds__(256) router_logits_splith_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   const __nv_bfloat16* __restrict__ wr,
                                                                   const float* __restrict__ bias, int M,
                                                                   int H, int E, float* __restrict__ logits) {
  __shared__ float red[8][RS_TB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x;
  const int t0 = blockIdx.y * RS_TB;
  const int nt = min(RS_TB, M - t0);
  float acc[RS_TB];
#pragma unroll
  for (int i = 0; i < RS_TB; ++i) acc[i] = 0.f;
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e) * H);
  const int h8n = H >> 3;
  for (int h8 = threadIdx.x; h8 < h8n; h8 += blockDim.x) {
    const uint4 w8 = __ldg(wrow + h8);
#pragma unroll
    for (int i = 0; i < RS_TB; ++i) {
      if (i < nt) {
        const uint4 x8 = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + i) * H) + h8);
        acc[i] += dot8_bf16(w8, x8);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < RS_TB; ++i) {
    const float v = warp_sum(acc[i]);
    if (lane == 0) red[warp][i] = v;
  }
  __syncthreads();
  if (threadIdx.x < nt) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
    logits[static_cast<size_t>(t0 + threadIdx.x) * E + e] = s + (bias ? bias[e] : 0.f);
  }
}

// ---------------------------------------------------------------- top-k + weights
// One warp per token.  Each lane holds experts lane, lane+32, ... (E <= 256).
// Selection: k rounds of a warp arg-max on (logit desc, expert asc).
// Weights: softmax over the k selected logits (equal to the full softmax
// renormalised over the selection).  Also counts pairs per sort key.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits,
                                                  const int32_t* __restrict__ adapter_ids, int M,
                                                  int E, int k, int L, int32_t* __restrict__ topk_ids,
                                                  float* __restrict__ topk_w,
                                                  int32_t* __restrict__ key_count,
                                                  int32_t* __restrict__ a_key, int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= M) return;
  float v[8];
  bool used[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? logits[static_cast<size_t>(t) * E + e] : -INFINITY;
    used[i] = (e >= E);
  }
  int a = adapter_ids[t];
  if (a < -1 || a >= L) {
    if (lane == 0) set_status(status, MOE_LORA_ERR_DEVICE_CHECK, t);
    a = -1;
  }
  const int ap = (a >= 0) ? a : L;
  if (lane == 0) a_key[t] = ap;

  float top_v0 = 0.f, denom = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (!used[i] && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (be == lane + 32 * i) used[i] = true;
    }
    if (j == 0) top_v0 = bv;
    const float ex = expf(bv - top_v0);
    denom += ex;
    if (lane == 0) {
      topk_ids[static_cast<size_t>(t) * k + j] = be;
      topk_w[static_cast<size_t>(t) * k + j] = ex;  // normalised below
      atomicAdd(key_count + be * (L + 1) + ap, 1);
    }
  }
  __syncwarp();
  const float inv = 1.0f / denom;
  for (int j = lane; j < k; j += 32) topk_w[static_cast<size_t>(t) * k + j] *= inv;
}

// ---------------------------------------------------------------- stable scatter
// One block per expert e.  (1) Exclusive prefix of the key counts gives the CSR
// offsets of e's L+1 keys.  (2) The 8 warps split the tokens into 8 contiguous
// ranges; each warp counts its pairs per adapter key, the counts are prefixed over
// warps, then each warp walks its range in token order and places its pairs with a
// warp match on the key: positions are stable (ascending token within a key).
__global__ void __launch_bounds__(256) sort_scatter_kernel(const int32_t* __restrict__ topk_ids,
                                                          const int32_t* __restrict__ a_key,
                                                          const int32_t* __restrict__ key_count,
                                                          int M, int k, int E, int L,
                                                          int32_t* __restrict__ sorted_pairs,
                                                          int32_t* __restrict__ seg_offsets) {
  constexpr int NW = 8;
  __shared__ int s_red[NW];
  __shared__ int s_off[65];
  __shared__ int s_wcnt[NW][65];
  __shared__ int s_run[NW][65];
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LA = L + 1;
  const int base_keys = e * LA;

  // (1) sum of counts of all keys before this expert
  int part = 0;
  for (int i = threadIdx.x; i < base_keys; i += blockDim.x) part += key_count[i];
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) s_red[warp] = part;
  for (int i = threadIdx.x; i < NW * 65; i += blockDim.x) {
    (&s_wcnt[0][0])[i] = 0;
    (&s_run[0][0])[i] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int base = 0;
    for (int w = 0; w < NW; ++w) base += s_red[w];
    for (int a = 0; a < LA; ++a) {
      s_off[a] = base;
      seg_offsets[base_keys + a] = base;
      base += key_count[base_keys + a];
    }
    if (e == E - 1) seg_offsets[E * LA] = base;
  }

  // (2a) per-warp counts
  const int chunk = (M + NW - 1) / NW;
  const int tb = warp * chunk, te = min(M, tb + chunk);
  for (int t = tb + lane; t < te; t += 32) {
    for (int j = 0; j < k; ++j) {
      if (topk_ids[static_cast<size_t>(t) * k + j] == e) {
        atomicAdd(&s_wcnt[warp][a_key[t]], 1);
        break;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < LA) {
    int acc = 0;
    for (int w = 0; w < NW; ++w) {
      const int c = s_wcnt[w][threadIdx.x];
      s_wcnt[w][threadIdx.x] = acc;  // becomes the warp's exclusive base for this key
      acc += c;
    }
  }
  __syncthreads();

  // (2b) stable placement
  for (int tb32 = tb; tb32 < te; tb32 += 32) {
    const int t = tb32 + lane;
    int jf = -1, ap = 0;
    if (t < te) {
      for (int j = 0; j < k; ++j)
        if (topk_ids[static_cast<size_t>(t) * k + j] == e) {
          jf = j;
          break;
        }
      ap = a_key[t];
    }
    const int keyv = (jf >= 0) ? ap : (LA + lane);
    const unsigned peers = __match_any_sync(0xffffffffu, keyv);
    if (jf >= 0) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = s_off[ap] + s_wcnt[warp][ap] + s_run[warp][ap] + rank;
      sorted_pairs[pos] = t * k + jf;
    }
    __syncwarp();
    if (jf >= 0 && (peers & ((1u << lane) - 1u)) == 0) s_run[warp][ap] += __popc(peers);
    __syncwarp();
  }
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  const int nk = a.E * (a.L + 1);
  cudaError_t err = cudaMemsetAsync(a.key_count, 0, sizeof(int32_t) * nk, st);
  if (err != cudaSuccess) return err;
  if (a.M == 0) {
    return cudaMemsetAsync(a.seg_offsets, 0, sizeof(int32_t) * (nk + 1), st);
  }
  const float* lg = a.logits_in;
  if (lg == nullptr) {
    ProfScope ps(K_ROUTE_LOGITS, st);
    if (a.M <= 256) {
      dim3 grid(a.E, (a.M + RS_TB - 1) / RS_TB);
      router_logits_splith_kernel<<<grid, 256, 0, st>>>(a.x, a.w_router, a.bias, a.M, a.H, a.E, a.logits);
    } else {
      dim3 grid((a.M + RT_TB - 1) / RT_TB, (a.E + RT_EB - 1) / RT_EB);
      router_logits_kernel<<<grid, 256, 0, st>>>(a.x, a.w_router, a.bias, a.M, a.H, a.E, a.logits);
    }
    count_launch();
    lg = a.logits;
  } else if (a.logits_out != nullptr) {
    err = cudaMemcpyAsync(a.logits_out, a.logits_in, sizeof(float) * a.M * a.E,
                          cudaMemcpyDeviceToDevice, st);
    if (err != cudaSuccess) return err;
  }
  {
    ProfScope ps(K_TOPK, st);
    topk_kernel<<<(a.M + 7) / 8, 256, 0, st>>>(lg, a.adapter_ids, a.M, a.E, a.k, a.L, a.topk_ids,
                                               a.topk_w, a.key_count, a.a_key, a.status);
    count_launch();
  }
  {
    ProfScope ps(K_SORT, st);
    sort_scatter_kernel<<<a.E, 256, 0, st>>>(a.topk_ids, a.a_key, a.key_count, a.M, a.k, a.E, a.L,
                                             a.sorted_pairs, a.seg_offsets);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace mlb
