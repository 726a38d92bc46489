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

#include <atomic>

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
    if (be >= E) {  // only NaN logits remain: flag the token, keep the indices in range
      if (lane == 0) set_status(status, MOE_LORA_ERR_DEVICE_CHECK, t);
      be = j % E;
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
// Slot j of token t routed to expert e, or -1: the token's k ids read as 16-byte
// vectors when k is a multiple of 4 (one load chain per token instead of k).
__device__ __forceinline__ int slot_of(const int32_t* __restrict__ topk_ids, int t, int k, int e) {
  const int32_t* row = topk_ids + static_cast<size_t>(t) * k;
  if ((k & 3) == 0 && k <= 16) {
    int4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (4 * q < k) v[q] = __ldg(reinterpret_cast<const int4*>(row) + q);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (4 * q < k) {
        if (v[q].x == e) return 4 * q;
        if (v[q].y == e) return 4 * q + 1;
        if (v[q].z == e) return 4 * q + 2;
        if (v[q].w == e) return 4 * q + 3;
      }
    return -1;
  }
  for (int j = 0; j < k; ++j)
    if (row[j] == e) return j;
  return -1;
}

// One block per expert e.  (1) Exclusive prefix of the key counts gives the CSR
// offsets of e's L+1 keys.  (2) The 16 warps split the tokens into 16 contiguous
// ranges; each warp counts its pairs per adapter key, the counts are prefixed over
// warps, then each warp walks its range in token order and places its pairs with a
// warp match on the key: positions are stable (ascending token within a key).
__global__ void __launch_bounds__(512) sort_scatter_kernel(const int32_t* __restrict__ topk_ids,
                                                          const int32_t* __restrict__ a_key,
                                                          const int32_t* __restrict__ key_count,
                                                          int M, int k, int E, int L,
                                                          int32_t* __restrict__ sorted_pairs,
                                                          int32_t* __restrict__ seg_offsets) {
  constexpr int NW = 16;
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
  for (int t = tb + lane; t < te; t += 32)
    if (slot_of(topk_ids, t, k, e) >= 0) atomicAdd(&s_wcnt[warp][a_key[t]], 1);
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
      jf = slot_of(topk_ids, t, k, e);
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

// ---------------------------------------------------------------- one-launch routing
// Small batches (M k <= RF_MAX_PAIRS): logits, top-k, weights, key counts, CSR offsets
// and the stable placement in ONE launch, so that a decode step pays one kernel instead
// of three.  Three phases, handed over by tickets (a_key[0, n_tb) per token block and
// a_key[n_tb] for all blocks, zeroed on the host before the launch):
//   1. CTA (expert block of RF_EB, token block of RF_TB) computes its logits, the 8
//      warps splitting H (128-bit loads, shuffle + fixed-order shared-memory sum);
//   2. the last CTA of a token block runs the top-k of its RF_TB tokens, one warp per
//      token as in topk_kernel (given logits: one CTA per token block starts here);
//   3. the last token block counts the pair keys in shared memory, scans them into
//      seg_offsets and places the pairs stably: one warp walks the pairs in order and
//      a warp match on the key ranks each pair among the earlier pairs of its key
//      (pairs of one token have distinct keys, so pair order is token order).
constexpr int RF_EB = 4;
constexpr int RF_TB = 8;
constexpr int RF_MAX_PAIRS = 1024;

// key counts [E (L+1)], pair keys [M k], unnormalised weights [RF_TB][k], pair ranks [M k]
size_t route_fused_smem(int E, int L, int M, int k) {
  return (static_cast<size_t>(E) * (L + 1) + 2 * static_cast<size_t>(M) * k + static_cast<size_t>(RF_TB) * k) * 4;
}

// Order-preserving unsigned key of a logit for the arg-max: larger logit, larger key;
// +0 and -0 share a key (they compare equal); NaN gets 0, the key of "not a candidate",
// since a NaN logit never wins a comparison.  -inf stays a candidate (key >= 1).
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (v != v) return 0u;
  if ((b & 0x7fffffffu) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// true in exactly one CTA: the one whose arrival completes `ticket` to `count`
__device__ __forceinline__ bool arrive_last(int* ticket, int count, int* s_flag) {
  __syncthreads();  // every write of this CTA is issued
  if (threadIdx.x == 0) {
    __threadfence();
    *s_flag = (atomicAdd(ticket, 1) == count - 1);
  }
  __syncthreads();
  if (!*s_flag) return false;
  __threadfence();
  return true;
}

__global__ void __launch_bounds__(256) route_fused_kernel(const RouteArgs a, const float* lg_in, int n_eb) {
  extern __shared__ int rf_smem[];
  __shared__ float s_red[8][RF_EB * RF_TB];
  __shared__ int s_scan[8];
  __shared__ int s_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tb = (a.M + RF_TB - 1) / RF_TB;
  int* tickets = a.a_key;
  const int LA = a.L + 1;
  const int nk = a.E * LA;
  const int mk = a.M * a.k;
  int* s_cnt = rf_smem;
  int* s_key = s_cnt + nk;
  float* s_w = reinterpret_cast<float*>(s_key + mk);
  const float* lg = lg_in;
  int tb;
  if (lg == nullptr) {
    // ---- phase 1: logits of experts [e0, e0 + 4) x tokens [t0, t0 + 8)
    const int eb = blockIdx.x % n_eb;
    tb = blockIdx.x / n_eb;
    const int e0 = eb * RF_EB, t0 = tb * RF_TB;
    const int ne = min(RF_EB, a.E - e0), nt = min(RF_TB, a.M - t0);
    float acc[RF_EB][RF_TB];
#pragma unroll
    for (int g = 0; g < RF_EB; ++g)
#pragma unroll
      for (int i = 0; i < RF_TB; ++i) acc[g][i] = 0.f;
    const int h8 = a.H / 8;
    const int per = (h8 + 7) / 8;
    const int c0 = warp * per, c1 = min(h8, c0 + per);
    const uint4* w4 = reinterpret_cast<const uint4*>(a.w_router);
    const uint4* x4 = reinterpret_cast<const uint4*>(a.x);
    for (int cc = c0 + lane; cc < c1; cc += 32) {
      uint4 wv[RF_EB], xv[RF_TB];
#pragma unroll
      for (int g = 0; g < RF_EB; ++g) wv[g] = __ldg(w4 + static_cast<size_t>(e0 + (g < ne ? g : 0)) * h8 + cc);
#pragma unroll
      for (int i = 0; i < RF_TB; ++i) xv[i] = __ldg(x4 + static_cast<size_t>(t0 + (i < nt ? i : 0)) * h8 + cc);
#pragma unroll
      for (int g = 0; g < RF_EB; ++g)
#pragma unroll
        for (int i = 0; i < RF_TB; ++i) acc[g][i] += dot8_bf16(wv[g], xv[i]);
    }
#pragma unroll
    for (int g = 0; g < RF_EB; ++g)
#pragma unroll
      for (int i = 0; i < RF_TB; ++i) {
        const float v = warp_sum(acc[g][i]);
        if (lane == 0) s_red[warp][g * RF_TB + i] = v;
      }
    __syncthreads();
    if (threadIdx.x < RF_EB * RF_TB) {
      const int g = threadIdx.x / RF_TB, i = threadIdx.x - g * RF_TB;
      if (g < ne && i < nt) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += s_red[w][threadIdx.x];
        a.logits[static_cast<size_t>(t0 + i) * a.E + e0 + g] = sum + (a.bias ? a.bias[e0 + g] : 0.f);
      }
    }
    if (!arrive_last(tickets + tb, n_eb, &s_flag)) return;
    lg = a.logits;
  } else {
    tb = blockIdx.x;
  }

  // ---- phase 2: top-k of the token block, one warp per token.  Each step takes the
  // largest logit left (the smallest expert id among equal ones) with two warp
  // reductions: the largest order-preserving key, then the smallest id holding it.
  const int t = tb * RF_TB + warp;
  if (t < a.M) {
    uint32_t kv[8];  // candidate keys; 0 once taken, for NaN and for ids >= E
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      kv[i] = (e < a.E) ? logit_key(__ldcg(lg + static_cast<size_t>(t) * a.E + e)) : 0u;
    }
    int ad = a.adapter_ids[t];
    if (ad < -1 || ad >= a.L) {
      if (lane == 0) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, t);
      ad = -1;
    }
    float top_v0 = 0.f, denom = 0.f;
    float* wrow = s_w + warp * a.k;
    for (int j = 0; j < a.k; ++j) {
      uint32_t lk = 0u, le = 0xffffffffu;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (kv[i] > lk) {  // ascending i: the lane's smallest id among its largest keys
          lk = kv[i];
          le = static_cast<uint32_t>(lane + 32 * i);
        }
      const uint32_t bk = __reduce_max_sync(0xffffffffu, lk);
      int be = static_cast<int>(__reduce_min_sync(0xffffffffu, (bk != 0u && lk == bk) ? le : 0xffffffffu));
      float bv;
      if (bk == 0u) {  // only NaN logits remain: flag the token, keep the indices in range
        if (lane == 0) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, t);
        be = j % a.E;
        bv = -INFINITY;
      } else {
        bv = key_logit(bk);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (be == lane + 32 * i) kv[i] = 0u;
      }
      if (j == 0) top_v0 = bv;
      const float ex = expf(bv - top_v0);
      denom += ex;
      if (lane == 0) {
        a.topk_ids[t * a.k + j] = be;
        wrow[j] = ex;
      }
    }
    __syncwarp();
    const float inv = 1.0f / denom;
    for (int j = lane; j < a.k; j += 32) a.topk_w[t * a.k + j] = wrow[j] * inv;
  }
  // one token block (M <= 8): this CTA is the only one past phase 2, and a block barrier
  // makes its top-k visible to its phase 3
  if (n_tb == 1) __syncthreads();
  else if (!arrive_last(tickets + n_tb, n_tb, &s_flag)) return;

  // ---- phase 3: key counts, CSR offsets, stable placement (one CTA)
  for (int i = threadIdx.x; i < nk; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < mk; p += blockDim.x) {
    const int tt = p / a.k;
    int ad = a.adapter_ids[tt];
    if (ad < -1 || ad >= a.L) ad = -1;
    const int key = __ldcg(a.topk_ids + p) * LA + (ad >= 0 ? ad : a.L);
    s_key[p] = key;
    atomicAdd(&s_cnt[key], 1);
  }
  __syncthreads();
  const int per = (nk + blockDim.x - 1) / blockDim.x;
  const int q0 = threadIdx.x * per, q1 = min(nk, q0 + per);
  int local = 0;
  for (int q = q0; q < q1; ++q) local += s_cnt[q];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  int base = incl - local;
  for (int w = 0; w < warp; ++w) base += s_scan[w];
  for (int q = q0; q < q1; ++q) {
    const int c = s_cnt[q];
    s_cnt[q] = base;
    a.seg_offsets[q] = base;
    base += c;
  }
  if (threadIdx.x == 0) a.seg_offsets[nk] = mk;
  // rank of each pair among the earlier pairs of its 32-pair chunk with the same key, and
  // for the first of them the chunk's count of that key (all warps, one chunk each)
  int* s_rank = reinterpret_cast<int*>(s_w + RF_TB * a.k);
  const unsigned lt = (1u << lane) - 1u;
  for (int p0 = warp * 32; p0 < mk; p0 += 8 * 32) {
    const int p = p0 + lane;
    const int key = (p < mk) ? s_key[p] : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    if (p < mk) s_rank[p] = __popc(peers & lt) | (((peers & lt) == 0u) ? __popc(peers) << 16 : 0);
  }
  __syncthreads();
  // stable placement, chunk after chunk: a pair goes to its key's next free slot plus its
  // rank; the chunk's first pair of each key then moves that key's slot on
  if (warp == 0) {
    for (int p0 = 0; p0 < mk; p0 += 32) {
      const int p = p0 + lane;
      const int key = (p < mk) ? s_key[p] : 0;
      const int rk = (p < mk) ? s_rank[p] : 0;
      if (p < mk) a.sorted_pairs[s_cnt[key] + (rk & 0xffff)] = p;
      __syncwarp();
      if (p < mk && (rk >> 16) != 0) s_cnt[key] += rk >> 16;
      __syncwarp();
    }
  }
}

int route_fused_tickets(int M, int k) {
  return (M > 0 && static_cast<long long>(M) * k <= RF_MAX_PAIRS) ? (M + RF_TB - 1) / RF_TB + 1 : 0;
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  const int nk = a.E * (a.L + 1);
  if (a.M == 0) return cudaMemsetAsync(a.seg_offsets, 0, sizeof(int32_t) * (nk + 1), st);
  if (static_cast<long long>(a.M) * a.k <= RF_MAX_PAIRS) {
    // one launch; a_key[0, n_tb] holds the tickets (zeroed here unless the caller's
    // status clear covered them)
    const int n_tb = (a.M + RF_TB - 1) / RF_TB;
    cudaError_t err = a.tickets_zeroed ? cudaSuccess : cudaMemsetAsync(a.a_key, 0, sizeof(int32_t) * (n_tb + 1), st);
    if (err != cudaSuccess) return err;
    const size_t smem = route_fused_smem(a.E, a.L, a.M, a.k);
    // the raised shared-memory limit is a per-device function attribute
    static std::atomic<bool> attr_set[kMaxDevices];
    const int dev = current_device_index();
    if (dev < 0) return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
      const int most = static_cast<int>(route_fused_smem(256, 64, 1, RF_MAX_PAIRS));  // E = 256, L = 64, caps
      err = cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      if (err != cudaSuccess) return err;
      attr_set[dev].store(true, std::memory_order_release);
    }
    if (a.logits_in != nullptr && a.logits_out != nullptr) {
      err = cudaMemcpyAsync(a.logits_out, a.logits_in, sizeof(float) * a.M * a.E, cudaMemcpyDeviceToDevice, st);
      if (err != cudaSuccess) return err;
    }
    const int n_eb = (a.E + RF_EB - 1) / RF_EB;
    const int grid = a.logits_in ? n_tb : n_eb * n_tb;
    ProfScope ps(K_ROUTE, st);
    route_fused_kernel<<<grid, 256, smem, st>>>(a, a.logits_in, n_eb);
    count_launch();
    return cudaGetLastError();
  }
  cudaError_t err = cudaMemsetAsync(a.key_count, 0, sizeof(int32_t) * nk, st);
  if (err != cudaSuccess) return err;
  const float* lg = a.logits_in;
  if (lg == nullptr && a.M >= 256 && tensor_map_encode_available()) {
    // large batches: logits on the tensor cores (the grouped GEMM with one group, W_r
    // rows in the MMA M slot, tokens in N, fp32 logits + bias in the epilogue)
    GemmArgs g{};
    g.epi = EPI_LOGITS;
    g.K = a.H;
    g.E = 1;
    g.group_offsets = nullptr;
    g.rows_per_group = a.E;
    g.n_out = a.E;
    g.total_rows = a.M;
    g.out_f32 = a.logits;
    g.bias = a.bias;
    g.status = a.status;
    g.w = a.w_router;
    g.b = a.x;
    g.bn = 32;
    g.num_sms = a.num_sms;
    err = launch_gemm_tc(g, st);
    if (err != cudaSuccess) return err;
    lg = a.logits;
  } else if (lg == nullptr) {
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
    sort_scatter_kernel<<<a.E, 512, 0, st>>>(a.topk_ids, a.a_key, a.key_count, a.M, a.k, a.E, a.L,
                                             a.sorted_pairs, a.seg_offsets);
    count_launch();
  }
  return cudaGetLastError();
}

}  // namespace mlb
