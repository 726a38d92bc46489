// Segmented LoRA kernels on CUDA cores (SGMV), the fp32 dense base GEMM and the
// fixed-order top-k combine.
//
// SGMV: tokens grouped into contiguous segments per adapter, each segment gathers
// its adapter's weights ([Punica review page], "提案手法").  The shrink z = xA has
// few outputs (r) and a long reduction (h_in), so the reduction is split over the
// 32 lanes of a warp and combined with shuffles ([vLLM MoE-LoRA page],
// "Otimizações em Nível de Kernel": split-K); A rows are read with 128-bit coalesced
// loads.  The expand adds zB into the output in the same pass (fused add, same
// section).  These kernels are HBM/L2-bound streams of adapter slices: no tensor
// cores (r <= 128 outputs per token).
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

namespace mlb {

constexpr int SH_RB = 8;  // max rows per shrink CTA

// largest q with off[q] <= s < off[q+1]; -1 when s lies outside [off[0], off[nseg])
__device__ __forceinline__ int find_segment(const int32_t* off, int nseg, int s) {
  if (nseg <= 0 || s < off[0] || s >= off[nseg]) return -1;
  int lo = 0, hi = nseg;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= s) lo = mid;
    else hi = mid;
  }
  return lo;
}

template <bool F32>
__global__ void __launch_bounds__(256) shrink_kernel(const ShrinkArgs a) {
  __shared__ int s_seg[SH_RB];
  __shared__ int s_src[SH_RB];
  __shared__ int s_ad[SH_RB];
  __shared__ int s_e[SH_RB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * a.rows_per_cta;
  const int nr = min(a.rows_per_cta, a.nrows - row0);
  if (nr <= 0) return;

  // offsets sanity (strided over the grid): monotone, start 0, end nrows
  for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < a.nseg; q += gridDim.x * blockDim.x)
    if (a.seg_offsets[q] > a.seg_offsets[q + 1]) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, q);
  if (blockIdx.x == 0 && threadIdx.x == 0 &&
      (a.seg_offsets[0] != 0 || a.seg_offsets[a.nseg] != a.nrows))
    set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, -1);

  if (threadIdx.x < nr) {
    const int s = row0 + threadIdx.x;
    const int q = find_segment(a.seg_offsets, a.nseg, s);
    int ad = -1, e = 0;
    if (q >= 0) {
      if (a.seg_adapter != nullptr) {
        ad = a.seg_adapter[q];
      } else {
        e = q / (a.L + 1);
        const int ap = q - e * (a.L + 1);
        ad = (ap == a.L) ? -1 : ap;
      }
      if (ad < -1 || ad >= a.L) {
        set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, s);
        ad = -1;
      }
    }
    s_seg[threadIdx.x] = (ad >= 0) ? q : -1;
    s_ad[threadIdx.x] = ad;
    s_e[threadIdx.x] = e;
    s_src[threadIdx.x] = a.gather ? a.gather[s] / a.gather_div : s;
    if (a.row_adapter) a.row_adapter[s] = ad;
  }
  __syncthreads();

  const size_t K = a.K;
  if (a.gather_dst != nullptr) {  // bf16 rows, 16 B per thread
    const int c16 = a.K / 8;
    for (int idx = threadIdx.x; idx < nr * c16; idx += blockDim.x) {
      const int i = idx / c16, c = idx - i * c16;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.src) +
                                                           s_src[i] * K) + c);
      reinterpret_cast<uint4*>(a.gather_dst + (row0 + i) * K)[c] = v;
    }
  }

  // runs of rows sharing one segment
  int i0 = 0;
  while (i0 < nr) {
    int i1 = i0 + 1;
    while (i1 < nr && s_seg[i1] == s_seg[i0]) ++i1;
    const int n = i1 - i0;
    const int ad = s_ad[i0];
    if (ad < 0) {
      for (int idx = threadIdx.x; idx < n * a.r; idx += blockDim.x)
        a.z[static_cast<size_t>(row0 + i0) * a.r + idx] = 0.f;
    } else {
      const size_t abase = (static_cast<size_t>(ad) * a.E + s_e[i0]) * a.r * K;
      for (int i = warp; i < a.r; i += 8) {
        float acc[SH_RB];
#pragma unroll
        for (int j = 0; j < SH_RB; ++j) acc[j] = 0.f;
        if constexpr (F32) {
          const float4* arow = reinterpret_cast<const float4*>(static_cast<const float*>(a.lora_a) + abase + i * K);
          for (int c = lane; c < a.K / 4; c += 32) {
            const float4 w4 = __ldg(arow + c);
#pragma unroll
            for (int j = 0; j < SH_RB; ++j) {
              if (j < n) {
                const float4 x4 = __ldg(reinterpret_cast<const float4*>(
                                            static_cast<const float*>(a.src) + s_src[i0 + j] * K) + c);
                acc[j] += w4.x * x4.x + w4.y * x4.y + w4.z * x4.z + w4.w * x4.w;
              }
            }
          }
        } else {
          const uint4* arow = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.lora_a) + abase + i * K);
          for (int c = lane; c < a.K / 8; c += 32) {
            const uint4 w8 = __ldg(arow + c);
#pragma unroll
            for (int j = 0; j < SH_RB; ++j) {
              if (j < n) {
                const uint4 x8 = __ldg(reinterpret_cast<const uint4*>(
                                           static_cast<const __nv_bfloat16*>(a.src) + s_src[i0 + j] * K) + c);
                acc[j] += dot8_bf16(w8, x8);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < SH_RB; ++j) {
          const float v = warp_sum(acc[j]);
          if (lane == 0 && j < n) a.z[static_cast<size_t>(row0 + i0 + j) * a.r + i] = v;
        }
      }
    }
    i0 = i1;
  }
}

cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t st) {
  if (a.nrows <= 0) return cudaSuccess;
  const int rb = a.rows_per_cta < 1 ? 1 : (a.rows_per_cta > SH_RB ? SH_RB : a.rows_per_cta);
  ShrinkArgs b = a;
  b.rows_per_cta = rb;
  const int grid = (a.nrows + rb - 1) / rb;
  ProfScope ps(K_SHRINK, st);
  if (a.src_f32) shrink_kernel<true><<<grid, 256, 0, st>>>(b);
  else shrink_kernel<false><<<grid, 256, 0, st>>>(b);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------- expand (dense API)
constexpr int EX_RB = 8;

template <bool F32>
__global__ void __launch_bounds__(256) expand_kernel(const ExpandArgs a) {
  constexpr int V = F32 ? 4 : 8;  // features per thread (16-byte loads of B)
  __shared__ int s_ad[EX_RB];
  const int row0 = blockIdx.x * EX_RB;
  const int nr = min(EX_RB, a.T - row0);
  if (threadIdx.x < nr) {
    const int s = row0 + threadIdx.x;
    const int q = find_segment(a.seg_offsets, a.nseg, s);
    int ad = (q >= 0) ? a.seg_adapter[q] : -1;
    if (ad < -1 || ad >= a.L) {
      set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, s);
      ad = -1;
    }
    s_ad[threadIdx.x] = ad;
  }
  __syncthreads();
  const int f = (blockIdx.y * blockDim.x + threadIdx.x) * V;
  if (f >= a.h_out) return;
  for (int j = 0; j < nr; ++j) {
    const int ad = s_ad[j];
    if (ad < 0) continue;
    const int s = row0 + j;
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    const float* zr = a.z + static_cast<size_t>(s) * a.r;
    for (int i = 0; i < a.r; ++i) {
      const float zi = zr[i];
      const size_t off = (static_cast<size_t>(ad) * a.r + i) * a.h_out + f;
      if constexpr (F32) {
        const float4 b4 = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(a.lora_b) + off));
        acc[0] += zi * b4.x;
        acc[1] += zi * b4.y;
        acc[2] += zi * b4.z;
        acc[3] += zi * b4.w;
      } else {
        float bf[8];
        unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.lora_b) + off)), bf);
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] += zi * bf[v];
      }
    }
    const size_t yoff = static_cast<size_t>(s) * a.h_out + f;
    if constexpr (F32) {
      float4* yp = reinterpret_cast<float4*>(static_cast<float*>(a.y) + yoff);
      float4 y4 = *yp;
      y4.x += acc[0];
      y4.y += acc[1];
      y4.z += acc[2];
      y4.w += acc[3];
      *yp = y4;
    } else {
      uint4* yp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) + yoff);
      float yf[8];
      unpack8_bf16(*yp, yf);
      *yp = make_uint4(pack2_bf16(yf[0] + acc[0], yf[1] + acc[1]), pack2_bf16(yf[2] + acc[2], yf[3] + acc[3]),
                       pack2_bf16(yf[4] + acc[4], yf[5] + acc[5]), pack2_bf16(yf[6] + acc[6], yf[7] + acc[7]));
    }
  }
}

cudaError_t launch_expand(const ExpandArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const int V = a.f32 ? 4 : 8;
  dim3 grid((a.T + EX_RB - 1) / EX_RB, (a.h_out + 256 * V - 1) / (256 * V));
  ProfScope ps(K_EXPAND, st);
  if (a.f32) expand_kernel<true><<<grid, 256, 0, st>>>(a);
  else expand_kernel<false><<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------- fp32 dense GEMM + expand
// Tile: 32 tokens x 64 features, K staged through shared memory 32 at a time.
__global__ void __launch_bounds__(256) dense_f32_kernel(const DenseF32Args a) {
  __shared__ float xs[32][33];
  __shared__ float ws[64][33];
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  const int t0 = blockIdx.y * 32, f0 = blockIdx.x * 64;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int k0 = 0; k0 < a.h_in; k0 += 32) {
    for (int idx = tid; idx < 32 * 32; idx += 256) {
      const int rr = idx >> 5, kk = idx & 31;
      const int t = t0 + rr, k = k0 + kk;
      xs[rr][kk] = (t < a.T && k < a.h_in) ? a.x[static_cast<size_t>(t) * a.h_in + k] : 0.f;
    }
    for (int idx = tid; idx < 64 * 32; idx += 256) {
      const int rr = idx >> 5, kk = idx & 31;
      const int f = f0 + rr, k = k0 + kk;
      ws[rr][kk] = (f < a.h_out && k < a.h_in) ? a.w[static_cast<size_t>(f) * a.h_in + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float x0 = xs[ty * 2][kk], x1 = xs[ty * 2 + 1][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float wv = ws[tx * 4 + j][kk];
        acc[0][j] += x0 * wv;
        acc[1][j] += x1 * wv;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int t = t0 + ty * 2 + u;
    if (t >= a.T) continue;
    const int ad = (a.row_adapter != nullptr && a.z != nullptr) ? a.row_adapter[t] : -1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int f = f0 + tx * 4 + j;
      if (f >= a.h_out) continue;
      float v = acc[u][j];
      if (ad >= 0) {
        const float* zr = a.z + static_cast<size_t>(t) * a.r;
        const float* bp = a.lora_b + static_cast<size_t>(ad) * a.r * a.h_out + f;
        for (int i = 0; i < a.r; ++i) v += zr[i] * bp[static_cast<size_t>(i) * a.h_out];
      }
      a.y[static_cast<size_t>(t) * a.h_out + f] = v;
    }
  }
}

cudaError_t launch_dense_f32(const DenseF32Args& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  dim3 grid((a.h_out + 63) / 64, (a.T + 31) / 32);
  ProfScope ps(K_DENSE_F32, st);
  dense_f32_kernel<<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------- top-k combine
// y[t, :] = sum_{j=0..k-1} o[t*k + j, :], summed in j order (run-to-run identical).
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ o, int M, int k, int H,
                                                     __nv_bfloat16* __restrict__ y) {
  const int t = blockIdx.x;
  const int f = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (f >= H) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* base = o + static_cast<size_t>(t) * k * H + f;
  for (int j = 0; j < k; ++j) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(base + static_cast<size_t>(j) * H));
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  uint2 out = make_uint2(pack2_bf16(acc.x, acc.y), pack2_bf16(acc.z, acc.w));
  *reinterpret_cast<uint2*>(y + static_cast<size_t>(t) * H + f) = out;
}

cudaError_t launch_combine(const float* o, int M, int k, int H, __nv_bfloat16* y, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  dim3 grid(M, (H / 4 + 255) / 256);
  ProfScope ps(K_COMBINE, st);
  combine_kernel<<<grid, 256, 0, st>>>(o, M, k, H, y);
  count_launch();
  return cudaGetLastError();
}

}  // namespace mlb
