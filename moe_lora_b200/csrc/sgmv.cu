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
#include <algorithm>

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

// One CTA per segment q (blockIdx.x < nseg) and row-chunk lane blockIdx.y: the CTA
// handles chunks y, y + gridDim.y, ... of SH_RB rows of segment q, so the segment's
// A slice is read from HBM once and then from L1/L2.  blockIdx.x == nseg handles the
// rows no segment covers (only possible with offsets that do not span [0, nrows)):
// no adapter, z = 0.
template <bool F32>
__global__ void __launch_bounds__(256) shrink_kernel(const ShrinkArgs a) {
  __shared__ int s_src[SH_RB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = blockIdx.x;
  const size_t K = a.K;

  if (blockIdx.y == 0) {  // offsets sanity, strided over the segments
    if (threadIdx.x == 0 && q < a.nseg && a.seg_offsets[q] > a.seg_offsets[q + 1])
      set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, q);
    if (q == 0 && threadIdx.x == 0 && (a.seg_offsets[0] != 0 || a.seg_offsets[a.nseg] != a.nrows))
      set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, -1);
  }

  int lo, hi, ad = -1, e = 0;
  if (q < a.nseg) {
    lo = a.seg_offsets[q];
    hi = min(a.seg_offsets[q + 1], a.nrows);
    lo = max(lo, 0);
    if (a.seg_adapter != nullptr) {
      ad = a.seg_adapter[q];
    } else {
      e = q / (a.L + 1);
      const int ap = q - e * (a.L + 1);
      ad = (ap == a.L) ? -1 : ap;
    }
    if (ad < -1 || ad >= a.L) {
      if (threadIdx.x == 0 && blockIdx.y == 0) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, q);
      ad = -1;
    }
  } else {
    lo = 0;  // uncovered rows: before the first offset and after the last
    hi = a.nrows;
  }
  const int first = (q < a.nseg) ? lo : 0;
  const int s_begin = a.seg_offsets[0], s_end = a.seg_offsets[a.nseg];
  if (q == a.nseg && s_begin <= 0 && s_end >= a.nrows) return;  // every row is covered
  const size_t abase = (ad >= 0) ? (static_cast<size_t>(ad) * a.E + e) * a.r * K : 0;

  for (int c = blockIdx.y; first + c * SH_RB < hi; c += gridDim.y) {
    const int r0 = first + c * SH_RB;
    const int n = min(SH_RB, hi - r0);
    __syncthreads();  // s_src of the previous chunk is no longer read
    if (threadIdx.x < SH_RB) {
      const int s = r0 + threadIdx.x;
      int src = -1;
      if (threadIdx.x < n) {
        const bool mine = (q < a.nseg) || s < s_begin || s >= s_end;
        if (mine) {
          src = a.gather ? a.gather[s] / a.gather_div : s;
          if (a.row_adapter) a.row_adapter[s] = ad;
        }
      }
      s_src[threadIdx.x] = src;
    }
    __syncthreads();
    if (a.gather_dst != nullptr) {  // bf16 rows, 16 B per thread
      const int c16 = a.K / 8;
      for (int idx = threadIdx.x; idx < n * c16; idx += blockDim.x) {
        const int i = idx / c16, cc = idx - i * c16;
        if (s_src[i] < 0) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.src) +
                                                             s_src[i] * K) + cc);
        reinterpret_cast<uint4*>(a.gather_dst + (r0 + i) * K)[cc] = v;
      }
    }
    if (ad < 0) {
      for (int idx = threadIdx.x; idx < n * a.r; idx += blockDim.x)
        if (s_src[idx / a.r] >= 0) a.z[static_cast<size_t>(r0) * a.r + idx] = 0.f;
      continue;
    }
    for (int i = warp; i < a.r; i += 8) {
      float acc[SH_RB];
#pragma unroll
      for (int j = 0; j < SH_RB; ++j) acc[j] = 0.f;
      if constexpr (F32) {
        const float4* arow = reinterpret_cast<const float4*>(static_cast<const float*>(a.lora_a) + abase + i * K);
        for (int cc = lane; cc < a.K / 4; cc += 32) {
          const float4 w4 = __ldg(arow + cc);
#pragma unroll
          for (int j = 0; j < SH_RB; ++j) {
            if (j < n) {
              const float4 x4 = __ldg(reinterpret_cast<const float4*>(
                                          static_cast<const float*>(a.src) + s_src[j] * K) + cc);
              acc[j] += w4.x * x4.x + w4.y * x4.y + w4.z * x4.z + w4.w * x4.w;
            }
          }
        }
      } else {
        const uint4* arow = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.lora_a) + abase + i * K);
        for (int cc = lane; cc < a.K / 8; cc += 32) {
          const uint4 w8 = __ldg(arow + cc);
#pragma unroll
          for (int j = 0; j < SH_RB; ++j) {
            if (j < n) {
              const uint4 x8 = __ldg(reinterpret_cast<const uint4*>(
                                         static_cast<const __nv_bfloat16*>(a.src) + s_src[j] * K) + cc);
              acc[j] += dot8_bf16(w8, x8);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < SH_RB; ++j) {
        const float v = warp_sum(acc[j]);
        if (lane == 0 && j < n) a.z[static_cast<size_t>(r0 + j) * a.r + i] = v;
      }
    }
  }
}

cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t st) {
  if (a.nrows <= 0) return cudaSuccess;
  // spread long segments over a few CTAs; one CTA per segment at decode sizes
  long long chunks = (a.nrows + SH_RB - 1) / SH_RB;
  int ysplit = static_cast<int>(chunks / (a.nseg > 0 ? a.nseg : 1));
  ysplit = ysplit < 1 ? 1 : (ysplit > 16 ? 16 : ysplit);
  dim3 grid(a.nseg + 1, ysplit);
  ProfScope ps(K_SHRINK, st);
  if (a.src_f32) shrink_kernel<true><<<grid, 256, 0, st>>>(a);
  else shrink_kernel<false><<<grid, 256, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------- e4m3 activation planes
// s = amax(|x|) / 448 per row (1 for an all-zero row); hi = RNE_sat(x / s) and
// lo = RNE_sat((x - hi s) / (s / 16)) in OCP e4m3, so that x = s hi + (s / 16) lo up to a
// relative 2^-8; the FP8-weight GEMM multiplies both planes on the kind::f8f6f4 tensor
// core.  |x / s| <= 448 and |(x - hi s) / (s / 16)| <= 448 by construction.
// One warp quantises one bf16 row of K elements into the two e4m3 planes (see below).
// copy_row (if set) also receives the bf16 row itself.
// The two e4m3 planes of 8 bf16 values (one 16-byte chunk) at scale s: hi = e4m3(v / s)
// and lo = e4m3((v - hi s) 16 / s), 8 bytes each.
__device__ __forceinline__ void quant8(const uint4 raw, float s, float inv, float inv_lo, uint2& hq8, uint2& lq8) {
  float f[8];
  unpack8_bf16(raw, f);
  uint32_t hq[2], lq[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t hw = 0, lw = 0;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int v = 4 * h + 2 * pr;
      const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(make_float2(f[v] * inv, f[v + 1] * inv),
                                                              __NV_SATFINITE, __NV_E4M3);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(q, __NV_E4M3);
      const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      const __nv_fp8x2_storage_t ql = __nv_cvt_float2_to_fp8x2(
          make_float2((f[v] - d.x * s) * inv_lo, (f[v + 1] - d.y * s) * inv_lo), __NV_SATFINITE, __NV_E4M3);
      hw |= static_cast<uint32_t>(q) << (16 * pr);
      lw |= static_cast<uint32_t>(ql) << (16 * pr);
    }
    hq[h] = hw;
    lq[h] = lw;
  }
  hq8 = make_uint2(hq[0], hq[1]);
  lq8 = make_uint2(lq[0], lq[1]);
}

__device__ __forceinline__ void quant_row_warp(const __nv_bfloat16* src_row, int K, uint8_t* hi_row, uint8_t* lo_row,
                                               float* scale2, int lane, __nv_bfloat16* copy_row = nullptr) {
  const uint4* xr = reinterpret_cast<const uint4*>(src_row);
  const int k8 = K / 8;
  float amax = 0.f;
  for (int c = lane; c < k8; c += 32) {
    float f[8];
    unpack8_bf16(__ldg(xr + c), f);
#pragma unroll
    for (int v = 0; v < 8; ++v) amax = fmaxf(amax, fabsf(f[v]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? amax / 448.f : 1.f;
  const float inv = 1.f / s, inv_lo = 16.f / s;
  for (int c = lane; c < k8; c += 32) {
    const uint4 raw = __ldg(xr + c);
    if (copy_row != nullptr) reinterpret_cast<uint4*>(copy_row)[c] = raw;
    uint2 hq, lq;
    quant8(raw, s, inv, inv_lo, hq, lq);
    reinterpret_cast<uint2*>(hi_row)[c] = hq;
    reinterpret_cast<uint2*>(lo_row)[c] = lq;
  }
  if (lane == 0) {
    scale2[0] = s;
    scale2[1] = s / 16.f;
  }
}

// ---------------------------------------------------------------- segmented LoRA for the GEMMs
// One fused streaming kernel per projection ([Punica review page], "提案手法": SGMV;
// [vLLM MoE-LoRA page], "O Papel da Multi-LoRA": shrink z = xA then expand zB, and
// "Otimizações em Nível de Kernel": split-K for the shrink, fused add of the expand).
// CTA = (work item, feature slice); an item is a chunk of up to rb rows of one segment
// (launch_lora_plan lists the chunks of the non-empty segments).  For its chunk the CTA
//   1. shrinks: warp w owns K slice (w mod KS) of rank rows (w / KS) + (8 / KS) m;
//      lanes stream 128-bit chunks of A and of the rows, split-K over lanes (shuffle)
//      and over the KS warps of a rank row (fixed-order sum in shared memory), so z
//      stays on chip;
//   2. expands: each thread owns 8 features of the slice, streams IB rows of B at a
//      time and writes delta = z B (fp32), which the GEMM epilogue adds to its tile.
// Segments without an adapter write delta = 0 (early exit of the LoRA work).  The
// CTAs of feature slice 0 also copy the gathered source rows (gate_up operand).
constexpr int LF_RB_MAX = 8;   // rows per chunk (4 or 8, chosen on the host)
constexpr int LF_NI = 4;       // rank rows per warp pass

struct SegInfo {
  int lo, hi, ad, e;
};

__device__ __forceinline__ SegInfo segment_info(const LoraDeltaArgs& a, int q, bool report) {
  SegInfo si;
  if (report && threadIdx.x == 0) {
    if (a.seg_offsets[q] > a.seg_offsets[q + 1]) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, q);
    if (q == 0 && (a.seg_offsets[0] != 0 || a.seg_offsets[a.nseg] != a.nrows))
      set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, -1);
  }
  si.lo = max(a.seg_offsets[q], 0);
  si.hi = min(a.seg_offsets[q + 1], a.nrows);
  si.e = 0;
  if (a.seg_adapter != nullptr) {
    si.ad = a.seg_adapter[q];
  } else {
    si.e = q / (a.L + 1);
    const int ap = q - si.e * (a.L + 1);
    si.ad = (ap == a.L) ? -1 : ap;
  }
  if (si.ad < -1 || si.ad >= a.L) {
    if (report && threadIdx.x == 0) set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, q);
    si.ad = -1;
  }
  return si;
}

// Source row of gathered row s: gather[s] / gather_div, or s without a gather.  An index
// outside [0, nsrc) (a corrupted pair index) is flagged and replaced by row 0.
__device__ __forceinline__ int gather_src(const LoraDeltaArgs& a, int s) {
  if (a.gather == nullptr) return s;
  const int v = a.gather[s] / a.gather_div;
  if (v < 0 || v >= a.nsrc) {
    set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, s);
    return 0;
  }
  return v;
}

// Partial shrink of one warp: rank rows i0 + istep g (g < LF_NI) over the 16-byte
// chunks [c0, c1) of K, for the chunk's rows j < RB (rows j >= n repeat row 0 and
// are dropped).  out[j * r + i] receives the warp's partial sums.
template <int RB, int U>
__device__ __forceinline__ void shrink_part(const __nv_bfloat16* aseg, const __nv_bfloat16* src, int K,
                                            const int* s_src, int n, int i0, int istep, int c0, int c1,
                                            int lane, float* out, int r) {
  float acc[LF_NI][RB];
#pragma unroll
  for (int g = 0; g < LF_NI; ++g)
#pragma unroll
    for (int j = 0; j < RB; ++j) acc[g][j] = 0.f;
  // 16-byte chunk offsets of the rank rows and of the source rows
  const uint4* a4 = reinterpret_cast<const uint4*>(aseg);
  const uint4* x4 = reinterpret_cast<const uint4*>(src);
  const int k8 = K / 8;
  uint32_t xo[RB];
#pragma unroll
  for (int j = 0; j < RB; ++j) xo[j] = static_cast<uint32_t>(s_src[j < n ? j : 0]) * k8;
  const uint32_t ao = static_cast<uint32_t>(i0) * k8, astep = static_cast<uint32_t>(istep) * k8;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  for (int base = c0; base < c1; base += 32 * U) {
    uint4 w8[U][LF_NI], x8[U][RB];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int cc = base + lane + 32 * u;
      const bool ok = cc < c1;
#pragma unroll
      for (int g = 0; g < LF_NI; ++g) w8[u][g] = ok ? __ldg(a4 + (ao + g * astep + cc)) : zero4;
#pragma unroll
      for (int j = 0; j < RB; ++j) x8[u][j] = ok ? __ldg(x4 + (static_cast<size_t>(xo[j]) + cc)) : zero4;
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int g = 0; g < LF_NI; ++g)
#pragma unroll
        for (int j = 0; j < RB; ++j) acc[g][j] += dot8_bf16(w8[u][g], x8[u][j]);
  }
#pragma unroll
  for (int g = 0; g < LF_NI; ++g)
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const float v = warp_sum(acc[g][j]);
      if (lane == 0 && j < n) out[j * r + i0 + istep * g] = v;
    }
}

// Row of delta that gathered row s writes: s itself, or scatter[s] (the routing pair of
// sorted row s, for a delta the combine reads in pair order).  An index outside
// [0, nrows) is flagged and the row is not written (-1).
__device__ __forceinline__ int delta_row(const LoraDeltaArgs& a, int s) {
  if (a.scatter == nullptr) return s;
  const int d = a.scatter[s];
  if (d < 0 || d >= a.nrows) {
    set_status(a.status, MOE_LORA_ERR_DEVICE_CHECK, s);
    return -1;
  }
  return d;
}

// Where the expand reads B for delta features [f, f + 8): the column pointer, its row
// stride, the B rows (rank) and the first z value they pair with.  Fused adapters: the
// slot's r rows of NB features.  Separate gate and up adapters (split_I = I): the slot holds
// the gate adapter's r_exp rows of I features, then the up adapter's; gate features pair
// with z[0, r_exp), up features with z[r_exp, 2 r_exp).
struct BCol {
  const __nv_bfloat16* p;
  int stride, zoff;
};

__device__ __forceinline__ BCol expand_bcol(const LoraDeltaArgs& a, size_t slot, int f) {
  BCol c;
  if (a.split_I == 0) {
    c.p = a.lora_b + slot * a.r_exp * a.NB + f;
    c.stride = a.NB;
    c.zoff = 0;
  } else {
    const bool up = f >= a.split_I;
    c.p = a.lora_b + (slot * 2 + (up ? 1 : 0)) * a.r_exp * a.split_I + (up ? f - a.split_I : f);
    c.stride = a.split_I;
    c.zoff = up ? a.r_exp : 0;
  }
  return c;
}

// delta[row(r0 + j)][f..f+8) = scale sum_i z[j][zoff + i] B_i[f..f+8) for j < n; IB rows of
// B in flight.
template <int RB, int IB>
__device__ __forceinline__ void expand_thread(const LoraDeltaArgs& a, const BCol& bc, const float* s_z, int n,
                                              int r0, int f) {
  float acc[RB][8];
#pragma unroll
  for (int j = 0; j < RB; ++j)
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[j][v] = 0.f;
  for (int i0 = 0; i0 < a.r_exp; i0 += IB) {
    uint4 b8[IB];
#pragma unroll
    for (int u = 0; u < IB; ++u)
      b8[u] = __ldg(reinterpret_cast<const uint4*>(bc.p + static_cast<size_t>(i0 + u) * bc.stride));
#pragma unroll
    for (int u = 0; u < IB; ++u) {
      float bf[8];
      unpack8_bf16(b8[u], bf);
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        const float zj = s_z[j * a.r + bc.zoff + i0 + u];
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[j][v] = fmaf(zj, bf[v], acc[j][v]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    const int row = j < n ? delta_row(a, r0 + j) : -1;
    if (row >= 0) {
      float4* d = reinterpret_cast<float4*>(a.delta + static_cast<size_t>(row) * a.NB + f);
      d[0] = make_float4(a.scale * acc[j][0], a.scale * acc[j][1], a.scale * acc[j][2], a.scale * acc[j][3]);
      d[1] = make_float4(a.scale * acc[j][4], a.scale * acc[j][5], a.scale * acc[j][6], a.scale * acc[j][7]);
    }
  }
}

// z[j][i] (into s_z) over the 16-byte K chunks [kc0, kc1): warps split the chunks ks
// ways and the rank rows 8 / ks ways; fixed-order sum of the ks partials.
template <int RB, int U>
__device__ __forceinline__ void shrink_chunk(const LoraDeltaArgs& a, const __nv_bfloat16* aseg, const int* s_src,
                                             int n, int ks, float* s_part, float* s_z, int kc0, int kc1) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ig = warp / ks, kp = warp - ig * ks;
  const int istep = 8 / ks;                 // rank-row groups
  const int per = (kc1 - kc0 + ks - 1) / ks;
  const int c0 = kc0 + kp * per, c1 = min(kc1, c0 + per);
  float* out = (ks == 1) ? s_z : s_part + kp * (LF_RB_MAX * a.r);
  for (int m0 = 0; ig + istep * m0 < a.r; m0 += LF_NI)
    shrink_part<RB, U>(aseg, a.src, a.K, s_src, n, ig + istep * m0, istep, c0, c1, lane, out, a.r);
  if (ks > 1) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < n * a.r; idx += blockDim.x) {
      float s = 0.f;
      for (int p = 0; p < ks; ++p) s += s_part[p * (LF_RB_MAX * a.r) + idx];
      s_z[idx] = s;
    }
  }
}

// RBMAX = rows per chunk (the host's rb); 4 keeps the decode kernel at three CTAs per SM.
template <int RBMAX>
__device__ __forceinline__ void lora_fused_body(const LoraDeltaArgs& a, int item_idx, int ks, int slice, int* s_src,
                                                float* s_z, float* s_part) {
  constexpr int rb = RBMAX;
  const int2 item = a.items[item_idx];
  SegInfo si = segment_info(a, item.x, false);
  si.lo = item.y;  // this CTA's chunk of the segment
  si.hi = min(si.hi, item.y + rb);
  const size_t K = a.K;
  const bool lora = a.delta != nullptr && a.r > 0;
  const bool do_gather = a.gather_dst != nullptr && blockIdx.y == 0;
  const bool do_quant = a.q_hi != nullptr && blockIdx.y == 0;
  if (!do_gather && !do_quant && !lora) return;
  const int f_lo = blockIdx.y * slice, f_hi = min(a.NB, f_lo + slice);
  const size_t slot = static_cast<size_t>(si.ad < 0 ? 0 : si.ad) * a.E + si.e;
  const __nv_bfloat16* aseg = a.lora_a + slot * a.r * K;
  if (lora && a.split_I == 0 && si.ad >= 0 && threadIdx.x < a.r && f_hi > f_lo) {
    // the expand's B rows head for L2 while the shrink streams A: the two loads overlap
    prefetch_l2_bulk(a.lora_b + (slot * a.r + threadIdx.x) * a.NB + f_lo, static_cast<uint32_t>(f_hi - f_lo) * 2u);
  }
  for (int c = blockIdx.z; si.lo + c * rb < si.hi; c += gridDim.z) {
    const int r0 = si.lo + c * rb;
    const int n = min(rb, si.hi - r0);
    __syncthreads();  // s_src / s_z of the previous chunk are no longer read
    if (threadIdx.x < LF_RB_MAX)
      s_src[threadIdx.x] = (threadIdx.x < n) ? gather_src(a, r0 + threadIdx.x) : 0;
    __syncthreads();
    if (do_gather) {
      const int c16 = a.K / 8;
      for (int idx = threadIdx.x; idx < n * c16; idx += blockDim.x) {
        const int j = idx / c16, cc = idx - j * c16;
        reinterpret_cast<uint4*>(a.gather_dst + (r0 + j) * K)[cc] =
            __ldg(reinterpret_cast<const uint4*>(a.src + s_src[j] * K) + cc);
      }
    }
    if (do_quant) {  // e4m3 experts: the activation planes of the chunk's rows
      const int w = threadIdx.x >> 5;
      if (w < n)
        quant_row_warp(a.src + s_src[w] * K, a.K, a.q_hi + (r0 + w) * K, a.q_lo + (r0 + w) * K,
                       a.q_scales + 2 * static_cast<size_t>(r0 + w), threadIdx.x & 31);
    }
    if (!lora) continue;
    if (si.ad < 0) {
      if (a.delta == nullptr) continue;  // shrink only: the GEMM skips rows without an adapter
      const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
      const int w4 = (f_hi - f_lo) / 4;
      for (int idx = threadIdx.x; idx < n * w4; idx += blockDim.x) {
        const int j = idx / w4, cc = idx - j * w4;
        const int row = delta_row(a, r0 + j);
        if (row >= 0) reinterpret_cast<float4*>(a.delta + static_cast<size_t>(row) * a.NB + f_lo)[cc] = z4;
      }
      continue;
    }
    const int k8 = a.K / 8;
    if (n <= 1) shrink_chunk<1, RBMAX == 4 ? 2 : 3>(a, aseg, s_src, n, ks, s_part, s_z, 0, k8);
    else if (n <= 2) shrink_chunk<2, 2>(a, aseg, s_src, n, ks, s_part, s_z, 0, k8);
    else if (RBMAX == 4 || n <= 4) shrink_chunk<4, 1>(a, aseg, s_src, n, ks, s_part, s_z, 0, k8);
    else shrink_chunk<8, 1>(a, aseg, s_src, n, ks, s_part, s_z, 0, k8);
    __syncthreads();
    for (int f = f_lo + threadIdx.x * 8; f < f_hi; f += blockDim.x * 8) {
      const BCol bc = expand_bcol(a, slot, f);
      if (n <= 1) {
        expand_thread<1, 8>(a, bc, s_z, n, r0, f);
      } else if (n <= 2) {
        expand_thread<2, 8>(a, bc, s_z, n, r0, f);
      } else if (RBMAX == 4 || n <= 4) {
        expand_thread<4, 8>(a, bc, s_z, n, r0, f);
      } else {
        expand_thread<8, 8>(a, bc, s_z, n, r0, f);
      }
    }
  }
}

// With programmatic dependent launch: the kernel behind this one (the GEMM that adds the
// delta in its epilogue) may start at once, and a kernel launched behind another one
// (pdl_end_wait) does not finish before that one has, so the launches after it still
// see a completed stream.
template <int RBMAX>
__global__ void __launch_bounds__(256, RBMAX == 4 ? 3 : 2) lora_fused_kernel(const LoraDeltaArgs a, int ks, int slice) {
  __shared__ int s_src[LF_RB_MAX];
  __shared__ float s_z[LF_RB_MAX * 128];
  __shared__ float s_part[64 * LF_RB_MAX];  // ks * r == 64 whenever ks > 1
  static_assert(sizeof(s_src) + sizeof(s_z) + sizeof(s_part) + 1024 <= kLoraCoresidentSmem,
                "the LoRA CTA must fit beside a GEMM CTA");
  if (a.pdl_trigger) pdl_trigger();
  if (a.pdl_after_plan) pdl_wait();  // the work list comes from the kernel ahead
  const int count = *a.item_count;  // a grid smaller than the work list walks it with a stride
  for (int it = blockIdx.x; it < count; it += gridDim.x) {
    lora_fused_body<RBMAX>(a, it, ks, slice, s_src, s_z, s_part);
    __syncthreads();  // the next item reuses s_src / s_z
  }
  if (a.pdl_secondary) pdl_wait();
}

// ---- split form for adapters with long A rows (r K >= 64 Ki elements): the shrink runs
// on CTAs (segment, K slice of LS_KSLICE, row-chunk lane), each writing fp32 partials
// z_part[slice][row][r]; then one CTA per (segment, feature slice, row-chunk lane) sums
// the partials in slice order (deterministic) and expands (delta) or stores z (bf16).
// Short load chains per CTA, and four to eight times the CTAs of the fused kernel.
constexpr int LS_KSLICE = 1024;

template <int RBMAX>
__global__ void __launch_bounds__(256, RBMAX == 4 ? 3 : 2) lora_shrink_part_kernel(const LoraDeltaArgs a, int ks) {
  constexpr int rb = RBMAX;
  __shared__ int s_src[LF_RB_MAX];
  __shared__ float s_z[LF_RB_MAX * 128];
  __shared__ float s_part[64 * LF_RB_MAX];
  if (blockIdx.x >= *a.item_count) return;
  const int2 item = a.items[blockIdx.x];
  SegInfo si = segment_info(a, item.x, false);
  si.lo = item.y;
  si.hi = min(si.hi, item.y + rb);
  const size_t K = a.K;
  const bool do_gather = a.gather_dst != nullptr && blockIdx.y == 0;
  const bool do_quant = a.q_hi != nullptr && blockIdx.y == 0;
  if (!do_gather && !do_quant && si.ad < 0) return;
  const int k8 = a.K / 8;
  const int kc0 = blockIdx.y * (LS_KSLICE / 8), kc1 = min(k8, kc0 + LS_KSLICE / 8);
  const size_t slot = static_cast<size_t>(si.ad < 0 ? 0 : si.ad) * a.E + si.e;
  const __nv_bfloat16* aseg = a.lora_a + slot * a.r * K;
  float* zp = a.z_part + static_cast<size_t>(blockIdx.y) * a.nrows * a.r;
  if (a.delta != nullptr && a.split_I == 0 && si.ad >= 0 && blockIdx.y == 0 && threadIdx.x < a.r) {
    // the expand kernel's B rows head for L2 while the shrink streams A
    prefetch_l2_bulk(a.lora_b + (slot * a.r + threadIdx.x) * a.NB, static_cast<uint32_t>(a.NB) * 2u);
  }
  for (int c = blockIdx.z; si.lo + c * rb < si.hi; c += gridDim.z) {
    const int r0 = si.lo + c * rb;
    const int n = min(rb, si.hi - r0);
    __syncthreads();
    if (threadIdx.x < LF_RB_MAX)
      s_src[threadIdx.x] = (threadIdx.x < n) ? gather_src(a, r0 + threadIdx.x) : 0;
    __syncthreads();
    if (do_gather) {
      for (int idx = threadIdx.x; idx < n * k8; idx += blockDim.x) {
        const int j = idx / k8, cc = idx - j * k8;
        reinterpret_cast<uint4*>(a.gather_dst + (r0 + j) * K)[cc] =
            __ldg(reinterpret_cast<const uint4*>(a.src + s_src[j] * K) + cc);
      }
    }
    if (do_quant) {  // e4m3 experts: the activation planes of the chunk's rows
      const int w = threadIdx.x >> 5;
      if (w < n)
        quant_row_warp(a.src + s_src[w] * K, a.K, a.q_hi + (r0 + w) * K, a.q_lo + (r0 + w) * K,
                       a.q_scales + 2 * static_cast<size_t>(r0 + w), threadIdx.x & 31);
    }
    if (si.ad < 0) continue;
    if (n <= 1) shrink_chunk<1, RBMAX == 4 ? 2 : 3>(a, aseg, s_src, n, ks, s_part, s_z, kc0, kc1);
    else if (n <= 2) shrink_chunk<2, 2>(a, aseg, s_src, n, ks, s_part, s_z, kc0, kc1);
    else if (RBMAX == 4 || n <= 4) shrink_chunk<4, 1>(a, aseg, s_src, n, ks, s_part, s_z, kc0, kc1);
    else shrink_chunk<8, 1>(a, aseg, s_src, n, ks, s_part, s_z, kc0, kc1);
    __syncthreads();
    for (int idx = threadIdx.x; idx < n * a.r; idx += blockDim.x) zp[static_cast<size_t>(r0) * a.r + idx] = s_z[idx];
  }
}

template <int RBMAX>
__global__ void __launch_bounds__(256, RBMAX == 4 ? 3 : 2) lora_expand_part_kernel(const LoraDeltaArgs a, int nks,
                                                                                    int slice) {
  constexpr int rb = RBMAX;
  __shared__ float s_z[LF_RB_MAX * 128];
  if (blockIdx.x >= *a.item_count) return;
  const int2 item = a.items[blockIdx.x];
  SegInfo si = segment_info(a, item.x, false);
  si.lo = item.y;
  si.hi = min(si.hi, item.y + rb);
  const int f_lo = blockIdx.y * slice, f_hi = min(a.NB, f_lo + slice);
  const size_t slot = static_cast<size_t>(si.ad < 0 ? 0 : si.ad) * a.E + si.e;
  const size_t pstride = static_cast<size_t>(a.nrows) * a.r;
  for (int c = blockIdx.z; si.lo + c * rb < si.hi; c += gridDim.z) {
    const int r0 = si.lo + c * rb;
    const int n = min(rb, si.hi - r0);
    if (si.ad < 0) {
      if (a.delta == nullptr) continue;  // z only: the GEMM skips rows without an adapter
      const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
      const int w4 = (f_hi - f_lo) / 4;
      for (int idx = threadIdx.x; idx < n * w4; idx += blockDim.x) {
        const int j = idx / w4, cc = idx - j * w4;
        const int row = delta_row(a, r0 + j);
        if (row >= 0) reinterpret_cast<float4*>(a.delta + static_cast<size_t>(row) * a.NB + f_lo)[cc] = z4;
      }
      continue;
    }
    __syncthreads();  // s_z of the previous chunk is no longer read
    for (int idx = threadIdx.x; idx < n * a.r; idx += blockDim.x) {
      const float* zp = a.z_part + static_cast<size_t>(r0) * a.r + idx;
      float sum = 0.f;
      for (int ky = 0; ky < nks; ++ky) sum += __ldcg(zp + ky * pstride);
      s_z[idx] = sum;
    }
    __syncthreads();
    if (a.delta == nullptr) continue;
    for (int f = f_lo + threadIdx.x * 8; f < f_hi; f += blockDim.x * 8) {
      const BCol bc = expand_bcol(a, slot, f);
      if (n <= 1) expand_thread<1, 8>(a, bc, s_z, n, r0, f);
      else if (n <= 2) expand_thread<2, 8>(a, bc, s_z, n, r0, f);
      else if (RBMAX == 4 || n <= 4) expand_thread<4, 8>(a, bc, s_z, n, r0, f);
      else expand_thread<8, 8>(a, bc, s_z, n, r0, f);
    }
  }
}

int lora_rows_per_chunk(int nrows, int nseg) { return (nrows >= 8LL * (nseg > 0 ? nseg : 1)) ? 8 : 4; }

int lora_items_bound(int nrows, int nseg, int rb) {
  return (nrows + rb - 1) / rb + (nseg < nrows ? nseg : nrows);
}

// Work list of the LoRA kernels: one item (segment q, first row) per chunk of up to rb
// rows of every non-empty segment, in segment order; also the sanity checks of the
// offsets and adapter ids (device status).  One CTA: contiguous ranges of segments per
// thread, block-wide exclusive scan of the item counts.
__global__ void __launch_bounds__(1024) lora_plan_kernel(const int32_t* __restrict__ off,
                                                         const int32_t* __restrict__ seg_adapter, int nseg, int L,
                                                         int nrows, int rb, int2* __restrict__ items,
                                                         int* __restrict__ count, int cap, int* status,
                                                         int adapters_only, int clear_status) {
  __shared__ int s_scan[32];
  pdl_trigger();  // a LoRA kernel launched behind this one may start (it waits for the list)
  if (clear_status) {  // the call's first kernel: its status block starts at zero
    for (int i = threadIdx.x; i < static_cast<int>(kStatusBytes / 4); i += blockDim.x) status[i] = 0;
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (nseg + blockDim.x - 1) / blockDim.x;
  const int q0 = threadIdx.x * per, q1 = min(nseg, q0 + per);
  if (threadIdx.x == 0 && (off[0] != 0 || off[nseg] != nrows)) set_status(status, MOE_LORA_ERR_DEVICE_CHECK, -1);
  // adapters_only: skip segments without an adapter (dense: id -1; MoE keys: a' = L)
  auto listed = [&](int q) {
    if (!adapters_only) return true;
    if (seg_adapter != nullptr) return seg_adapter[q] >= 0 && seg_adapter[q] < L;
    return q % (L + 1) != L;
  };
  int local = 0;
  for (int q = q0; q < q1; ++q) {
    const int a0 = off[q], a1 = off[q + 1];
    if (a0 > a1) set_status(status, MOE_LORA_ERR_DEVICE_CHECK, q);
    if (seg_adapter != nullptr && (seg_adapter[q] < -1 || seg_adapter[q] >= L))
      set_status(status, MOE_LORA_ERR_DEVICE_CHECK, q);
    const int lo = max(a0, 0), hi = min(a1, nrows);
    if (hi > lo && listed(q)) local += (hi - lo + rb - 1) / rb;
  }
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
    const int lo = max(off[q], 0), hi = min(off[q + 1], nrows);
    if (!listed(q)) continue;
    for (int r0 = lo; r0 < hi; r0 += rb, ++base)
      if (base < cap) items[base] = make_int2(q, r0);
  }
  if (threadIdx.x == blockDim.x - 1) *count = min(base, cap);
}

cudaError_t launch_lora_plan(const LoraDeltaArgs& a, cudaStream_t st) {
  if (a.nrows <= 0) return cudaSuccess;
  ProfScope ps(K_LORA, st);
  lora_plan_kernel<<<1, 1024, 0, st>>>(a.seg_offsets, a.seg_adapter, a.nseg, a.L, a.nrows, a.rb, a.items,
                                       a.item_count, a.items_bound, a.status, 0, a.clear_status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_lora_plan_all(const int32_t* seg_offsets, const int32_t* seg_adapter, int nseg, int L, int nrows,
                                 int rb, int2* items, int* count, int cap, int* status, cudaStream_t st,
                                 bool clear_status) {
  if (nrows <= 0) return cudaSuccess;
  ProfScope ps(K_LORA, st);
  lora_plan_kernel<<<1, 1024, 0, st>>>(seg_offsets, seg_adapter, nseg, L, nrows, rb, items, count, cap, status, 0,
                                       clear_status ? 1 : 0);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_lora_delta(const LoraDeltaArgs& args, cudaStream_t st) {
  LoraDeltaArgs a = args;
  if (a.r_exp == 0) a.r_exp = a.r;
  if (a.nrows <= 0) return cudaSuccess;
  if (a.r > 128 || a.r % 8 != 0 || a.NB % 8 != 0) return cudaErrorInvalidValue;
  if (a.items == nullptr || a.item_count == nullptr || (a.rb != 4 && a.rb != 8)) return cudaErrorInvalidValue;
  const bool lora = a.delta != nullptr && a.r > 0;
  if (!lora && a.gather_dst == nullptr && a.q_hi == nullptr) return cudaSuccess;  // nothing to do
  if (a.q_hi != nullptr && a.K % 16 != 0) return cudaErrorInvalidValue;
  const int bound = a.items_bound;
  // K split of the shrink over warps: every warp owns 8 rank rows (r <= 64)
  const int ks = lora ? (a.r >= 64 ? 1 : 64 / a.r) : 1;
  // feature slices of the expand: enough CTAs for two per SM when the items are few
  int nsplit = 1;
  if (lora && a.delta != nullptr) {
    const long long want = (2LL * (a.num_sms > 0 ? a.num_sms : 148) + bound - 1) / std::max(1, bound);
    const long long cap = std::max(1, a.NB / 512);
    nsplit = static_cast<int>(std::max(1LL, std::min(want, cap)));
  }
  int slice = (a.NB + nsplit - 1) / nsplit;
  slice = (slice + 7) / 8 * 8;
  nsplit = (a.NB + slice - 1) / slice;
  const int nks = (a.K + LS_KSLICE - 1) / LS_KSLICE;
  const bool pdl = a.pdl_trigger || a.pdl_secondary || a.pdl_after_plan;  // overlapped: one kernel
  if (!pdl && lora && a.z_part != nullptr && static_cast<long long>(a.r) * a.K >= 65536 && nks > 1 &&
      static_cast<long long>(nks) * a.nrows * a.r <= a.z_part_cap) {
    ProfScope ps(a.prof_id, st);
    dim3 g1(bound, nks);
    if (a.rb == 8) lora_shrink_part_kernel<8><<<g1, 256, 0, st>>>(a, ks);
    else lora_shrink_part_kernel<4><<<g1, 256, 0, st>>>(a, ks);
    dim3 g2(bound, a.delta != nullptr ? nsplit : 1);
    if (a.rb == 8) lora_expand_part_kernel<8><<<g2, 256, 0, st>>>(a, nks, slice);
    else lora_expand_part_kernel<4><<<g2, 256, 0, st>>>(a, nks, slice);
    count_launch(2);
    return cudaGetLastError();
  }
  dim3 grid(bound, nsplit);
  if (pdl) {
    // running beside a GEMM (one CTA of it per SM): at most one CTA per SM, so that every
    // CTA is resident at once (the GEMM behind a triggering kernel launches only when all
    // of its CTAs have started) and fits beside the GEMM.  Few work items (small batches):
    // the features are split into slices so that the SMs share the B stream, each slice
    // CTA redoing the item's shrink (A from L2 after the first); many items: one CTA per
    // SM walks the list, whole rows of features per item.
    const int sms = std::max(1, a.num_sms);
    int ns = lora ? std::max(1, std::min(sms / std::max(1, bound), std::max(1, a.NB / 256))) : 1;
    slice = ((a.NB + ns - 1) / ns + 7) / 8 * 8;
    ns = (a.NB + slice - 1) / slice;
    grid = dim3(std::max(1, std::min(bound, sms / ns)), ns);
  }
  ProfScope ps(a.prof_id, st);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (a.pdl_secondary || a.pdl_after_plan) ? 1 : 0;
  const cudaError_t e = a.rb == 8 ? cudaLaunchKernelEx(&cfg, lora_fused_kernel<8>, a, ks, slice)
                                  : cudaLaunchKernelEx(&cfg, lora_fused_kernel<4>, a, ks, slice);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---------------------------------------------------------------- row gather
// dst[i] = src[gather[i] / div]: one warp per row, 16-byte loads and stores, four in
// flight per lane.  A source index outside [0, nsrc) (corrupted pairs) gives a zero row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ src, int nsrc,
                                                         const int32_t* __restrict__ gather, int div, int rows,
                                                         int K, __nv_bfloat16* __restrict__ dst,
                                                         int* __restrict__ clear_status) {
  if (clear_status != nullptr && blockIdx.x == 0)  // the call's first kernel: its status block
    for (int i = threadIdx.x; i < static_cast<int>(kStatusBytes / 4); i += blockDim.x) clear_status[i] = 0;
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * 8;
  const int k8 = K / 8;
  for (int row = blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += nw) {
    const int s = gather[row] / div;
    const bool ok = s >= 0 && s < nsrc;
    const uint4* sp = reinterpret_cast<const uint4*>(src + static_cast<size_t>(ok ? s : 0) * K);
    uint4* dp = reinterpret_cast<uint4*>(dst + static_cast<size_t>(row) * K);
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    for (int c = lane; c < k8; c += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (ok && c + 32 * u < k8) ? __ldg(sp + c + 32 * u) : z4;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c + 32 * u < k8) dp[c + 32 * u] = v[u];
    }
  }
}

cudaError_t launch_gather_rows(const __nv_bfloat16* src, int nsrc, const int32_t* gather, int div, int rows, int K,
                               __nv_bfloat16* dst, cudaStream_t st, int* clear_status) {
  if (rows <= 0) return cudaSuccess;
  if (K % 8 != 0 || div <= 0) return cudaErrorInvalidValue;
  int grid = (rows + 7) / 8;
  if (grid > 148 * 8) grid = 148 * 8;
  ProfScope ps(K_GATHER, st);
  gather_rows_kernel<<<grid, 256, 0, st>>>(src, nsrc, gather, div, rows, K, dst, clear_status);
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

// ---------------------------------------------------------------- activation planes (standalone)
// One warp per row (quant_row_warp); used when no LoRA kernel reads the rows.
__global__ void __launch_bounds__(256) quant_planes_kernel(const __nv_bfloat16* __restrict__ src, int rows, int K,
                                                          uint8_t* __restrict__ hi, uint8_t* __restrict__ lo,
                                                          float* __restrict__ scales) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = blockIdx.x * 8 + warp; row < rows; row += gridDim.x * 8)
    quant_row_warp(src + static_cast<size_t>(row) * K, K, hi + static_cast<size_t>(row) * K,
                   lo + static_cast<size_t>(row) * K, scales + 2 * static_cast<size_t>(row), lane);
}

// The e4m3 planes of gathered rows: row i of the planes is quantised from
// src[gather[i] / div] (a zero row for an index outside [0, nsrc)).
__global__ void __launch_bounds__(256) gather_quant_kernel(const __nv_bfloat16* __restrict__ src, int nsrc,
                                                          const int32_t* __restrict__ gather, int div, int rows,
                                                          int K, uint8_t* __restrict__ hi, uint8_t* __restrict__ lo,
                                                          float* __restrict__ scales,
                                                          __nv_bfloat16* __restrict__ copy,
                                                          int* __restrict__ clear_status) {
  if (clear_status != nullptr && blockIdx.x == 0)  // the call's first kernel: its status block
    for (int i = threadIdx.x; i < static_cast<int>(kStatusBytes / 4); i += blockDim.x) clear_status[i] = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = blockIdx.x * 8 + warp; row < rows; row += gridDim.x * 8) {
    const int sr = gather[row] / div;
    if (sr < 0 || sr >= nsrc) {
      for (int c = lane; c < K / 16; c += 32) {
        reinterpret_cast<uint4*>(hi + static_cast<size_t>(row) * K)[c] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(lo + static_cast<size_t>(row) * K)[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (copy != nullptr)
        for (int c = lane; c < K / 8; c += 32)
          reinterpret_cast<uint4*>(copy + static_cast<size_t>(row) * K)[c] = make_uint4(0u, 0u, 0u, 0u);
      if (lane == 0) {
        scales[2 * static_cast<size_t>(row)] = 0.f;
        scales[2 * static_cast<size_t>(row) + 1] = 0.f;
      }
      continue;
    }
    quant_row_warp(src + static_cast<size_t>(sr) * K, K, hi + static_cast<size_t>(row) * K,
                   lo + static_cast<size_t>(row) * K, scales + 2 * static_cast<size_t>(row), lane,
                   copy != nullptr ? copy + static_cast<size_t>(row) * K : nullptr);
  }
}

// Rows of up to 8192 elements: one CTA per row, the row's 16-byte chunks held in
// registers (U per thread), so each row is read once; the same arithmetic as
// quant_row_warp (the row maximum does not depend on the order it is taken in).  gather
// null: row i of src; an index outside [0, nsrc) gives zero planes and zero scales.
template <int U>
__global__ void __launch_bounds__(256) quant_rows_kernel(const __nv_bfloat16* __restrict__ src, int nsrc,
                                                        const int32_t* __restrict__ gather, int div, int rows, int K,
                                                        uint8_t* __restrict__ hi, uint8_t* __restrict__ lo,
                                                        float* __restrict__ scales, __nv_bfloat16* __restrict__ copy,
                                                        int* __restrict__ clear_status) {
  __shared__ float s_amax[8];
  if (clear_status != nullptr && blockIdx.x == 0)  // the call's first kernel: its status block
    for (int i = threadIdx.x; i < static_cast<int>(kStatusBytes / 4); i += blockDim.x) clear_status[i] = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k8 = K / 8;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const int sr = gather != nullptr ? gather[row] / div : row;
    const bool ok = sr >= 0 && sr < nsrc;
    const uint4* xr = reinterpret_cast<const uint4*>(src + static_cast<size_t>(ok ? sr : 0) * K);
    uint4 raw[U];
    float amax = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + 256 * u;
      raw[u] = (ok && c < k8) ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
      float f[8];
      unpack8_bf16(raw[u], f);
#pragma unroll
      for (int v = 0; v < 8; ++v) amax = fmaxf(amax, fabsf(f[v]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) s_amax[warp] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = fmaxf(amax, s_amax[w]);
    const float s = amax > 0.f ? amax / 448.f : 1.f;
    const float inv = 1.f / s, inv_lo = 16.f / s;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = threadIdx.x + 256 * u;
      if (c < k8) {
        if (copy != nullptr) reinterpret_cast<uint4*>(copy + static_cast<size_t>(row) * K)[c] = raw[u];
        uint2 hq, lq;
        quant8(raw[u], s, inv, inv_lo, hq, lq);  // zero chunks give zero bytes
        reinterpret_cast<uint2*>(hi + static_cast<size_t>(row) * K)[c] = hq;
        reinterpret_cast<uint2*>(lo + static_cast<size_t>(row) * K)[c] = lq;
      }
    }
    if (threadIdx.x == 0) {
      scales[2 * static_cast<size_t>(row)] = ok ? s : 0.f;
      scales[2 * static_cast<size_t>(row) + 1] = ok ? s / 16.f : 0.f;
    }
    __syncthreads();  // s_amax is rewritten for the next row
  }
}

// quant_rows_kernel for K <= 8192 (one row per CTA), else the warp-per-row kernels
static cudaError_t launch_quant_rows(const __nv_bfloat16* src, int nsrc, const int32_t* gather, int div, int rows,
                                     int K, uint8_t* hi, uint8_t* lo, float* scales, __nv_bfloat16* copy,
                                     int* clear_status, cudaStream_t st) {
  const int k8 = K / 8;
  const int grid = rows < 148 * 8 ? rows : 148 * 8;
  if (k8 <= 256) quant_rows_kernel<1><<<grid, 256, 0, st>>>(src, nsrc, gather, div, rows, K, hi, lo, scales, copy, clear_status);
  else if (k8 <= 512) quant_rows_kernel<2><<<grid, 256, 0, st>>>(src, nsrc, gather, div, rows, K, hi, lo, scales, copy, clear_status);
  else quant_rows_kernel<4><<<grid, 256, 0, st>>>(src, nsrc, gather, div, rows, K, hi, lo, scales, copy, clear_status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather_quant(const __nv_bfloat16* src, int nsrc, const int32_t* gather, int div, int rows, int K,
                                uint8_t* hi, uint8_t* lo, float* scales, __nv_bfloat16* copy, cudaStream_t st,
                                int* clear_status) {
  if (rows <= 0) return cudaSuccess;
  if (K % 16 != 0 || div <= 0) return cudaErrorInvalidValue;
  ProfScope ps(K_QUANT, st);
  if (K / 8 <= 1024) return launch_quant_rows(src, nsrc, gather, div, rows, K, hi, lo, scales, copy, clear_status, st);
  int grid = (rows + 7) / 8;
  if (grid > 148 * 8) grid = 148 * 8;
  gather_quant_kernel<<<grid, 256, 0, st>>>(src, nsrc, gather, div, rows, K, hi, lo, scales, copy, clear_status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quant_planes(const __nv_bfloat16* src, int rows, int K, uint8_t* hi, uint8_t* lo, float* scales,
                                cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (K % 16 != 0) return cudaErrorInvalidValue;
  ProfScope ps(K_QUANT, st);
  if (K / 8 <= 1024) return launch_quant_rows(src, rows, nullptr, 1, rows, K, hi, lo, scales, nullptr, nullptr, st);
  int grid = (rows + 7) / 8;
  if (grid > 148 * 8) grid = 148 * 8;
  quant_planes_kernel<<<grid, 256, 0, st>>>(src, rows, K, hi, lo, scales);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------- top-k combine
// y[t, :] = sum_{j=0..k-1} o[t*k + j, :], summed in fp32 in j order (run-to-run identical);
// o holds the weighted per-pair outputs in bf16.  Thread = 8 features (16-byte loads).
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ o, int M, int k, int H,
                                                     const float* __restrict__ delta,
                                                     const __nv_bfloat16* __restrict__ delta_bf16,
                                                     const float* __restrict__ topk_w,
                                                     __nv_bfloat16* __restrict__ y) {
  const int t = blockIdx.x;
  const int f = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
  if (f >= H) return;
  float acc[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) acc[v] = 0.f;
  const __nv_bfloat16* base = o + static_cast<size_t>(t) * k * H + f;
  for (int j0 = 0; j0 < k; j0 += 8) {  // 8 slot rows (and their bf16 deltas) in flight
    uint4 v8[8], d8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v8[u] = (j0 + u < k) ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(j0 + u) * H))
                           : make_uint4(0u, 0u, 0u, 0u);
    if (delta_bf16 != nullptr) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const size_t pr = static_cast<size_t>(t) * k + j0 + u;
        d8[u] = (j0 + u < k) ? __ldg(reinterpret_cast<const uint4*>(delta_bf16 + pr * H + f))
                             : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // summed in slot order
      if (j0 + u < k) {
        float fv[8];
        unpack8_bf16(v8[u], fv);
        const size_t pr = static_cast<size_t>(t) * k + j0 + u;
        if (delta != nullptr) {  // the down LoRA delta of the pair, weighted here
          const float w = topk_w[pr];
          const float4* dp = reinterpret_cast<const float4*>(delta + pr * H + f);
          const float4 d0 = __ldg(dp), d1 = __ldg(dp + 1);
          fv[0] += w * d0.x;
          fv[1] += w * d0.y;
          fv[2] += w * d0.z;
          fv[3] += w * d0.w;
          fv[4] += w * d1.x;
          fv[5] += w * d1.y;
          fv[6] += w * d1.z;
          fv[7] += w * d1.w;
        } else if (delta_bf16 != nullptr) {
          const float w = topk_w[pr];
          float dv[8];
          unpack8_bf16(d8[u], dv);
#pragma unroll
          for (int v = 0; v < 8; ++v) fv[v] += w * dv[v];
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] += fv[v];
      }
    }
  }
  *reinterpret_cast<uint4*>(y + static_cast<size_t>(t) * H + f) =
      make_uint4(pack2_bf16(acc[0], acc[1]), pack2_bf16(acc[2], acc[3]), pack2_bf16(acc[4], acc[5]),
                 pack2_bf16(acc[6], acc[7]));
}

cudaError_t launch_combine(const __nv_bfloat16* o, int M, int k, int H, const float* delta,
                           const __nv_bfloat16* delta_bf16, const float* topk_w, __nv_bfloat16* y, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if ((delta != nullptr || delta_bf16 != nullptr) && topk_w == nullptr) return cudaErrorInvalidValue;
  dim3 grid(M, (H / 8 + 255) / 256);
  ProfScope ps(K_COMBINE, st);
  combine_kernel<<<grid, 256, 0, st>>>(o, M, k, H, delta, delta_bf16, topk_w, y);
  count_launch();
  return cudaGetLastError();
}

}  // namespace mlb
