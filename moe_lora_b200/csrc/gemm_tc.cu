// Tensor-core grouped GEMM for the expert (or dense) projections, sm_100a.
//
// Operand swap: the MMA's 128-row M slot takes 128 weight rows (output features)
// and its N slot the tokens of one expert, so that a decode batch of a few tokens
// per expert still fills the tensor core's M dimension ([SageMaker MoE kernels
// page], first item: transpose so the large expert dimension is the first operand).
// The LoRA expand z B and the base output are added in the epilogue, in registers,
// before anything is stored ([vLLM MoE-LoRA page], "Otimizações em Nível de
// Kernel": the LoRA add fused into the expand; "Implementação Técnica no vLLM":
// fused_moe_lora).  gate_up tiles pair 64 gate rows with the matching 64 up rows so
// the SiLU-and-mul gate is applied before act leaves the SM; down tiles multiply by
// the routing weight and store one fp32 row per routing pair for the fixed-order
// combine (expert aggregation, [SageMaker MoE kernels page], second item).
//
// Structure (one CTA per SM, persistent over a device-side tile list):
//   warp 0      TMA producer: weight tile 128 x 64 (two 64-row boxes) and token
//               tile BN x 64 per stage, 128-byte swizzle, mbarrier transaction count
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in TMEM),
//               M = 128, N = BN, K = 16 x 4 per stage; commits free the smem stage
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, LoRA expand, activation,
//               stores; two TMEM accumulators so the epilogue of tile i overlaps
//               the MMAs of tile i+1
// Every mbarrier wait is bounded; on expiry the CTA records MOE_LORA_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace mlb {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kMaxGroups = 256;
constexpr int kMaxR = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

struct TcParams {
  int epi;
  int K;
  int E;
  const int32_t* group_offsets;
  int group_stride;
  int rows_per_group;
  int n_out;
  int I;
  const float* z;
  const int32_t* row_adapter;
  const __nv_bfloat16* lora_b;
  int r;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  const int32_t* sorted_pairs;
  const float* topk_w;
  const float* w_scales;
  int scale_idx;
  int* status;
  int m_tiles;
  int stages;
};

// Non-pipeline shared memory, placed after the stage ring.
struct SmemMisc {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t tdone;
  uint32_t tmem_base;
  int abort_flag;
  int chunk_pref[kMaxGroups + 1];
  int grp_off[kMaxGroups + 1];
  float ebuf[kBM][33];
  float zs[32 * kMaxR];
  int col_ad[32];
  int col_pair[32];
  float col_w[32];
};

template <int BN>
struct TileCfg {
  static constexpr int kBTileBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kATileBytes + kBTileBytes;
  static constexpr int kAccStride = BN < 32 ? 32 : BN;  // TMEM columns per accumulator
  static constexpr int kTmemCols = 2 * kAccStride;      // power of two >= 32
};

struct TileInfo {
  int g, mt, row0, nvalid;
};

__device__ __forceinline__ TileInfo decode_tile(const SmemMisc& sm, int t, int m_tiles, int E, int BN) {
  TileInfo ti;
  const int c = t / m_tiles;
  ti.mt = t - c * m_tiles;
  int lo = 0, hi = E;  // largest g with chunk_pref[g] <= c (chunk_pref[E] > c)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sm.chunk_pref[mid] <= c) lo = mid;
    else hi = mid;
  }
  ti.g = lo;
  ti.row0 = sm.grp_off[lo] + (c - sm.chunk_pref[lo]) * BN;
  ti.nvalid = min(BN, sm.grp_off[lo + 1] - ti.row0);
  return ti;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmb,
                   const TcParams p) {
  using Cfg = TileCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemMisc& sm = *reinterpret_cast<SmemMisc*>(smem + p.stages * Cfg::kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;
  volatile int* abort_flag = &sm.abort_flag;

  // ---- setup: barriers, TMEM, tile list prefix
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kEpiThreads);
    }
    mbar_init(&sm.tdone, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmw);
    tma_prefetch_desc(&tmb);
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, Cfg::kTmemCols);
  for (int g = threadIdx.x; g <= p.E; g += blockDim.x)
    sm.grp_off[g] = p.group_offsets[static_cast<size_t>(g) * p.group_stride];
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix of chunks per group (E <= 256: 8 per lane, then a warp scan)
    int cnt[8];
    int tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = lane * 8 + i;
      int c = 0;
      if (g < p.E) {
        const int n = sm.grp_off[g + 1] - sm.grp_off[g];
        c = n > 0 ? (n + BN - 1) / BN : 0;
      }
      cnt[i] = c;
      tot += c;
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - tot;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = lane * 8 + i;
      if (g < p.E) sm.chunk_pref[g] = run;
      run += cnt[i];
    }
    if (lane == 31) sm.chunk_pref[p.E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int total_tiles = sm.chunk_pref[p.E] * p.m_tiles;
  const int nk = (p.K + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled_mask = 0, last_parity = 0;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x) {
        const TileInfo ti = decode_tile(sm, t, p.m_tiles, p.E, BN);
        int wrow0, wrow1;
        if (p.epi == EPI_GATEUP) {
          wrow0 = ti.g * p.rows_per_group + ti.mt * 64;
          wrow1 = ti.g * p.rows_per_group + p.I + ti.mt * 64;
        } else {
          wrow0 = ti.g * p.rows_per_group + ti.mt * kBM;
          wrow1 = wrow0 + 64;
        }
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort_flag, p.status, kWaitLimitNs, 1)) break;
          uint8_t* a_s = smem + stage * Cfg::kStageBytes;
          uint8_t* b_s = a_s + kATileBytes;
          mbar_arrive_expect_tx(&sm.full[stage], Cfg::kStageBytes);
          tma_load_2d(a_s, &tmw, &sm.full[stage], kb * kBK, wrow0);
          tma_load_2d(a_s + kATileBytes / 2, &tmw, &sm.full[stage], kb * kBK, wrow1);
          tma_load_2d(b_s, &tmb, &sm.full[stage], kb * kBK, ti.row0);
          filled_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let our own copies land before the CTA exits
        for (int s = 0; s < S; ++s)
          if (filled_mask & (1u << s)) {
            volatile int dummy = 0;
            mbar_wait(&sm.full[s], (last_parity >> s) & 1u, &dummy, nullptr, kWaitLimitNs / 4, 0);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int t = blockIdx.x; t < total_tiles && !*abort_flag; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait(&sm.tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, kWaitLimitNs, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * Cfg::kAccStride;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status, kWaitLimitNs, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * Cfg::kStageBytes);
          const uint32_t b_addr = a_addr + kATileBytes;
          const uint64_t adesc = umma_desc_sw128(a_addr);
          const uint64_t bdesc = umma_desc_sw128(b_addr);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&sm.empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&sm.tfull[buf]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(&sm.tdone);
      volatile int dummy = 0;
      mbar_wait(&sm.tdone, 0, &dummy, nullptr, kWaitLimitNs, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;   // 0..127
    const int g4 = warp & 3;           // TMEM lane quarter this warp may access
    const int m = g4 * 32 + lane;      // accumulator row = weight row within the tile
    int it = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++it) {
      const TileInfo ti = decode_tile(sm, t, p.m_tiles, p.E, BN);
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const bool got = mbar_wait(&sm.tfull[buf], use & 1u, abort_flag, p.status, kWaitLimitNs, 4);
      if (!named_bar_and(2, kEpiThreads, got)) break;  // the four warps leave together
      tc_fence_after();

      // weight row (within the group's rows) held by this thread, and whether it is real
      int wrow, feat;
      bool row_ok;
      if (p.epi == EPI_GATEUP) {
        feat = ti.mt * 64 + (m & 63);
        wrow = (m < 64) ? feat : p.I + feat;
        row_ok = feat < p.I;
      } else {
        feat = ti.mt * kBM + m;
        wrow = feat;
        row_ok = feat < p.n_out;
      }
      float scale = 1.f;
      if (p.w_scales != nullptr) scale = p.w_scales[ti.g * 2 + p.scale_idx];

      for (int c0 = 0; c0 < ti.nvalid; c0 += 32) {
        named_bar_sync(1, kEpiThreads);
        const int ncol = min(32, ti.nvalid - c0);
        if (et < 32) {
          const int s = ti.row0 + c0 + et;
          const bool valid = et < ncol;
          sm.col_ad[et] = (valid && p.row_adapter != nullptr) ? p.row_adapter[s] : -1;
          if (p.epi == EPI_DOWN) {
            const int pr = valid ? p.sorted_pairs[s] : 0;
            sm.col_pair[et] = pr;
            sm.col_w[et] = valid ? p.topk_w[pr] : 0.f;
          }
        }
        if (p.z != nullptr) {
          for (int idx = et; idx < 32 * p.r; idx += kEpiThreads) {
            const int n = idx / p.r;
            sm.zs[idx] = (n < ncol) ? p.z[static_cast<size_t>(ti.row0 + c0 + n) * p.r + (idx - n * p.r)] : 0.f;
          }
        }
        named_bar_sync(1, kEpiThreads);

        float v[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(g4 * 32) << 16) + buf * Cfg::kAccStride + c0, v);
#pragma unroll
        for (int n = 0; n < 32; ++n) v[n] *= scale;

        if (row_ok && p.z != nullptr) {
#pragma unroll
          for (int n = 0; n < 32; ++n) {
            const int ad = sm.col_ad[n];
            if (ad >= 0) {
              const __nv_bfloat16* bcol = p.lora_b + (static_cast<size_t>(ad) * p.E + ti.g) * p.r * p.rows_per_group + wrow;
              const float* zr = &sm.zs[n * p.r];
              float acc = 0.f;
              for (int i = 0; i < p.r; ++i)
                acc = fmaf(zr[i], __bfloat162float(bcol[static_cast<size_t>(i) * p.rows_per_group]), acc);
              v[n] += acc;
            }
          }
        }

        if (p.epi == EPI_GATEUP) {
#pragma unroll
          for (int n = 0; n < 32; ++n) sm.ebuf[m][n] = v[n];
          named_bar_sync(1, kEpiThreads);
          const int n = et >> 2;
          const int fq = (et & 3) * 16;
          if (n < ncol) {
            __nv_bfloat16* dst = p.out_bf16 + static_cast<size_t>(ti.row0 + c0 + n) * p.I + ti.mt * 64 + fq;
            const int fbase = ti.mt * 64 + fq;
            uint32_t packed[8];
#pragma unroll
            for (int f = 0; f < 16; f += 2) {
              const float a0 = silu(sm.ebuf[fq + f][n]) * sm.ebuf[64 + fq + f][n];
              const float a1 = silu(sm.ebuf[fq + f + 1][n]) * sm.ebuf[64 + fq + f + 1][n];
              packed[f >> 1] = pack2_bf16(a0, a1);
            }
            if (fbase + 16 <= p.I) {
              uint4* d4 = reinterpret_cast<uint4*>(dst);
              d4[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              d4[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            } else {
              for (int f = 0; f < 16 && fbase + f < p.I; ++f) {
                const uint32_t w2 = packed[f >> 1];
                const uint16_t h = (f & 1) ? static_cast<uint16_t>(w2 >> 16) : static_cast<uint16_t>(w2 & 0xFFFF);
                reinterpret_cast<uint16_t*>(dst)[f] = h;
              }
            }
          }
        } else if (p.epi == EPI_DOWN) {
          if (row_ok) {
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol)
                p.out_f32[static_cast<size_t>(sm.col_pair[n]) * p.n_out + feat] = v[n] * sm.col_w[n];
          }
        } else {
          if (row_ok) {
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol)
                p.out_bf16[static_cast<size_t>(ti.row0 + c0 + n) * p.n_out + feat] = __float2bfloat16_rn(v[n]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

// ---------------------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

bool tensor_map_encode_available() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

CUresult encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                        CUtensorMapSwizzle swz) {
  if (!tensor_map_encode_available()) return CUDA_ERROR_NOT_SUPPORTED;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int BN>
static cudaError_t launch_bn(const GemmArgs& a, cudaStream_t st) {
  using Cfg = TileCfg<BN>;
  const int misc = static_cast<int>(sizeof(SmemMisc));
  const int budget = 232448 - 1024 - misc;
  int stages = budget / Cfg::kStageBytes;
  stages = stages > 8 ? 8 : stages;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + static_cast<size_t>(stages) * Cfg::kStageBytes + misc;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem > 232448 ? 232448 : smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap tmw, tmb;
  const uint64_t wrows = static_cast<uint64_t>(a.E) * a.rows_per_group;
  if (encode_tmap_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w, a.K, wrows, static_cast<uint64_t>(a.K) * 2,
                     kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tmap_2d(&tmb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b, a.K, a.total_rows,
                     static_cast<uint64_t>(a.K) * 2, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  TcParams p;
  p.epi = a.epi;
  p.K = a.K;
  p.E = a.E;
  p.group_offsets = a.group_offsets;
  p.group_stride = a.group_stride;
  p.rows_per_group = a.rows_per_group;
  p.n_out = a.n_out;
  p.I = a.I;
  p.z = a.z;
  p.row_adapter = a.row_adapter;
  p.lora_b = a.lora_b;
  p.r = a.r;
  p.out_bf16 = a.out_bf16;
  p.out_f32 = a.out_f32;
  p.sorted_pairs = a.sorted_pairs;
  p.topk_w = a.topk_w;
  p.w_scales = a.w_scales;
  p.scale_idx = a.scale_idx;
  p.status = a.status;
  p.m_tiles = (a.epi == EPI_GATEUP) ? (a.I + 63) / 64 : (a.n_out + kBM - 1) / kBM;
  p.stages = stages;
  const long long chunks_ub = (a.total_rows + BN - 1) / BN + a.E;
  const long long tiles_ub = chunks_ub * p.m_tiles;
  int grid = a.num_sms;
  if (tiles_ub < grid) grid = static_cast<int>(tiles_ub);
  if (grid < 1) grid = 1;
  ProfScope ps(a.epi == EPI_GATEUP ? K_GEMM_GATEUP : (a.epi == EPI_DOWN ? K_GEMM_DOWN : K_GEMM_DENSE), st);
  gemm_tc_kernel<BN><<<grid, kThreads, smem, st>>>(tmw, tmb, p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxGroups || a.r > kMaxR || a.w_fp8) return cudaErrorInvalidValue;
  switch (a.bn) {
    case 16: return launch_bn<16>(a, st);
    case 32: return launch_bn<32>(a, st);
    case 64: return launch_bn<64>(a, st);
    case 128: return launch_bn<128>(a, st);
    case 256: return launch_bn<256>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mlb
