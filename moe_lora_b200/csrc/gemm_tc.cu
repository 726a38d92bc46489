// Tensor-core grouped GEMM for the expert (or dense) projections, sm_100a.
//
// Operand swap: the MMA's 128-row M slot takes 128 weight rows (output features)
// and its N slot the tokens of one expert, so that a decode batch of a few tokens
// per expert still fills the tensor core's M dimension ([SageMaker MoE kernels
// page], first item: transpose so the large expert dimension is the first operand).
// The LoRA expand runs inside the tile as extra MMA K steps: for every adapter segment
// that meets the tile, B_a^T (MN-major TMA boxes of 64 features x r rank rows) times
// the segment's z rows (written by the shrink kernel, zero outside the segment) is
// accumulated before anything is stored ([vLLM MoE-LoRA page], "Otimizações em Nível
// de Kernel": the LoRA add fused into the base output; "Implementação Técnica no
// vLLM": fused_moe_lora), so no LoRA delta round-trips through HBM.  gate_up tiles pair 64 gate rows
// with the matching 64 up rows so SiLU-and-mul is applied before act leaves the SM;
// down tiles multiply by the routing weight and store one fp32 row per routing pair
// for the fixed-order combine (expert aggregation, [SageMaker MoE kernels page],
// second item).  FP8 (e4m3) expert weights stay one byte per weight in HBM, in the TMA
// ring and in the MMA: the activations are split exactly into two e4m3 planes
// (hi = RNE(x / s), lo = RNE((x - hi s) / (s / 16)), per-row s), one kind::f8f6f4 MMA
// of N = 2 BN takes both planes (stacked token rows) into adjacent TMEM columns, so
// the weight tile is read from shared memory once per K step, and the epilogue combines
// s_w (s acc_hi + s/16 acc_lo) (per-tensor scale, [SageMaker MoE kernels page],
// second item).
//
// Structure (one CTA per SM, persistent over a device-side tile list):
//   warp 0      TMA producer: weight tile 128 x 64 bf16 (or 128 x 128 e4m3) per stage as
//               two 64-row boxes, and the token tile(s) of the same K range; then one
//               LoRA stage per (segment, 64 rank rows): B^T boxes by TMA, the z tile
//               written by the warp in the 128-byte swizzle
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16) or kind::f8f6f4 (e4m3),
//               M = 128, N = BN (rows of a ragged last chunk rounded up to 16); LoRA
//               stages kind::f16 with A MN-major (into a third accumulator for e4m3,
//               which the epilogue adds unscaled and re-zeroes); commits free the stage
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, + LoRA delta, activation,
//               stores; two TMEM accumulators so the epilogue of tile i overlaps the
//               MMAs of tile i+1
//   warp 6      epilogue loader: one tile ahead of the epilogue, the per-column data
//               (pair ids, routing weights, activation plane scales) and, for N tiles
//               <= 64, a TMA of the tile's LoRA delta into a two-slot shared-memory ring
// Every mbarrier wait is bounded; on expiry the CTA records MOE_LORA_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <mutex>

namespace mlb {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiThreads = 128;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kMaxGroups = 256;
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
  const float* delta;
  int delta_cols;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  const float* bias;
  int total_rows;
  const int32_t* sorted_pairs;
  const float* topk_w;
  const float* w_scales;
  int scale_idx;
  int* status;
  const float* b_scales;  // e4m3: [rows][2] = (s, s / 16) of the activation planes
  int m_tiles;
  int stages;
  // LoRA expand as extra K steps of the tile (bf16 weights): for every adapter segment
  // that meets the tile, acc[f][t] += sum_i B_a[i][f] z[t][i]
  const __nv_bfloat16* z;       // [total_rows][r] bf16, null = no fused expand
  int r;
  int rbox;                     // K rows per LoRA stage: min(64, r rounded up to 16)
  const int32_t* lseg_off;      // segment CSR; group g's candidates at g * lseg_stride
  int lseg_stride;
  int lseg_count;
  const int32_t* lseg_adapter;  // adapter of candidate c (null: adapter = c)
  int L;
  // stream-K (few tiles): CTA b takes the (tile, K stage) iterations
  // [b T / G, (b + 1) T / G) of T = tiles * stages; a CTA that starts inside a tile writes
  // its partial accumulator to sk_part[b] and raises sk_flag[b]; the CTA holding the
  // tile's first stages adds the partials in CTA order and runs the epilogue
  int sk;
  float* sk_part;               // [grid][128][BN] fp32
  int* sk_flag;                 // [grid], zero on entry, zero again on exit
  // item tiles (LoRA shrink on the tensor cores): tile t = items[t] = (segment key q,
  // first row); A rows = slot (a E + e) * r of LoRA A, N = the segment's rows there
  const int2* items;
  const int* item_count;
  int iE;
  int m_tiles2;                 // CTA pairs: pairs of 128-row tiles
};

// A unit of work: tile t, K stages [k0, k1).
struct Unit {
  int t, k0, k1;
};
struct UnitIter {
  long long pos, end;
  int t;
};

__device__ __forceinline__ long long sk_start(long long b, long long T, long long G) { return b * T / G; }
// CTA whose stream-K range holds iteration i
__device__ __forceinline__ int sk_owner(long long i, long long T, long long G) {
  return static_cast<int>(((i + 1) * G + T - 1) / T - 1);
}

// CTA bb's stream-K range is non-empty (it holds at least one iteration)
__device__ __forceinline__ bool sk_busy(long long bb, long long T, long long G) {
  return sk_start(bb, T, G) < sk_start(bb + 1, T, G);
}

// CTA pairs: unit index space is per cluster (two CTAs walk the same units)
__device__ __forceinline__ int unit_cta(const TcParams& p) { return p.m_tiles2 ? blockIdx.x >> 1 : blockIdx.x; }
__device__ __forceinline__ int unit_ctas(const TcParams& p) { return p.m_tiles2 ? gridDim.x >> 1 : gridDim.x; }

__device__ __forceinline__ UnitIter unit_begin(const TcParams& p, int total_tiles, int nk) {
  UnitIter it;
  it.t = unit_cta(p);
  const long long T = static_cast<long long>(total_tiles) * nk;
  it.pos = sk_start(blockIdx.x, T, gridDim.x);
  it.end = sk_start(blockIdx.x + 1, T, gridDim.x);
  return it;
}

__device__ __forceinline__ bool unit_next(const TcParams& p, int total_tiles, int nk, UnitIter& it, Unit& u) {
  if (!p.sk) {
    if (it.t >= total_tiles) return false;
    u.t = it.t;
    u.k0 = 0;
    u.k1 = nk;
    it.t += unit_ctas(p);
    return true;
  }
  if (it.pos >= it.end) return false;
  u.t = static_cast<int>(it.pos / nk);
  u.k0 = static_cast<int>(it.pos - static_cast<long long>(u.t) * nk);
  u.k1 = static_cast<int>(min(static_cast<long long>(nk), u.k0 + (it.end - it.pos)));
  it.pos += u.k1 - u.k0;
  return true;
}

// Non-pipeline shared memory, placed after the stage rings.
struct SmemCore {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t sfull[2];
  uint64_t sempty[2];
  uint64_t tdone;
  uint32_t tmem_base;
  int abort_flag;
  int chunk_pref[kMaxGroups + 1];
  int grp_off[kMaxGroups + 1];
  float ebuf[kBM][33];
  // in-GEMM LoRA expand: LoRA stages of the producer's unit it (mod 16), and per ring
  // stage holding a LoRA stage its MMA's first tile column and N
  int tile_nls[16];
  int lstage_col[16];
  int lstage_n[16];
};

// Epilogue prefetch slot, filled one tile ahead by the loader warp: the tile's pair ids,
// routing weights and plane scales, and (N tiles <= 64) its LoRA delta [2 halves][BN][64].
template <int BN>
struct EpiSlot {
  float delta[BN <= 64 ? 2 * BN * 64 : 4];
  int col_pair[BN];
  float col_w[BN];
  float col_sh[BN];
  float col_sl[BN];
};

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

// TWO: the CTA pair (cta_group::2) computes 256 weight rows x BN tokens; each CTA holds
// its 128 weight rows and half of the BN token rows.
template <int BN, bool W8, bool TWO = false>
struct TileCfg {
  static constexpr int kKB = W8 ? 128 : 64;                  // K per stage (128 bytes per row)
  static constexpr int kBRows = TWO ? BN / 2 : BN;           // token rows held by this CTA
  static constexpr int kBTileBytes = kBRows * 128;           // one token tile (or plane)
  static constexpr int kStageBytes = kATileBytes + (W8 ? 2 : 1) * kBTileBytes;
  static constexpr int kAccStride = BN < 32 ? 32 : BN;       // TMEM columns per accumulator
  static constexpr int kAccPerBuf = W8 ? 3 : 1;              // e4m3: hi, lo and LoRA accumulators
  static constexpr int kTmemCols = pow2_at_least(2 * kAccPerBuf * kAccStride);
  static constexpr bool kPrefetch = BN <= 64;                // LoRA delta prefetched into the slots
  static constexpr int kSlotBytes = static_cast<int>((sizeof(EpiSlot<BN>) + 1023) / 1024 * 1024);
  static constexpr int kThreads = 224;
  static_assert(!W8 || kPrefetch, "e4m3 weights use N tiles <= 64");
  static_assert(!TWO || (!W8 && BN >= 128), "CTA pairs: bf16 weights, N tiles of 128 or 256");
};

struct TileInfo {
  int g, mt, row0, nvalid;
};

__device__ __forceinline__ TileInfo decode_tile(const SmemCore& sm, int t, int m_tiles, int E, int BN) {
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

// Tile of the LoRA shrink: g = the (adapter, expert) slot, rows from the work item.
__device__ __forceinline__ TileInfo item_tile(const TcParams& p, int t, int BN) {
  TileInfo ti;
  const int2 it = p.items[t];
  if (p.lseg_adapter != nullptr) {  // dense segments: one group, adapter per segment
    ti.g = p.lseg_adapter[it.x];
  } else {                          // MoE keys q = e (L + 1) + a
    const int LA = p.L + 1;
    const int e = it.x / LA, a = it.x - e * LA;
    ti.g = a * p.iE + e;
  }
  ti.mt = 0;
  ti.row0 = it.y;
  ti.nvalid = max(0, min(BN, p.lseg_off[it.x + 1] - it.y));
  return ti;
}

// delta column (weight row within the group) of accumulator row m in tile column block f0
__device__ __forceinline__ int delta_col(int epi, int m, int f0, int I) {
  if (epi == EPI_GATEUP) return (m < 64) ? f0 + m : I + f0 + (m - 64);
  return f0 + m;
}

// Adapter segments meeting a tile's rows [row0, row0 + nvalid): the segments of group g
// are candidates c in [0, lseg_count) with ascending row ranges
// [off[c], off[c + 1]), off = lseg_off + g * lseg_stride.  The producer and the MMA
// issuer walk the same sequence, so they agree on the stages of every tile.
struct LoraSeg {
  int c;        // next candidate
  int end;      // tile end row
  int lo, hi;   // rows of the current segment inside the tile
  int slot;     // (adapter, group) slice of B: row block slot * r
  int c_start;  // first tile column of the MMA (multiple of 32)
  int n;        // MMA N (multiple of 16)
};

__device__ __forceinline__ void lora_seg_begin(const TcParams& p, const TileInfo& ti, LoraSeg& s) {
  const int32_t* off = p.lseg_off + static_cast<size_t>(ti.g) * p.lseg_stride;
  int lo = 0, hi = p.lseg_count;  // smallest c with off[c + 1] > row0
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (off[mid + 1] > ti.row0) hi = mid;
    else lo = mid + 1;
  }
  s.c = lo;
  s.end = ti.row0 + ti.nvalid;
}

// MMA columns of a segment [lo, hi) inside the tile: from the 32-aligned column at or
// below lo, N rounded up to 16 (CTA pairs: 32, N / 2 rows per CTA)
__device__ __forceinline__ void seg_cols(const TcParams& p, const TileInfo& ti, LoraSeg& s) {
  s.c_start = ((s.lo - ti.row0) >> 5) << 5;
  const int na = p.m_tiles2 ? 31 : 15;
  s.n = (s.hi - ti.row0 - s.c_start + na) & ~na;
}

// Advances to the next segment with an adapter; false when the tile has no more.
__device__ __forceinline__ bool lora_seg_next(const TcParams& p, const TileInfo& ti, LoraSeg& s) {
  const int32_t* off = p.lseg_off + static_cast<size_t>(ti.g) * p.lseg_stride;
  while (s.c < p.lseg_count) {
    const int c = s.c++;
    const int a0 = off[c], a1 = off[c + 1];
    if (a0 >= s.end) return false;
    const int lo = max(a0, ti.row0), hi = min(a1, s.end);
    if (hi <= lo) continue;
    const int ad = p.lseg_adapter ? p.lseg_adapter[c] : c;
    if (ad < 0 || ad >= p.L) continue;
    s.lo = lo;
    s.hi = hi;
    s.slot = ad * p.E + ti.g;
    seg_cols(p, ti, s);
    return true;
  }
  return false;
}

// Warp-parallel view of the segments that meet a tile: lane l loads candidate
// base + 32 h + l (h < 2) in one round of independent loads, and a ballot marks the
// candidates that meet the tile with an adapter.  Candidates past base + 64 (only with
// very many segments per group) are walked one at a time from global memory.
struct SegScan {
  uint32_t mask0, mask1;
  int lo0, hi0, slot0, lo1, hi1, slot1;  // this lane's candidate of chunk 0 / chunk 1
  int rest;                             // first candidate after the chunks that may meet the tile, or -1
};

__device__ __forceinline__ void seg_scan(const TcParams& p, const TileInfo& ti, int lane, SegScan& sc) {
  const int32_t* off = p.lseg_off + static_cast<size_t>(ti.g) * p.lseg_stride;
  const int end = ti.row0 + ti.nvalid;
  int base = 0;
  if (p.lseg_count > 64) {  // smallest c with off[c + 1] > row0
    int lo = 0, hi = p.lseg_count;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (off[mid + 1] > ti.row0) hi = mid;
      else lo = mid + 1;
    }
    base = lo;
  }
  int lo[2], hi[2], slot[2];
  bool v[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = base + 32 * h + lane;
    v[h] = false;
    lo[h] = hi[h] = slot[h] = 0;
    if (c < p.lseg_count) {
      const int a0 = off[c], a1 = off[c + 1];
      const int ad = p.lseg_adapter ? p.lseg_adapter[c] : c;
      lo[h] = max(a0, ti.row0);
      hi[h] = min(a1, end);
      v[h] = hi[h] > lo[h] && ad >= 0 && ad < p.L;
      slot[h] = ad * p.E + ti.g;
    }
  }
  sc.mask0 = __ballot_sync(0xffffffffu, v[0]);
  sc.mask1 = __ballot_sync(0xffffffffu, v[1]);
  sc.lo0 = lo[0], sc.hi0 = hi[0], sc.slot0 = slot[0];
  sc.lo1 = lo[1], sc.hi1 = hi[1], sc.slot1 = slot[1];
  const int nx = base + 64;
  sc.rest = (nx < p.lseg_count && off[nx] < end) ? nx : -1;
}

struct SegIter {
  int h;
  uint32_t m;
  bool in_rest;
  LoraSeg ls;
};

__device__ __forceinline__ SegIter seg_iter_begin(const SegScan& sc) {
  SegIter it;
  it.h = 0;
  it.m = sc.mask0;
  it.in_rest = false;
  return it;
}

// Next segment of the tile (warp-uniform: every lane of the warp calls it together).
__device__ __forceinline__ bool seg_iter_next(const TcParams& p, const TileInfo& ti, const SegScan& sc, SegIter& it,
                                              LoraSeg& out) {
  while (it.h < 2) {
    if (it.m == 0) {
      if (++it.h == 1) it.m = sc.mask1;
      continue;
    }
    const int b = __ffs(it.m) - 1;
    it.m &= it.m - 1;
    const bool h1 = it.h == 1;
    out.lo = __shfl_sync(0xffffffffu, h1 ? sc.lo1 : sc.lo0, b);
    out.hi = __shfl_sync(0xffffffffu, h1 ? sc.hi1 : sc.hi0, b);
    out.slot = __shfl_sync(0xffffffffu, h1 ? sc.slot1 : sc.slot0, b);
    seg_cols(p, ti, out);
    return true;
  }
  if (sc.rest < 0) return false;
  if (!it.in_rest) {
    it.in_rest = true;
    it.ls.c = sc.rest;
    it.ls.end = ti.row0 + ti.nvalid;
  }
  if (!lora_seg_next(p, ti, it.ls)) return false;
  out = it.ls;
  return true;
}

// LZ: the in-GEMM LoRA expand is compiled in (launches with z); without it the kernel
// carries none of that code.
template <int BN, bool W8, bool TWO, bool LZ>
__global__ void __launch_bounds__(TileCfg<BN, W8, TWO>::kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmb,
                   const __grid_constant__ CUtensorMap tml, const __grid_constant__ CUtensorMap tmd,
                   const __grid_constant__ CUtensorMap tmlb, const TcParams p) {
  // tml: the lo activation plane (e4m3 weights); tmlb: LoRA B viewed as [L * E * r][NB]
  const bool lz = LZ && p.z != nullptr;
  // (MN-major boxes of 64 features x rbox rank rows)
  using Cfg = TileCfg<BN, W8, TWO>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;                                 // stages: [A tile][token tile(s)]
  uint8_t* slots = ring + p.stages * Cfg::kStageBytes;  // epilogue prefetch slots
  SmemCore& sm = *reinterpret_cast<SmemCore*>(slots + 2 * Cfg::kSlotBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;
  volatile int* abort_flag = &sm.abort_flag;
  // CTA pairs: rank 0 (leader) issues the MMAs for both; the barriers the MMA consumes
  // live in the leader's shared memory
  const uint32_t rank = TWO ? cluster_ctarank() : 0;
  auto leader_bar = [&](uint64_t* bar) -> uint32_t { return TWO ? mapa_shared(smem_u32(bar), 0) : smem_u32(bar); };

  // ---- setup: barriers, TMEM, tile list prefix
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sm.full[s], TWO ? 2 : 1);  // pair: the leader's and the peer's producer
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], TWO ? 2 * kEpiThreads : kEpiThreads);
      mbar_init(&sm.sfull[b], 1);
      mbar_init(&sm.sempty[b], kEpiThreads);
    }
    mbar_init(&sm.tdone, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmw);
    tma_prefetch_desc(&tmb);
    if (W8) tma_prefetch_desc(&tml);
    if (lz) tma_prefetch_desc(&tmlb);
    if (p.delta != nullptr) tma_prefetch_desc(&tmd);
  }
  if (warp == 1) {
    if constexpr (TWO) tmem_alloc_pair(&sm.tmem_base, Cfg::kTmemCols);
    else tmem_alloc(&sm.tmem_base, Cfg::kTmemCols);
  }
  for (int g = threadIdx.x; g <= p.E; g += blockDim.x)
    sm.grp_off[g] = p.group_offsets ? p.group_offsets[static_cast<size_t>(g) * p.group_stride]
                                    : (g == 0 ? 0 : p.total_rows);
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
  if constexpr (TWO) cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  if constexpr (W8) {
    // the LoRA accumulators start at zero; the epilogue re-zeroes one after reading it
    if (lz && warp >= 2 && warp < 6) {
      for (int b = 0; b < 2; ++b)
        for (int c = 0; c < Cfg::kAccStride; c += 32)
          tmem_zero_32x32b_x32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) +
                               (b * Cfg::kAccPerBuf + 2) * Cfg::kAccStride + c);
      tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
  }
  const int total_tiles =
      p.items ? *p.item_count : sm.chunk_pref[p.E] * (TWO ? p.m_tiles2 : p.m_tiles);
  // this CTA's tile of a unit (pairs: the unit is a pair of 128-row tiles, rank picks one)
  auto tile_of = [&](int t) -> TileInfo {
    if (p.items) return item_tile(p, t, BN);
    TileInfo ti = decode_tile(sm, t, TWO ? p.m_tiles2 : p.m_tiles, p.E, BN);
    if constexpr (TWO) ti.mt = 2 * ti.mt + static_cast<int>(rank);
    return ti;
  };
  const int nk = (p.K + Cfg::kKB - 1) / Cfg::kKB;  // stages per tile

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 issues the TMA copies.  The whole warp fills the z tiles of LoRA stages
    // with cp.async (zero-fill outside the segment) whose completion is tracked by the
    // stage's full barrier (cp.async.mbarrier.arrive), so the producer never waits for
    // them; the MMA thread issues a proxy fence before it reads such a stage.  CTA pairs
    // signal the leader's barrier, which cp.async cannot: there the stage is completed
    // (copies waited for, fence, remote arrive) when the producer would otherwise block.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t filled_mask = 0, last_parity = 0;
    uint32_t pend_mask = 0;  // LoRA stages whose z copies are issued but not yet arrived
    bool ok = true;
    auto flush_lora = [&]() {
      if (pend_mask != 0) {
        cp_async_wait_all();
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA
        __syncwarp();
        if (lane == 0)
          for (int s2 = 0; s2 < S; ++s2)
            if (pend_mask & (1u << s2)) {
              if constexpr (TWO) mbar_arrive_cluster(leader_bar(&sm.full[s2]));
              else mbar_arrive(&sm.full[s2]);
            }
        pend_mask = 0;
      }
    };
    // warp-uniform wait for a free ring slot
    auto acquire = [&](int where) -> bool {
      bool got = true;
      if (lane == 0) got = mbar_try_wait(&sm.empty[stage], phase ^ 1u);
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        flush_lora();
        if (lane == 0) got = mbar_wait(&sm.empty[stage], phase ^ 1u, abort_flag, p.status, kWaitLimitNs, where);
        got = __shfl_sync(0xffffffffu, got, 0);
      }
      return got;
    };
    UnitIter uit = unit_begin(p, total_tiles, nk);
    Unit u;
    int itp = 0;  // unit index, the same sequence as the MMA thread's
    while (ok && unit_next(p, total_tiles, nk, uit, u)) {
      if (__shfl_sync(0xffffffffu, *abort_flag != 0, 0)) break;  // warp-uniform
      const TileInfo ti = tile_of(u.t);
      int wrow0, wrow1;
      if (p.epi == EPI_GATEUP) {
        wrow0 = ti.g * p.rows_per_group + ti.mt * 64;
        wrow1 = ti.g * p.rows_per_group + p.I + ti.mt * 64;
      } else if (p.epi == EPI_ZOUT) {
        wrow0 = ti.g * p.r;  // the slot's A rows
        wrow1 = wrow0 + 64;
      } else {
        wrow0 = ti.g * p.rows_per_group + ti.mt * kBM;
        wrow1 = wrow0 + 64;
      }
      // r <= 64: the second 64-row half of A is not needed (accumulator rows >= r are
      // never read), so it is not loaded
      const bool a_half = p.epi == EPI_ZOUT && p.r <= 64;
      const bool lora = lz;
      const int nb = u.k1 - u.k0;  // base stages of the unit
      // LoRA stages (in-GEMM expand), after the unit's base stages: A = B_a^T (MN-major:
      // 64 gate/low + 64 up/high features x rbox rank rows), B = the segment's z rows in
      // tile columns [c_start, c_start + n), zero outside the segment.  Their count goes
      // to shared memory before the last base stage's arrival and each one's MMA columns
      // before its own, for the MMA thread.  (Spreading them between the base stages
      // measured slower: mixed MMA kinds slowed the tensor pipe more than the earlier
      // loads saved.)
      const int lf0 = (p.epi == EPI_GATEUP) ? ti.mt * 64 : ti.mt * kBM;
      const int lcol1 = (p.epi == EPI_GATEUP) ? p.I + lf0 : lf0 + 64;
      const int kch = p.rbox / 8;  // 16-byte chunks of a z row per stage
      const int per = lora ? (p.r + 63) / 64 : 0;
      SegScan sc;
      int nls = 0;
      for (int i = 0; i < nb; ++i) {
        // the segment scan waits for global loads: midway, while the ring is full
        if (lora && i == nb / 2) {
          seg_scan(p, ti, lane, sc);
          nls = (__popc(sc.mask0) + __popc(sc.mask1)) * per;
          if (sc.rest >= 0) {  // very many segments: count the rest one by one
            LoraSeg rs;
            rs.c = sc.rest;
            rs.end = ti.row0 + ti.nvalid;
            while (lora_seg_next(p, ti, rs)) nls += per;
          }
          if (lane == 0) sm.tile_nls[itp & 15] = nls;
        }
        const int kb = u.k0 + i;
        ok = acquire(1);
        if (!ok) break;
        if (lane == 0) {
          uint8_t* a_s = ring + stage * Cfg::kStageBytes;
          uint8_t* b_s = a_s + kATileBytes;
          const int kc = kb * Cfg::kKB;  // first K element of the stage
          if constexpr (TWO) {
            // both CTAs' copies complete on the leader's barrier: the leader expects the
            // pair's bytes, the peer adds its arrival
            const uint32_t fb = leader_bar(&sm.full[stage]);
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[stage], 2 * Cfg::kStageBytes);
            tma_load_2d_pair(a_s, &tmw, fb, kc, wrow0);
            tma_load_2d_pair(a_s + kATileBytes / 2, &tmw, fb, kc, wrow1);
            // MMA N = the tile's rows rounded to 32; the peer holds columns [N/2, N)
            const int n_pair = min(BN, (ti.nvalid + 31) & ~31);
            tma_load_2d_pair(b_s, &tmb, fb, kc, ti.row0 + static_cast<int>(rank) * (n_pair / 2));
            if (rank != 0) mbar_arrive_cluster(fb);
          } else {
            mbar_arrive_expect_tx(&sm.full[stage], Cfg::kStageBytes - (a_half ? kATileBytes / 2 : 0));
            tma_load_2d(a_s, &tmw, &sm.full[stage], kc, wrow0);
            if (!a_half) tma_load_2d(a_s + kATileBytes / 2, &tmw, &sm.full[stage], kc, wrow1);
            tma_load_2d(b_s, &tmb, &sm.full[stage], kc, ti.row0);
            if constexpr (W8) tma_load_2d(b_s + Cfg::kBTileBytes, &tml, &sm.full[stage], kc, ti.row0);
          }
          filled_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok && nls > 0) {
        SegIter si = seg_iter_begin(sc);
        LoraSeg ls;
        while (ok && seg_iter_next(p, ti, sc, si, ls)) {  // warp-uniform
          for (int kh = 0; kh < per; ++kh) {
            ok = acquire(9);
            if (!ok) break;
            uint8_t* a_s = ring + stage * Cfg::kStageBytes;
            uint8_t* b_s = a_s + kATileBytes;
            if (lane == 0) {
              sm.lstage_col[stage] = ls.c_start;
              sm.lstage_n[stage] = ls.n;
              const int krow = ls.slot * p.r + kh * 64;
              if constexpr (TWO) {
                const uint32_t fb = leader_bar(&sm.full[stage]);
                if (rank == 0) mbar_expect_tx(&sm.full[stage], 2 * 2 * p.rbox * 128);
                tma_load_2d_pair(a_s, &tmlb, fb, lf0, krow);
                tma_load_2d_pair(a_s + p.rbox * 128, &tmlb, fb, lcol1, krow);
              } else {
                mbar_expect_tx(&sm.full[stage], 2 * p.rbox * 128);
                tma_load_2d(a_s, &tmlb, &sm.full[stage], lf0, krow);
                tma_load_2d(a_s + p.rbox * 128, &tmlb, &sm.full[stage], lcol1, krow);
              }
              filled_mask |= 1u << stage;
              last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            }
            // pairs: this CTA holds rows [rank n / 2, (rank + 1) n / 2) of the unit's n columns
            const int n_h = TWO ? ls.n / 2 : ls.n;
            const int col_base = ls.c_start + static_cast<int>(rank) * n_h;
            for (int idx = lane; idx < n_h * kch; idx += 32) {
              const int j = idx / kch, c = idx - j * kch;
              const int row = ti.row0 + col_base + j;
              const int el = kh * 64 + c * 8;
              const bool valid = row >= ls.lo && row < ls.hi && el < p.r;
              const __nv_bfloat16* src = valid ? p.z + static_cast<size_t>(row) * p.r + el : p.z;
              cp_async_16_zfill(b_s + j * 128 + ((c ^ (j & 7)) << 4), src, valid);  // 128-byte swizzle
            }
            if constexpr (TWO) {
              pend_mask |= 1u << stage;
            } else {
              cp_async_mbar_arrive(&sm.full[stage]);     // each lane: +1 now, -1 when its copies land
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.full[stage]);  // the stage's counted arrival
            }
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      ++itp;
    }
    flush_lora();  // every issued stage gets its arrival, also on the abort path
    cp_async_wait_all();  // no copy into this CTA's shared memory outlives the producer
    if (lane == 0 && *abort_flag && rank == 0) {  // pairs: the leader's barriers count both CTAs' copies
      // let our own copies land before the CTA exits
      for (int s = 0; s < S; ++s)
        if (filled_mask & (1u << s)) {
          volatile int dummy = 0;
          mbar_wait(&sm.full[s], (last_parity >> s) & 1u, &dummy, nullptr, kWaitLimitNs / 4, 0);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // pairs: the leader issues the MMAs of both CTAs (M = 256: its 128 rows and the
    // peer's), commits reach both CTAs' barriers; the peer waits for the last commit
    if (lane == 0 && TWO && rank != 0) {
      volatile int dummy = 0;
      mbar_wait(&sm.tdone, 0, &dummy, nullptr, kWaitLimitNs, 0);
    } else if (lane == 0) {
      constexpr int kMM = TWO ? 2 * kBM : kBM;  // MMA M
      auto commit = [&](uint64_t* bar) {
        if constexpr (TWO) umma_commit_pair(bar, 3);
        else umma_commit(bar);
      };
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      UnitIter uit = unit_begin(p, total_tiles, nk);
      Unit u;
      for (; !*abort_flag && unit_next(p, total_tiles, nk, uit, u); ++it) {
        // the last chunk of a group is ragged: N = its rows rounded up to 16, so a
        // skewed expert load does not pay MMAs on padding rows
        const TileInfo ti = tile_of(u.t);
        // e4m3: the hi and lo planes sit back to back in the ring, so one instruction of
        // N = 2 BN covers both and each weight tile is read from shared memory once
        const int n_mma = TWO ? min(BN, (ti.nvalid + 31) & ~31) : min(BN, (ti.nvalid + 15) & ~15);
        const uint32_t idesc = W8 ? umma_idesc_e4m3(kBM, 2 * BN) : umma_idesc_bf16(kMM, n_mma);
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait(&sm.tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, kWaitLimitNs, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * Cfg::kAccPerBuf * Cfg::kAccStride;
        bool ok = true;
        for (int kb = u.k0; kb < u.k1; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status, kWaitLimitNs, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(ring + stage * Cfg::kStageBytes);
          const uint64_t adesc = umma_desc_sw128(a_addr);
          const uint64_t bdesc = umma_desc_sw128(a_addr + kATileBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
            const uint32_t acc = (kb != u.k0 || k != 0) ? 1u : 0u;
            if constexpr (W8) {
              umma_e4m3(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);  // columns [0, BN) hi, [BN, 2 BN) lo
            } else if constexpr (TWO) {
              umma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
            } else {
              umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
            }
          }
          commit(&sm.empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok && lz) {
          // e4m3 weights: LoRA goes to its own accumulator (no weight or plane scale).
          // The count and each stage's columns come from the producer's shared-memory
          // records, so no segment table is read on this thread's critical path.
          const uint32_t d_lora = d_tmem + (W8 ? 2 * Cfg::kAccStride : 0);
          const int nls = static_cast<volatile int*>(sm.tile_nls)[it & 15];
          for (int j = 0; j < nls; ++j) {
            if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status, kWaitLimitNs, 10)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if constexpr (!TWO) fence_proxy_async_smem();  // z written by cp.async (generic proxy)
            const int c_start = static_cast<volatile int*>(sm.lstage_col)[stage];
            const int n_l = static_cast<volatile int*>(sm.lstage_n)[stage];
            const uint32_t lidesc = umma_idesc_bf16_amn(kMM, n_l);
            const uint32_t a_addr = smem_u32(ring + stage * Cfg::kStageBytes);
            const uint64_t adesc = umma_desc_mn_sw128(a_addr, p.rbox * 128);
            const uint64_t bdesc = umma_desc_sw128(a_addr + kATileBytes);
            for (int kk = 0; kk < p.rbox / 16; ++kk) {  // 16 rank rows (2048 B of A) per instruction
              if constexpr (TWO) umma_bf16_pair(d_lora + c_start, adesc + 128 * kk, bdesc + 2 * kk, lidesc, 1u);
              else umma_bf16(d_lora + c_start, adesc + 128 * kk, bdesc + 2 * kk, lidesc, 1u);
            }
            commit(&sm.empty[stage]);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        commit(&sm.tfull[buf]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      commit(&sm.tdone);
      volatile int dummy = 0;
      mbar_wait(&sm.tdone, 0, &dummy, nullptr, kWaitLimitNs, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;   // 0..127
    const int g4 = warp & 3;           // TMEM lane quarter this warp may access
    const int m = g4 * 32 + lane;      // accumulator row = weight row within the tile
    int it = 0;
    UnitIter uit = unit_begin(p, total_tiles, nk);
    Unit u;
    const long long skT = static_cast<long long>(total_tiles) * nk;
    for (; unit_next(p, total_tiles, nk, uit, u); ++it) {
      const TileInfo ti = tile_of(u.t);
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      bool got = mbar_wait(&sm.tfull[buf], use & 1u, abort_flag, p.status, kWaitLimitNs, 4);
      got = got && mbar_wait(&sm.sfull[buf], use & 1u, abort_flag, p.status, kWaitLimitNs, 7);
      // stream-K roles: a later part stores its partial; the first part of a split tile
      // waits (bounded) for the later parts' flags, then adds their partials in CTA order
      const bool sk_store = p.sk && u.k0 != 0;
      int sk_b1 = 0, sk_b2 = -1;  // CTAs holding the later parts of this tile
      if (p.sk && u.k0 == 0 && u.k1 != nk) {
        sk_b1 = static_cast<int>(blockIdx.x) + 1;
        sk_b2 = sk_owner(static_cast<long long>(u.t) * nk + nk - 1, skT, gridDim.x);
        if (got && et == 0) {
          const uint64_t t0 = globaltimer_ns();
          for (int bb = sk_b1; bb <= sk_b2 && got; ++bb) {
            if (!sk_busy(bb, skT, gridDim.x)) continue;  // empty range: holds no part
            while (ld_acquire_gpu(p.sk_flag + bb) == 0) {
              if (*abort_flag) {
                got = false;
                break;
              }
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                set_status(p.status, MOE_LORA_ERR_TIMEOUT, 11);
                got = false;
                break;
              }
            }
          }
        }
      }
      if (!named_bar_and(2, kEpiThreads, got)) break;  // the four warps leave together
      tc_fence_after();

      const int f0 = (p.epi == EPI_GATEUP) ? ti.mt * 64 : ti.mt * kBM;
      int feat;
      bool row_ok;
      if (p.epi == EPI_GATEUP) {
        feat = f0 + (m & 63);
        row_ok = feat < p.I;
      } else {
        feat = f0 + m;
        row_ok = feat < p.n_out;
      }
      const int dcol = delta_col(p.epi, m, f0, p.I);
      float scale = 1.f;
      if (p.w_scales != nullptr) scale = p.w_scales[ti.g * 2 + p.scale_idx];
      const EpiSlot<BN>* slot = reinterpret_cast<const EpiSlot<BN>*>(slots + buf * Cfg::kSlotBytes);

      for (int c0 = 0; c0 < ti.nvalid; c0 += 32) {
        named_bar_sync(1, kEpiThreads);  // the previous chunk is done with smem
        const int ncol = min(32, ti.nvalid - c0);
        float v[32];
        const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(g4 * 32) << 16) +
                               buf * Cfg::kAccPerBuf * Cfg::kAccStride + c0;
        tmem_ld_32x32b_x32(t_acc, v);
        if constexpr (W8) {
          float vl[32];
          tmem_ld_32x32b_x32(t_acc + BN, vl);
#pragma unroll
          for (int n = 0; n < 32; ++n)
            if (c0 + n < BN) v[n] = scale * (v[n] * slot->col_sh[c0 + n] + vl[n] * slot->col_sl[c0 + n]);
          if (lz) {
            tmem_ld_32x32b_x32(t_acc + 2 * Cfg::kAccStride, vl);
#pragma unroll
            for (int n = 0; n < 32; ++n) v[n] += vl[n];
          }
        } else {
#pragma unroll
          for (int n = 0; n < 32; ++n) v[n] *= scale;
        }
        if (sk_store) {  // later part of a split tile: keep the partial, nothing else
          float4* dst = reinterpret_cast<float4*>(p.sk_part + (static_cast<size_t>(blockIdx.x) * kBM + m) * BN + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (c0 + 4 * q < BN) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          continue;
        }
        for (int bb = sk_b1; bb <= sk_b2; ++bb) {  // first part: add the later parts in order
          if (!sk_busy(bb, skT, gridDim.x)) continue;
          const float4* src = reinterpret_cast<const float4*>(p.sk_part + (static_cast<size_t>(bb) * kBM + m) * BN + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (c0 + 4 * q < BN) {
              const float4 w4 = __ldcg(src + q);
              v[4 * q] += w4.x;
              v[4 * q + 1] += w4.y;
              v[4 * q + 2] += w4.z;
              v[4 * q + 3] += w4.w;
            }
        }
        if (p.delta != nullptr) {
          if constexpr (Cfg::kPrefetch) {
            const float* dl = slot->delta + ((m >> 6) * BN + c0) * 64 + (m & 63);
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (c0 + n < BN) v[n] += dl[n * 64];
          } else if (dcol < p.delta_cols) {
            const float* dg = p.delta + static_cast<size_t>(ti.row0 + c0) * p.delta_cols + dcol;
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol) v[n] += dg[static_cast<size_t>(n) * p.delta_cols];
          }
        }

        if (p.epi == EPI_GATEUP) {
#pragma unroll
          for (int n = 0; n < 32; ++n) sm.ebuf[m][n] = v[n];
          named_bar_sync(1, kEpiThreads);
          const int n = et >> 2;
          const int fq = (et & 3) * 16;
          if (n < ncol) {
            __nv_bfloat16* dst = p.out_bf16 + static_cast<size_t>(ti.row0 + c0 + n) * p.I + f0 + fq;
            const int fbase = f0 + fq;
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
            const int* cp = slot->col_pair + c0;
            const float* cw = slot->col_w + c0;
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol) p.out_f32[static_cast<size_t>(cp[n]) * p.n_out + feat] = v[n] * cw[n];
          }
        } else if (p.epi == EPI_ZOUT) {
          if (m < p.r) {
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol) p.out_bf16[static_cast<size_t>(ti.row0 + c0 + n) * p.r + m] = __float2bfloat16_rn(v[n]);
          }
        } else if (p.epi == EPI_LOGITS) {
          if (row_ok) {
            const float b = p.bias ? p.bias[feat] : 0.f;
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol) p.out_f32[static_cast<size_t>(ti.row0 + c0 + n) * p.n_out + feat] = v[n] + b;
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
      if constexpr (W8) {
        if (lz)
          for (int c = 0; c < Cfg::kAccStride; c += 32)
            tmem_zero_32x32b_x32(tmem_base + (static_cast<uint32_t>(g4 * 32) << 16) +
                                 (buf * Cfg::kAccPerBuf + 2) * Cfg::kAccStride + c);
      }
      if (sk_store || sk_b2 >= sk_b1) {
        __threadfence();                 // this thread's partial row is visible GPU-wide
        named_bar_sync(1, kEpiThreads);  // every partial row stored / every partial read
        if (et == 0) {
          if (sk_store) {
            __threadfence();
            st_release_gpu(p.sk_flag + blockIdx.x, 1);
          } else {
            for (int bb = sk_b1; bb <= sk_b2; ++bb) p.sk_flag[bb] = 0;  // consumed: re-armed for the next launch
          }
        }
      }
      tc_fence_before();
      if constexpr (TWO) mbar_arrive_cluster(leader_bar(&sm.tempty[buf]));  // the leader's MMA reuses it
      else mbar_arrive(&sm.tempty[buf]);
      mbar_arrive(&sm.sempty[buf]);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ epilogue loader
    {
      uint32_t issued_mask = 0, issued_parity = 0;
      int it = 0;
      UnitIter uit = unit_begin(p, total_tiles, nk);
      Unit u;
      for (; unit_next(p, total_tiles, nk, uit, u); ++it) {
        const TileInfo ti = tile_of(u.t);
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        const bool got = mbar_wait(&sm.sempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, kWaitLimitNs, 8);
        if (!__all_sync(0xffffffffu, got)) break;
        EpiSlot<BN>* slot = reinterpret_cast<EpiSlot<BN>*>(slots + buf * Cfg::kSlotBytes);
        if constexpr (Cfg::kPrefetch) {
          if (lane == 0 && p.delta != nullptr) {
            const int f0 = (p.epi == EPI_GATEUP) ? ti.mt * 64 : ti.mt * kBM;
            const int c1 = (p.epi == EPI_GATEUP) ? p.I + f0 : f0 + 64;
            mbar_expect_tx(&sm.sfull[buf], 2 * BN * 64 * 4);
            tma_load_2d(slot->delta, &tmd, &sm.sfull[buf], f0, ti.row0);
            tma_load_2d(slot->delta + BN * 64, &tmd, &sm.sfull[buf], c1, ti.row0);
            issued_mask |= 1u << buf;
            issued_parity = (issued_parity & ~(1u << buf)) | ((use & 1u) << buf);
          }
        }
        if (p.epi == EPI_DOWN) {
          for (int n = lane; n < BN; n += 32) {
            const int pr = n < ti.nvalid ? p.sorted_pairs[ti.row0 + n] : 0;
            slot->col_pair[n] = pr;
            slot->col_w[n] = n < ti.nvalid ? p.topk_w[pr] : 0.f;
          }
        }
        if (W8) {
          for (int n = lane; n < BN; n += 32) {
            const bool v = n < ti.nvalid;
            slot->col_sh[n] = v ? p.b_scales[2 * static_cast<size_t>(ti.row0 + n)] : 0.f;
            slot->col_sl[n] = v ? p.b_scales[2 * static_cast<size_t>(ti.row0 + n) + 1] : 0.f;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sfull[buf]);
      }
      if (lane == 0 && *abort_flag) {
        for (int b = 0; b < 2; ++b)
          if (issued_mask & (1u << b)) {
            volatile int dummy = 0;
            mbar_wait(&sm.sfull[b], (issued_parity >> b) & 1u, &dummy, nullptr, kWaitLimitNs / 4, 0);
          }
      }
    }
  }

  tc_fence_before();
  if constexpr (TWO) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (TWO) tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    else tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
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

template <int BN, bool W8, bool TWO = false>
static cudaError_t launch_bn(const GemmArgs& a, cudaStream_t st) {
  using Cfg = TileCfg<BN, W8, TWO>;
  const int fixed = static_cast<int>(sizeof(SmemCore)) + 2 * Cfg::kSlotBytes;
  const int budget = 232448 - 1024 - fixed;
  int stages = budget / Cfg::kStageBytes;
  stages = stages > 8 ? 8 : stages;
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + static_cast<size_t>(stages) * Cfg::kStageBytes + fixed;
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  // the raised shared-memory limit is a per-device function attribute
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, W8, TWO, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_tc_kernel<BN, W8, TWO, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               232448);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tmw, tmb, tml, tmd, tmlb;
  const uint64_t wrows = static_cast<uint64_t>(a.E) * a.rows_per_group;
  if (W8) {
    if (encode_tmap_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w, a.K, wrows, static_cast<uint64_t>(a.K), 128, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_tmap_2d(&tmb, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_hi, a.K, a.total_rows, static_cast<uint64_t>(a.K),
                       128, BN, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_tmap_2d(&tml, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.b_lo, a.K, a.total_rows, static_cast<uint64_t>(a.K),
                       128, BN, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    if (encode_tmap_2d(&tmw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w, a.K, wrows, static_cast<uint64_t>(a.K) * 2, kBK,
                       64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_tmap_2d(&tmb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b, a.K, a.total_rows,
                       static_cast<uint64_t>(a.K) * 2, kBK, Cfg::kBRows, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tml = tmb;  // unused
  }
  if (a.z != nullptr) {  // LoRA B as [L * E * r][delta_cols], boxes 64 features x rbox rows
    const int rbox = a.r >= 64 ? 64 : (a.r + 15) / 16 * 16;
    if (encode_tmap_2d(&tmlb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_b, a.delta_cols,
                       static_cast<uint64_t>(a.L) * a.E * a.r, static_cast<uint64_t>(a.delta_cols) * 2, 64, rbox,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    tmlb = tmb;  // unused
  }
  if (a.delta != nullptr && Cfg::kPrefetch) {
    if (encode_tmap_2d(&tmd, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.delta, a.delta_cols, a.total_rows,
                       static_cast<uint64_t>(a.delta_cols) * 4, 64, BN, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    tmd = tmb;  // unused
  }
  TcParams p;
  p.epi = a.epi;
  p.K = a.K;
  p.E = a.E;
  p.group_offsets = a.group_offsets;
  p.group_stride = a.group_stride;
  p.rows_per_group = a.rows_per_group;
  p.n_out = a.n_out;
  p.I = a.I;
  p.delta = a.delta;
  p.delta_cols = a.delta_cols;
  p.out_bf16 = a.out_bf16;
  p.out_f32 = a.out_f32;
  p.bias = a.bias;
  p.total_rows = a.total_rows;
  p.sorted_pairs = a.sorted_pairs;
  p.topk_w = a.topk_w;
  p.w_scales = a.w_scales;
  p.scale_idx = a.scale_idx;
  p.status = a.status;
  p.b_scales = a.b_scales;
  p.m_tiles = (a.epi == EPI_GATEUP) ? (a.I + 63) / 64 : (a.n_out + kBM - 1) / kBM;
  p.stages = stages;
  p.z = a.z;
  p.r = a.r;
  p.rbox = a.r >= 64 ? 64 : (a.r + 15) / 16 * 16;
  p.lseg_off = a.lseg_off;
  p.lseg_stride = a.lseg_stride;
  p.lseg_count = a.lseg_count;
  p.lseg_adapter = a.lseg_adapter;
  p.L = a.L;
  p.items = a.items;
  p.item_count = a.item_count;
  p.iE = a.iE;
  p.m_tiles2 = TWO ? (p.m_tiles + 1) / 2 : 0;
  const long long chunks_ub = (a.total_rows + BN - 1) / BN + a.E;
  const long long tiles_ub = a.items ? a.items_bound : chunks_ub * (TWO ? p.m_tiles2 : p.m_tiles);
  int grid = a.num_sms;
  // stream-K when the tiles would leave SMs idle or unbalanced (< two waves)
  p.sk = 0;
  p.sk_part = a.sk_part;
  p.sk_flag = a.sk_flag;
  // Opt-in (MOE_LORA_STREAMK=1), for fewer than two tiles per SM.  Measured on the dense
  // decode GEMM (86 tiles): all SMs stream but each at half the rate, 40.6 us against
  // 36.3 us for 86 whole tiles, so whole tiles stay the default.
  const char* skv = std::getenv("MOE_LORA_STREAMK");
  const bool sk_want = skv != nullptr && std::atoi(skv) != 0 && tiles_ub < 2LL * grid;
  if (!TWO && a.sk_part != nullptr && a.sk_flag != nullptr && a.z == nullptr && BN <= 64 && sk_want &&
      grid <= a.sk_slots && static_cast<long long>(grid) * kBM * BN <= a.sk_part_cap) {
    p.sk = 1;
  } else if (TWO) {
    grid = (grid / 2 < tiles_ub ? grid / 2 : static_cast<int>(tiles_ub)) * 2;  // whole pairs
  } else {
    if (tiles_ub < grid) grid = static_cast<int>(tiles_ub);
  }
  if (grid < (TWO ? 2 : 1)) grid = TWO ? 2 : 1;
  ProfScope ps(a.epi == EPI_GATEUP ? K_GEMM_GATEUP
               : a.epi == EPI_DOWN ? K_GEMM_DOWN
               : a.epi == EPI_LOGITS ? K_ROUTE_LOGITS
               : a.epi == EPI_ZOUT ? K_LORA : K_GEMM_DENSE, st);
  if constexpr (TWO) {  // clusters of two CTAs (the MMA pair)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = a.z != nullptr
                        ? cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, W8, TWO, true>, tmw, tmb, tml, tmd, tmlb, p)
                        : cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, W8, TWO, false>, tmw, tmb, tml, tmd, tmlb, p);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  } else {
    if (a.z != nullptr) gemm_tc_kernel<BN, W8, TWO, true><<<grid, Cfg::kThreads, smem, st>>>(tmw, tmb, tml, tmd, tmlb, p);
    else gemm_tc_kernel<BN, W8, TWO, false><<<grid, Cfg::kThreads, smem, st>>>(tmw, tmb, tml, tmd, tmlb, p);
    count_launch();
    return cudaGetLastError();
  }
}

// N tiles of 128 and 256 on CTA pairs (cta_group::2), opt-in with MOE_LORA_PAIR=1.  On a
// prefill-shaped case (256 rows per expert, H = 4096) the pair kernel is correct but
// slower than one CTA per tile (gate_up 283 us against 156 us, tensor pipe active 17.5%),
// so single-CTA tiles stay the default.
static bool pairs_on() {
  const char* v = std::getenv("MOE_LORA_PAIR");
  return v != nullptr && std::atoi(v) != 0;
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxGroups) return cudaErrorInvalidValue;
  if (a.delta != nullptr && a.delta_cols % 8 != 0) return cudaErrorInvalidValue;
  if (a.epi == EPI_ZOUT && (a.items == nullptr || a.item_count == nullptr || a.lseg_off == nullptr || a.w_fp8 ||
                            a.r <= 0 || a.r > 128 || a.z != nullptr || a.delta != nullptr))
    return cudaErrorInvalidValue;
  if (a.z != nullptr) {
    if (a.delta != nullptr || a.lora_b == nullptr || a.lseg_off == nullptr || a.r <= 0 ||
        a.r > 128 || a.r % 8 != 0 || a.delta_cols % 8 != 0 || a.L <= 0)
      return cudaErrorInvalidValue;
  }
  if (a.w_fp8) {
    if (a.b_hi == nullptr || a.b_lo == nullptr || a.b_scales == nullptr) return cudaErrorInvalidValue;
    switch (a.bn) {
      case 16: return launch_bn<16, true>(a, st);
      case 32: return launch_bn<32, true>(a, st);
      default: return launch_bn<64, true>(a, st);
    }
  }
  switch (a.bn) {
    case 16: return launch_bn<16, false>(a, st);
    case 32: return launch_bn<32, false>(a, st);
    case 64: return launch_bn<64, false>(a, st);
    case 128: return pairs_on() ? launch_bn<128, false, true>(a, st) : launch_bn<128, false>(a, st);
    case 256: return pairs_on() ? launch_bn<256, false, true>(a, st) : launch_bn<256, false>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mlb
