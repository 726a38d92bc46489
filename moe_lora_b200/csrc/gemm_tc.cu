// Tensor-core grouped GEMM for the expert (or dense) projections, sm_100a.
//
// Operand swap: the MMA's 128-row M slot takes 128 weight rows (output features)
// and its N slot the tokens of one expert, so that a decode batch of a few tokens
// per expert still fills the tensor core's M dimension ([SageMaker MoE kernels
// page], first item: transpose so the large expert dimension is the first operand).
// The LoRA delta of each row (from the segmented LoRA kernels) is added by the
// epilogue before anything is stored ([vLLM MoE-LoRA page], "Otimizações em Nível de
// Kernel": the LoRA add fused into the base output): an fp32 delta prefetched by TMA
// into shared memory (decode tiles), or a bf16 delta read row by row (prefill tiles).
// gate_up tiles pair 64 gate rows with the matching 64 up rows so SiLU-and-mul is
// applied before act leaves the SM; down tiles multiply by the routing weight and store
// one bf16 row per routing pair for the fixed-order combine (expert aggregation,
// [SageMaker MoE kernels page], second item).  FP8 (e4m3) expert weights stay one byte
// per weight in HBM, in the TMA ring and in the MMA: the activations are split exactly
// into two e4m3 planes (hi = RNE(x / s), lo = RNE((x - hi s) / (s / 16)), per-row s),
// one kind::f8f6f4 MMA of N = 2 BN takes both planes (stacked token rows) into adjacent
// TMEM columns, so the weight tile is read from shared memory once per K step, and the
// epilogue combines s_w (s acc_hi + s/16 acc_lo) (per-tensor scale, [SageMaker MoE
// kernels page], second item).
//
// Structure (one CTA per SM, persistent over a device-side tile list):
//   warp 0      TMA producer: weight tile 128 x 64 bf16 (or 128 x 128 e4m3) per K block as
//               two 64-row boxes, and the token tile(s) of the same K range; two K blocks
//               per stage for decode-sized tiles (256-byte runs of every weight row)
//   warp 1      MMA issuer: tcgen05.mma kind::f16 (bf16) or kind::f8f6f4 (e4m3),
//               M = 128, N = BN (rows of a ragged last chunk rounded up to 16); commits
//               free the stage
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, + LoRA delta, activation,
//               stores; two TMEM accumulators so the epilogue of tile i overlaps the
//               MMAs of tile i+1
//   warp 6      epilogue loader: one tile ahead of the epilogue, the per-column data
//               (pair ids, routing weights, activation plane scales) and, for N tiles
//               <= 64, a TMA of the tile's fp32 LoRA delta into a two-slot ring
// N tiles of 256 (prefill) run on CTA pairs (a cluster of two, tcgen05 cta_group::2):
// the pair computes 256 weight rows x 256 tokens, each CTA staging its own 128 weight
// rows and half of the token rows (the MMA reads both halves), so every staged byte
// feeds twice the MMA work; the leader CTA's thread issues the MMAs of both and alone
// expects the pair's bytes on its stage barriers, its commits reach both CTAs, and both
// CTAs' epilogues release the accumulator on the leader's barrier.
// Every mbarrier wait is bounded; on expiry the CTA records MOE_LORA_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cstdlib>
#include <mutex>

namespace mlb {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiThreads = 128;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kMaxGroups = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr bool kPairDefault = true;                // CTA pairs for N tiles of 256

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
  const __nv_bfloat16* delta_bf16;  // [total_rows][delta_cols] bf16, read in the epilogue
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
  // limit of every bounded wait (ns); test_stall: CTA 0 never issues the copies of its
  // first stage, so the MMA's wait runs out and the abort path runs (tests only)
  uint64_t wait_ns;
  int test_stall;
  int pdl_trigger;    // let the next kernel launch at once
  int pdl_secondary;  // launched behind the LoRA kernel: whatever reads its delta waits for it
  int pdl_end_wait;   // launched behind a kernel whose output it does not read: it waits for
                      // that kernel only before it exits, so the launches after it see both done
  // base stages hold kpb consecutive K blocks (sub-stages of TileCfg::kStageBytes): two
  // give 256-byte runs of every weight row per stage at decode, which the memory system
  // streams faster than 128-byte runs
  int kpb;
  int stage_bytes;    // kpb * TileCfg::kStageBytes
  // epilogue slots: two (the loader fills tile i+1's while the epilogue reads tile i's)
  // or one (wide fp32 deltas, where shared memory is better spent on ring stages)
  int nslots, slot_bytes;
  int slot_delta;     // the loader TMA-prefetches the fp32 delta into the slots
};

// A unit of work: tile t, K stages [k0, k1) (every unit is a whole tile).
struct Unit {
  int t, k0, k1;
};
struct UnitIter {
  int t;
};

// persistent tile loop: CTA b takes tiles b, b + G, b + 2 G, ...; with CTA pairs both
// CTAs of a cluster walk the same units (pair b / 2 of G / 2)
template <bool TWO>
__device__ __forceinline__ UnitIter unit_begin() {
  UnitIter it;
  it.t = TWO ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  return it;
}

template <bool TWO>
__device__ __forceinline__ bool unit_next(int total_tiles, int nk, UnitIter& it, Unit& u) {
  if (it.t >= total_tiles) return false;
  u.t = it.t;
  u.k0 = 0;
  u.k1 = nk;
  it.t += TWO ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
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
  short chunk_rows[kMaxGroups];  // token rows per chunk of group g (<= the tile's)
  float ebuf[kBM][33];
};

// Epilogue prefetch slot, filled one tile ahead by the loader warp: the tile's pair ids,
// routing weights and plane scales, and (N tiles <= 64, fp32 LoRA delta) its delta
// [2 halves][BN][64].  Without a delta a slot ends before `delta` (TcParams::slot_bytes).
template <int BN>
struct EpiSlot {
  int col_pair[BN];
  float col_w[BN];
  float col_sh[BN];
  float col_sl[BN];
  float delta[BN <= 64 ? 2 * BN * 64 : 4];  // 128-byte aligned: 16 BN bytes in
};

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

// TWO: a CTA pair (cta_group::2) computes 256 weight rows x BN tokens; each CTA holds its
// 128 weight rows and half of the BN token rows of every stage.
// NS (not swapped, for the operand-swap comparison): tokens in the MMA's M slot (chunks of
// kNsTok = 128 token rows), weight rows in N (BN = 256: for gate_up 128 gate rows and the
// matching 128 up rows, for down 256 output rows).
constexpr int kNsTok = 128;
template <int BN, bool W8, bool TWO = false, bool NS = false>
struct TileCfg {
  static constexpr int kKB = W8 ? 128 : 64;                  // K per stage (128 bytes per row)
  // token rows held by this CTA: pairs of bf16 tiles split the tokens, pairs of e4m3 tiles
  // split the planes (the leader stages the hi plane, its peer the lo plane, all BN rows)
  static constexpr int kBRows = (TWO && !W8) ? BN / 2 : BN;
  static constexpr int kBTileBytes = kBRows * 128;           // one token tile (or plane)
  static constexpr int kStageBytes = kATileBytes + ((W8 && !TWO) ? 2 : 1) * kBTileBytes;
  static constexpr int kAccStride = BN < 32 ? 32 : BN;       // TMEM columns per accumulator
  static constexpr int kAccPerBuf = W8 ? 2 : 1;              // e4m3: hi and lo side by side (N = 2 BN)
  static constexpr int kTmemCols = pow2_at_least(2 * kAccPerBuf * kAccStride);
  static constexpr bool kPrefetch = BN <= 64;                // LoRA delta prefetched into the slots
  static constexpr int kThreads = 224;
  static_assert(!W8 || BN <= 128, "e4m3 weights use N tiles <= 128 (hi and lo planes: N = 2 BN)");
  static_assert(!TWO || (!W8 && BN == 256) || (W8 && BN == 128), "CTA pairs: bf16 N tiles of 256, e4m3 of 128");
  static_assert(!NS || (!W8 && !TWO && BN == 256), "tokens in M: bf16 weights, 256 weight rows in N");
  static constexpr int kTokRows = NS ? kNsTok : BN;          // token rows per tile
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
  const int cr = sm.chunk_rows[lo];
  ti.row0 = sm.grp_off[lo] + (c - sm.chunk_pref[lo]) * cr;
  ti.nvalid = min(cr, sm.grp_off[lo + 1] - ti.row0);
  return ti;
}

// delta column (weight row within the group) of accumulator row m in tile column block f0
__device__ __forceinline__ int delta_col(int epi, int m, int f0, int I) {
  if (epi == EPI_GATEUP) return (m < 64) ? f0 + m : I + f0 + (m - 64);
  return f0 + m;
}

template <int BN, bool W8, bool TWO, bool NS>
__global__ void __launch_bounds__(TileCfg<BN, W8, TWO, NS>::kThreads, BN <= 64 ? 2 : 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmw, const __grid_constant__ CUtensorMap tmb,
                   const __grid_constant__ CUtensorMap tml, const __grid_constant__ CUtensorMap tmd,
                   const TcParams p) {
  // tml: the lo activation plane (e4m3 weights); tmd: the fp32 LoRA delta (N tiles <= 64)
  using Cfg = TileCfg<BN, W8, TWO, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;                                 // stages: [A tile][token tile(s)]
  uint8_t* slots = ring + p.stages * p.stage_bytes;  // epilogue prefetch slots
  SmemCore& sm = *reinterpret_cast<SmemCore*>(slots + p.nslots * p.slot_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.stages;
  volatile int* abort_flag = &sm.abort_flag;
  // CTA pairs: rank 0 (the leader) issues the MMAs of both CTAs; the stage and TMEM
  // barriers it consumes live in its shared memory
  const uint32_t rank = TWO ? cluster_ctarank() : 0u;
  auto leader_bar = [&](uint64_t* bar) -> uint32_t { return TWO ? mapa_shared(smem_u32(bar), 0) : smem_u32(bar); };

  if (p.pdl_trigger) pdl_trigger();
  // ---- setup: barriers, TMEM, tile list prefix
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], TWO ? 2 * kEpiThreads : kEpiThreads);  // pairs: both CTAs' epilogues
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
    if (W8 || TWO) tma_prefetch_desc(&tml);
    if (p.delta != nullptr || (TWO && !W8)) tma_prefetch_desc(&tmd);
  }
  if (warp == 1) {
    if constexpr (TWO) tmem_alloc_pair(&sm.tmem_base, Cfg::kTmemCols);
    else tmem_alloc(&sm.tmem_base, Cfg::kTmemCols);
  }
  // group offsets clamped to [0, total_rows]: offsets that are out of range or not
  // monotone (flagged by the work-list kernel) can leave rows uncomputed, never make a
  // tile reach outside the operands
  for (int g = threadIdx.x; g <= p.E; g += blockDim.x)
    sm.grp_off[g] = p.group_offsets ? min(max(p.group_offsets[static_cast<size_t>(g) * p.group_stride], 0), p.total_rows)
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
        c = n > 0 ? (n + Cfg::kTokRows - 1) / Cfg::kTokRows : 0;
        // a group whose last chunk would hold less than half a tile splits its rows evenly
        // over its chunks instead (rounded up to 16): the small last chunk would cost
        // about as many MMA issue slots as a full one
        int cr = Cfg::kTokRows;
        if (c >= 2 && n - (c - 1) * Cfg::kTokRows < Cfg::kTokRows / 2) {
          cr = min(Cfg::kTokRows, ((n + c - 1) / c + 15) & ~15);
          c = (n + cr - 1) / cr;  // every chunk keeps at least one row
        }
        sm.chunk_rows[g] = static_cast<short>(cr);
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
  // pairs: a unit is a pair of 128-row weight tiles (an even count per group), rank picks one
  const int unit_m = TWO ? p.m_tiles / 2 : p.m_tiles;
  const int total_tiles = sm.chunk_pref[p.E] * unit_m;
  auto tile_of = [&](int t) -> TileInfo {
    TileInfo ti = decode_tile(sm, t, unit_m, p.E, Cfg::kTokRows);
    if constexpr (TWO) ti.mt = 2 * ti.mt + static_cast<int>(rank);
    return ti;
  };
  const int nk = (p.K + Cfg::kKB * p.kpb - 1) / (Cfg::kKB * p.kpb);  // stages per tile

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 issues the TMA copies of every stage: the weight tile (two 64-row boxes:
    // for gate_up the 64 gate rows and the matching 64 up rows) and the token tile(s) of
    // the same K range, kpb K blocks per stage.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t filled_mask = 0, last_parity = 0;
    bool ok = true;
    UnitIter uit = unit_begin<TWO>();
    Unit u;
    int itp = 0;  // unit index, the same sequence as the MMA thread's
    while (ok && unit_next<TWO>(total_tiles, nk, uit, u)) {
      if (*abort_flag) break;
      const TileInfo ti = tile_of(u.t);
      int wrow0, wrow1;
      if constexpr (NS) {  // 128-row weight boxes: gate and up halves, or two halves of 256 rows
        if (p.epi == EPI_GATEUP) {
          wrow0 = ti.g * p.rows_per_group + ti.mt * 128;
          wrow1 = ti.g * p.rows_per_group + p.I + ti.mt * 128;
        } else {
          wrow0 = ti.g * p.rows_per_group + ti.mt * 256;
          wrow1 = wrow0 + 128;
        }
      } else if (p.epi == EPI_GATEUP) {
        wrow0 = ti.g * p.rows_per_group + ti.mt * 64;
        wrow1 = ti.g * p.rows_per_group + p.I + ti.mt * 64;
      } else {
        wrow0 = ti.g * p.rows_per_group + ti.mt * kBM;
        wrow1 = wrow0 + 64;
      }
      for (int kb = u.k0; kb < u.k1; ++kb) {
        if (lane == 0) ok = mbar_wait(&sm.empty[stage], phase ^ 1u, abort_flag, p.status, p.wait_ns, 1);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const bool stall = p.test_stall && blockIdx.x == 0 && itp == 0 && kb == u.k0;  // never arrives
        if (lane == 0 && !stall) {
          uint8_t* a_s = ring + stage * p.stage_bytes;
          const int kc = kb * Cfg::kKB * p.kpb;  // first K element of the stage
          const int nj = min(p.kpb, (p.K - kc + Cfg::kKB - 1) / Cfg::kKB);  // sub-stages inside K
          if constexpr (TWO && W8) {
            // e4m3 pairs: the MMA's N is both planes (2 BN rows); the leader stages the hi
            // plane of the chunk's BN token rows, its peer the lo plane
            const uint32_t fb = leader_bar(&sm.full[stage]);
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[stage], 2u * nj * Cfg::kStageBytes);
            for (int j = 0; j < nj; ++j) {
              uint8_t* aj = a_s + j * Cfg::kStageBytes;
              const int kcj = kc + j * Cfg::kKB;
              tma_load_2d_pair(aj, &tmw, fb, kcj, wrow0);
              tma_load_2d_pair(aj + kATileBytes / 2, &tmw, fb, kcj, wrow1);
              tma_load_2d_pair(aj + kATileBytes, rank == 0 ? &tmb : &tml, fb, kcj, ti.row0);
            }
          } else if constexpr (TWO) {
            // both CTAs' copies complete on the leader's barrier, which expects the pair's
            // bytes; the MMA's N is the tile's rows rounded to 32, the peer holds [N/2, N)
            const uint32_t fb = leader_bar(&sm.full[stage]);
            const int n_pair = min(BN, (ti.nvalid + 31) & ~31);
            // each CTA's half of the token rows from the smallest box that holds it (32, 64
            // or 128 rows), so a ragged chunk does not stream the next group's rows
            const int half = n_pair / 2;
            const CUtensorMap* bm = half <= 32 ? &tml : half <= 64 ? &tmd : &tmb;
            const uint32_t bbytes = (half <= 32 ? 32u : half <= 64 ? 64u : 128u) * 128u;
            if (rank == 0) mbar_arrive_expect_tx(&sm.full[stage], 2u * nj * (kATileBytes + bbytes));
            for (int j = 0; j < nj; ++j) {
              uint8_t* aj = a_s + j * Cfg::kStageBytes;
              const int kcj = kc + j * Cfg::kKB;
              tma_load_2d_pair(aj, &tmw, fb, kcj, wrow0);
              tma_load_2d_pair(aj + kATileBytes / 2, &tmw, fb, kcj, wrow1);
              tma_load_2d_pair(aj + kATileBytes, bm, fb, kcj, ti.row0 + static_cast<int>(rank) * half);
            }
          } else if constexpr (NS) {
            // A = the chunk's 128 token rows, B = the two 128-row weight boxes
            mbar_arrive_expect_tx(&sm.full[stage], nj * Cfg::kStageBytes);
            for (int j = 0; j < nj; ++j) {
              uint8_t* aj = a_s + j * Cfg::kStageBytes;
              const int kcj = kc + j * Cfg::kKB;
              tma_load_2d(aj, &tmb, &sm.full[stage], kcj, ti.row0);
              tma_load_2d(aj + kATileBytes, &tmw, &sm.full[stage], kcj, wrow0);
              tma_load_2d(aj + kATileBytes + Cfg::kBTileBytes / 2, &tmw, &sm.full[stage], kcj, wrow1);
            }
          } else {
          mbar_arrive_expect_tx(&sm.full[stage], nj * Cfg::kStageBytes);
          for (int j = 0; j < nj; ++j) {  // sub-stage j: K block kc + j kKB
            uint8_t* aj = a_s + j * Cfg::kStageBytes;
            uint8_t* bj = aj + kATileBytes;
            const int kcj = kc + j * Cfg::kKB;
            tma_load_2d(aj, &tmw, &sm.full[stage], kcj, wrow0);
            tma_load_2d(aj + kATileBytes / 2, &tmw, &sm.full[stage], kcj, wrow1);
            tma_load_2d(bj, &tmb, &sm.full[stage], kcj, ti.row0);
            if constexpr (W8) tma_load_2d(bj + Cfg::kBTileBytes, &tml, &sm.full[stage], kcj, ti.row0);
          }
          }
          filled_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      ++itp;
    }
    if (lane == 0 && *abort_flag) {
      // let our own copies land before the CTA exits (pairs: the peer's copies complete on
      // the leader's barriers, so the peer gives them a fixed 50 us)
      if (TWO && rank != 0) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 50000ull) {
        }
      } else {
        for (int s = 0; s < S; ++s)
          if (filled_mask & (1u << s)) {
            volatile int dummy = 0;
            mbar_wait(&sm.full[s], (last_parity >> s) & 1u, &dummy, nullptr, p.wait_ns / 4, 0);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // pairs: the leader issues the MMAs of both CTAs (M = 256: its 128 rows and the
    // peer's); its commits arrive on the barrier at the same offset in both CTAs
    if (lane == 0 && (!TWO || rank == 0)) {
      auto commit = [&](uint64_t* bar) {
        if constexpr (TWO) umma_commit_pair(bar, 3);
        else umma_commit(bar);
      };
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      UnitIter uit = unit_begin<TWO>();
      Unit u;
      for (; !*abort_flag && unit_next<TWO>(total_tiles, nk, uit, u); ++it) {
        // the last chunk of a group is ragged: N = its rows rounded up to 16, so a
        // skewed expert load does not pay MMAs on padding rows
        const TileInfo ti = tile_of(u.t);
        // e4m3: the hi and lo planes sit back to back in the ring, so one instruction of
        // N = 2 BN covers both and each weight tile is read from shared memory once
        const int n_mma = NS ? BN : TWO ? min(BN, (ti.nvalid + 31) & ~31) : min(BN, (ti.nvalid + 15) & ~15);
        const uint32_t idesc = W8 ? umma_idesc_e4m3(TWO ? 2 * kBM : kBM, 2 * BN) : umma_idesc_bf16(TWO ? 2 * kBM : kBM, n_mma);
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait(&sm.tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, p.wait_ns, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * Cfg::kAccPerBuf * Cfg::kAccStride;
        bool ok = true;
        for (int kb = u.k0; kb < u.k1; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status, p.wait_ns, 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nj = min(p.kpb, (p.K - kb * p.kpb * Cfg::kKB + Cfg::kKB - 1) / Cfg::kKB);
          for (int j = 0; j < nj; ++j) {
            const uint32_t a_addr = smem_u32(ring + stage * p.stage_bytes) + j * Cfg::kStageBytes;
            const uint64_t adesc = umma_desc_sw128(a_addr);
            const uint64_t bdesc = umma_desc_sw128(a_addr + kATileBytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
              const uint32_t acc = (kb != u.k0 || j != 0 || k != 0) ? 1u : 0u;
              if constexpr (W8 && TWO) {
                umma_e4m3_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);  // hi from the leader, lo from the peer
              } else if constexpr (W8) {
                umma_e4m3(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);  // columns [0, BN) hi, [BN, 2 BN) lo
              } else if constexpr (TWO) {
                umma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
              } else {
                umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
              }
            }
          }
          commit(&sm.empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        commit(&sm.tfull[buf]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      if constexpr (TWO) umma_commit_pair(&sm.tdone, 1);
      else commit(&sm.tdone);
      volatile int dummy = 0;
      mbar_wait(&sm.tdone, 0, &dummy, nullptr, p.wait_ns, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;   // 0..127
    const int g4 = warp & 3;           // TMEM lane quarter this warp may access
    const int m = g4 * 32 + lane;      // accumulator row = weight row within the tile
    int it = 0;
    UnitIter uit = unit_begin<TWO>();
    Unit u;
    for (; unit_next<TWO>(total_tiles, nk, uit, u); ++it) {
      const TileInfo ti = tile_of(u.t);
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int sb = p.nslots == 2 ? buf : 0;  // epilogue slot and its use count
      const uint32_t su = p.nslots == 2 ? use : static_cast<uint32_t>(it);
      bool got = mbar_wait(&sm.tfull[buf], use & 1u, abort_flag, p.status, p.wait_ns, 4);
      got = got && mbar_wait(&sm.sfull[sb], su & 1u, abort_flag, p.status, p.wait_ns, 7);
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
      const EpiSlot<BN>* slot = reinterpret_cast<const EpiSlot<BN>*>(slots + sb * p.slot_bytes);

      if constexpr (NS) {
        // tokens in the TMEM lanes: thread m holds token row row0 + m, the columns are
        // weight rows (gate_up: 128 gate columns, then the matching 128 up columns)
        const int row = ti.row0 + m;
        const bool tok_ok = m < ti.nvalid;
        const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(g4 * 32) << 16) + buf * Cfg::kAccPerBuf * Cfg::kAccStride;
        if (p.epi == EPI_GATEUP) {
          for (int c0 = 0; c0 < 128; c0 += 32) {
            float gv[32], uv[32];
            tmem_ld_32x32b_x32(t_acc + c0, gv);
            tmem_ld_32x32b_x32(t_acc + 128 + c0, uv);
            const int f = ti.mt * 128 + c0;
            if (!tok_ok || f >= p.I) continue;
#pragma unroll
            for (int n = 0; n < 32; ++n) {
              gv[n] *= scale;
              uv[n] *= scale;
            }
            if (p.delta_bf16 != nullptr) {  // this row's 32 gate and 32 up delta values
              if (p.pdl_secondary) pdl_wait();  // the delta comes from the kernel ahead
              const __nv_bfloat16* dr = p.delta_bf16 + static_cast<size_t>(row) * p.delta_cols;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (f + 8 * q + 8 > p.I) break;
                float dg[8], du[8];
                unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(dr + f + 8 * q)), dg);
                unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(dr + p.I + f + 8 * q)), du);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  gv[8 * q + e] += dg[e];
                  uv[8 * q + e] += du[e];
                }
              }
            }
            uint32_t packed[16];
#pragma unroll
            for (int n = 0; n < 16; ++n)
              packed[n] = pack2_bf16(silu(gv[2 * n]) * uv[2 * n], silu(gv[2 * n + 1]) * uv[2 * n + 1]);
            __nv_bfloat16* dst = p.out_bf16 + static_cast<size_t>(row) * p.I + f;
            if (f + 32 <= p.I) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(dst)[q] =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
            } else {
              for (int n = 0; n < 32 && f + n < p.I; ++n)
                reinterpret_cast<uint16_t*>(dst)[n] =
                    static_cast<uint16_t>((n & 1) ? (packed[n >> 1] >> 16) : (packed[n >> 1] & 0xFFFFu));
            }
          }
        } else {  // EPI_DOWN: the routing pair of this row, weighted
          int pr = 0;
          float w = 0.f;
          if (tok_ok) {
            pr = p.sorted_pairs[row];
            if (pr < 0 || pr >= p.total_rows) {  // a corrupted pair index is not followed
              set_status(p.status, MOE_LORA_ERR_DEVICE_CHECK, row);
              pr = -1;
            } else {
              w = p.topk_w[pr];
            }
          }
          for (int c0 = 0; c0 < 256; c0 += 32) {
            float v[32];
            tmem_ld_32x32b_x32(t_acc + c0, v);
            const int f = ti.mt * 256 + c0;
            if (!tok_ok || pr < 0 || f >= p.n_out) continue;
            uint32_t packed[16];
#pragma unroll
            for (int n = 0; n < 16; ++n) packed[n] = pack2_bf16(w * scale * v[2 * n], w * scale * v[2 * n + 1]);
            __nv_bfloat16* dst = p.out_bf16 + static_cast<size_t>(pr) * p.n_out + f;
            if (f + 32 <= p.n_out) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(dst)[q] =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
            } else {
              for (int n = 0; n < 32 && f + n < p.n_out; ++n)
                reinterpret_cast<uint16_t*>(dst)[n] =
                    static_cast<uint16_t>((n & 1) ? (packed[n >> 1] >> 16) : (packed[n >> 1] & 0xFFFFu));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.tempty[buf]);
        mbar_arrive(&sm.sempty[sb]);
        continue;
      }

      // bf16 delta [rows][delta_cols] (token-major): lane L of a warp loads row c0 + L's 32
      // delta columns of the warp (64 contiguous bytes, one chunk ahead), the warp passes
      // them through its own 32 rows of ebuf, and lane m takes column m (its feature)
      const bool dbf = p.delta_bf16 != nullptr;
      const int dcol_w = delta_col(p.epi, g4 * 32, f0, p.I);  // the warp's first delta column
      uint4 draw[4];
      auto dload = [&](int cbase) {
        const int row = cbase + lane;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool ok = row < ti.nvalid && dcol_w + 8 * q + 8 <= p.delta_cols;
          draw[q] = ok ? __ldg(reinterpret_cast<const uint4*>(p.delta_bf16 + static_cast<size_t>(ti.row0 + row) *
                                                                                p.delta_cols + dcol_w + 8 * q))
                       : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      if (dbf && p.pdl_secondary) pdl_wait();  // the delta comes from the kernel ahead
      if (dbf) dload(0);
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
        } else {
#pragma unroll
          for (int n = 0; n < 32; ++n) v[n] *= scale;
        }
        if (p.delta != nullptr) {
          if (Cfg::kPrefetch && p.slot_delta) {
            const float* dl = slot->delta + ((m >> 6) * BN + c0) * 64 + (m & 63);
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (c0 + n < BN) v[n] += dl[n * 64];
          } else if (dcol < p.delta_cols) {
            if (p.pdl_secondary) pdl_wait();  // the delta comes from the kernel ahead
            const float* dg = p.delta + static_cast<size_t>(ti.row0 + c0) * p.delta_cols + dcol;
#pragma unroll
            for (int n = 0; n < 32; ++n)
              if (n < ncol) v[n] += dg[static_cast<size_t>(n) * p.delta_cols];
          }
        } else if (dbf) {
          // transpose through the warp's own ebuf rows (34 bf16 per staged row: no bank
          // conflicts either way); the previous chunk's readers are past the barrier above
          uint32_t* stg = reinterpret_cast<uint32_t*>(&sm.ebuf[g4 * 32][0]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            stg[lane * 17 + 4 * q] = draw[q].x;
            stg[lane * 17 + 4 * q + 1] = draw[q].y;
            stg[lane * 17 + 4 * q + 2] = draw[q].z;
            stg[lane * 17 + 4 * q + 3] = draw[q].w;
          }
          __syncwarp();
          const uint16_t* colp = reinterpret_cast<const uint16_t*>(stg) + lane;
#pragma unroll
          for (int n = 0; n < 32; ++n) v[n] += bf2f_bits(colp[n * 34]);
          __syncwarp();
          if (c0 + 32 < ti.nvalid) dload(c0 + 32);  // the next chunk's rows fly meanwhile
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
          // through ebuf (thread m's 32 columns into row m), then lane n of warp g4 writes
          // the 32 features [32 g4, 32 g4 + 32) of token column n as four 16-byte runs, so
          // a routing pair's row leaves as whole 64-byte pieces
#pragma unroll
          for (int n = 0; n < 32; ++n) sm.ebuf[m][n] = v[n];
          named_bar_sync(1, kEpiThreads);
          const int n = lane;
          const int fbase = f0 + g4 * 32;
          if (n < ncol && fbase < p.n_out) {
            const float w = slot->col_w[c0 + n];
            __nv_bfloat16* dst = p.out_bf16 + static_cast<size_t>(slot->col_pair[c0 + n]) * p.n_out + fbase;
            uint32_t packed[16];
#pragma unroll
            for (int f = 0; f < 16; ++f)
              packed[f] = pack2_bf16(w * sm.ebuf[g4 * 32 + 2 * f][n], w * sm.ebuf[g4 * 32 + 2 * f + 1][n]);
            if (fbase + 32 <= p.n_out) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(dst)[q] =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
            } else {
              for (int f = 0; f < 32 && fbase + f < p.n_out; ++f)
                reinterpret_cast<uint16_t*>(dst)[f] =
                    static_cast<uint16_t>((f & 1) ? (packed[f >> 1] >> 16) : (packed[f >> 1] & 0xFFFFu));
            }
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
      tc_fence_before();
      if constexpr (TWO) mbar_arrive_remote(leader_bar(&sm.tempty[buf]));  // the leader's MMA reuses it
      else mbar_arrive(&sm.tempty[buf]);
      mbar_arrive(&sm.sempty[sb]);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ epilogue loader
    {
      // the LoRA delta (and nothing else this kernel reads) comes from the kernel ahead:
      // the loader waits for it only when it prefetches the delta
      if (p.pdl_secondary && p.slot_delta && p.delta != nullptr) pdl_wait();
      uint32_t issued_mask = 0, issued_parity = 0;
      int it = 0;
      UnitIter uit = unit_begin<TWO>();
      Unit u;
      for (; unit_next<TWO>(total_tiles, nk, uit, u); ++it) {
        const TileInfo ti = tile_of(u.t);
        const int buf = p.nslots == 2 ? (it & 1) : 0;
        const uint32_t use = p.nslots == 2 ? static_cast<uint32_t>(it >> 1) : static_cast<uint32_t>(it);
        const bool got = mbar_wait(&sm.sempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, p.wait_ns, 8);
        if (!__all_sync(0xffffffffu, got)) break;
        EpiSlot<BN>* slot = reinterpret_cast<EpiSlot<BN>*>(slots + buf * p.slot_bytes);
        if constexpr (Cfg::kPrefetch) {
          if (lane == 0 && p.delta != nullptr && p.slot_delta) {
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
            int pr = n < ti.nvalid ? p.sorted_pairs[ti.row0 + n] : 0;
            const bool pv = pr >= 0 && pr < p.total_rows;  // a corrupted pair index is not followed
            if (!pv && n < ti.nvalid) set_status(p.status, MOE_LORA_ERR_DEVICE_CHECK, ti.row0 + n);
            pr = pv ? pr : 0;
            slot->col_pair[n] = pr;
            slot->col_w[n] = (n < ti.nvalid && pv) ? p.topk_w[pr] : 0.f;
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
            mbar_wait(&sm.sfull[b], (issued_parity >> b) & 1u, &dummy, nullptr, p.wait_ns / 4, 0);
          }
      }
    }
  }

  if (p.pdl_end_wait) pdl_wait();
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

template <int BN, bool W8, bool TWO = false, bool NS = false>
static cudaError_t launch_bn(const GemmArgs& a, cudaStream_t st) {
  using Cfg = TileCfg<BN, W8, TWO, NS>;
  // two K blocks per stage for the weight-streaming (decode) tiles, and for CTA pairs
  // (64 KB stages: eight MMAs of M = 256 between the commits that free a stage)
  const int kpb = ((BN <= 64 || TWO) && a.K > Cfg::kKB) ? 2 : 1;
  const int m_tiles = NS ? ((a.epi == EPI_GATEUP) ? (a.I + 127) / 128 : (a.n_out + 255) / 256)
                         : (a.epi == EPI_GATEUP) ? (a.I + 63) / 64 : (a.n_out + kBM - 1) / kBM;
  if (TWO && m_tiles % 2 != 0) return cudaErrorInvalidValue;  // whole pairs of weight tiles
  if (NS && (a.delta != nullptr || (a.epi != EPI_GATEUP && a.epi != EPI_DOWN))) return cudaErrorInvalidValue;
  // epilogue slots: the fp32 delta part only when the loader prefetches it (whole tiles,
  // N <= 64); one slot instead of two where that buys another ring stage
  const bool dslot = a.delta != nullptr && Cfg::kPrefetch;
  const int slot_bytes = static_cast<int>(((dslot ? sizeof(EpiSlot<BN>) : offsetof(EpiSlot<BN>, delta)) + 1023) /
                                          1024 * 1024);
  const int stage_bytes = kpb * Cfg::kStageBytes;
  // overlapped with the SIMT LoRA kernel (PDL: launched behind one, or letting one start)
  // the GEMM leaves room for one of its CTAs on every SM (228 KB per SM, 1 KB reserved per
  // CTA), so both run side by side; behind the tensor-core LoRA kernel (pdl_full_smem)
  // nothing shares an SM, and a GEMM CTA starts on each SM that kernel has left
  const bool coloc = (a.pdl_secondary || a.pdl_trigger) && !a.pdl_full_smem;
  const int smem_cap = coloc ? 228 * 1024 - 1024 - kLoraCoresidentSmem : 232448;
  auto stages_for = [&](int ns) {
    const int s = (smem_cap - 1024 - static_cast<int>(sizeof(SmemCore)) - ns * slot_bytes) / stage_bytes;
    return s > 8 ? 8 : s;
  };
  const int nslots = stages_for(1) > stages_for(2) ? 1 : 2;
  const int stages = stages_for(nslots);
  if (stages < 2) return cudaErrorInvalidConfiguration;
  const int fixed = static_cast<int>(sizeof(SmemCore)) + nslots * slot_bytes;
  const size_t smem = 1024 + static_cast<size_t>(stages) * stage_bytes + fixed;
  if (smem > 232448) return cudaErrorInvalidConfiguration;
  // the raised shared-memory limit is a per-device function attribute
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    const cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, W8, TWO, NS>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tmw, tmb, tml, tmd;
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
                       NS ? 128 : 64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
        encode_tmap_2d(&tmb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b, a.K, a.total_rows,
                       static_cast<uint64_t>(a.K) * 2, kBK, NS ? kNsTok : Cfg::kBRows,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tml = tmb;  // unused
    if constexpr (TWO) {  // token boxes of 32 and 64 rows for ragged chunks (tml, tmd)
      if (encode_tmap_2d(&tml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b, a.K, a.total_rows,
                         static_cast<uint64_t>(a.K) * 2, kBK, 32, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
          encode_tmap_2d(&tmd, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.b, a.K, a.total_rows,
                         static_cast<uint64_t>(a.K) * 2, kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  if (TWO && !W8) {
    // tmd holds the 64-row token box (pairs take no fp32 delta)
  } else if (a.delta != nullptr && Cfg::kPrefetch) {
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
  p.delta_bf16 = a.delta_bf16;
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
  p.m_tiles = m_tiles;
  p.stages = stages;
  p.wait_ns = a.test_stall_ms > 0 ? static_cast<uint64_t>(a.test_stall_ms) * 1000000ull : kWaitLimitNs;
  p.test_stall = a.test_stall_ms > 0 ? 1 : 0;
  p.pdl_trigger = a.pdl_trigger;
  p.pdl_secondary = a.pdl_secondary;
  p.pdl_end_wait = a.pdl_end_wait;
  p.kpb = kpb;
  p.stage_bytes = stage_bytes;
  p.nslots = nslots;
  p.slot_bytes = slot_bytes;
  p.slot_delta = dslot ? 1 : 0;
  const long long chunks_ub = (a.total_rows + Cfg::kTokRows - 1) / Cfg::kTokRows + a.E;
  const long long tiles_ub = chunks_ub * (TWO ? p.m_tiles / 2 : p.m_tiles);
  int grid = a.num_sms;
  if constexpr (TWO) {  // whole clusters of two CTAs
    grid = (grid / 2 < tiles_ub ? grid / 2 : static_cast<int>(tiles_ub)) * 2;
    if (grid < 2) grid = 2;
  } else {
    if (tiles_ub < grid) grid = static_cast<int>(tiles_ub);
    if (grid < 1) grid = 1;
  }
  ProfScope ps(a.epi == EPI_GATEUP ? K_GEMM_GATEUP
               : a.epi == EPI_DOWN ? K_GEMM_DOWN
               : a.epi == EPI_LOGITS ? K_ROUTE_LOGITS
               : K_GEMM_DENSE, st);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cfg::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if constexpr (TWO) {  // clusters of two CTAs: the MMA pair
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (a.pdl_secondary || a.pdl_end_wait) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, W8, TWO, NS>, tmw, tmb, tml, tmd, p);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st) {
  if (a.E > kMaxGroups) return cudaErrorInvalidValue;
  if (a.delta != nullptr && a.delta_cols % 8 != 0) return cudaErrorInvalidValue;
  if (a.delta_bf16 != nullptr && a.delta != nullptr) return cudaErrorInvalidValue;
  if (a.w_fp8) {
    if (a.b_hi == nullptr || a.b_lo == nullptr || a.b_scales == nullptr) return cudaErrorInvalidValue;
    switch (a.bn) {
      case 16: return launch_bn<16, true>(a, st);
      case 32: return launch_bn<32, true>(a, st);
      case 64: return launch_bn<64, true>(a, st);
      default: {
        // CTA pairs (M = 256): each CTA stages one plane, so a stage holds one weight tile
        // and one plane and every staged byte feeds twice the MMA work
        const int m_tiles = (a.epi == EPI_GATEUP) ? (a.I + 63) / 64 : (a.n_out + kBM - 1) / kBM;
        const char* v = std::getenv("MOE_LORA_PAIR");
        const bool pair = (v != nullptr ? std::atoi(v) != 0 : kPairDefault) && m_tiles % 2 == 0 && a.K > 128 &&
                          (a.epi == EPI_GATEUP || a.epi == EPI_DOWN);
        return pair ? launch_bn<128, true, true>(a, st) : launch_bn<128, true>(a, st);
      }
    }
  }
  switch (a.bn) {
    case 16: return launch_bn<16, false>(a, st);
    case 32: return launch_bn<32, false>(a, st);
    case 64: return launch_bn<64, false>(a, st);
    case 128: return launch_bn<128, false>(a, st);
    case 256: {
      // N tiles of 256 on CTA pairs (tcgen05 cta_group::2, M = 256): per CTA and stage one
      // 16 KB weight tile and half of the token tile, so the same shared memory holds more
      // stages and each byte staged feeds twice the MMA work.  MOE_LORA_PAIR=0|1 overrides.
      const int m_tiles = (a.epi == EPI_GATEUP) ? (a.I + 63) / 64 : (a.n_out + kBM - 1) / kBM;
      // MOE_LORA_SWAP=0: tokens in M and weights in N (the operand-swap comparison)
      const char* sw = std::getenv("MOE_LORA_SWAP");
      if (sw != nullptr && std::atoi(sw) == 0 && a.delta == nullptr && (a.epi == EPI_GATEUP || a.epi == EPI_DOWN))
        return launch_bn<256, false, false, true>(a, st);
      const char* v = std::getenv("MOE_LORA_PAIR");
      const bool pair = (v != nullptr ? std::atoi(v) != 0 : kPairDefault) && m_tiles % 2 == 0 && a.K > kBK &&
                        (a.epi == EPI_GATEUP || a.epi == EPI_DOWN || a.epi == EPI_DENSE);
      return pair ? launch_bn<256, false, true>(a, st) : launch_bn<256, false>(a, st);
    }
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mlb
