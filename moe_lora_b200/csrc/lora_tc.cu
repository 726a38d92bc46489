// Tensor-core segmented LoRA (SGMV) for long adapter segments, sm_100a.
//
// For every work item (a chunk of up to kLtN rows of one adapter segment, [Punica
// review page], "提案手法": segmented gather), one CTA computes
//   shrink  z = x A_a            on tcgen05: A_a (r rows of the slot, K-major) in the MMA's
//                                M slot, the segment's rows in N, K = h_in streamed by TMA
//                                ([vLLM MoE-LoRA page], "O Papel da Multi-LoRA": z = xA)
//   expand  delta = z B_a        on tcgen05: B_a^T (feature-contiguous, MN-major boxes of
//                                64 features x r rank rows) in M, z in N (MN-major, written
//                                from TMEM into shared memory), K = r
// so z never leaves the SM, and writes delta (bf16, [rows][features]) for the grouped
// GEMM's epilogue to add before the activation ("Otimizações em Nível de Kernel": the
// LoRA add fused into the base output).  Rows of segments without an adapter get
// delta = 0 (early exit of the LoRA work, "Otimizações em Nível de Execução").
//
// Both products are many small MMAs (N = the item's rows, a few dozen), and one thread
// issuing them, with the commits that free its stages, keeps the tensor pipe idle much of
// the time; two issuing threads on one SM get about 1.5-1.8x the MMAs through.  So the
// shrink and the expand have an issuer each, fed by rings of their own, and the shrink of
// item i + 1 runs while the expand of item i does.
//
// Structure (one CTA per SM, persistent over the device-side work list, 12 warps):
//   warp 0      claims items (a queue of kLtQ slots) and loads the shrink stages: A_a box +
//               the rows' box (one of six heights, so a short segment does not load 128
//               rows), several K blocks per stage
//   warp 1      shrink MMAs into the z accumulator (TMEM columns [0, 128))
//   warp 2      loads the expand stages: B_a^T boxes of 64 features
//   warp 3      expand MMAs into three rotating accumulators (TMEM columns [128, 512);
//               several feature blocks side by side in one when the segment is short)
//   warps 4..7  delta epilogue: expand accumulators -> bf16 delta rows in global memory
//   warps 8..11 z: the z accumulator -> bf16 -> one of two shared-memory z tiles (the
//               expand's B operand), so the shrink of the next item can start at once
// Every mbarrier wait is bounded; on expiry the CTA records MOE_LORA_ERR_TIMEOUT,
// drains its own copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"
#include "prof.h"

#include <atomic>

namespace mlb {

constexpr int kLtThreads = 384;
constexpr int kLtEpi = 128;                        // delta epilogue threads (warps 4..7)
constexpr int kLtZ = 128;                          // z threads (warps 8..11)
constexpr int kLtAcc = 3;                          // expand accumulators
constexpr int kLtMaxStages = 8;
constexpr int kLtQ = 4;                            // item queue slots
constexpr int kLtQConsumers = 5;                   // shrink MMA, expand loader, expand MMA, delta, z
constexpr uint64_t kLtWaitNs = 2000000000ull;      // 2 s

struct LoraTcParams {
  const int2* items;          // (segment q, first row): chunks of <= kLtN rows, every segment
  const int* item_count;
  const int32_t* seg_off;     // [nseg + 1]
  int nseg;
  const int32_t* seg_adapter; // dense: adapter of segment q; null: MoE keys q = e (L + 1) + a'
  int L, E;                   // slot of (adapter a, group e) = a E + e (dense: E = 1, e = 0)
  int K, r, rbox, F, nrows;
  int s_stages, s_stage_bytes;  // shrink ring
  // expand ring: stages of bps feature blocks (expand_bytes each), so the expand issuer
  // commits a stage after several blocks' MMAs (a commit costs about as much as several
  // small MMAs)
  int e_stages, e_stage_bytes, bps, expand_bytes;
  int ztile_bytes;            // one z tile: 2 blocks of 64 rows x rbox ranks, MN-major
  __nv_bfloat16* delta;       // [nrows][F]
  const int32_t* scatter;     // delta row of row s: scatter[s] (pair order); null = s
  int* status;
  int* work_counter;          // next unclaimed work item (zero on entry)
  const __nv_bfloat16* lora_b;  // [L E r][F] (split: [L E 2 r_exp][split_I]): the expand's B rows
  // separate gate and up adapters (split_I = I > 0): the shrink's r = 2 r_exp rows are the
  // gate adapter's then the up adapter's; gate features take B rows against z[0, r_exp)
  // and zeros against z[r_exp, r), up features the other way round
  int split_I;
  int r_exp;
  float scale;                // multiplies every delta value
  int pdl_trigger;            // the kernel behind this one (PDL) may launch at once
};

struct LtItem {
  int lo, hi, n, n_mma, box, slot;
  int kpb;                    // K blocks of 64 per shrink stage (short segments: several)
  bool lora;                  // the segment has an adapter (else delta = 0 rows)
};

struct LtSmem {
  uint64_t sfull[kLtMaxStages];   // shrink ring
  uint64_t sempty[kLtMaxStages];
  uint64_t efull[kLtMaxStages];   // expand ring
  uint64_t eempty[kLtMaxStages];
  uint64_t zfull;             // shrink accumulated (shrink MMA -> z warps)
  uint64_t zfree;             // z accumulator read out (z warps -> shrink MMA)
  uint64_t zready[2];         // z tile b written (z warps -> expand MMA)
  uint64_t zdone[2];          // the MMAs reading z tile b completed (expand MMA -> z warps)
  uint64_t tfull[kLtAcc];
  uint64_t tempty[kLtAcc];
  uint64_t sdone, edone;      // each issuer's last MMAs completed (before TMEM is freed)
  uint64_t qfull[kLtQ];       // work-item queue: warp 0 claims items ...
  uint64_t qempty[kLtQ];      // ... and the five consumers release the slot
  int q[kLtQ];
  LtItem qi[kLtQ];            // the claimed items, decoded once
  uint32_t tmem_base;
  int abort_flag;
  int rowmap[kLtN];           // delta row of each row of the delta epilogue's current item
};

constexpr int kLtStgPitch = 80;               // bytes per staged row of 32 bf16 (16-byte aligned)
constexpr int kLtStgWarp = 32 * kLtStgPitch;  // one epilogue warp's staging block

// heights of the rows' box (a short segment loads no more rows than it needs, to the next
// multiple of 8 or 16; the shrink MMA's N rounds up to 16 and reads past a 24-row box into
// rows whose z columns are never used)
constexpr int kLtBoxes = 6;
__device__ __forceinline__ int lt_box_rows(int box) {
  return box == 0 ? 16 : box == 1 ? 24 : box == 2 ? 32 : box == 3 ? 48 : box == 4 ? 64 : 128;
}

// Work item `it`: rows [lo, hi) of segment q with hi - lo <= kLtN.
__device__ __forceinline__ LtItem lt_item(const LoraTcParams& p, int it) {
  LtItem t;
  const int2 w = p.items[it];
  const int q = w.x;
  t.lo = max(w.y, 0);
  t.hi = (q >= 0 && q < p.nseg) ? min(min(p.seg_off[q + 1], t.lo + kLtN), p.nrows) : t.lo;
  t.n = max(0, t.hi - t.lo);
  t.n_mma = (t.n + 15) & ~15;
  t.box = t.n <= 16 ? 0 : t.n <= 24 ? 1 : t.n <= 32 ? 2 : t.n <= 48 ? 3 : t.n <= 64 ? 4 : 5;
  int ad, e = 0;
  if (p.seg_adapter != nullptr) {
    ad = (q >= 0 && q < p.nseg) ? p.seg_adapter[q] : -1;
  } else {
    e = q / (p.L + 1);
    const int ap = q - e * (p.L + 1);
    ad = (ap == p.L) ? -1 : ap;
  }
  t.lora = ad >= 0 && ad < p.L && t.n > 0;
  t.slot = t.lora ? ad * p.E + e : 0;
  // a shrink stage holds as many (A box, rows box) pairs as fit, up to 4: short segments
  // then keep as many bytes in flight as long ones
  t.kpb = min(4, max(1, p.s_stage_bytes / (p.r * 128 + lt_box_rows(t.box) * 128)));
  return t;
}

// Row of delta written for gathered row s: s, or scatter[s] (the routing pair of sorted
// row s, for a delta the combine reads in pair order); -1 (not written) for an index
// outside [0, nrows).
__device__ __forceinline__ int lt_delta_row(const LoraTcParams& p, int s) {
  if (p.scatter == nullptr) return s;
  const int d = p.scatter[s];
  return (d >= 0 && d < p.nrows) ? d : -1;
}

// Next item of the queue for a consumer: waits for slot qi, reads it, releases it (one
// arrival per consumer role).  False when the wait ran out.
__device__ __forceinline__ bool lt_take(LtSmem& sm, int qi, int& it, LtItem& t, volatile int* abort_flag, int* status,
                                        int where, bool release) {
  const int qs = qi % kLtQ;
  if (!mbar_wait(&sm.qfull[qs], static_cast<uint32_t>(qi / kLtQ) & 1u, abort_flag, status, kLtWaitNs, where))
    return false;
  it = static_cast<volatile int*>(sm.q)[qs];
  t = sm.qi[qs];
  if (release) mbar_arrive(&sm.qempty[qs]);
  return true;
}

__global__ void __launch_bounds__(kLtThreads, 1)
    lora_tc_kernel(const __grid_constant__ CUtensorMap tmx16, const __grid_constant__ CUtensorMap tmx24,
                   const __grid_constant__ CUtensorMap tmx32, const __grid_constant__ CUtensorMap tmx48,
                   const __grid_constant__ CUtensorMap tmx64, const __grid_constant__ CUtensorMap tmx128,
                   const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                   const LoraTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sring = smem;                                   // shrink stages
  uint8_t* ering = sring + p.s_stages * p.s_stage_bytes;   // expand stages
  uint8_t* zs = ering + p.e_stages * p.e_stage_bytes;      // two z tiles
  uint8_t* stg = zs + 2 * p.ztile_bytes;                   // delta staging: 4 warps x 32 rows
  LtSmem& sm = *reinterpret_cast<LtSmem*>(stg + 4 * kLtStgWarp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;
  // the GEMM behind this kernel takes each SM this kernel leaves; only what reads the delta
  // waits for this kernel to finish
  if (p.pdl_trigger) pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.s_stages; ++s) {
      mbar_init(&sm.sfull[s], 1);
      mbar_init(&sm.sempty[s], 1);
    }
    for (int s = 0; s < p.e_stages; ++s) {
      mbar_init(&sm.efull[s], 1);
      mbar_init(&sm.eempty[s], 1);
    }
    mbar_init(&sm.zfull, 1);
    mbar_init(&sm.zfree, kLtZ);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.zready[b], kLtZ);
      mbar_init(&sm.zdone[b], 1);
    }
    for (int b = 0; b < kLtAcc; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kLtEpi);
    }
    mbar_init(&sm.sdone, 1);
    mbar_init(&sm.edone, 1);
    for (int b = 0; b < kLtQ; ++b) {
      mbar_init(&sm.qfull[b], 1);
      mbar_init(&sm.qempty[b], kLtQConsumers);
    }
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmx16);
    tma_prefetch_desc(&tmx24);
    tma_prefetch_desc(&tmx32);
    tma_prefetch_desc(&tmx48);
    tma_prefetch_desc(&tmx64);
    tma_prefetch_desc(&tmx128);
    tma_prefetch_desc(&tma);
  }
  if (warp == 2 && lane == 0) tma_prefetch_desc(&tmb);
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);  // z: [0, 128); expand: 3 x 128 after it
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm.tmem_base;
  const int count = *p.item_count;
  const int nk = (p.K + 63) / 64;           // shrink K blocks per item
  const int nf = (p.F + 127) / 128;         // expand feature blocks per item
  const uint32_t zlbo = static_cast<uint32_t>(p.rbox) * 128u;  // z tile: 64-row blocks apart

  if (warp == 0) {
    // ------------------------------------------------------------ claims + shrink loads
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled_mask = 0, last_parity = 0;
      bool ok = true;
      // items are claimed one at a time from a global counter (their costs differ with the
      // segment's rows): the CTAs finish together
      for (int qi = 0; ok; ++qi) {
        const int qs = qi % kLtQ;
        if (!mbar_wait(&sm.qempty[qs], (static_cast<uint32_t>(qi / kLtQ) & 1u) ^ 1u, abort_flag, p.status,
                       kLtWaitNs, 20))
          break;
        int it = atomicAdd(p.work_counter, 1);
        if (it >= count) it = -1;
        const LtItem t = it >= 0 ? lt_item(p, it) : LtItem{};
        sm.q[qs] = it;
        sm.qi[qs] = t;
        mbar_arrive(&sm.qfull[qs]);
        if (it < 0) break;
        if (!t.lora) continue;
        const int arow = t.slot * p.r;
        const CUtensorMap* xm = t.box == 0 ? &tmx16 : t.box == 1 ? &tmx24 : t.box == 2 ? &tmx32
                              : t.box == 3 ? &tmx48 : t.box == 4 ? &tmx64 : &tmx128;
        const uint32_t xbytes = static_cast<uint32_t>(lt_box_rows(t.box)) * 128u;
        const uint32_t pair = static_cast<uint32_t>(p.r) * 128u + xbytes;  // one (A, rows) box pair
        // the item's B_a rows head for L2 in pieces, one per shrink stage, so the expand
        // stages later load from L2 while HBM streams the next item
        const int brow = p.split_I ? p.split_I : p.F;  // elements per B row
        const uint8_t* bslot = reinterpret_cast<const uint8_t*>(p.lora_b + static_cast<size_t>(arow) * brow);
        const uint32_t bbytes = static_cast<uint32_t>(p.r) * static_cast<uint32_t>(brow) * 2u;
        const int nstg = (nk + t.kpb - 1) / t.kpb;
        const uint32_t bpiece = (bbytes / nstg + 15u) & ~15u;
        uint32_t boff = 0;
        for (int kb = 0; kb < nk; kb += t.kpb) {
          if (!mbar_wait(&sm.sempty[stage], phase ^ 1u, abort_flag, p.status, kLtWaitNs, 21)) {
            ok = false;
            break;
          }
          if (boff < bbytes) {
            prefetch_l2_bulk(bslot + boff, min(bpiece, bbytes - boff));
            boff += bpiece;
          }
          uint8_t* s = sring + stage * p.s_stage_bytes;
          const int np = min(t.kpb, nk - kb);
          mbar_arrive_expect_tx(&sm.sfull[stage], pair * static_cast<uint32_t>(np));
          for (int j = 0; j < np; ++j) {
            tma_load_2d(s + j * pair, &tma, &sm.sfull[stage], (kb + j) * 64, arow);
            tma_load_2d(s + j * pair + p.r * 128, xm, &sm.sfull[stage], (kb + j) * 64, t.lo);
          }
          filled_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == p.s_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let our own copies land before the CTA exits
        for (int s = 0; s < p.s_stages; ++s)
          if (filled_mask & (1u << s)) {
            volatile int dummy = 0;
            mbar_wait(&sm.sfull[s], (last_parity >> s) & 1u, &dummy, nullptr, kLtWaitNs / 4, 0);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ shrink MMAs
    if (lane == 0) {
      int stage = 0, li = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t tz = tmem_base;
      for (int qi = 0; ok && !*abort_flag; ++qi) {
        int it;
        LtItem t;
        if (!lt_take(sm, qi, it, t, abort_flag, p.status, 28, true) || it < 0) break;
        if (!t.lora) continue;
        // the z accumulator is free once the z warps have read the previous item's
        if (!mbar_wait(&sm.zfree, (static_cast<uint32_t>(li) & 1u) ^ 1u, abort_flag, p.status, kLtWaitNs, 23)) break;
        tc_fence_after();
        // z[i][j] = sum_k A[i][k] x[j][k]; rows i >= r of the accumulator are unused
        const uint32_t idesc = umma_idesc_bf16(128, t.n_mma);
        const uint32_t pair = static_cast<uint32_t>(p.r) * 128u + static_cast<uint32_t>(lt_box_rows(t.box)) * 128u;
        for (int kb = 0; kb < nk; kb += t.kpb) {
          if (!mbar_wait(&sm.sfull[stage], phase, abort_flag, p.status, kLtWaitNs, 22)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int np = min(t.kpb, nk - kb);
          for (int j = 0; j < np; ++j) {
            const uint32_t a_addr = smem_u32(sring + stage * p.s_stage_bytes) + j * pair;
            const uint64_t adesc = umma_desc_sw128(a_addr);
            const uint64_t bdesc = umma_desc_sw128(a_addr + p.r * 128);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16(tz, adesc + 2 * k, bdesc + 2 * k, idesc, (kb + j > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&sm.sempty[stage]);
          if (++stage == p.s_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&sm.zfull);
        ++li;
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(&sm.sdone);
      volatile int dummy = 0;
      mbar_wait(&sm.sdone, 0, &dummy, nullptr, kLtWaitNs, 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ expand loads
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled_mask = 0, last_parity = 0;
      bool ok = true;
      const int zrow = p.L * p.E * p.r;  // first row past B (a box there reads zeros)
      for (int qi = 0; ok && !*abort_flag; ++qi) {
        int it;
        LtItem t;
        if (!lt_take(sm, qi, it, t, abort_flag, p.status, 30, true) || it < 0) break;
        if (!t.lora) continue;
        const int arow = t.slot * p.r;
        for (int fb0 = 0; fb0 < nf; fb0 += p.bps) {
          if (!mbar_wait(&sm.eempty[stage], phase ^ 1u, abort_flag, p.status, kLtWaitNs, 31)) {
            ok = false;
            break;
          }
          const int nb = min(p.bps, nf - fb0);
          mbar_arrive_expect_tx(&sm.efull[stage], static_cast<uint32_t>(nb) * 2u * static_cast<uint32_t>(p.rbox) * 128u);
          for (int jb = 0; jb < nb; ++jb) {
            const int fb = fb0 + jb;
            uint8_t* s = ering + stage * p.e_stage_bytes + jb * p.expand_bytes;
            if (p.split_I == 0) {
              tma_load_2d(s, &tmb, &sm.efull[stage], fb * 128, arow);
              tma_load_2d(s + p.rbox * 128, &tmb, &sm.efull[stage], fb * 128 + 64, arow);
            } else {
              // each 64-feature box: K rows [0, r_exp) then [r_exp, 2 r_exp), one of them the
              // adapter's B rows and the other zeros (a box past the tensor's last row)
              for (int h = 0; h < 2; ++h) {
                const int f = fb * 128 + 64 * h;
                const bool up = f >= p.split_I;
                const int fc = up ? f - p.split_I : f;
                uint8_t* bx = s + h * (p.rbox * 128);
                tma_load_2d(bx, &tmb, &sm.efull[stage], fc, up ? zrow : arow);
                tma_load_2d(bx + p.r_exp * 128, &tmb, &sm.efull[stage], fc, up ? arow + p.r_exp : zrow);
              }
            }
          }
          filled_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == p.e_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < p.e_stages; ++s)
          if (filled_mask & (1u << s)) {
            volatile int dummy = 0;
            mbar_wait(&sm.efull[s], (last_parity >> s) & 1u, &dummy, nullptr, kLtWaitNs / 4, 0);
          }
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ expand MMAs
    if (lane == 0) {
      int stage = 0, acc_i = 0, li = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t tz = tmem_base;
      for (int qi = 0; ok && !*abort_flag; ++qi) {
        int it;
        LtItem t;
        if (!lt_take(sm, qi, it, t, abort_flag, p.status, 32, true) || it < 0) break;
        if (!t.lora) continue;
        const int zb = li & 1;
        if (!mbar_wait(&sm.zready[zb], static_cast<uint32_t>(li >> 1) & 1u, abort_flag, p.status, kLtWaitNs, 33)) break;
        tc_fence_after();
        // delta[j][f] = sum_i B[i][f] z[i][j], one feature block of 128 per MMA group
        const uint32_t lidesc = umma_idesc_bf16(128, t.n_mma) | (1u << 15) | (1u << 16);  // A and B MN-major
        const uint64_t zdesc = umma_desc_mn_sw128(smem_u32(zs + zb * p.ztile_bytes), zlbo);
        // feature blocks side by side in an accumulator (n_mma columns each): a short
        // segment's whole expand fits in the three accumulators
        const int bpb = 128 / t.n_mma, ng = (nf + bpb - 1) / bpb;
        int bsub = 0;  // block within the current expand stage
        for (int g = 0; g < ng && ok; ++g, ++acc_i) {
          const int buf = acc_i % kLtAcc;
          const uint32_t use = static_cast<uint32_t>(acc_i / kLtAcc);
          if (!mbar_wait(&sm.tempty[buf], (use & 1u) ^ 1u, abort_flag, p.status, kLtWaitNs, 24)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int j = 0; j < bpb && g * bpb + j < nf; ++j) {
            if (bsub == 0) {
              if (!mbar_wait(&sm.efull[stage], phase, abort_flag, p.status, kLtWaitNs, 25)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint64_t adesc =
                umma_desc_mn_sw128(smem_u32(ering + stage * p.e_stage_bytes + bsub * p.expand_bytes), zlbo);
            const uint32_t td = tz + 128 + buf * 128 + j * t.n_mma;
            for (int kk = 0; kk < p.rbox / 16; ++kk)  // 16 rank rows (2048 B) per instruction
              umma_bf16(td, adesc + 128 * kk, zdesc + 128 * kk, lidesc, kk > 0 ? 1u : 0u);
            if (++bsub == p.bps || g * bpb + j == nf - 1) {  // the stage's last block: release it
              bsub = 0;
              umma_commit(&sm.eempty[stage]);
              if (++stage == p.e_stages) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
          if (!ok) break;
          umma_commit(&sm.tfull[buf]);
        }
        if (!ok) break;
        umma_commit(&sm.zdone[zb]);  // z tile zb may be rewritten once these MMAs complete
        ++li;
      }
      umma_commit(&sm.edone);
      volatile int dummy = 0;
      mbar_wait(&sm.edone, 0, &dummy, nullptr, kLtWaitNs, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ delta epilogue
    const int et = threadIdx.x - 128;     // 0..127
    const int g4 = warp & 3;              // TMEM lane quarter this warp may access
    const uint32_t lane_off = static_cast<uint32_t>(g4 * 32) << 16;
    int acc_i = 0;
    for (int qi = 0;; ++qi) {
      int it = -1;
      LtItem t{};
      const bool gq = lt_take(sm, qi, it, t, abort_flag, p.status, 29, false);
      if (!named_bar_and(3, kLtEpi, gq)) break;  // every thread has read the slot
      if (et == 0) mbar_arrive(&sm.qempty[qi % kLtQ]);
      if (it < 0) break;
      if (t.n <= 0) continue;
      // the item's delta rows, read once (the previous item's readers are past the
      // queue barrier above)
      for (int j = et; j < t.n; j += kLtEpi) sm.rowmap[j] = lt_delta_row(p, t.lo + j);
      named_bar_sync(3, kLtEpi);
      if (!t.lora) {  // no adapter: delta = 0 on the segment's rows, a warp per row
        const int f8 = p.F / 8;
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        for (int j = warp - 4; j < t.n; j += 4) {
          const int row = sm.rowmap[j];
          if (row < 0) continue;
          uint4* d = reinterpret_cast<uint4*>(p.delta + static_cast<size_t>(row) * p.F);
          for (int c = lane; c < f8; c += 32) d[c] = z4;
        }
        continue;
      }
      // expand accumulators -> delta rows (thread = feature, one store per row: a warp
      // writes 32 consecutive features of a row)
      bool stop = false;
      const int bpb = 128 / t.n_mma, ng = (nf + bpb - 1) / bpb;
      for (int g = 0; g < ng; ++g, ++acc_i) {
        const int buf = acc_i % kLtAcc;
        const uint32_t use = static_cast<uint32_t>(acc_i / kLtAcc);
        const bool got = mbar_wait(&sm.tfull[buf], use & 1u, abort_flag, p.status, kLtWaitNs, 27);
        if (!named_bar_and(3, kLtEpi, got)) {
          stop = true;
          break;
        }
        tc_fence_after();
        // accumulator column c holds row c % n_mma of feature block g bpb + c / n_mma; the
        // warp's 32 features x 32 columns go through its staging block (column writes),
        // then out as 16-byte runs of 8 features per row
        const int cols = min(bpb, nf - g * bpb) * t.n_mma;
        uint8_t* wst = stg + (g4 * kLtStgWarp);
        for (int c0 = 0; c0 < cols; c0 += 32) {
          float v[32];
          tmem_ld_32x32b_x32(tmem_base + lane_off + 128 + buf * 128 + c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            *reinterpret_cast<__nv_bfloat16*>(wst + j * kLtStgPitch + 2 * lane) = __float2bfloat16_rn(p.scale * v[j]);
          __syncwarp();
          // the 32 columns span at most two feature blocks (n_mma >= 16)
          const int blk0 = c0 / t.n_mma, tr0 = c0 - blk0 * t.n_mma;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int idx = lane + 32 * i;
            const int j = idx >> 2, q = idx & 3;
            const int c = c0 + j;
            int blk = blk0, tr = tr0 + j;
            if (tr >= t.n_mma) {
              tr -= t.n_mma;
              ++blk;
            }
            const int f8 = (g * bpb + blk) * 128 + g4 * 32 + 8 * q;
            const int row = (c < cols && tr < t.n && f8 + 8 <= p.F) ? sm.rowmap[tr] : -1;
            if (row >= 0)
              *reinterpret_cast<uint4*>(p.delta + static_cast<size_t>(row) * p.F + f8) =
                  *reinterpret_cast<const uint4*>(wst + j * kLtStgPitch + 16 * q);
          }
          __syncwarp();
        }
        tc_fence_before();
        mbar_arrive(&sm.tempty[buf]);
      }
      if (stop) break;
    }
  } else {
    // ------------------------------------------------------------ z: TMEM -> shared memory
    // z tile: MN-major with the 128-byte swizzle, block b of 64 rows at b rbox 128, rank row
    // i at i 128, 16-byte chunk c at (c ^ (i & 7))
    const int zt = threadIdx.x - 256;     // 0..127
    const int g4 = warp & 3;
    const int m = g4 * 32 + lane;         // rank row of the accumulator
    const uint32_t lane_off = static_cast<uint32_t>(g4 * 32) << 16;
    int li = 0;
    for (int qi = 0;; ++qi) {
      int it = -1;
      LtItem t{};
      const bool gq = lt_take(sm, qi, it, t, abort_flag, p.status, 34, false);
      if (!named_bar_and(4, kLtZ, gq)) break;
      if (zt == 0) mbar_arrive(&sm.qempty[qi % kLtQ]);
      if (it < 0) break;
      if (!t.lora) continue;
      const int zb = li & 1;
      bool got = mbar_wait(&sm.zfull, static_cast<uint32_t>(li) & 1u, abort_flag, p.status, kLtWaitNs, 26);
      // the MMAs that read this tile two items ago have completed
      got = got && mbar_wait(&sm.zdone[zb], (static_cast<uint32_t>(li >> 1) & 1u) ^ 1u, abort_flag, p.status,
                             kLtWaitNs, 35);
      if (!named_bar_and(4, kLtZ, got)) break;
      tc_fence_after();
      uint8_t* zt_base = zs + zb * p.ztile_bytes;
      if (g4 * 32 < p.rbox) {
        for (int c0 = 0; c0 < t.n_mma; c0 += 32) {
          float v[32];
          tmem_ld_32x32b_x32(tmem_base + lane_off + c0, v);
          if (m < p.rbox) {
            uint8_t* rowp = zt_base + (c0 >> 6) * (p.rbox * 128) + m * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int chunk = ((c0 & 63) >> 3) + q;
              if (c0 + 8 * q >= t.n_mma) break;
              uint4 w;
              if (m < p.r) {
                w = make_uint4(pack2_bf16(v[8 * q], v[8 * q + 1]), pack2_bf16(v[8 * q + 2], v[8 * q + 3]),
                               pack2_bf16(v[8 * q + 4], v[8 * q + 5]), pack2_bf16(v[8 * q + 6], v[8 * q + 7]));
              } else {
                w = make_uint4(0u, 0u, 0u, 0u);  // rank rows r..rbox-1 of the MMA's K
              }
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ (m & 7)) << 4)) = w;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.zfree);    // the shrink may overwrite the accumulator
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA
      mbar_arrive(&sm.zready[zb]);
      ++li;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// ---------------------------------------------------------------------------- host side

cudaError_t launch_lora_tc(const LoraTcArgs& a, cudaStream_t st) {
  if (a.nrows <= 0) return cudaSuccess;
  if (a.r < 8 || a.r > 128 || a.r % 8 != 0 || a.K % 8 != 0 || a.F % 8 != 0 || a.items == nullptr ||
      a.item_count == nullptr || a.delta == nullptr || a.src == nullptr || a.lora_a == nullptr || a.work_counter == nullptr ||
      a.lora_b == nullptr || a.L <= 0)
    return cudaErrorInvalidValue;
  // split: the shrink's rank is 2 r_exp and the expand's K the same (block-diagonal B)
  const int rbox = (a.r + 15) / 16 * 16;
  if (a.split_I != 0 && (a.split_I % 64 != 0 || a.r != 2 * a.r_exp || a.r % 16 != 0)) return cudaErrorInvalidValue;
  const int shrink_bytes = a.r * 128 + kLtN * 128;
  const int expand_bytes = 2 * rbox * 128;
  // after the rings: two z tiles, the delta staging, barriers; the shrink MMA reads 128 A
  // rows (16 KB) from each box pair's start, which may reach past the shrink ring into the
  // expand ring
  const int ztile = 2 * rbox * 128;
  const int tail = 2 * ztile + 4 * kLtStgWarp + static_cast<int>(sizeof(LtSmem));
  // the two rings share what is left, in proportion to the bytes an item streams through
  // each (shrink: the A rows and the rows' boxes over K; expand: the B boxes over F), at
  // least two stages each; expand stages of about 16 KB (one or more 64-feature-pair
  // blocks), shrink stages that hold at least the largest box pair
  const int bps = std::max(1, std::min(4, 16384 / expand_bytes));
  const int e_stage_bytes = bps * expand_bytes;
  const int rings = 232448 - 1024 - tail;
  const double s_item = static_cast<double>((a.K + 63) / 64) * (a.r + 32) * 128.0;  // rows boxes of ~32
  const double e_item = static_cast<double>((a.F + 127) / 128) * expand_bytes;
  int e_stages = static_cast<int>(rings * (e_item / (s_item + e_item)) / e_stage_bytes);
  e_stages = std::max(2, std::min(kLtMaxStages, e_stages));
  while (e_stages > 2 && rings - e_stages * e_stage_bytes < 2 * shrink_bytes) --e_stages;
  const int avail = rings - e_stages * e_stage_bytes;
  int s_stages = 4;
  int s_stage_bytes = avail / s_stages / 1024 * 1024;
  while (s_stages > 2 && s_stage_bytes < shrink_bytes) {
    --s_stages;
    s_stage_bytes = avail / s_stages / 1024 * 1024;
  }
  if (s_stage_bytes < shrink_bytes || e_stage_bytes < expand_bytes) return cudaErrorInvalidConfiguration;
  const size_t smem = 1024 + static_cast<size_t>(s_stages) * s_stage_bytes +
                      static_cast<size_t>(e_stages) * e_stage_bytes + tail;
  if (smem > 232448) return cudaErrorInvalidConfiguration;

  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(lora_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  CUtensorMap tx[kLtBoxes], ta, tb;
  const uint32_t box_rows[kLtBoxes] = {16, 24, 32, 48, 64, 128};
  for (int b = 0; b < kLtBoxes; ++b)
    if (encode_tmap_2d(&tx[b], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.src, a.K, a.nrows,
                       static_cast<uint64_t>(a.K) * 2, 64, box_rows[b], CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  const uint64_t slot_rows = static_cast<uint64_t>(a.L) * a.E * a.r;
  if (encode_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_a, a.K, slot_rows, static_cast<uint64_t>(a.K) * 2,
                     64, a.r, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS ||
      encode_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_b, a.split_I ? a.split_I : a.F, slot_rows,
                     static_cast<uint64_t>(a.split_I ? a.split_I : a.F) * 2, 64, a.split_I ? a.r_exp : rbox,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  LoraTcParams p;
  p.items = a.items;
  p.item_count = a.item_count;
  p.seg_off = a.seg_offsets;
  p.nseg = a.nseg;
  p.seg_adapter = a.seg_adapter;
  p.L = a.L;
  p.E = a.E;
  p.K = a.K;
  p.r = a.r;
  p.rbox = rbox;
  p.F = a.F;
  p.nrows = a.nrows;
  p.s_stages = s_stages;
  p.s_stage_bytes = s_stage_bytes;
  p.e_stages = e_stages;
  p.e_stage_bytes = e_stage_bytes;
  p.bps = bps;
  p.expand_bytes = expand_bytes;
  p.ztile_bytes = ztile;
  p.delta = a.delta;
  p.scatter = a.scatter;
  p.status = a.status;
  p.work_counter = a.work_counter;
  p.lora_b = a.lora_b;
  p.split_I = a.split_I;
  p.r_exp = a.split_I ? a.r_exp : a.r;
  p.scale = a.scale;
  p.pdl_trigger = a.pdl_trigger;
  int grid = a.num_sms > 0 ? a.num_sms : 148;
  if (a.items_bound < grid) grid = a.items_bound;
  if (grid < 1) grid = 1;
  ProfScope ps(a.prof_id, st);
  lora_tc_kernel<<<grid, kLtThreads, smem, st>>>(tx[0], tx[1], tx[2], tx[3], tx[4], tx[5], ta, tb, p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace mlb
