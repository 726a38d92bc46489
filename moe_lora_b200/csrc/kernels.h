// Host-side launch interfaces between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_lora.h"

namespace mlb {

struct RouteArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* w_router;
  const float* bias;
  const float* logits_in;
  const int32_t* adapter_ids;
  int M, H, E, k, L;
  float* logits;          // where computed logits go (logits_out or workspace)
  float* logits_out;      // may be null
  int32_t* topk_ids;
  float* topk_w;
  int32_t* sorted_pairs;
  int32_t* seg_offsets;
  int32_t* key_count;     // workspace [E*(L+1)]
  int32_t* a_key;         // workspace [max(M, ceil(M / 8) + 1)]: adapter keys, or the
                          // tickets of the one-launch routing
  int* status;
  int num_sms;
  int tickets_zeroed = 0;  // the caller's status clear already zeroed the tickets
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
// Tickets (ints at a_key) of the one-launch routing for M tokens of k pairs, or 0 when the
// routing takes the multi-kernel path.
int route_fused_tickets(int M, int k);

// Segmented shrink z[s] = src_row(s) . A_seg(s)^T (SIMT: 128-bit loads, warp-shuffle
// split-K reduction).  Segments come either from a dense (offsets, adapter) table or
// from MoE keys q = e*(L+1) + a' (seg_adapter == null).
struct ShrinkArgs {
  const void* src;            // rows [*, K], f32 or bf16
  bool src_f32;
  const int32_t* gather;      // if set: source row of output row s = gather[s] / gather_div
  int gather_div;
  __nv_bfloat16* gather_dst;  // if set: copy of the gathered source row (bf16 rows [nrows, K])
  int nrows, K, r;
  const int32_t* seg_offsets; // [nseg+1]
  int nseg;
  const int32_t* seg_adapter; // dense: [nseg]; null: MoE key decode
  int L, E;
  const void* lora_a;         // dense [L][r][K]; MoE [L][E][r][K] (same dtype as src)
  float* z;                   // [nrows][r]
  int32_t* row_adapter;       // out: adapter per row (-1 none), may be null
  int rows_per_cta;
  int* status;
};
cudaError_t launch_shrink(const ShrinkArgs& a, cudaStream_t st);

// Segmented LoRA for the GEMMs: per segment, gather the source rows (optional) and
// shrink z = src . A^T; then either write z (bf16) for a GEMM that runs the expand as
// extra MMA K steps, or expand delta = z . B into an fp32 buffer that the GEMM epilogue
// adds (rows without an adapter get delta = 0).  bf16 only; one kernel launch.
// Shared memory a CTA of the SIMT LoRA kernel needs on an SM beside a GEMM CTA (its
// static arrays and the driver's per-CTA reservation): a GEMM launched behind that kernel
// leaves this much free.
constexpr int kLoraCoresidentSmem = 8192;

struct LoraDeltaArgs {
  const __nv_bfloat16* src;   // rows [*, K]
  const int32_t* gather;      // if set: source row of output row s = gather[s] / gather_div
  int gather_div;
  int nsrc;                   // source rows (bound of the gathered indices)
  __nv_bfloat16* gather_dst;  // if set: copy of the gathered source row
  int nrows, K, r, NB;        // NB = delta features per row
  const int32_t* seg_offsets; // [nseg+1]
  int nseg;
  const int32_t* seg_adapter; // dense: [nseg]; null: MoE key decode
  int L, E;
  const __nv_bfloat16* lora_a;  // MoE [L][E][r][K]; dense [L][r][K]
  const __nv_bfloat16* lora_b;  // MoE [L][E][r][NB]; dense [L][r][NB]
  float* delta;               // [nrows][NB] (expand in this kernel) or null
  // e4m3 experts: the two activation planes of the source rows (in row order), written
  // by the CTAs of feature slice / K slice 0 (see launch_quant_planes); null otherwise
  uint8_t* q_hi;
  uint8_t* q_lo;
  float* q_scales;            // [nrows][2]
  float* z_part;              // optional scratch for the split form: [ceil(K / 1024)][nrows][r]
  long long z_part_cap;       // floats available at z_part
  // work list (launch_lora_plan): one item (segment, first row) per chunk of rb rows
  int2* items;                // [items_bound]
  int* item_count;
  int items_bound;            // lora_items_bound(nrows, nseg, rb)
  int rb;                     // lora_rows_per_chunk(nrows, nseg)
  int* status;
  int num_sms;
  // delta row of gathered row s: scatter[s] (a routing pair, so that the combine reads
  // delta in pair order) instead of s; null = s
  const int32_t* scatter;
  // expand: r_exp rank rows of B per delta feature (r for fused adapters); split_I > 0:
  // separate gate and up adapters (A = the 2 r_exp rows of both, B = [2][r_exp][split_I]);
  // every delta value is multiplied by scale; r_exp = 0 means r
  int r_exp = 0;
  int split_I = 0;
  float scale = 1.f;
  int prof_id = 11;  // measurement hook id of the launch (K_LORA or K_LORA_DOWN)
  // programmatic dependent launch: pdl_trigger lets the next kernel start right away;
  // pdl_secondary launches this one behind the running kernel ahead of it, and the
  // kernel then waits for that kernel before it exits; pdl_after_plan launches it behind
  // the work-list kernel, whose list it waits for before reading it.  Any of them forces
  // the one-kernel form.
  int pdl_trigger;
  int pdl_secondary;
  int pdl_after_plan = 0;
  int clear_status = 0;  // launch_lora_plan: zero the status block first (the call's first kernel)
};
int lora_rows_per_chunk(int nrows, int nseg);
int lora_items_bound(int nrows, int nseg, int rb);
cudaError_t launch_lora_plan(const LoraDeltaArgs& a, cudaStream_t st);
cudaError_t launch_lora_delta(const LoraDeltaArgs& a, cudaStream_t st);

// Tensor-core segmented LoRA for long segments: per work item (a chunk of up to kLtN
// rows of one segment) shrink z = src A_a and expand delta = z B_a on tcgen05, z kept on
// chip; delta rows (bf16, [nrows][F]) for the grouped GEMM's epilogue.  Items of
// segments without an adapter write delta = 0 rows.  Work list: lora_plan over every
// segment with chunks of kLtN rows.
constexpr int kLtN = 128;
struct LoraTcArgs {
  const __nv_bfloat16* src;     // rows [nrows][K] (gathered x, or act)
  int nrows, K, r, F;
  const int32_t* seg_offsets;   // [nseg + 1]
  int nseg;
  const int32_t* seg_adapter;   // dense: [nseg]; null: MoE keys q = e (L + 1) + a'
  int L, E;
  const __nv_bfloat16* lora_a;  // MoE [L][E][r][K]; dense [L][r][K]
  const __nv_bfloat16* lora_b;  // MoE [L][E][r][F]; dense [L][r][F]
  const int2* items;
  const int* item_count;
  int items_bound;
  __nv_bfloat16* delta;         // [nrows][F]
  const int32_t* scatter;       // delta row of gathered row s: scatter[s] (pair order); null = s
  int* status;
  int* work_counter;            // int in device memory, zero before the launch (work claiming)
  int num_sms;
  // separate gate and up adapters: split_I = I (a multiple of 64), r = 2 r_exp (A holds
  // both adapters' rows), B [L][E][2][r_exp][I]; 0 = one fused adapter (B [..][r][F])
  int split_I = 0;
  int r_exp = 0;                // 0 means r
  float scale = 1.f;            // multiplies every delta value
  int prof_id = 11;             // measurement hook id of the launch (K_LORA or K_LORA_DOWN)
  int pdl_trigger = 0;          // the kernel behind this one (PDL) may launch at once
};
cudaError_t launch_lora_tc(const LoraTcArgs& a, cudaStream_t st);

// dst[i] = src[gather[i] / div] for i < rows (bf16 rows of K elements; a source index
// outside [0, nsrc) gives a zero row).
// clear_status (if set): the call's status block, zeroed by the kernel's first CTA before
// any later kernel of the call runs (so the first kernel of a call replaces a memset).
cudaError_t launch_gather_rows(const __nv_bfloat16* src, int nsrc, const int32_t* gather, int div, int rows, int K,
                               __nv_bfloat16* dst, cudaStream_t st, int* clear_status = nullptr);
// Work list of every non-empty segment (with or without an adapter), chunks of rb rows.
// clear_status: zero the status block first (the plan kernel is then the call's first).
cudaError_t launch_lora_plan_all(const int32_t* seg_offsets, const int32_t* seg_adapter, int nseg, int L, int nrows,
                                 int rb, int2* items, int* count, int cap, int* status, cudaStream_t st,
                                 bool clear_status = false);

// y[t] += z[t] . B_a(t) for dense segments (f32 or bf16 y and B).
struct ExpandArgs {
  const float* z;
  const void* lora_b;         // [L][r][h_out]
  bool f32;
  const int32_t* seg_offsets;
  int nseg;
  const int32_t* seg_adapter;
  int L, T, h_out, r;
  void* y;
  int* status;
};
cudaError_t launch_expand(const ExpandArgs& a, cudaStream_t st);

// fp32 SIMT base GEMM with the LoRA expand fused in its epilogue:
// y[t][f] = sum_k x[t][k] W[f][k] + sum_i z[t][i] B[a(t)][i][f].
struct DenseF32Args {
  const float* x;
  const float* w;
  const float* lora_b;        // [L][r][h_out]
  const float* z;             // [T][r]
  const int32_t* row_adapter; // [T]
  int T, h_in, h_out, r, L;
  float* y;
};
cudaError_t launch_dense_f32(const DenseF32Args& a, cudaStream_t st);

// Tensor-core grouped GEMM with operand swap: the weight rows fill the 128-row MMA
// M slot, the tokens of one expert (or of the dense batch) the N slot.
enum EpiKind : int { EPI_GATEUP = 0, EPI_DOWN = 1, EPI_DENSE = 2, EPI_LOGITS = 3 };

struct GemmArgs {
  int epi;
  bool w_fp8;
  int K;                       // reduction length
  int E;                       // groups (experts); 1 for dense
  const int32_t* group_offsets;  // row offsets of group g at group_offsets[g * group_stride];
                               // null: one group of total_rows rows
  int group_stride;
  int rows_per_group;          // weight rows per expert (2I for gate_up, H for down, h_out)
  int n_out;                   // output features per group (I for gate_up, H, h_out)
  int I;                       // gate_up: gate/up split
  int total_rows;              // rows of the B operand tensor
  // LoRA delta added in the epilogue: [total_rows][delta_cols] fp32, column = weight row
  // within the group (gate_up: gate rows [0, I), up rows [I, 2I)); null = no LoRA
  const float* delta;
  int delta_cols;
  // the same as a bf16 delta (from the tensor-core LoRA kernel), read by the epilogue
  // straight from global memory; exclusive with delta
  const __nv_bfloat16* delta_bf16;
  // epilogue outputs
  __nv_bfloat16* out_bf16;     // gate_up: act [rows][I]; down: o [pairs][H] (weighted); dense: y [T][h_out]
  float* out_f32;              // logits: [rows][n_out]
  const float* bias;           // logits: [n_out] or null
  const int32_t* sorted_pairs; // down: pair index of each sorted row
  const float* topk_w;         // down: routing weight per pair
  const float* w_scales;       // fp8: [E][2]
  int scale_idx;               // 0 gate_up, 1 down
  int* status;
  // operands
  const void* w;               // weights [E*rows_per_group][K]
  const __nv_bfloat16* b;      // bf16 weights: token rows [total_rows][K]
  const uint8_t* b_hi;         // e4m3 weights: token rows as two e4m3 planes [total_rows][K]
  const uint8_t* b_lo;
  const float* b_scales;       // [total_rows][2] = (s, s / 16)
  int bn;                      // N tile (16..256)
  int num_sms;
  // tests only: > 0 makes CTA 0 skip the copies of its first stage and shortens every
  // bounded wait to this many milliseconds (the MMA's wait runs out: MOE_LORA_ERR_TIMEOUT)
  int test_stall_ms;
  // programmatic dependent launch: pdl_trigger lets the next kernel start right away;
  // pdl_secondary launches the GEMM behind the running kernel ahead of it (the LoRA
  // kernel that writes the fp32 delta): only the epilogue's loader waits for that kernel,
  // so the weight stream and the MMAs start at once
  int pdl_trigger;
  int pdl_secondary;
  // launched behind a kernel whose output it does not read (PDL): it waits for that
  // kernel only before it exits
  int pdl_end_wait = 0;
  // the kernel ahead holds its SMs' shared memory (the tensor-core LoRA kernel): keep the
  // full shared memory, nothing runs beside this kernel's CTAs
  int pdl_full_smem = 0;
};
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st);

// Rows of bf16 values as two e4m3 planes: hi = RNE(x / s), lo = RNE((x - hi s) / (s / 16)),
// s = amax(row) / 448; scales[row] = (s, s / 16).
cudaError_t launch_quant_planes(const __nv_bfloat16* src, int rows, int K, uint8_t* hi, uint8_t* lo, float* scales,
                                cudaStream_t st);

// y[t] = sum_j (o[t*k + j] + w[t*k + j] delta[t*k + j])  (o bf16, already weighted; delta
// in pair order, fp32 or bf16, optional), fixed j order, fp32 sum, bf16 out.
cudaError_t launch_combine(const __nv_bfloat16* o, int M, int k, int H, const float* delta,
                           const __nv_bfloat16* delta_bf16, const float* topk_w, __nv_bfloat16* y, cudaStream_t st);
// The e4m3 activation planes of gathered rows (see launch_quant_planes): plane row i from
// src[gather[i] / div]; copy (if set) also receives the gathered bf16 rows.
cudaError_t launch_gather_quant(const __nv_bfloat16* src, int nsrc, const int32_t* gather, int div, int rows, int K,
                                uint8_t* hi, uint8_t* lo, float* scales, __nv_bfloat16* copy, cudaStream_t st,
                                int* clear_status = nullptr);

// Host state that CUDA keeps per device (function attributes, SM counts, capability)
// is cached per device index, for processes that drive several GPUs.
constexpr int kMaxDevices = 64;
// The current device's index in [0, kMaxDevices), or -1 when there is none.
int current_device_index();
// MOE_LORA_OK on an sm_100a device; the library's status code otherwise (message set).
moe_lora_status check_current_device();

// driver entry point for tensor map encoding (resolved once)
bool tensor_map_encode_available();
CUresult encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                        uint32_t box_rows, CUtensorMapSwizzle swz);

}  // namespace mlb
