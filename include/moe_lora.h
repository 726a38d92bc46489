/*
 * moe_lora.h -- C ABI of libmoe_lora.so: batched multi-tenant LoRA on a
 * Mixture-of-Experts FFN layer, and dense segmented LoRA (SGMV), for NVIDIA B200
 * (sm_100a).
 *
 * Sources of the operations (web pages, cited by page and section):
 *   [vLLM MoE-LoRA page]   "vllm-moe-lora-sagemaker-bedrock" (wp.cloudtroop.com.br):
 *       "Entendendo os Modelos MoE"     router, experts, gate_up then down, aggregation
 *       "O Papel da Multi-LoRA"         y = xW + xAB, shrink z = xA, expand zB
 *       "Implementação Técnica no vLLM" fused_moe_lora; expert routing x adapter selection
 *       "Otimizações em Nível de Kernel" split-K shrink, fused add in expand
 *   [SageMaker MoE kernels page] "aws-sagemaker-moe-kernel-optimizations" (aib.vote):
 *       first item: top-k = 8, operand swap so the wide expert dim fills the MMA M slot;
 *       second item: FP8 per-tensor MoE, scale + GEMM + expert aggregation in one pass.
 *   [Punica review page]   "Punica: Multi-Tenant LoRA Serving" (nubint.ai):
 *       "提案手法" segmented gather matrix-vector multiplication (SGMV).
 *
 * Conventions for every call
 *   - Pointers are DEVICE pointers unless stated otherwise; the caller allocates and
 *     owns every buffer (inputs, outputs, workspace).  The library never allocates,
 *     frees or synchronises inside a call (moe_lora_check_status excepted).
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  No host read-back happens inside a call.
 *   - Every tensor must be 16-byte aligned; rows are dense (row stride = row length).
 *   - Host-side validation errors return at once with nothing enqueued.  Launch
 *     failures return MOE_LORA_ERR_CUDA.  moe_lora_last_error() gives the message.
 *   - Data-dependent errors found on the device (an adapter id >= L, offsets that are
 *     not monotone, a bounded wait that ran out) do not trap: the kernel records a
 *     status word in the workspace and skips the offending work.  The call clears that
 *     word first; moe_lora_check_status() reads it.
 *   - bf16 = bfloat16; e4m3 = OCP FP8 E4M3 ("fn": max 448, no infinities).
 *   - Weight storage (K-major: each row is one output feature, contiguous over the
 *     reduction dim): expert gate_up w_gu [E][2I][H] with the gate in rows [0, I) and
 *     the up projection in rows [I, 2I); expert down w_d [E][H][I]; dense W [h_out][h_in].
 *     LoRA A is stored transposed as [.. ][r][h_in]; LoRA B as [.. ][r][h_out].
 *   - Adapter scaling: y = xW + s (xA)B with s = 1 unless moe_lora_forward's format sets
 *     a per-projection scale (an alpha / r factor).
 *
 * Environment switches (read at each call; none changes a result beyond rounding order)
 *   MOE_LORA_EXPAND=delta|tc    where the LoRA work of the grouped GEMMs runs: "delta", the
 *                               segmented CUDA-core LoRA kernel writes fp32 deltas (decode:
 *                               gate_up's added by the GEMM epilogue, down's by the
 *                               combine); "tc", the tensor-core LoRA kernel (shrink and
 *                               expand on tcgen05, z on chip) writes bf16 deltas (prefill).
 *                               Default: "tc" above 64 rows per expert, "delta" below.
 *   MOE_LORA_PAIR=0|1           N tiles of 256 on CTA pairs (tcgen05 cta_group::2, M = 256);
 *                               default 1.
 *   MOE_LORA_SWAP=0             tiles of 256 with tokens in the MMA's M (128 tokens x 256 weight
 *                               rows per CTA) instead of weights in M; bf16 weights and the
 *                               tensor-core LoRA placement only (default: weights in M).
 *   MOE_LORA_FORCE_BN=16|32|64|128|256  the GEMM's token tile (default: from the mean rows
 *                               per group: <= 12 -> 16, <= 24 -> 32, <= 64 -> 64, <= 96 -> 128,
 *                               else 256).
 */
#ifndef MOE_LORA_H
#define MOE_LORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_LORA_API __attribute__((visibility("default")))
#else
#define MOE_LORA_API
#endif

typedef struct CUstream_st* moe_lora_stream;  /* same handle as cudaStream_t */

typedef enum {
  MOE_LORA_OK = 0,
  MOE_LORA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad enum      */
  MOE_LORA_ERR_UNSUPPORTED = 2,   /* valid but outside the supported shape range      */
  MOE_LORA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed                */
  MOE_LORA_ERR_DEVICE_CHECK = 4,  /* a device-side data check failed (see above)      */
  MOE_LORA_ERR_TIMEOUT = 5        /* a bounded device-side wait ran out               */
} moe_lora_status;

typedef enum { ML_F32 = 0, ML_BF16 = 1, ML_E4M3 = 2 } ml_dtype;

typedef enum {
  MOE_LORA_OP_ROUTE = 0,
  MOE_LORA_OP_FORWARD = 1,
  MOE_LORA_OP_SGMV_SHRINK = 2,
  MOE_LORA_OP_SGMV_EXPAND = 3,
  MOE_LORA_OP_DENSE = 4,
  MOE_LORA_OP_FORWARD_BF16 = 5,  /* moe_lora_forward with ML_BF16 experts only  */
  MOE_LORA_OP_FORWARD_E4M3 = 6   /* moe_lora_forward with ML_E4M3 experts only  */
} moe_lora_op;

/* Supported ranges (outside them: MOE_LORA_ERR_UNSUPPORTED).
 *   r in {8, 16, 32, 64, 128}; 1 <= k <= E <= 256; 0 <= L <= 64;
 *   H, I, h_in, h_out multiples of 8 (16-byte rows); M*k <= 2^20. */

/* ---------------------------------------------------------------------------------
 * moe_lora_route -- router logits, softmax top-k with renormalised weights, and the
 * stable (expert, adapter) sort of the M*k routing pairs.
 *
 * Defines: a router sends each token to its most relevant experts ([vLLM MoE-LoRA
 * page], "Entendendo os Modelos MoE"); top-k with k = 8 ([SageMaker MoE kernels
 * page], first item); expert routing and adapter selection are the two sparsity
 * sources the MoE-LoRA kernel combines ([vLLM MoE-LoRA page], "Implementação
 * Técnica no vLLM"), hence the sort by (expert, adapter).
 *
 *   x          bf16 [M, H] tokens; may be NULL when logits_in is given.
 *   w_router   bf16 [E, H] router weight (row e = expert e); NULL with logits_in.
 *   bias       fp32 [E] per-expert logit bias, or NULL.
 *   logits_in  fp32 [M, E] precomputed logits, or NULL to compute l = x W_r^T + bias
 *              (fp32 accumulation).
 *   adapter_ids int32 [M]: adapter of each token in [0, L), or -1 = no adapter.
 *   logits_out fp32 [M, E] or NULL: the logits the selection used.
 *   topk_ids   int32 [M, k]: the k experts of largest logit, descending; equal
 *              logits go to the lower expert index.
 *   topk_w     fp32 [M, k]: softmax over all E logits, renormalised over the k
 *              selected (equal to the softmax of the k selected logits).
 *   sorted_pairs int32 [M*k]: the pair indices p = t*k + j sorted stably by key
 *              e*(L+1) + a' (a' = a(t) if a(t) >= 0 else L); ascending p within a key.
 *   seg_offsets int32 [E*(L+1)+1]: CSR offsets of the keys into sorted_pairs.
 *   workspace  >= moe_lora_workspace_size(MOE_LORA_OP_ROUTE, M, H, 0, E, k, L, 0) bytes.
 * Outputs are bit-exact and deterministic for given logits.  An adapter id outside
 * [-1, L) sets MOE_LORA_ERR_DEVICE_CHECK and is treated as -1.  M = 0: OK, nothing
 * enqueued except the zeroing of seg_offsets.
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status moe_lora_route(
    const void* x, const void* w_router, const float* bias, const float* logits_in,
    const int32_t* adapter_ids, int M, int H, int E, int k, int L,
    float* logits_out, int32_t* topk_ids, float* topk_w,
    int32_t* sorted_pairs, int32_t* seg_offsets,
    void* workspace, size_t workspace_bytes, moe_lora_stream stream);

/* Layout and scaling of the adapters given to moe_lora_forward (NULL: the defaults,
 * which are {0, 1.0f, 1.0f}).  Each projection carries its own adapter on the pages
 * ([vLLM MoE-LoRA page], "O Papel da Multi-LoRA": one A and one B per projection).
 *   gate_up_split  0: one adapter on the fused gate_up projection,
 *                     lora_a_gu [L][E][r][H], lora_b_gu [L][E][r][2I];
 *                  1: separate gate and up adapters, lora_a_gu [L][E][2][r][H] and
 *                     lora_b_gu [L][E][2][r][I] (index 0 = gate, 1 = up); needs r <= 64.
 *   scale_gu       multiplies the gate_up delta (both halves), e.g. alpha / r.
 *   scale_d        multiplies the down delta. */
typedef struct {
  int gate_up_split;
  float scale_gu;
  float scale_d;
} moe_lora_adapter_format;

/* ---------------------------------------------------------------------------------
 * moe_lora_forward -- the MoE FFN with per-(adapter, expert) LoRA on gate_up and
 * down, and the top-k weighted combine.  For every routing pair p = (t, j), with
 * e = topk_ids[t, j] and a = a(t):
 *   h   = s_gu[e] * W_gu[e] x_t + [a >= 0] c_gu (x_t A_gu[a,e]) B_gu[a,e]   (2I)
 *   act = silu(h[0:I]) * h[I:2I],  silu(g) = g / (1 + exp(-g))             (I)
 *   o   = s_d[e] * W_d[e] act + [a >= 0] c_d (act A_d[a,e]) B_d[a,e]        (H)
 * (c_gu, c_d: the format's scales; with separate gate and up adapters the gate half of
 * the gate_up delta is (x_t A_gate) B_gate and the up half (x_t A_up) B_up)
 *   y_t = sum_j topk_w[t, j] * o_(t, j)      (fixed j order: deterministic)
 * Defines: expert gate_up/down ([vLLM MoE-LoRA page], "Entendendo os Modelos MoE"),
 * y = xW + xAB per projection, per expert and per adapter ("O Papel da Multi-LoRA"),
 * shrink/expand fused with the base MoE GEMMs ("Implementação Técnica no vLLM",
 * fused_moe_lora); FP8 per-tensor scaled experts with scale, GEMM and expert
 * aggregation in one pass ([SageMaker MoE kernels page], second item).
 *
 *   x            bf16 [M, H].
 *   topk_w, sorted_pairs, seg_offsets: as written by moe_lora_route for the same
 *                M, E, k, L (the adapter of every pair is read from its key).
 *   w_gateup     [E][2I][H], w_down [E][H][I], of type w_dtype (ML_BF16 or ML_E4M3).
 *   w_scales     fp32 [E][2] = (s_gu, s_d) per expert when w_dtype = ML_E4M3; NULL
 *                for ML_BF16 (scales 1).
 *   lora_a_gu    bf16 [L][E][r][H];  lora_b_gu bf16 [L][E][r][2I] (split: see above);
 *   lora_a_d     bf16 [L][E][r][I];  lora_b_d  bf16 [L][E][r][H]  (NULL iff L = 0).
 *   format       adapter layout and scales, or NULL for the defaults.
 *   y            bf16 [M, H] output (overwritten).
 *   workspace    >= moe_lora_workspace_size(MOE_LORA_OP_FORWARD, M, H, I, E, k, L, r)
 *                (either expert type), or the smaller size of MOE_LORA_OP_FORWARD_BF16 /
 *                MOE_LORA_OP_FORWARD_E4M3 for that expert type.
 * Intermediates (gathered rows, z, act, per-pair outputs) live in the workspace.
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status moe_lora_forward(
    const void* x, int M, int H, int I, int E, int k, int L, int r,
    const float* topk_w, const int32_t* sorted_pairs, const int32_t* seg_offsets,
    const void* w_gateup, const void* w_down, ml_dtype w_dtype, const float* w_scales,
    const void* lora_a_gu, const void* lora_b_gu, const void* lora_a_d, const void* lora_b_d,
    const moe_lora_adapter_format* format, void* y, void* workspace, size_t workspace_bytes,
    moe_lora_stream stream);

/* ---------------------------------------------------------------------------------
 * sgmv_shrink -- segmented gather matrix-vector shrink: z_t = x_t A_{a(s)} for every
 * token t in segment s = [seg_offsets[s], seg_offsets[s+1]), a(s) = seg_adapter[s].
 * Defines: SGMV over contiguous per-adapter segments ([Punica review page],
 * "提案手法"); shrink z = xA with split-K reduction ([vLLM MoE-LoRA page],
 * "O Papel da Multi-LoRA", "Otimizações em Nível de Kernel").
 *
 *   x           [T, h_in] of type dt (ML_F32 or ML_BF16).
 *   lora_a      [L][r][h_in] of type dt.
 *   seg_offsets int32 [S+1], non-decreasing, seg_offsets[0] = 0, seg_offsets[S] = T.
 *   seg_adapter int32 [S], in [-1, L); -1 = no adapter (z rows set to 0).
 *   z           fp32 [T, r] output (overwritten).
 *   workspace   >= moe_lora_workspace_size(MOE_LORA_OP_SGMV_SHRINK, T, h_in, 0, 1, 1, L, r).
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status sgmv_shrink(
    const void* x, const void* lora_a, const int32_t* seg_offsets, const int32_t* seg_adapter,
    int S, int T, int h_in, int r, int L, ml_dtype dt, float* z,
    void* workspace, size_t workspace_bytes, moe_lora_stream stream);

/* ---------------------------------------------------------------------------------
 * sgmv_expand -- y_t += z_t B_{a(s)} per segment (fused add into the base output:
 * [vLLM MoE-LoRA page], "Otimizações em Nível de Kernel"; SGMV per [Punica review
 * page], "提案手法").  Tokens of segments with adapter -1 are left unchanged.
 *
 *   z           fp32 [T, r];  lora_b [L][r][h_out] of type dt;
 *   y           [T, h_out] of type dt, read and written in place.
 *   workspace   >= moe_lora_workspace_size(MOE_LORA_OP_SGMV_EXPAND, T, 0, h_out, 1, 1, L, r).
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status sgmv_expand(
    const float* z, const void* lora_b, const int32_t* seg_offsets, const int32_t* seg_adapter,
    int S, int T, int h_out, int r, int L, ml_dtype dt, void* y,
    void* workspace, size_t workspace_bytes, moe_lora_stream stream);

/* ---------------------------------------------------------------------------------
 * dense_lora_forward -- one dense projection with segmented multi-LoRA:
 *   y_t = W x_t + [a(t) >= 0] (x_t A_a(t)) B_a(t)
 * ([vLLM MoE-LoRA page], "O Papel da Multi-LoRA"; batched across adapters by
 * segments as in SGMV, [Punica review page]).  ML_BF16 runs the base GEMM on the
 * tensor cores with the expand fused into its epilogue; ML_F32 runs on CUDA cores.
 *
 *   x [T, h_in], w [h_out][h_in], lora_a [L][r][h_in], lora_b [L][r][h_out], all dt;
 *   segments as in sgmv_shrink;  y [T, h_out] of type dt (overwritten).
 *   workspace >= moe_lora_workspace_size(MOE_LORA_OP_DENSE, T, h_in, h_out, 1, 1, L, r).
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status dense_lora_forward(
    const void* x, const void* w, const void* lora_a, const void* lora_b,
    const int32_t* seg_offsets, const int32_t* seg_adapter, int S, int T,
    int h_in, int h_out, int r, int L, ml_dtype dt, void* y,
    void* workspace, size_t workspace_bytes, moe_lora_stream stream);

/* ---------------------------------------------------------------------------------
 * moe_lora_route_noalloc -- moe_lora_route for callers that cannot allocate device
 * memory.  The pages have no counterpart to this entry point; it exists for callers
 * that receive only their input and output buffers from a host framework (a plugin
 * or custom-op interface with no workspace) and may not call cudaMalloc themselves,
 * because an allocation can synchronise the device, is not allowed during stream
 * capture, or would break a memory budget planned in advance.
 *
 * Arguments, outputs and results are those of moe_lora_route, without the workspace.
 * The scratch (status word, per-key counts, per-token keys, and the logits when
 * logits_out is NULL) lives in one fixed array of about 1.07 MiB that the library
 * defines; every GPU that loads the library holds it until the process exits.
 *   - Limits: M <= 1024, k <= E <= 256, L <= 64; larger sizes return
 *     MOE_LORA_ERR_UNSUPPORTED with nothing enqueued.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.
 *   - Every call uses the same array and leaves its contents behind; each call clears
 *     what must start at zero.  Calls that overlap on the GPU (concurrent streams, or
 *     several host threads on one device) race on the array and must be serialised by
 *     the caller.
 *   - Nothing is allocated or freed.  Device-side data checks (an adapter id outside
 *     [-1, L)) are applied as in moe_lora_route, but their status word is not readable
 *     through this entry point.
 * ------------------------------------------------------------------------------- */
MOE_LORA_API moe_lora_status moe_lora_route_noalloc(
    const void* x, const void* w_router, const float* bias, const float* logits_in,
    const int32_t* adapter_ids, int M, int H, int E, int k, int L,
    float* logits_out, int32_t* topk_ids, float* topk_w,
    int32_t* sorted_pairs, int32_t* seg_offsets, moe_lora_stream stream);

/* Workspace bytes for one call of `op` (arguments not used by the op are ignored;
 * for the SGMV/dense ops pass T as M, h_in as H and h_out as I).  Returns 0 for an
 * unknown op. */
MOE_LORA_API size_t moe_lora_workspace_size(int op, int M, int H, int I, int E, int k, int L, int r);

/* Synchronises `stream`, returns the device status word recorded in `workspace` by
 * the last call that used it (MOE_LORA_OK if none), and clears it.  Host only. */
MOE_LORA_API moe_lora_status moe_lora_check_status(void* workspace, moe_lora_stream stream);

/* Thread-local message for the last non-OK status returned on this thread. */
MOE_LORA_API const char* moe_lora_last_error(void);

/* Measurement hooks (off by default; used by benchmarks, never by the hot path).
 * moe_lora_profile_enable(n) creates a pool of 2n CUDA events and from then on
 * records one event pair around each kernel launch of the library, on the launch's
 * stream, for up to n launches; n = 0 disables and frees the pool.  Kernel ids:
 *   0 router logits, 1 top-k, 2 sort, 3 SGMV shrink, 4 gate_up GEMM, 5 down GEMM,
 *   6 combine, 7 SGMV expand, 8 fp32 dense GEMM, 9 dense bf16 GEMM,
 *   10 e4m3 activation planes, 11 segmented LoRA of gate_up (or dense) and the LoRA
 *   work lists, 12 one-launch routing (small batches), 13 segmented LoRA of down,
 *   14 token-row gather into (expert, adapter) order.
 * Launches captured into a CUDA graph record their events as graph nodes, so every
 * replay of the graph re-records them (the last replay's times are read).
 * moe_lora_profile_read() waits for the recorded events and returns the summed
 * device time (ms) and the number of recorded launches of one kernel id.
 * moe_lora_launch_count() counts every kernel launch of the library since load. */
MOE_LORA_API moe_lora_status moe_lora_profile_enable(int max_launches);
MOE_LORA_API moe_lora_status moe_lora_profile_read(int kernel_id, double* total_ms, int* launches);
MOE_LORA_API long long moe_lora_launch_count(void);

/* Library version string, e.g. "moe_lora_b200 0.1 sm_100a". */
MOE_LORA_API const char* moe_lora_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LORA_H */
