/*
 * moeffn.h -- C ABI of the quantized gated FFN / Mixture-of-Experts layer
 * library for NVIDIA B200 (sm_100a), libmoeffn.so.
 *
 * The layer computed is the FFN half of a transformer layer as three model
 * families run it in the turbospark-runtime pages:
 *
 *   h = down_proj( act(gate_proj @ m) * (up_proj @ m) )
 *     llama / Mistral dense layer: x = x + h (raw residual add only)
 *       -- turbospark-runtime 0.3.0, src/families/llama/dense.rs, module doc
 *          formula box and encode_llama_layer_dense;
 *     Gemma shared-expert branch: h1 = RMSNorm(h) * w, eps 1e-6
 *       -- turbospark-runtime 0.1.0, src/families/gemma4/shared_expert.rs,
 *          encode_shared_expert_branch[_batched];
 *     Qwen-style routed MoE: top-k experts per token, phase-2 accumulator
 *       seeded with the sigmoid-gated shared expert, ranks added in pair order,
 *       then one raw residual add
 *       -- turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs, module doc
 *          and encode_qwen_layer_moe_batched.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees them and keeps none after the call returns (plans excepted:
 *    a plan keeps the expert weight pointers until moe_plan_destroy).
 *  - Activations are bf16 (uint16 bit patterns), token-major [M][H], rows
 *    contiguous. x must not alias the output (on the pages the normed input
 *    may not be written by any dispatch encoded between its norm and its use).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronize the host. No call reads results
 *    back to the host (the reference's blocking router readback is not
 *    reproduced).
 *  - Hot calls allocate no memory: scratch comes from the caller's workspace
 *    (`ws`, `ws_bytes`, 256-byte aligned, size from the *_workspace_bytes
 *    queries). Its contents need no initialisation and are garbage after.
 *  - Arguments are validated on the host before any launch. Unsupported
 *    combinations are refused with MOEFFN_ERR_UNSUPPORTED and a message; there
 *    is no fallback path (the pages refuse unsupported inputs rather than run
 *    a lesser path).
 *  - On error the return value is negative and moeffn_last_error() gives a
 *    thread-local message. CUDA launch errors map to MOEFFN_ERR_CUDA.
 *
 * Weight formats (struct moeffn_qweight, W[rows][cols], y = W x):
 *  - MOEFFN_Q_INT8_ROW: q = int8 [rows][cols]; scale = fp16 [rows]; min = NULL.
 *    W[n][k] = q[n][k] * scale[n]. cols % 16 == 0.
 *  - MOEFFN_Q_INT4_AFFINE_G32: q = uint8 [rows][cols/2], element 2j in the low
 *    nibble of byte j, 2j+1 in the high nibble; scale, min = fp16
 *    [rows][cols/32]. W[n][k] = q * scale[n][k/32] + min[n][k/32]. cols % 32 == 0.
 *  - MOEFFN_Q_Q4_K: the K-quant block type of Q4_K_M files (turbospark-runtime
 *    0.3.0, src/families/llama/dense.rs: encode_gemv_any resolves the block
 *    type of each tensor), in the public GGUF layout, which the pages do not
 *    spell out. q = [rows][cols/256] super-blocks of 144 bytes: fp16 d (bytes
 *    0-1), fp16 dmin (2-3), the 6-bit scale and min of the eight 32-weight
 *    sub-blocks packed in bytes 4-15, then 128 code bytes in four runs of 32
 *    (run c: weights 64c..64c+31 in the low nibbles, 64c+32..64c+63 in the
 *    high nibbles). W = fp32(d * scale_j * q - dmin * min_j). scale = min =
 *    NULL. cols % 256 == 0. Dense layers only (ffn_dense, ffn_shared_expert),
 *    each of gate/up and down independently.
 *  - MOEFFN_BF16 / MOEFFN_F32: plain [rows][cols] in q (router, gate vector).
 *  All base pointers 16-byte aligned.
 */
#ifndef MOEFFN_H
#define MOEFFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* moeffn_stream_t; /* same type as cudaStream_t */

typedef enum {
  MOEFFN_OK = 0,
  MOEFFN_ERR_INVALID = -1,     /* null pointer, bad shape, misalignment */
  MOEFFN_ERR_UNSUPPORTED = -2, /* valid but not built (format, size limit) */
  MOEFFN_ERR_WORKSPACE = -3,   /* workspace missing or too small */
  MOEFFN_ERR_CUDA = -4         /* CUDA error (message has its string) */
} moeffn_status;

typedef enum {
  MOEFFN_Q_INT8_ROW = 1,
  MOEFFN_Q_INT4_AFFINE_G32 = 2,
  MOEFFN_BF16 = 3,
  MOEFFN_F32 = 4,
  MOEFFN_Q_Q4_K = 5
} moeffn_qformat;

typedef enum { MOEFFN_ACT_SILU = 0, MOEFFN_ACT_GELU_TANH = 1 } moeffn_act;

typedef enum {
  MOEFFN_KIND_DENSE = 1,   /* ffn_dense */
  MOEFFN_KIND_SHARED = 2,  /* ffn_shared_expert */
  MOEFFN_KIND_ROUTER = 3,  /* moe_router_topk */
  MOEFFN_KIND_MOE = 4      /* moe_layer (prefer moe_workspace_bytes) */
} moeffn_kind;

typedef struct moeffn_qweight {
  int32_t format;     /* moeffn_qformat */
  int32_t rows;       /* N: output features */
  int32_t cols;       /* K: reduction length */
  const void* q;      /* codes or plain values, see the format list above */
  const void* scale;  /* fp16, NULL for BF16/F32 */
  const void* min;    /* fp16, INT4 only, else NULL */
} moeffn_qweight;

/* One gated FFN: gate, up [I][H]; down [H][I]; all of one quantized format. */
typedef struct moeffn_ffn {
  moeffn_qweight gate, up, down;
} moeffn_ffn;

/* Workspace bytes for a call of `kind` with M token rows, hidden size H,
 * intermediate width I, E experts and top_k ranks (E, top_k ignored for the
 * dense kinds). For MOEFFN_KIND_MOE pass I = max(expert width, shared width).
 * Returns 0 for invalid arguments. */
size_t moeffn_workspace_bytes(int kind, int M, int H, int I, int E, int top_k);

/* Thread-local text of the last error (empty string if none). */
const char* moeffn_last_error(void);

/* Dense llama-style FFN plus raw residual add, in place:
 *   residual[t] = bf16(residual[t] + bf16(down(bf16(act(gate x_t) * (up x_t)))))
 * turbospark-runtime 0.3.0, src/families/llama/dense.rs,
 * encode_llama_layer_dense (gate and up GEMVs on the normed input, gated
 * activation, down GEMV into h2, residual add into x).
 * w: gate/up rows = I, cols = H; down rows = H, cols = I; INT8 or INT4 formats.
 * x, residual: [M][H] bf16. act: moeffn_act. M >= 1. */
int ffn_dense(const moeffn_ffn* w, const uint16_t* x, uint16_t* residual, int M, int act,
              void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* ffn_dense with the layer's input norm folded in:
 *   m = bf16(x / sqrt(mean(x^2) + eps) * norm_w)   (fp32, over the H columns)
 *   residual[t] = bf16(residual[t] + bf16(down(bf16(act(gate m_t) * (up m_t)))))
 * with x = residual (read before it is updated). turbospark-runtime 0.3.0,
 * src/families/llama/dense.rs, module doc formula box (the input norm
 * m = rms_norm(x, post_attention_layernorm), there encoded by the caller)
 * and encode_llama_layer_dense; the norm is the one the pages encode as
 * encode_rms_norm_bf16w. norm_w: [H] bf16, 16-byte aligned; eps >= 0.
 * Few token rows: the norm runs inside the gate/up kernel's staging of the
 * token rows (no launch of its own); more rows: one small launch writes m into
 * the workspace first. Workspace and errors as ffn_dense. */
int ffn_dense_prenorm(const moeffn_ffn* w, const uint16_t* norm_w, float eps, uint16_t* residual, int M,
                      int act, void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* Dense FFN plus residual add without a caller workspace. No counterpart on
 * the pages. For callers that cannot allocate device memory at the point of
 * the call: code inside a stream capture that must not add allocations,
 * runtimes that budget all device memory before they start, plugins handed
 * only input and output pointers. Computes exactly what ffn_dense computes,
 * with its scratch in a fixed array inside the library that is
 * MOEFFN_NOALLOC_SCRATCH_BYTES long and stays allocated on every GPU that
 * loads the library until the process exits. Allocates nothing. A call whose
 * scratch need (moeffn_workspace_bytes of MOEFFN_KIND_DENSE) is larger than
 * the array returns MOEFFN_ERR_WORKSPACE before any launch. The first call on
 * a device looks up the array's device address there (with that device
 * current); make that first call before any stream capture. Every call uses
 * the same array: calls that can overlap on the GPU (other streams, other
 * host threads) race on it and must be serialized by the caller. */
#define MOEFFN_NOALLOC_SCRATCH_BYTES (4u << 20)
int ffn_dense_noalloc(const moeffn_ffn* w, const uint16_t* x, uint16_t* residual, int M, int act,
                      moeffn_stream_t stream);

/* Gemma shared-expert branch with its trailing post-FFN RMSNorm:
 *   h1[t] = bf16(h / sqrt(mean(h^2) + eps) * norm_w), h = bf16(FFN(x_t))
 * turbospark-runtime 0.1.0, src/families/gemma4/shared_expert.rs,
 * encode_shared_expert_branch and encode_shared_expert_branch_batched
 * (RMS_EPS = 1e-6, weight post_feedforward_layernorm_1).
 * norm_w: [H] bf16. h1_out: [M][H] bf16 (written, not read). */
int ffn_shared_expert(const moeffn_ffn* w, const uint16_t* x, const uint16_t* norm_w, float eps,
                      uint16_t* h1_out, int M, int act, void* ws, size_t ws_bytes,
                      moeffn_stream_t stream);

/* Router GEMV, top-k softmax and (optionally) the expert-grouped pair order.
 * logits[t][e] = router[e] . x[t] (fp32). Ranks r = 0..top_k-1 ordered by
 * (logit desc, expert asc); topk_w[t][r] = fp16(softmax over the k selected
 * logits), stored as float. perm lists pair indices p = t*top_k + r grouped by
 * expert, stable in p; expert_offsets[e]..[e+1] is expert e's range of perm.
 * turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs: router logits
 * readback, router_topk_gemma4 with per_expert_ones, routes in PAIR order.
 * router: MOEFFN_F32 or MOEFFN_BF16, rows = E (<= 1024), cols = H (% 8 == 0).
 * logits_out [M][E], perm [M*top_k], expert_offsets [E+1] may be NULL
 * (expert_offsets is required when perm is given). top_k in 1..16, <= E. */
int moe_router_topk(const moeffn_qweight* router, const uint16_t* x, int M, int top_k,
                    float* logits_out, int32_t* topk_idx, float* topk_w, int32_t* perm,
                    int32_t* expert_offsets, void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* Description of a routed MoE layer (host memory; read by moe_plan_create). */
typedef struct moeffn_moe_desc {
  int32_t num_experts;                /* E */
  int32_t top_k;                      /* k */
  int32_t act;                        /* moeffn_act */
  moeffn_qweight router;              /* F32 or BF16 [E][H] */
  const moeffn_ffn* experts;          /* host array [E]; INT4-affine only */
  const moeffn_ffn* shared;           /* NULL: no shared expert (routed sum starts at 0) */
  const moeffn_qweight* shared_gate;  /* BF16 [1][H]; required with `shared` in the Qwen form */
  /* Gemma form of the routed layer (turbospark-runtime 0.3.0,
   * src/families/qwen/moe_batch.rs, module doc: Gemma's routed sum starts
   * from nothing, its shared branch joins in the tail after a norm, and
   * router_topk_gemma4 takes a learned per-expert scale;
   * turbospark-runtime 0.1.0, src/families/gemma4/shared_expert.rs: the
   * shared branch is the FFN then post_feedforward_layernorm_1). Appended
   * fields; all zero for the Qwen form. */
  const float* expert_scale;          /* device fp32 [E]: routing weight of expert e is
                                         fp16(softmax * expert_scale[e]); NULL: ones */
  const uint16_t* shared_post_norm;   /* device bf16 [H], 16-byte aligned: the shared expert is not
                                         gated and does not seed the sum; its output s becomes
                                         h1 = bf16(s / sqrt(mean(s^2) + eps) * w) and the tail is
                                         residual = bf16(residual + bf16(y + h1)), y the routed sum
                                         from 0. Requires `shared`, forbids `shared_gate`. NULL:
                                         the Qwen form. */
  float shared_post_norm_eps;         /* eps of that norm (the pages: 1e-6) */
} moeffn_moe_desc;

typedef struct moeffn_moe_plan moeffn_moe_plan;

/* Validates the description and copies the expert pointer tables to the
 * device (the only library-owned memory). Blocking; not for the hot path. */
int moe_plan_create(const moeffn_moe_desc* desc, moeffn_moe_plan** plan);
int moe_plan_destroy(moeffn_moe_plan* plan);
size_t moe_workspace_bytes(const moeffn_moe_plan* plan, int M);

/* Routed MoE layer plus its single raw residual add, in place:
 *   y[t] = bf16( ((seed[t] + w_0 d_0) + w_1 d_1) + ... )  (fp32, rank order)
 *   residual[t] = bf16(residual[t] + y[t])
 * seed = bf16(bf16(shared(x_t)) * sigmoid(shared_gate . x_t)), or 0.
 * Gemma form (shared_post_norm given): seed = 0 and
 *   residual[t] = bf16(residual[t] + bf16(y[t] + h1[t])), h1 the normed shared branch.
 * turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs, module doc (phase 2
 * starts its accumulator from the gated shared-expert output; the tail has no
 * sandwich norm) and encode_qwen_layer_moe_batched.
 * topk_idx_out: optional [M][k] int32 copy of the selected experts. */
int moe_layer(moeffn_moe_plan* plan, const uint16_t* x, uint16_t* residual, int M, int32_t* topk_idx_out,
              void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* moe_layer with the layer's input norm folded in: the router kernel forms
 * m = bf16(x / sqrt(mean(x^2) + eps) * norm_w) from x = residual, uses it for
 * the logits (and the shared-expert gate) and stores it in the workspace for
 * the expert and shared-expert projections; then as moe_layer. Sources as
 * ffn_dense_prenorm and moe_layer. norm_w: [H] bf16, 16-byte aligned. */
int moe_layer_prenorm(moeffn_moe_plan* plan, const uint16_t* norm_w, float eps, uint16_t* residual, int M,
                      int32_t* topk_idx_out, void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* ---- Expert-parallel MoE: the routed layer split at its exchange points ----
 * The batched pass of turbospark-runtime 0.3.0, src/families/qwen/moe_batch.rs
 * (encode_qwen_layer_moe_batched) groups the (token, rank) pairs by expert,
 * runs phase 1 (gate/up + activation) and phase 2 (down) per expert of the
 * union, and sums the expert outputs onto the gated shared-expert seed in rank
 * order. With the experts spread over GPUs (a contiguous block of E / world
 * experts per rank), each pair's token row goes to its expert's GPU after the
 * grouping and its down output comes back before the sum. The three calls
 * below are the GPU work between those two exchanges, which are the caller's
 * (e.g. NCCL all-to-alls); the result equals moe_layer's up to the fp32
 * summation order of the down projection's K splits. The Gemma form is not
 * covered. */

/* Dispatch order: rows_out[s] = x[perm[s] / top_k], expert_out[s] =
 * topk_idx[perm[s]] for the M*top_k pair slots s, with topk_idx and perm as
 * moe_router_topk writes them (pairs in expert order, so each owning rank's
 * pairs are one contiguous block, of expert_offsets[(r+1)*E/world] -
 * expert_offsets[r*E/world] rows). x: [M][H] bf16, 16-byte aligned;
 * topk_idx, perm: [M*top_k] int32; rows_out: [M*top_k][H] bf16, 16-byte
 * aligned; expert_out: [M*top_k] int32. H a multiple of 8. */
int moe_dispatch_rows(const uint16_t* x, const int32_t* topk_idx, const int32_t* perm, int M, int top_k, int H,
                      uint16_t* rows_out, int32_t* expert_out, moeffn_stream_t stream);

/* Workspace bytes of moe_experts_grouped for R rows on this plan (0 if invalid). */
size_t moe_experts_workspace_bytes(const moeffn_moe_plan* plan, int R);

/* Phases 1 and 2 of the plan's experts over R rows given in any order (as
 * they arrived from the ranks): d_out[i] = down_e(bf16(act(gate_e . rows[i]) *
 * (up_e . rows[i]))) in fp32, the down projection's K splits summed in split
 * order, with e = row_expert[i] - expert_base; a row whose e is outside
 * [0, E) gives a zero row. The rows are grouped by expert on the device (a
 * stable counting sort), then run as moe_layer's grouped GEMV or tensor-core
 * GEMM over the union of experts present. A plan holding one rank's block
 * of experts (router and top_k unused here; its shared expert is not run)
 * does exactly that rank's expert work; a plan holding only a shared expert
 * gives its down output with row_expert all zero. rows: [R][H] bf16;
 * row_expert: [R] int32; d_out: [R][H] fp32; rows and d_out 16-byte aligned;
 * at most 1024 experts per plan. R = 0 returns at once. */
int moe_experts_grouped(moeffn_moe_plan* plan, const uint16_t* rows, int R, const int32_t* row_expert,
                        int expert_base, float* d_out, void* ws, size_t ws_bytes, moeffn_stream_t stream);

/* Workspace bytes of moe_combine (the inverse of perm). */
size_t moe_combine_workspace_bytes(int M, int top_k);

/* moe_layer's seeded rank-ordered sum and raw residual add, from the expert
 * outputs of every pair:
 *   y[t] = bf16( ((seed[t] + w_0 d_{t,0}) + w_1 d_{t,1}) + ... )  (fp32, rank order)
 *   residual[t] = bf16(residual[t] + y[t])
 * with d_{t,r} the row of d at the slot s where perm[s] = t*top_k + r, w =
 * topk_w, seed[t] = bf16(bf16(shared_d[t]) * sigmoid(gate_logit[t])), or 0
 * when shared_d is null. d: [M*top_k][H] fp32 in perm's slot order (as
 * moe_dispatch_rows sent the rows); perm: [M*top_k] int32; topk_w: [M][top_k]
 * fp32; shared_d: [M][H] fp32 (moe_experts_grouped on a shared-expert plan) or
 * null; gate_logit: [M] fp32 (moe_router_topk's logits with the shared gate
 * vector as a one-row router), required with shared_d; residual: [M][H] bf16,
 * updated in place. d, shared_d, residual 16-byte aligned; H a multiple of 4. */
int moe_combine(const float* d, const int32_t* perm, const float* topk_w, int M, int top_k, int H,
                const float* shared_d, const float* gate_logit, uint16_t* residual, void* ws, size_t ws_bytes,
                moeffn_stream_t stream);

/* Failure detection. Pipeline waits inside the kernels are bounded (about one
 * second); a wait that runs out sets a bit in a device fault word and the
 * kernel finishes without its result instead of hanging. Returns the word
 * (bit 0: a pipeline barrier wait timed out; bit 1: a launch with an invalid
 * pipeline depth was refused) and clears it if `clear` != 0.
 * Synchronous (a device-to-host copy); not for the hot path. */
unsigned int moeffn_device_faults(int clear);

/* ---- Per-launch timing (tracing) ------------------------------------------
 * No counterpart on the pages (they time host phases with PhaseCounters).
 * Off by default. While enabled, every kernel launch of the library is
 * bracketed by two CUDA events on its stream (a small gap per launch).
 * moeffn_profile_read waits for the recorded events and returns, per kernel
 * name (names: '\n'-separated, truncated to names_len), the number of
 * launches and their summed device time in ms since the previous read, then
 * clears the records. Not thread-safe across concurrent callers' reads. */
int moeffn_profile_enable(int on);
int moeffn_profile_read(char* names, int names_len, int32_t* counts, float* total_ms, int max_kernels,
                        int* n_kernels);

/* ---- Test exports: feed identical inputs to single steps. ---------------- */

/* Dequantize W on the device with the kernels' own conversion: out_f32
 * [rows][cols] (exact q*scale(+min)) and/or out_bf16 [rows][cols] (round to
 * nearest even of the fp32 value). Either output may be NULL. */
int moeffn_test_dequant(const moeffn_qweight* w, float* out_f32, uint16_t* out_bf16, moeffn_stream_t stream);

/* Top-k, softmax weights and grouped permutation from given fp32 logits
 * [M][E] (device). union_out [E] and n_union_out [1] may be NULL. */
int moeffn_test_topk_from_logits(const float* logits, int M, int E, int top_k, int32_t* topk_idx,
                                 float* topk_w, int32_t* perm, int32_t* expert_offsets,
                                 int32_t* union_out, int32_t* n_union_out, moeffn_stream_t stream);

/* Failure injection for tests of the failure detection above (no counterpart
 * on the pages). One-shot: applies to the next ffn_dense / ffn_shared_expert
 * call whose gate/up projection runs the weight-streaming GEMV, then clears.
 *  kind 1: that launch's producer issues no weight stage from stage `value`
 *          on, as if it had died; the consumers' bounded waits run out after
 *          `wait_us` microseconds, set bit 0 of the fault word and the kernel
 *          finishes without its result (no copy is left in flight).
 *  kind 2: that launch gets ring depth `value` (1..8); a depth the kernel
 *          cannot use (not a multiple of its consumer group count) is refused
 *          by the kernel, which sets bit 1 and returns at once.
 *  kind 0: cancel a pending injection.
 * wait_us: 1..1000000. The call's outputs are garbage; the next call is not
 * affected. Returns MOEFFN_ERR_INVALID for other arguments. Not thread-safe. */
int moeffn_test_inject_gemv_fault(int kind, int value, unsigned int wait_us);

#ifdef __cplusplus
}
#endif

#endif /* MOEFFN_H */
