/*
 * moe.h - C ABI of libmoe.so: the forward pass of one sparse Mixture-of-Experts
 * layer on an NVIDIA B200 (sm_100a).
 *
 * What the layer computes (the reviewed pages, cited by title and section):
 *  - Token-choice top-k routing over m experts; R&Q ("A Replicate-and-Quantize
 *    Strategy for Plug-and-Play Load Balancing of Sparse Mixture-of-Experts
 *    LLMs") applies to top-1, top-2 and shared-expert routing ("If this is
 *    right"), and its Definition 1 counts n_j, the tokens routed to expert j.
 *  - The Load Imbalance Score LIS = m * max_j n_j / (n k) (R&Q, Definition 1;
 *    1 is perfectly balanced, larger is more skewed).
 *  - Expert-centric scheduling: (token, expert) tasks are sorted into one
 *    contiguous group per active expert and each group runs as a grouped GEMM
 *    (OmniMoE, "An Efficient MoE by Orchestrating Atomic Experts at Scale",
 *    "What carries the argument" and Fig. 3).
 *  - SwiGLU experts with W_gate, W_up, W_down and a SiLU gate (FloE, "On-the-Fly
 *    MoE Inference on Memory-constrained GPU", "What carries the argument";
 *    OmniMoE Sec. 2.1), or Switch-style two-matrix ReLU experts.
 *  - Always-on shared experts added with weight 1 (OmniMoE's shared dense MLP
 *    branch; R&Q's shared-expert routing).
 *  - The atomic-expert variant: a Cartesian Product Router (OmniMoE Sec. 2.2,
 *    Eq. 8), exact top-K over the implicit grid (OmniMoE App. A) and atomic
 *    experts sigma(x w_in^T) w_out (OmniMoE Eq. 4).
 *
 * Conventions for every call:
 *  - Pointers named x, w_*, out, ... are DEVICE pointers owned by the caller;
 *    config structs and scalar out-parameters (bytes, moe_status_t*) are HOST
 *    pointers. The library allocates no device memory; scratch comes from the
 *    caller's workspace `ws` of `ws_bytes` bytes (size it with
 *    moe_workspace_size / moe_atomic_workspace_size, zero it once before first
 *    use: its first 4 bytes hold the device status word).
 *  - Layouts are row-major with nn.Linear [out, in] weights:
 *      x [T, d]; w_router [m, d]; bias [m] fp32;
 *      w_gate, w_up [m, f, d]; w_down [m, d, f];   (ReLU experts: w_gate = W1, w_up = NULL, w_down = W2)
 *      ws_gate, ws_up [n_shared, f_shared, d]; ws_down [n_shared, d, f_shared];
 *      topk_idx [T, k] int32; topk_w [T, k] fp32; logits [T, m] fp32;
 *      counts [m] int32; offsets [m + 1] int32; perm, inv_perm [T k] int32;
 *      x_perm [T k, d]; y_perm [T k, d] fp32; out [T, d] in the config dtype.
 *    Element type of x / weights / x_perm / out is cfg->dtype (fp32 or bf16).
 *  - Alignment: every device pointer must be 16-byte aligned; d, f and f_shared
 *    must be multiples of 8.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream), never synchronise the host, and may be captured in a CUDA graph.
 *  - Errors: arguments are checked on the host before any launch
 *    (MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE); a failed
 *    launch returns MOE_ERR_CUDA. Errors found on the device (an expert id
 *    outside [0, m): MOE_ERR_DEVICE_INDEX, and no write is issued for it; a
 *    bounded wait inside a kernel that ran out: MOE_ERR_TIMEOUT) are recorded
 *    in the status word of `ws` and read with moe_read_device_status.
 *  - Only sm_100 devices are supported (MOE_ERR_UNSUPPORTED elsewhere); there
 *    is no fallback path.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5,
  MOE_ERR_DEVICE_INDEX = 6
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;
typedef enum { MOE_SWIGLU = 0, MOE_RELU = 1 } moe_act_t;
typedef enum { MOE_ATOMIC_SILU = 0, MOE_ATOMIC_SIGMOID = 1 } moe_atomic_act_t;

/* One coarse-expert layer. T = tokens (the pages' n), d = d_model, f = d_ff of a
 * routed expert, m = routed experts (1..1024), k = experts per token (1..min(m, 32)),
 * n_shared / f_shared = always-on shared experts (0..8) and their d_ff.
 * renormalize != 0 divides the k gate weights by their sum. */
typedef struct {
  int32_t T, d, f, m, k, n_shared, f_shared;
  int32_t dtype;       /* moe_dtype_t */
  int32_t act;         /* moe_act_t */
  int32_t renormalize; /* 0 or 1 */
} moe_config_t;

/* Load diagnostics of one layer call (device memory, 16 bytes). */
typedef struct {
  int32_t max_count;     /* max_j n_j */
  int32_t argmax_expert; /* lowest j attaining it: the heavy hitter (R&Q Alg. 1) */
  double lis;            /* m * max_j n_j / (T k), one correctly rounded fp64 division */
} moe_lis_t;

/* Atomic-expert layer: N = Nr * Nc experts on a grid, K selected per token
 * (1..4096, at most N: decode budgets up to 64 use a staircase candidate set,
 * prefill budgets above 64 a radix selection over the whole grid; both exact),
 * Nr and Nc in 64..1024 and multiples of 8; dtype must be MOE_BF16. */
typedef struct {
  int32_t T, d, Nr, Nc, K;
  int32_t act;   /* moe_atomic_act_t */
  int32_t dtype; /* moe_dtype_t */
} moe_atomic_config_t;

/* Workspace bytes needed by every call below for this config (the maximum over
 * them, i.e. what moe_layer_forward needs). bytes: host out-parameter. */
MOE_API moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes);
MOE_API moe_status_t moe_atomic_workspace_size(const moe_atomic_config_t* cfg, size_t* bytes);

/* Router (R&Q's token-choice routing). logits = x w_router^T + bias (fp32,
 * fp32 accumulation; bias may be NULL), or logits_in verbatim when given (then x,
 * w_router and bias are ignored). top-k by (logit desc, expert index asc);
 * p = softmax over all m logits; topk_w[t,s] = p[idx] (or renormalised over the
 * k when cfg->renormalize). logits_out (nullable) receives the logits used. */
MOE_API moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                       const float* logits_in, float* logits_out, int32_t* topk_idx, float* topk_w, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/* Per-expert histogram n_j, segment offsets (exclusive prefix sum, m + 1
 * entries) and LIS (R&Q Definition 1). counts, offsets and lis are device
 * pointers; lis may be NULL. An id outside [0, m) sets MOE_ERR_DEVICE_INDEX in
 * the status word and nothing is written. */
MOE_API moe_status_t moe_histogram_lis(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                               moe_lis_t* lis, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Load Imbalance Score of a given histogram (R&Q Definition 1): lis->max_count =
 * max_j counts[j], lis->argmax_expert = the lowest j attaining it, lis->lis =
 * m * max / tasks (one fp64 division). For a histogram that spans more than one
 * call, e.g. the per-expert counts of every data-parallel rank's batch summed
 * across ranks, where tasks = the summed T k. counts [m] int32 and lis are device
 * pointers (counts 4-byte, lis 16-byte aligned); m in 1..1024 (MOE_ERR_UNSUPPORTED
 * above), tasks >= 1; no workspace. */
MOE_API moe_status_t moe_lis_from_counts(int32_t m, int64_t tasks, const int32_t* counts, moe_lis_t* lis,
                                         moe_stream_t stream);

/* Expert-centric permutation (OmniMoE Fig. 3). Task q = t k + s goes to
 * position pos = offsets[e] + (number of earlier tasks q' < q with the same
 * expert e): segments are contiguous and ordered by task id. Writes
 * perm[pos] = q, inv_perm[q] = pos and x_perm[pos, :] = x[q / k, :]. A task
 * whose id or position falls outside the segment given by `offsets` sets
 * MOE_ERR_DEVICE_INDEX; such a task keeps inv_perm[q] = -1 and its perm / x_perm
 * rows are not written (an id outside [0, m) anywhere leaves every inv_perm entry
 * at -1 and writes no perm or x_perm row). */
MOE_API moe_status_t moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* offsets,
                         void* x_perm, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Grouped expert FFN over the segments of x_perm (rows offsets[e]..offsets[e+1]
 * belong to expert e): y_perm[pos] = task_w[perm[pos]] * FFN_e(x_perm[pos]) with
 * FFN_e the SwiGLU (or ReLU) expert; task_w == NULL means weight 1 (perm is then
 * ignored). bf16 runs on the tcgen05 tensor cores (bf16 operands, fp32
 * accumulation, the hidden activation h rounded to bf16 between the two GEMMs);
 * fp32 runs on the CUDA cores in fp32. */
MOE_API moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                             const void* w_gate, const void* w_up, const void* w_down, const float* task_w,
                             const int32_t* perm, float* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Shared experts: y_shared[s, t, :] = FFN_s(x[t, :]) for s < cfg->n_shared,
 * y_shared fp32 [n_shared, T, d]. */
MOE_API moe_status_t moe_shared_ffn(const moe_config_t* cfg, const void* x, const void* ws_gate, const void* ws_up,
                            const void* ws_down, float* y_shared, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Combine: out[t] = sum_{s<k} y_perm[inv_perm[t k + s]] + sum_{s<n_shared}
 * y_shared[s, t] (y_shared may be NULL), summed in fp32 in that order and rounded
 * to cfg->dtype. */
MOE_API moe_status_t moe_combine(const moe_config_t* cfg, const float* y_perm, const int32_t* inv_perm,
                         const float* y_shared, void* out, moe_stream_t stream);

/* The whole layer in one call, on one stream with no host synchronisation:
 * route -> histogram/LIS -> permute -> grouped FFN (+ shared experts) -> combine.
 * Optional device outputs (each may be NULL): logits_out [T, m], topk_idx_out,
 * topk_w_out [T, k], counts_out [m], lis_out; and copies of the expert-centric
 * permutation the layer computed, as moe_histogram_lis / moe_permute define it
 * (OmniMoE Fig. 3): offsets_out [m + 1], perm_out [T k] (segment row -> task
 * t k + s), inv_perm_out [T k] (task -> segment row) and x_perm_out [T k, d]
 * (the permuted token rows, cfg->dtype). w_up / ws_up are NULL for ReLU; ws_* are
 * NULL when n_shared == 0. */
MOE_API moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                               const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                               const void* ws_up, const void* ws_down, void* out, float* logits_out,
                               int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, moe_lis_t* lis_out,
                               int32_t* offsets_out, int32_t* perm_out, int32_t* inv_perm_out, void* x_perm_out,
                               void* ws, size_t ws_bytes, moe_stream_t stream);

/* R&Q replica dispatch ("A Replicate-and-Quantize Strategy for Plug-and-Play Load
 * Balancing of Sparse Mixture-of-Experts LLMs", Sec. 2.5 and Algorithm 3, which
 * append a replica of the heavy-hitter but leave the router unchanged and give no
 * rule that sends tokens to it; the rule here is the one its review suggests:
 * the heavy-hitter's tokens alternate between the original and the replica).
 * Inputs are the outputs of moe_histogram_lis / moe_permute for topk_idx (m
 * experts): the heavy-hitter h = lis->argmax_expert (most tasks, lowest index on
 * ties); the tasks of h in their segment order (increasing task id t k + s) go
 * original, replica, original, ...; the replica is expert m.
 * idx_out [T, k] int32: experts in [0, m] after the split (every other task is
 * unchanged). Optional: counts_out [m + 1] (h keeps ceil(n_h / 2), the replica
 * gets floor(n_h / 2)); lis_out = Definition 1 over the m + 1 experts. All device
 * pointers; ws: moe_workspace_size(cfg) bytes. MOE_ERR_DEVICE_INDEX (device
 * status) if an id, h or a segment rank is out of range. Needs m + 1 <= 1024. */
MOE_API moe_status_t moe_replica_split(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* offsets,
                                       const int32_t* inv_perm, const moe_lis_t* lis, int32_t* idx_out,
                                       int32_t* counts_out, moe_lis_t* lis_out, void* ws, size_t ws_bytes,
                                       moe_stream_t stream);

/* moe_layer_forward with R&Q replica dispatch (bf16 only): route over the m
 * experts, split the heavy-hitter's tasks as moe_replica_split does, then run
 * the layer over m + 1 routed groups, the replica computing with the
 * heavy-hitter's own weights (the pages' replica is a quantised copy; low-precision
 * weights are not part of this call). The output therefore equals
 * moe_layer_forward's up to rounding order. Optional device outputs: logits_out
 * [T, m], topk_idx_out / topk_w_out [T, k] (the router's choice), dispatch_idx_out
 * [T, k] (after the split), counts_out [m + 1], lis_before_out (m experts),
 * lis_after_out (m + 1 experts). ws: moe_workspace_size() of the same config with
 * m + 1 experts. MOE_ERR_UNSUPPORTED for fp32 or m + 1 > 1024. */
MOE_API moe_status_t moe_layer_forward_replicated(
    const moe_config_t* cfg, const void* x, const void* w_router, const float* bias, const void* w_gate,
    const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down, void* out,
    float* logits_out, int32_t* topk_idx_out, float* topk_w_out, int32_t* dispatch_idx_out, int32_t* counts_out,
    moe_lis_t* lis_before_out, moe_lis_t* lis_after_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/* FloE contextual sparsity ("FloE: On-the-Fly MoE Inference on Memory-constrained
 * GPU", "Core claim", Sec. 3.2 and Eq. 6). bf16 SwiGLU layers without shared
 * experts only (MOE_ERR_UNSUPPORTED otherwise). For a task of expert e:
 * u = x W_up[e]^T; channel j is kept when |u_j| >= thresholds[e]; kept channels
 * compute g_j = x . W_gate[e][j] and h_j = g_j sigma(g_j) u_j, the others
 * contribute nothing; y = w * sum over kept j of h_j W_down[e][:, j]. Only the
 * gate rows and down columns of channels that some task of e keeps are read.
 *
 * moe_floe_pack_down: w_down_t [m, f, d] bf16 = W_down transposed per expert
 * (channel-major, so a kept channel is one contiguous row); a one-time layout. */
MOE_API moe_status_t moe_floe_pack_down(const moe_config_t* cfg, const void* w_down, void* w_down_t,
                                        moe_stream_t stream);

/* Per-expert thresholds from a calibration batch (Eq. 6, the empirical CDF of
 * |up-projection activations| at target sparsity s in [0, 1]): u_scratch
 * [T_calib, m f] fp32 receives u[t][e f + j] = x_calib[t] . W_up[e][j] for every
 * expert (tensor cores, fp32 accumulation); thresholds_out [m] fp32 = the
 * ceil(s n)-th smallest (at least the 1st) of the n = T_calib f values |u| of
 * each expert, found exactly. ws: moe_workspace_size(cfg) bytes (status word). */
MOE_API moe_status_t moe_floe_calibrate(const moe_config_t* cfg, const void* x_calib, int32_t T_calib,
                                        const void* w_up, double sparsity, float* u_scratch, float* thresholds_out,
                                        void* ws, size_t ws_bytes, moe_stream_t stream);

/* Workspace of moe_layer_forward_floe (host out-parameter). */
MOE_API moe_status_t moe_floe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* The layer with FloE sparse experts: route -> histogram/LIS -> permute -> dense
 * up projection (fp32 u) -> kept-channel lists -> gate rows and down rows of the
 * kept channels -> combine. thresholds [m] fp32 (device), w_down_t from
 * moe_floe_pack_down. Optional device outputs: topk_idx_out / topk_w_out
 * [T, k]; kept_out [m] int32 = channels read per expert; u_out [T k, f] fp32 =
 * u of each segment row and perm_out [T k] = the task of each row (for checks).
 * ws: moe_floe_workspace_size() bytes. */
MOE_API moe_status_t moe_layer_forward_floe(const moe_config_t* cfg, const void* x, const void* w_router,
                                            const float* bias, const void* w_gate, const void* w_up,
                                            const void* w_down_t, const float* thresholds, void* out,
                                            int32_t* topk_idx_out, float* topk_w_out, int32_t* kept_out,
                                            float* u_out, int32_t* perm_out, void* ws, size_t ws_bytes,
                                            moe_stream_t stream);

/* 8-bit expert weights (R&Q, "Free parameters": 8-bit expert copies for
 * LLaMA-MoE and DeepSeek; the format is not named there). Format: OCP E4M3 codes
 * (uint8: sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448)
 * with one fp32 scale per row. A row of values v becomes scale = fl32(max |v| /
 * 448) (1 for an all-zero row) and codes E4M3(fl32(v / scale)), rounded to
 * nearest even and saturating at +-448; the value of a code is E4M3(code) * scale.
 *
 * moe_quantize_e4m3: per-row quantization of a bf16 matrix src [rows, cols]
 * (device, row-major, 16-byte aligned) into codes [rows, cols] (device, 16-byte
 * aligned) and scales [rows] (device fp32). cols must be a multiple of 16
 * (MOE_ERR_UNSUPPORTED otherwise). Used once on the expert weights; outputs are
 * owned by the caller. Asynchronous on `stream`. */
MOE_API moe_status_t moe_quantize_e4m3(int64_t rows, int64_t cols, const void* src, uint8_t* codes, float* scales,
                                       moe_stream_t stream);

/* Quantized expert weights for moe_layer_forward_fp8: the bf16 weights of
 * moe_layer_forward passed through moe_quantize_e4m3 row by row (each output
 * channel its own scale). Device pointers; codes 16-byte aligned.
 *   gate, up  [m, f, d] codes, gate_scale / up_scale [m f]  (up: SwiGLU only)
 *   down      [m, d, f] codes, down_scale [m d]
 *   sh_gate, sh_up [n_shared, f_shared, d], scales [n_shared f_shared]
 *   sh_down   [n_shared, d, f_shared], sh_down_scale [n_shared d]
 * (sh_*: only with n_shared > 0; unused entries may be NULL). */
typedef struct {
  const uint8_t* gate;
  const float* gate_scale;
  const uint8_t* up;
  const float* up_scale;
  const uint8_t* down;
  const float* down_scale;
  const uint8_t* sh_gate;
  const float* sh_gate_scale;
  const uint8_t* sh_up;
  const float* sh_up_scale;
  const uint8_t* sh_down;
  const float* sh_down_scale;
} moe_fp8_experts_t;

/* Workspace of moe_layer_forward_fp8 (host out-parameter): moe_workspace_size()
 * plus the E4M3 rows of x and h. bf16 layers with d, f and f_shared multiples of
 * 16 only (MOE_ERR_UNSUPPORTED otherwise). */
MOE_API moe_status_t moe_fp8_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* moe_layer_forward with 8-bit experts. The router is the bf16 layer's (same
 * logits, top-k and gate weights, same histogram, LIS and permutation); every
 * projection of every routed and shared expert multiplies E4M3 operands on the
 * tensor cores (fp32 accumulation): the permuted token rows and the bf16 h rows
 * are quantized per row on the way in, and each product is scaled by its weight
 * row's and its activation row's scales. out [T, d] bf16. Optional outputs as in
 * moe_layer_forward, plus copies for inspection (all nullable, device): h_out
 * [T k, f] bf16 = the stored h of each segment row, h_shared_out [n_shared T,
 * f_shared] bf16, perm_out [T k] int32 = the task (t k + s) of each segment row.
 * ws: moe_fp8_workspace_size() bytes, 256-byte aligned. Stage events
 * (moe_set_stage_events) as in moe_layer_forward; the quantization of x rows
 * falls in stage 4-5 and that of h in 5-6. */
MOE_API moe_status_t moe_layer_forward_fp8(const moe_config_t* cfg, const void* x, const void* w_router,
                                           const float* bias, const moe_fp8_experts_t* wq, void* out,
                                           float* logits_out, int32_t* topk_idx_out, float* topk_w_out,
                                           int32_t* counts_out, moe_lis_t* lis_out, void* h_out,
                                           void* h_shared_out, int32_t* perm_out, void* ws, size_t ws_bytes,
                                           moe_stream_t stream);

/* Cartesian Product Router (OmniMoE Sec. 2.2, Eq. 8; App. A): lr = log_softmax(x
 * w_row^T), lc = log_softmax(x w_col^T) (fp32); expert (i, j) with flat id
 * i Nc + j scores S = fl32(lr_i + lc_j); idx_out [T, K] = the exact top-K of all
 * Nr Nc scores by (S desc, id asc), g_out [T, K] = softmax of the selected S.
 * row_logp_out [T, Nr] and col_logp_out [T, Nc] are optional (nullable). */
MOE_API moe_status_t moe_atomic_route(const moe_atomic_config_t* cfg, const void* x, const void* w_row, const void* w_col,
                              float* row_logp_out, float* col_logp_out, int32_t* idx_out, float* g_out, void* ws,
                              size_t ws_bytes, moe_stream_t stream);

/* Atomic experts (OmniMoE Eq. 4, Dynamic Expert Assembly): out[t] = sum_s
 * g[t,s] act(x_t . w_in[idx[t,s]]) w_out[idx[t,s]], act = SiLU or sigmoid;
 * w_in, w_out [Nr Nc, d] bf16; out [T, d] bf16. */
MOE_API moe_status_t moe_atomic_experts(const moe_atomic_config_t* cfg, const void* x, const void* w_in, const void* w_out,
                                const int32_t* idx, const float* g, void* out, void* ws, size_t ws_bytes,
                                moe_stream_t stream);

/* moe_atomic_route followed by moe_atomic_experts. idx_out, g_out nullable. */
MOE_API moe_status_t moe_atomic_forward(const moe_atomic_config_t* cfg, const void* x, const void* w_row, const void* w_col,
                                const void* w_in, const void* w_out, void* out, int32_t* idx_out, float* g_out,
                                void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_route without a workspace, for callers that cannot allocate device memory:
 * plugins that only see the tensors a host framework hands them (the framework
 * owns the allocator), or request paths that must not allocate (an allocation can
 * block or fail under memory pressure). (The reviewed pages have no counterpart:
 * this is a deployment convenience, not part of the method.) Same arguments and results as
 * moe_route, except that the status word and - when neither logits_in nor
 * logits_out is given - the router logits live in an 8 MiB array compiled into
 * the library, held on every GPU that loads it until the process exits. It
 * allocates nothing. Limits: T * m <= 2,097,088 when the logits go to that
 * array, else MOE_ERR_WORKSPACE is returned before any launch. The status word
 * is cleared at the start of each call and, when device_status_out (device
 * pointer, nullable) is given, copied there at the end (0 = ok, else a
 * moe_status_t). All calls on a device share the array: calls whose work overlaps
 * on the GPU race on it, so order them on one stream. The first call on each
 * device looks up the array's address; make it before any stream capture. */
MOE_API moe_status_t moe_route_static(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                                      const float* logits_in, float* logits_out, int32_t* topk_idx, float* topk_w,
                                      int32_t* device_status_out, moe_stream_t stream);

/* Synchronises `stream`, reads the status word of `ws` into *out (host) and
 * clears it. Returns MOE_ERR_CUDA if the synchronisation or copy fails. */
MOE_API moe_status_t moe_read_device_status(void* ws, moe_stream_t stream, moe_status_t* out);

/* Static string for a status code. */
MOE_API const char* moe_status_string(moe_status_t status);

/* Test hook: the time limit, in nanoseconds, of every bounded wait inside the
 * tensor-core kernels launched after this call (0 restores the default of 2 s).
 * Not thread-safe; meant for fault-injection tests. */
MOE_API moe_status_t moe_debug_set_wait_limit_ns(uint64_t ns);

/* Test hook: the grid-wide barrier of the decode-budget atomic-expert kernel
 * (moe_atomic_experts / moe_atomic_forward with T K < 16384) waits for n arrivals
 * more than its grid has, so with n > 0 it can only end at the bounded wait's
 * time limit: the kernel then records MOE_ERR_TIMEOUT and its blocks return
 * without the assembly phase. 0 (the default) restores the normal barrier. Not
 * thread-safe; meant for fault-injection tests. */
MOE_API moe_status_t moe_debug_set_barrier_extra(uint32_t n);

/* Profiling hook: when n > 0, every later moe_layer_forward records the n
 * cudaEvent_t handles in `events` (host array, caller-owned events) on its
 * stream at its stage boundaries, in order: 0 start, 1 router logits, 2 top-k,
 * 3 histogram/LIS/ranks, 4 row permutation, 5 up projection, 6 down projection,
 * 7 combine (n <= 8; extra stages are not recorded); moe_atomic_forward records
 * 0 start, 1 router projections, 2 grid top-K, 3 and 4 after the atomic-expert FFN (coefficients and
 * assembly are one launch);
 * moe_layer_forward_replicated records the stages of moe_layer_forward (3 is
 * after both sorts and the split).
 * A NULL entry skips that
 * boundary (a recorded event between two kernels stops the second one from
 * starting early, so record only the boundaries you time). n = 0 turns it off.
 * During a stream capture the records become external event-record nodes of
 * the graph (each replay records the events again).
 * The array is copied. Process-wide and not thread-safe; meant for benchmarks. */
MOE_API moe_status_t moe_set_stage_events(void* const* events, int n);

/* Number of kernels this library launched since the process started (host
 * counter; for benchmarks that report their launch count). */
MOE_API uint64_t moe_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
