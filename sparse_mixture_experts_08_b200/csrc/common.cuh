// Shared device helpers and internal launch interfaces of libmoe (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Record the first device-side error in the status word (later errors keep it).
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase with `parity` completed; false when the time
// limit ran out or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                          const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}


// Bulk copy global -> shared (the copy engine, no tensor map): bytes % 16 == 0, both
// addresses 16-byte aligned; completion counted on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- dependent launch
// Every kernel of the layer is launched with programmatic stream serialization:
// it tells the hardware at entry that its successor may be scheduled
// (launch_dependents), and waits for its predecessor's completion (and memory)
// right before reading that predecessor's outputs. The successor's launch and
// prologue then overlap this kernel's tail instead of following it.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- internal API
// Every launcher returns cudaSuccess or the launch error; arguments were checked
// by the C-ABI layer before.

enum Epi { EPI_LOGITS = 0, EPI_SWIGLU = 1, EPI_RELU = 2, EPI_DOWN = 3, EPI_ROUTE = 4,
           // the down projection with two consecutive feature blocks per tile sharing the
           // token rows (pair tiles only: 512 output features x up to 256 token rows)
           EPI_DOWN_DUAL = 5 };

// EPI_ROUTE: the router with tokens as the MMA's M rows (A = x) and all experts in
// one N tile (B = W_r, m <= 256 rows): each epilogue thread owns a token's logits.
constexpr int ROUTE_MAX_M = 256;
constexpr int ROUTE_MAX_K = 8;
// Each CTA streams one 128-token tile through its SM, so the fused router pays off
// only when the batch has tiles for most SMs; smaller batches keep the separate
// router, top-k and sort kernels (measured: slower fused at 2048 and 4096 tokens).
constexpr int ROUTE_MIN_T = 8192;
inline bool fused_route_ok(const moe_config_t& c) {
  return c.dtype == MOE_BF16 && c.m <= ROUTE_MAX_M && c.k <= ROUTE_MAX_K && c.T >= ROUTE_MIN_T;
}

// One class of problems for the grouped GEMM  out = epi(A_g . B_rows^T):
// A_g = rows [g*R, g*R + R) of a K-major weight matrix, B rows = one segment.
struct GemmClass {
  int n_groups;
  int R;                     // output features per group (rows of A per group)
  int K;                     // reduction length
  int ksplit;                // K is cut into ksplit contiguous ranges (partial outputs)
  int kb_per_split;          // k-blocks (64 bf16 or 128 E4M3 elements) per range
  const int* seg_off;        // device [n_groups + 1]: B/out rows of group g (nullable)
  int max_row;               // seg_off entries and perm values must lie in [0, max_row]
  int const_rows;            // rows per group when seg_off == nullptr
  int b_group_stride;        // B row start of group g when seg_off == nullptr
  int out_group_stride;      // out row start of group g when seg_off == nullptr
  void* out;                 // fp32 (LOGITS, DOWN) or the activation dtype (SWIGLU, RELU)
  long long out_ld;          // elements between output rows
  long long out_split_stride;// elements between k-split partial outputs
  const float* bias;         // LOGITS: bias[feature] (nullable)
  const float* row_w;        // DOWN: weight of output row `row` (nullable; preferred over task_w)
  const float* task_w;       // DOWN: row weight task_w[perm[row]] (nullable = 1)
  const int* perm;
  int scatter_k1;            // DOWN with top-1 routing: write bf16 out[perm[row]] (combine fused)
  const int* group_map;      // device [n_groups]: weight matrix of group g (nullable = g); values < n_wgroups
  int n_wgroups;             // weight matrices behind group_map
  // ROUTE: top-k selection in the epilogue (out = fp32 logits [T, m], nullable)
  int k_sel, renorm;
  int32_t* sel_idx;          // [T, k] experts by (logit desc, expert asc)
  float* sel_w;              // [T, k] gate weights
  int32_t* lrank;            // [T, k] rank of task (t, s) among the tile's tasks of its expert (nullable)
  int32_t* tile_cnt;         // [tiles][m] tasks per expert in each 128-token tile (with lrank)
  // 8-bit operands (launch_tc_gemm with f8): fp32 scale of each row of A (weight
  // rows, indexed like the A operand) and of B (activation rows)
  const float* a0_scale;
  const float* a1_scale;
  const float* b_scale;
  // SIMT path only (fp32 / bf16 element pointers, row-major)
  const void* a0;            // [n_groups * R, K]
  const void* a1;            // second matrix (SwiGLU up) or nullptr
  const void* b;             // [rows, K]
  long long a_ld, b_ld;      // elements between rows
};

struct GemmParams {
  GemmClass cls[2];
  int n_classes;
  int* status;
  unsigned long long wait_limit_ns;
};

// Tensor-core grouped GEMM (bf16 in, fp32 accumulate). Tensor maps are built
// from the pointers in `maps` (see tc_gemm.cu). mats = 2 for SwiGLU.
struct TcOperand {
  const void* ptr;     // bf16 (or E4M3 codes with f8) [rows, K] row-major
  long long rows;
  long long K;
};
struct TcMaps {
  TcOperand a0[2], a1[2], b[2];
};
// pair = two-CTA tiles (tcgen05.mma.cta_group::2, 256 weight rows x up to 256 token
// rows per tile; bf16 SwiGLU / ReLU / down projections with bn = 256 and no K split).
cudaError_t launch_tc_gemm(int epi, int bn, const TcMaps& maps, const GemmParams& p, int num_ctas,
                           cudaStream_t s, bool f8 = false, bool pair = false);
int tc_pick_bn(int epi, double avg_rows_per_group);
// Whether the expert GEMMs of a layer with this mean segment length run as pair tiles.
bool tc_pick_pair(double avg_rows_per_group);
// Router logits + top-k softmax (+ per-tile expert counts and task ranks when lrank
// and tile_cnt are given) in one tensor-core launch (EPI_ROUTE); logits nullable.
cudaError_t launch_route_topk(const moe_config_t& c, const void* x, const void* w_r, const float* bias, float* logits,
                              int32_t* idx, float* w, int32_t* lrank, int32_t* tile_cnt, int* status,
                              unsigned long long wait_limit_ns, cudaStream_t s);
int tc_max_groups();
// Router logits by the kernel that suits the batch (CUDA cores for fp32 or small
// batches, the tensor cores otherwise); the bounded waits use wait_limit_ns().
cudaError_t launch_router_logits(const moe_config_t& c, const void* x, const void* w_r, const float* bias,
                                 float* logits, int* status, cudaStream_t s);
// The current time limit of the bounded waits (moe_debug_set_wait_limit_ns).
unsigned long long wait_limit_ns();
// moe_route's device work (logits, top-k, gate weights) by the kernels that suit the
// batch; logits_scratch (T m floats) serves when logits_out is NULL and a kernel
// needs the logits in memory.
cudaError_t launch_route(const moe_config_t& c, const void* x, const void* w_r, const float* bias,
                         const float* logits_in, float* logits_out, float* logits_scratch, int32_t* idx, float* w,
                         int* status, cudaStream_t s, bool stage_marks);

// SIMT grouped linear (fp32 or bf16 inputs, fp32 math), same GemmParams.
cudaError_t launch_simt_gemm(int epi, int dtype, const GemmParams& p, int max_rows_per_group, cudaStream_t s);

// Routing
cudaError_t launch_simt_logits(int dtype, int T, int d, int m, const void* x, const void* w_r, const float* bias,
                               float* logits, cudaStream_t s);
// logits of a few bf16 tokens (T <= 64) against few experts (m <= 32): one block per token.
bool few_expert_logits_ok(int dtype, int T, int m);
cudaError_t launch_few_expert_logits(int T, int d, int m, const void* x, const void* w, const float* bias,
                                     float* logits, cudaStream_t s);
cudaError_t launch_topk_softmax(int T, int m, int k, int renorm, const float* logits, int32_t* idx, float* w,
                                cudaStream_t s);
// logits (nullable), top-k ids and gate weights in one launch: bf16 layers with m <= 16.
bool small_route_ok(int dtype, int m);
cudaError_t launch_small_route(int T, int d, int m, int k, int renorm, const void* x, const void* w, const float* bias,
                               float* logits, int32_t* idx, float* wout, cudaStream_t s);
// Stable counting sort of the tasks by expert: route_index (one block: per-range
// counts, offsets when mode & 1 (plus counts and LIS), range start positions
// `start` [R][m], R * (m + 1) <= 8192) and rank (one warp per range: perm,
// inv_perm, w_perm); permute_rows then copies the rows. route_ranges gives R, L.
void route_ranges(int Tk, int m, int* R, int* L);
cudaError_t launch_route_index(int mode, int T, int k, int m, const int32_t* idx, int32_t* counts, int32_t* offsets,
                               moe_lis_t* lis, int32_t* start, int* status, cudaStream_t s);
// offsets, counts, LIS, perm / inv_perm / w_perm and x_perm from the router's tile
// counts and ranks (EPI_ROUTE): one block per (128-token tile, column part).
cudaError_t launch_route_scatter(int dtype, int T, int k, int m, int d, const int32_t* tile_cnt, const int32_t* idx,
                                 const int32_t* lrank, const float* task_w, const void* x, int32_t* counts,
                                 int32_t* offsets, moe_lis_t* lis, int32_t* perm, int32_t* inv_perm, float* w_perm,
                                 void* x_perm, int* status, cudaStream_t s);
// max / argmax / LIS (R&Q Definition 1) of a given histogram counts[m] over `tasks` tasks.
cudaError_t launch_lis_from_counts(int m, long long tasks, const int32_t* counts, moe_lis_t* lis, cudaStream_t s);
// R&Q replica dispatch: tasks of the heavy-hitter (lis_in->argmax_expert) with an
// odd rank in its segment go to expert m; writes idx_out, the group -> weight map
// [m + 1] and, when given, counts [m + 1] and the LIS over m + 1 experts.
cudaError_t launch_replica_split(int T, int k, int m, const int32_t* idx, const int32_t* offsets,
                                 const int32_t* inv_perm, const moe_lis_t* lis_in, int32_t* idx_out, int32_t* gmap,
                                 int32_t* counts_out, moe_lis_t* lis_out, int* status, cudaStream_t s);
// FloE contextual sparsity (csrc/floe.cu)
cudaError_t launch_floe_pack(int m, int d, int f, const void* w, void* w_t, cudaStream_t s);
cudaError_t launch_floe_calib(int Tc, int m, int f, const float* u, double sparsity, float* thr, cudaStream_t s);
// keep lists, then the gate + down stream writing partial outputs y[slot][row][:]
// (row_splits[row] slots per row, at most max_slots)
cudaError_t launch_floe_sparse_ffn(int m, int d, int f, const int32_t* offsets, const void* x_perm,
                                   const void* w_gate, const void* w_down_t, const float* u, const float* thr,
                                   int32_t* list, int32_t* cnt, const float* row_w, float* y, long long y_split,
                                   int max_slots, int32_t* row_splits, int32_t* kept_out, int* status,
                                   unsigned long long lim, cudaStream_t s);
int floe_chunks(int f);
int floe_chunk_size();
int floe_max_slots(long long rows, int d);  // partial-output slots the workspace holds per row
bool floe_shape_ok(int d, int f);           // d <= 8192, f <= 65536
cudaError_t launch_rank(int T, int k, int m, const int32_t* idx, const int32_t* offsets, const int32_t* start,
                        const float* task_w, int32_t* perm, int32_t* inv_perm, float* w_perm, int* status,
                        cudaStream_t s);
cudaError_t launch_permute_rows(int dtype, int Tk, int k, int d, const void* x, const int32_t* inv_perm, void* x_perm,
                                cudaStream_t s);
cudaError_t launch_combine(int dtype, int T, int d, int k, int ksplit, const float* y_perm, long long y_split_stride,
                           const int32_t* inv_perm, int n_shared, const float* y_shared, long long ysh_split_stride,
                           void* out, cudaStream_t s, const int32_t* row_splits = nullptr);
cudaError_t launch_reduce_splits(long long n, int ksplit, const float* in, long long split_stride, float* out,
                                 cudaStream_t s);

// Atomic experts
cudaError_t launch_atomic_select(int T, int Nr, int Nc, int K, int ksplit, const float* zr, long long zr_split,
                                 const float* zc, long long zc_split, float* lr_out, float* lc_out, int32_t* idx,
                                 float* g, int* status, unsigned* bar_reset, cudaStream_t s);
// coef and assembly in one cooperative launch with a grid barrier on `bar` (zeroed
// by the preceding select kernel when bar_zeroed, else by a memset here)
cudaError_t launch_atomic_experts(int T, int d, int K, int act, const void* x, const void* w_in, const void* w_out,
                                  const int32_t* idx, const float* g, float* coef, void* out, long long n_experts,
                                  unsigned* bar, bool bar_zeroed, unsigned long long limit_ns, int* status,
                                  cudaStream_t s);
// Per-row E4M3 codes + fp32 scales of bf16 rows [rows, cols] (row strides in
// elements, multiples of 8; src 16-byte and dst 8-byte aligned).
cudaError_t launch_quantize_e4m3(long long rows, int cols, const void* src, long long src_ld, uint8_t* dst,
                                 long long dst_ld, float* scale, cudaStream_t s);
// Records the profiling hook's event i (moe_set_stage_events) on `s`, if one is set.
cudaError_t mark_stage_event(int i, cudaStream_t s);

int num_sms();
void count_launch(int n = 1);

}  // namespace moe
