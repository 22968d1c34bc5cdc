// FloE contextual sparsity for the expert FFN ("FloE: On-the-Fly MoE Inference on
// Memory-constrained GPU", "Core claim" and Sec. 3.2; threshold: Eq. 6 via the
// empirical CDF of |up-projection activations|). For a task of expert e:
//   u = x W_up[e]^T (dense, tensor cores, fp32), channel j kept when |u_j| >= t_e,
//   h_j = g_j sigma(g_j) u_j with g_j = x . W_gate[e][j] for kept j (0 otherwise),
//   y = w * sum over kept j of h_j W_down[e][:, j].
// Only the gate rows and down columns of kept channels are read. Per expert the
// kept set is the union over its tasks (each task still zeroes its own pruned
// channels), cut into chunks of FL_CHUNK channels so many blocks build it at once.
// W_down is read channel-major, W_down_t[e][j][:] = W_down[e][:, j] (a one-time
// layout: moe_floe_pack_down), so a kept channel is one contiguous row.
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace moe {

namespace {
constexpr unsigned FULL = 0xffffffffu;
constexpr int FL_CHUNK = 1024;      // channels per kept-list chunk
constexpr int FL_KEEP_THREADS = 256;
}  // namespace

// ------------------------------------------------------------------ W_down layout
// w_t[e][j][i] = w[e][i][j] for the m [d, f] matrices; 32 x 32 tiles via shared memory.
__global__ void floe_pack_kernel(int m, int d, int f, const __nv_bfloat16* __restrict__ w,
                                 __nv_bfloat16* __restrict__ w_t) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int e = blockIdx.z;
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const __nv_bfloat16* src = w + (long long)e * d * f;
  __nv_bfloat16* dst = w_t + (long long)e * f * d;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = i0 + r, j = j0 + threadIdx.x;
    if (i < d && j < f) tile[r][threadIdx.x] = src[(long long)i * f + j];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int j = j0 + r, i = i0 + threadIdx.x;
    if (i < d && j < f) dst[(long long)j * d + i] = tile[threadIdx.x][r];
  }
}

cudaError_t launch_floe_pack(int m, int d, int f, const void* w, void* w_t, cudaStream_t s) {
  const dim3 grid((f + 31) / 32, (d + 31) / 32, m);
  floe_pack_kernel<<<grid, dim3(32, 8), 0, s>>>(m, d, f, (const __nv_bfloat16*)w, (__nv_bfloat16*)w_t);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ calibration
// t_e = the r-th smallest |u| over the n = Tc f values u[t][e f + j] of expert e,
// r = max(1, ceil(s n)) (Eq. 6's empirical CDF at sparsity s): an exact radix
// select over the bit patterns of |u| (monotone for non-negative floats), most
// significant byte first; one block per expert.
__global__ void floe_calib_kernel(int Tc, int m, int f, const float* __restrict__ u, double sparsity,
                                  float* __restrict__ thr) {
  __shared__ unsigned hist[256];
  __shared__ uint32_t prefix_s, mask_s;
  __shared__ long long rank_s;
  const int e = blockIdx.x;
  const long long n = (long long)Tc * f;
  long long r = (long long)ceil(sparsity * (double)n);
  if (r < 1) r = 1;
  if (r > n) r = n;
  if (threadIdx.x == 0) {
    prefix_s = 0;
    mask_s = 0;
    rank_s = r;  // rank still to find among values matching the prefix (1-based)
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = prefix_s, mask = mask_s;
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
      const long long t = i / f, j = i - t * f;
      const uint32_t key = __float_as_uint(fabsf(u[t * (long long)m * f + (long long)e * f + j]));
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      long long rk = rank_s;
      int dgt = 0;
      for (; dgt < 255; ++dgt) {  // ascending digits: smallest values first
        if ((long long)hist[dgt] >= rk) break;
        rk -= hist[dgt];
      }
      rank_s = rk;
      prefix_s = prefix | ((uint32_t)dgt << shift);
      mask_s = mask | (255u << shift);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) thr[e] = __uint_as_float(prefix_s);
}

cudaError_t launch_floe_calib(int Tc, int m, int f, const float* u, double sparsity, float* thr, cudaStream_t s) {
  floe_calib_kernel<<<m, 1024, 0, s>>>(Tc, m, f, u, sparsity, thr);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ kept channels
// Block (expert e, chunk c): channels j in [c FL_CHUNK, ...) kept by any of e's
// segment rows (|u[r][j]| >= t_e), listed in ascending order: list[e][c][0..cnt).
__global__ void __launch_bounds__(FL_KEEP_THREADS)
    floe_keep_kernel(int m, int f, int nchunks, const int32_t* __restrict__ offsets, const float* __restrict__ u,
                     const float* __restrict__ thr, int32_t* __restrict__ list, int32_t* __restrict__ cnt,
                     int* status) {
  __shared__ int warp_n[FL_KEEP_THREADS / 32];
  __shared__ int base_s;
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.x, c = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  const float t = thr[e];
  int32_t* out = list + ((long long)e * nchunks + c) * FL_CHUNK;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int j0 = c * FL_CHUNK; j0 < min(f, (c + 1) * FL_CHUNK); j0 += FL_KEEP_THREADS) {
    const int j = j0 + threadIdx.x;
    bool keep = false;
    if (j < f && j < (c + 1) * FL_CHUNK)
      for (int r = r0; r < r1 && !keep; ++r) keep = fabsf(u[(long long)r * f + j]) >= t;
    const unsigned bal = __ballot_sync(FULL, keep);
    if (lane == 0) warp_n[warp] = __popc(bal);
    __syncthreads();
    int before = base_s, total = 0;
    for (int w = 0; w < FL_KEEP_THREADS / 32; ++w) {
      if (w < warp) before += warp_n[w];
      total += warp_n[w];
    }
    if (keep) out[before + __popc(bal & ((1u << lane) - 1u))] = j;
    __syncthreads();
    if (threadIdx.x == 0) base_s += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) cnt[e * nchunks + c] = base_s;
  (void)status;
}

// ------------------------------------------------------------------ gate + down
// One streaming pass over the kept channels. The grid (one block per SM plus one
// spare per expert) is shared out in proportion to each expert's work, its kept
// channels K_e times its passes over the segment rows: expert e gets cs_e channel
// ranges (at most the partial-output slots the workspace holds) times rs_e ranges of
// passes, every block computing the same plan from the keep counts. A block streams
// the gate row W_gate[e][j] and the down row W_down_t[e][j] of a few kept channels
// at a time into a ring of shared-memory stages with bulk async copies (one thread
// issues them, the stage's mbarrier counts the bytes), so several stages are in
// flight while the block computes on the oldest:
//   gate: g[r][j] = x_r . W_gate[e][j], each warp over its own slice of d, then the
//         slices added across warps in warp order; h[r][j] = g sigma(g) u[r][j] when
//         |u[r][j]| >= t_e, else 0;
//   down: acc[r][cols] += h[r][j] W_down_t[e][j][cols] over the warp's own columns.
// At the end of a pass the block writes w_r acc[r] to its partial slot; the combine
// adds an expert's cs_e slots in slot order (as split-K), and row_splits[row] = cs_e
// tells it how many there are.
//
// Two kernels do the arithmetic. For d <= 4096, floe_mma_kernel: warp-level bf16
// tensor-core MMAs with fp32 accumulation read the staged rows with ldmatrix
// (which takes any row address, so the rows stay as the bulk copy lays them down),
// 8 token rows per pass (the MMA's 8-wide side), h rounded to bf16 as the dense
// path's intermediate is. For wider rows, floe_stream_kernel: fp32 FMAs on the
// CUDA cores, 4 token rows per pass.
namespace {
constexpr int FS_THREADS = 256;
constexpr int FS_WARPS = FS_THREADS / 32;
constexpr int FS_ROWS = 4;                     // segment rows per pass (CUDA-core kernel)
constexpr int FS_MAX_STAGES = 8;
constexpr int FS_DYN_BYTES = 212 * 1024;       // dynamic shared memory: stages (+ staged token rows)
constexpr int FS_PLAN_BYTES = 2 * 1024 * 4;    // the plan's per-expert arrays, borrowed from the ring
constexpr int FS_MAX_M = 1024;
constexpr size_t FS_SLOT_BUDGET = 256u << 20;  // bytes of partial-output slots in the workspace
constexpr int FM_THREADS = 512;
constexpr int FM_WARPS = FM_THREADS / 32;
constexpr int FM_ROWS = 8;                     // segment rows per pass (MMA kernel)
constexpr int FM_CB = 4;                       // kept channels per stage (MMA kernel)
constexpr int FM_MAX_D = 4096;
constexpr int FS_ID_WIN = 2048;                // kept-channel ids staged in shared memory per block

// Staged rows are FS_PITCH(d) = 2d + 16 bytes apart: a stage holds the CB gate rows
// in slots 0..CB-1 and the down rows in slots CB..2CB-1, so the 8 tile rows an
// ldmatrix reads (8 consecutive slots) start 16 bytes apart in the bank cycle and
// cover all 32 banks; rows 2d bytes apart would all start on the same banks.
__host__ __device__ constexpr size_t fs_pitch(int d) { return (size_t)d * 2 + 16; }

struct FsShared {
  unsigned long long wsum;
  int nz, e, sp, cs;
};

__device__ __forceinline__ void unpack_bf16x8(const uint4 v, float (&o)[8]) {
  o[0] = __uint_as_float(v.x << 16);
  o[1] = __uint_as_float(v.x & 0xffff0000u);
  o[2] = __uint_as_float(v.y << 16);
  o[3] = __uint_as_float(v.y & 0xffff0000u);
  o[4] = __uint_as_float(v.z << 16);
  o[5] = __uint_as_float(v.z & 0xffff0000u);
  o[6] = __uint_as_float(v.w << 16);
  o[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Sum of NV per-lane values over the warp, scattered: afterwards lane l holds the
// total of value l / (32 / NV). Each level halves the values a lane keeps (the half
// picked by one lane bit) and adds the partner's copy of that half; the levels left
// after one value remains add plainly.
template <int NV>
__device__ __forceinline__ float warp_reduce_scatter(float (&p)[NV], int lane) {
#pragma unroll
  for (int lvl = 0; (NV >> lvl) > 1; ++lvl) {
    const int n = NV >> lvl, o = 16 >> lvl;
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int t = 0; t < n / 2; ++t) {
      const float keep = hi ? p[n / 2 + t] : p[t];
      const float send = hi ? p[t] : p[n / 2 + t];
      p[t] = keep + __shfl_xor_sync(FULL, send, o);
    }
  }
  float v = p[0];
#pragma unroll
  for (int o = 16 / NV; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

// ---- warp-level MMA operands (8x8 b16 tiles; each lane names one 16-byte tile row)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr)
               : "memory");
}
// D[16 x 8] += A[16 x 16] B[16 x 8], bf16 operands, fp32 accumulators
__device__ __forceinline__ void mma_bf16_k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
               "{%0, %1, %2, %3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D[16 x 8] += A[16 x 8] B[8 x 8]
__device__ __forceinline__ void mma_bf16_k8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
               "{%0, %1, %2, %3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(b0));
}

// The block plan (every thread calls it): expert of this block, or -1 for a spare
// block; sp = its place among the expert's cs * rs blocks (channel range sp % cs,
// pass range sp / cs). Block 0 also writes kept_out and row_splits.
__device__ int floe_plan(int m, int nchunks, int fr, int nblk, int max_slots, const int32_t* __restrict__ offsets,
                         const int32_t* __restrict__ cnt, int32_t* __restrict__ row_splits,
                         int32_t* __restrict__ kept_out, int* nb_s, int* start_s, FsShared& sh, int& sp, int& cs,
                         int& rs) {
  const int tid = threadIdx.x, nth = blockDim.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    sh.wsum = 0;
    sh.nz = 0;
    sh.e = -1;
    sh.sp = 0;
    sh.cs = 1;
  }
  __syncthreads();
  for (int e = tid; e < m; e += nth) {
    int K = 0;
    for (int c = 0; c < nchunks; ++c) K += cnt[e * nchunks + c];
    const int rows = offsets[e + 1] - offsets[e];
    const unsigned long long w = rows > 0 ? (unsigned long long)K * ((rows + fr - 1) / fr) : 0ull;
    if (w) {
      atomicAdd(&sh.wsum, w);
      atomicAdd(&sh.nz, 1);
    }
    nb_s[e] = K;
    start_s[e] = rows;
    if (blockIdx.x == 0 && kept_out) kept_out[e] = K;
  }
  __syncthreads();
  const unsigned long long W = sh.wsum;
  const long long B = max(1, nblk - sh.nz);  // blocks shared out; each non-empty expert gets one more at most
  for (int e = tid; e < m; e += nth) {
    const int K = nb_s[e], rows = start_s[e];
    const int groups = (rows + fr - 1) / fr;
    const unsigned long long w = rows > 0 ? (unsigned long long)K * groups : 0ull;
    int nb = 0;
    if (w) {
      const int want = (int)max(1ll, min((long long)(B * w / W), (long long)nblk));
      const int c = min(want, min(max_slots, K));
      const int r = min(groups, max(1, want / c));
      nb = c * r;
      start_s[e] = c;  // channel ranges of e, until the scan below overwrites it
    }
    nb_s[e] = nb;
    if (blockIdx.x == 0)
      for (int r = offsets[e]; r < offsets[e + 1]; ++r) row_splits[r] = w ? start_s[e] : 0;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of nb_s into start_s
    const int per = (m + 31) / 32, b0 = min(m, lane * per), b1 = min(m, b0 + per);
    int sum = 0;
    for (int e = b0; e < b1; ++e) sum += nb_s[e];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int e = b0; e < b1; ++e) {
      const int c = nb_s[e] ? start_s[e] : 0;
      start_s[e] = run;
      if (nb_s[e] && (int)blockIdx.x >= run && (int)blockIdx.x < run + nb_s[e]) {
        sh.e = e;
        sh.sp = (int)blockIdx.x - run;
        sh.cs = c;
      }
      run += nb_s[e];
    }
  }
  __syncthreads();
  const int e = sh.e;
  sp = sh.sp;
  cs = sh.cs;
  rs = e >= 0 ? nb_s[e] / cs : 1;
  return e;
}

// The copy side of the stream (warp 0): the bulk copies of an item's gate and down
// rows into its stage, one row per lane so the copies are issued in parallel (one
// thread issuing them one after another is measurably slower). The block's
// kept-channel ids come from a window staged in shared memory at the start (idw, the
// first FS_ID_WIN of its range); past the window (ranges that long only arise when
// the workspace holds few partial-output slots) they are looked up in the keep lists.
template <int CB>
struct FsProducer {
  const int* coff;
  const int* idw;
  const int32_t* list_e;
  const __nv_bfloat16* wg_e;
  const __nv_bfloat16* wd_e;
  unsigned char* ring;
  uint64_t* full;
  int (*ids)[CB];
  int g0, g1, nbatch, nstages, nchunks, d;
  int issued;

  __device__ int id_at(int g) const {
    if (g - g0 < FS_ID_WIN) return idw[g - g0];
    int c = 0;
    while (c + 1 < nchunks && coff[c + 1] <= g) ++c;
    return list_e[c * FL_CHUNK + (g - coff[c])];
  }
  // every lane of warp 0 calls this
  __device__ void issue(int it, int lane) {
    static_assert(2 * CB <= 32, "one row per lane");
    const int st = it % nstages, gb = g0 + (it % nbatch) * CB;
    const int nv = min(CB, g1 - gb);  // channels in this item (>= 1)
    const size_t row_bytes = (size_t)d * 2, pitch = fs_pitch(d);
    unsigned char* base = ring + (size_t)st * CB * 2 * pitch;
    if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)(nv * 2 * row_bytes));
    __syncwarp();
    if (lane < 2 * nv) {  // lane 2v: gate row of channel v (slot v); lane 2v + 1: its down row (slot CB + v)
      const int v = lane >> 1;
      const long long row = (long long)id_at(gb + v) * d;
      fence_proxy_async_smem();
      bulk_copy_g2s(base + (size_t)((lane & 1) ? CB + v : v) * pitch, (lane & 1) ? wd_e + row : wg_e + row,
                    (uint32_t)row_bytes, &full[st]);
    }
    if (lane < CB) ids[st][lane] = lane < nv ? id_at(gb + lane) : -1;
    if (lane == 0) issued = it + 1;
  }
};

// Block setup shared by both kernels: the expert's chunk offsets (coff), the stage
// mbarriers, the block's channel range [g0, g1) (range ci of cs) and its id window.
__device__ void floe_setup(int e, int nchunks, int nstages, int ci, int cs, const int32_t* __restrict__ cnt,
                           const int32_t* __restrict__ list_e, int* coff, int* idw, uint64_t* full, int& g0,
                           int& g1) {
  const int tid = threadIdx.x;
  if (tid == 0) {
    int tot = 0;
    for (int c = 0; c < nchunks; ++c) {
      coff[c] = tot;
      tot += cnt[e * nchunks + c];
    }
    coff[nchunks] = tot;
    for (int st = 0; st < nstages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int K = coff[nchunks];
  g0 = (int)((long long)K * ci / cs);
  g1 = (int)((long long)K * (ci + 1) / cs);
  for (int i = tid; i < min(g1 - g0, FS_ID_WIN); i += blockDim.x) {
    const int g = g0 + i;
    int c = 0;
    while (c + 1 < nchunks && coff[c + 1] <= g) ++c;
    idw[i] = list_e[c * FL_CHUNK + (g - coff[c])];
  }
  __syncthreads();
}
}  // namespace

// ---- CUDA-core variant (rows wider than 4096): every thread dots its 16-byte column
// chunks of the staged gate rows with the same chunks of the pass's token rows (held
// in registers); the block adds the partials (warp reduce-scatter, then across warps
// in warp order).
template <int DQ, int CB>  // DQ: 16-byte column chunks per thread (d <= 2048 DQ); CB: channels per stage
__global__ void __launch_bounds__(FS_THREADS, 1)
    floe_stream_kernel(int m, int d, int f, int nchunks, int nstages, int nblk, int max_slots,
                       const int32_t* __restrict__ offsets, const uint4* __restrict__ x_perm,
                       const __nv_bfloat16* __restrict__ w_gate, const __nv_bfloat16* __restrict__ w_down_t,
                       const float* __restrict__ u, const float* __restrict__ thr, const int32_t* __restrict__ list,
                       const int32_t* __restrict__ cnt, const float* __restrict__ row_w, float* __restrict__ y,
                       long long y_split, int32_t* __restrict__ row_splits, int32_t* __restrict__ kept_out,
                       int* status, unsigned long long lim) {
  constexpr int FR = FS_ROWS, NV = CB * FR;
  constexpr bool XP = DQ > 2;  // token rows kept as bf16 (unpacked per use) to stay in registers
  static_assert(32 % NV == 0, "gate values per stage");
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ uint64_t full[FS_MAX_STAGES];
  __shared__ int coff[64 + 1];
  __shared__ int idw[FS_ID_WIN];
  __shared__ int ids[FS_MAX_STAGES][CB];
  __shared__ float red[FS_WARPS][NV];
  __shared__ float hs[NV];
  __shared__ FsShared sh;
  __shared__ volatile int abort_s;
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int sp, cs, rs;
  // the plan's per-expert arrays borrow the ring before the first copy is issued
  const int e = floe_plan(m, nchunks, FR, nblk, max_slots, offsets, cnt, row_splits, kept_out,
                          reinterpret_cast<int*>(ring), reinterpret_cast<int*>(ring) + FS_MAX_M, sh, sp, cs, rs);
  if (e < 0) return;  // a spare block
  const int ci = sp % cs, ri = sp / cs;
  if (tid == 0) abort_s = 0;
  const int32_t* list_e = list + (long long)e * nchunks * FL_CHUNK;
  int g0, g1;
  floe_setup(e, nchunks, nstages, ci, cs, cnt, list_e, coff, idw, full, g0, g1);
  const int r0 = offsets[e], r1 = offsets[e + 1];
  const int groups = (r1 - r0 + FR - 1) / FR;
  const int ga = (int)((long long)groups * ri / rs), gb = (int)((long long)groups * (ri + 1) / rs);
  const int nbatch = (g1 - g0 + CB - 1) / CB;
  const int nitems = nbatch * (gb - ga);
  const float t_e = thr[e];
  const int d8 = d / 8;
  const size_t pitch = fs_pitch(d);
  const size_t stage_bytes = (size_t)CB * 2 * pitch;
  float* ys = y + (long long)ci * y_split;
  __shared__ FsProducer<CB> pr;  // thread 0's copy-side state, kept out of every thread's registers
  if (tid == 0) {
    pr.coff = coff;
    pr.idw = idw;
    pr.list_e = list_e;
    pr.wg_e = w_gate + (long long)e * f * d;
    pr.wd_e = w_down_t + (long long)e * f * d;
    pr.ring = ring;
    pr.full = full;
    pr.ids = ids;
    pr.g0 = g0;
    pr.g1 = g1;
    pr.nbatch = nbatch;
    pr.nstages = nstages;
    pr.nchunks = nchunks;
    pr.d = d;
    pr.issued = 0;
  }
  __syncthreads();
  if (warp == 0)
    for (int it = 0; it < min(nstages, nitems); ++it) pr.issue(it, lane);
  __syncthreads();

  float xr[FR][XP ? 1 : DQ][8], acc[FR][DQ][8];
  uint4 xp[FR][XP ? DQ : 1];
  // u of an item for lane v FR + r < NV of warp 1 (channel v, row r); warp 1 loads the
  // next item's while this one runs (its ids are in the ring by then: >= 3 stages)
  auto load_u = [&](int it2, int& idv, float& uv) {
    const int rg2 = r0 + (ga + it2 / nbatch) * FR, nr2 = min(FR, r1 - rg2);
    idv = -1;
    uv = 0.f;
    if (lane < NV) {
      idv = ids[it2 % nstages][lane / FR];
      if (idv >= 0 && lane % FR < nr2) uv = u[(long long)(rg2 + lane % FR) * f + idv];
    }
  };
  int id_cur = -1;
  float u_cur = 0.f;
  if (warp == 1 && nitems > 0) load_u(0, id_cur, u_cur);
  int it = 0;
  for (; it < nitems; ++it) {
    const int gi = ga + it / nbatch, bi = it % nbatch;
    const int st = it % nstages;
    const uint32_t par = (uint32_t)(it / nstages) & 1u;
    const int rg = r0 + gi * FR, nr = min(FR, r1 - rg);
    const unsigned char* base = ring + (size_t)st * stage_bytes;
    if (bi == 0) {  // a new pass: its token rows, zeroed accumulators
#pragma unroll
      for (int r = 0; r < FR; ++r)
#pragma unroll
        for (int q = 0; q < DQ; ++q) {
          const int c = tid + FS_THREADS * q;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (r < nr && c < d8) v = x_perm[(long long)(rg + r) * d8 + c];
          if constexpr (XP)
            xp[r][q] = v;
          else
            unpack_bf16x8(v, xr[r][q]);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[r][q][j] = 0.f;
        }
    }
    int id_nx = -1;
    float u_nx = 0.f;
    if (warp == 1 && it + 1 < nitems) load_u(it + 1, id_nx, u_nx);
    const bool ok = mbar_wait(&full[st], par, lim, &abort_s);
    if (!ok) {
      set_status(status, MOE_ERR_TIMEOUT);
      abort_s = 1;
    }
    float p[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) p[i] = 0.f;
    if (ok) {
#pragma unroll
      for (int v = 0; v < CB; ++v)
#pragma unroll
        for (int q = 0; q < DQ; ++q) {
          const int c = tid + FS_THREADS * q;
          if (c < d8) {
            float wv[8];
            unpack_bf16x8(*reinterpret_cast<const uint4*>(base + (size_t)v * pitch + (size_t)c * 16), wv);
#pragma unroll
            for (int r = 0; r < FR; ++r) {
              float xv[8];
              if constexpr (XP)
                unpack_bf16x8(xp[r][q], xv);
              else
#pragma unroll
                for (int j = 0; j < 8; ++j) xv[j] = xr[r][q][j];
#pragma unroll
              for (int j = 0; j < 8; ++j) p[v * FR + r] = fmaf(wv[j], xv[j], p[v * FR + r]);
            }
          }
        }
    }
    {
      const float v = warp_reduce_scatter<NV>(p, lane);
      if (lane % (32 / NV) == 0) red[warp][lane / (32 / NV)] = v;
    }
    __syncthreads();
    if (abort_s) break;
    if (warp == 0 && it >= 1 && it - 1 + nstages < nitems) pr.issue(it - 1 + nstages, lane);  // the previous stage is free
    if (warp == 1 && lane < NV) {  // off thread 0's warp, which issues copies meanwhile
      float g = 0.f;
#pragma unroll
      for (int w = 0; w < FS_WARPS; ++w) g += red[w][lane];
      hs[lane] = (id_cur >= 0 && lane % FR < nr && fabsf(u_cur) >= t_e) ? g / (1.f + expf(-g)) * u_cur : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int v = 0; v < CB; ++v) {
      if (ids[st][v] < 0) continue;
      float h[FR];
#pragma unroll
      for (int r = 0; r < FR; ++r) h[r] = hs[v * FR + r];
#pragma unroll
      for (int q = 0; q < DQ; ++q) {
        const int c = tid + FS_THREADS * q;
        if (c < d8) {
          float wv[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(base + (size_t)(CB + v) * pitch + (size_t)c * 16), wv);
#pragma unroll
          for (int r = 0; r < FR; ++r)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[r][q][j] = fmaf(h[r], wv[j], acc[r][q][j]);
        }
      }
    }
    if (bi == nbatch - 1) {  // the pass is complete: w_r acc to this block's slot
#pragma unroll
      for (int r = 0; r < FR; ++r) {
        if (r >= nr) break;
        const float wr = row_w ? row_w[rg + r] : 1.f;
#pragma unroll
        for (int q = 0; q < DQ; ++q) {
          const int c = tid + FS_THREADS * q;
          if (c < d8) {
            float4* o = reinterpret_cast<float4*>(ys + (long long)(rg + r) * d) + 2 * c;
            o[0] = make_float4(acc[r][q][0] * wr, acc[r][q][1] * wr, acc[r][q][2] * wr, acc[r][q][3] * wr);
            o[1] = make_float4(acc[r][q][4] * wr, acc[r][q][5] * wr, acc[r][q][6] * wr, acc[r][q][7] * wr);
          }
        }
      }
    }
    id_cur = id_nx;
    u_cur = u_nx;
  }
  if (tid == 0) {  // after an abort: let the copies still in flight land before the block exits
    const volatile int never = 0;
    for (int j = it; j < pr.issued; ++j)
      if (!mbar_wait(&full[j % nstages], (uint32_t)(j / nstages) & 1u, lim, &never)) break;
  }
  __syncthreads();
}

// ---- tensor-core variant (d <= 4096). Warp w owns the 16-column units
// [w KT, (w + 1) KT) of d, for the gate's reduction dimension and the down's output
// columns alike. Lane (g = lane / 4, t = lane % 4) holds, per unit u:
//   gate  (M = 16 token rows, 8 real; N = 8 channels, CB real; K = the unit):
//         A = x[g][16u + 2t, +1] and x[g][16u + 8 + 2t, +1], built once per pass and
//         kept in registers, or (XS, from 8 units per warp on, so that the registers
//         can hold the accumulators) as the pass's token rows staged in shared memory
//         and read through ldmatrix; B = the staged gate rows through ldmatrix (a
//         channel's row is a tile row); D = this warp's partial g[g][2t, 2t + 1];
//   down  (M = the unit's 16 columns; N = 8 token rows; K = 8 channels, CB real):
//         A = the staged down rows through ldmatrix.trans (channel = tile row, its 8
//         columns transposed into the fragment); B = h[g][2t, 2t + 1] as bf16;
//         D = acc[cols 16u + g, + 8][rows 2t, 2t + 1].
// Channels past CB or past the range, and columns past d, read a zero tile row.
// FULL: d = 256 KT, every warp's units all inside d (no column checks).
template <int KT, bool FULL, int CB, bool XS>
__global__ void __launch_bounds__(FM_THREADS, 1)
    floe_mma_kernel(int m, int d, int f, int nchunks, int nstages, int nblk, int max_slots,
                    const int32_t* __restrict__ offsets, const uint32_t* __restrict__ x_perm,
                    const __nv_bfloat16* __restrict__ w_gate, const __nv_bfloat16* __restrict__ w_down_t,
                    const float* __restrict__ u, const float* __restrict__ thr, const int32_t* __restrict__ list,
                    const int32_t* __restrict__ cnt, const float* __restrict__ row_w, float* __restrict__ y,
                    long long y_split, int32_t* __restrict__ row_splits, int32_t* __restrict__ kept_out, int* status,
                    unsigned long long lim) {
  constexpr int FR = FM_ROWS;
  static_assert(FR == 8 && CB >= 1 && CB <= 8 && FR * CB <= 32, "MMA shapes; one u value per lane of warp 1");
  static_assert(!FULL || KT % 2 == 0, "full tiles come in unit pairs");
  static_assert(!XS || KT % 2 == 0, "staged token rows are read in unit pairs");
  // dynamic: the stage ring, then (XS) the pass's token rows [FR][d]; the plan's
  // per-expert arrays borrow the ring before the first copy is issued
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ uint64_t full[FS_MAX_STAGES];
  __shared__ int coff[64 + 1];
  __shared__ int idw[FS_ID_WIN];
  __shared__ int ids[FS_MAX_STAGES][CB];
  __shared__ float red[FM_WARPS][FR][CB];
  __shared__ __align__(16) __nv_bfloat16 hs[FR][8];  // h[row][channel]; channels CB..7 stay 0
  __shared__ __align__(16) uint32_t zero_row[4];
  __shared__ FsShared sh;
  __shared__ volatile int abort_s;
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int sp, cs, rs;
  const int e = floe_plan(m, nchunks, FR, nblk, max_slots, offsets, cnt, row_splits, kept_out,
                          reinterpret_cast<int*>(ring), reinterpret_cast<int*>(ring) + FS_MAX_M, sh, sp, cs, rs);
  if (e < 0) return;  // a spare block
  const int ci = sp % cs, ri = sp / cs;
  if (tid == 0) abort_s = 0;
  const int32_t* list_e = list + (long long)e * nchunks * FL_CHUNK;
  int g0, g1;
  floe_setup(e, nchunks, nstages, ci, cs, cnt, list_e, coff, idw, full, g0, g1);
  if (tid < 4) zero_row[tid] = 0u;
  if (tid < FR * 8) hs[tid / 8][tid % 8] = __float2bfloat16_rn(0.f);
  const int r0 = offsets[e], r1 = offsets[e + 1];
  const int groups = (r1 - r0 + FR - 1) / FR;
  const int ga = (int)((long long)groups * ri / rs), gb = (int)((long long)groups * (ri + 1) / rs);
  const int nbatch = (g1 - g0 + CB - 1) / CB;
  const int nitems = nbatch * (gb - ga);
  const float t_e = thr[e];
  const uint32_t pitch = (uint32_t)fs_pitch(d);
  const uint32_t stage_bytes = (uint32_t)CB * 2 * pitch;
  float* ys = y + (long long)ci * y_split;
  __shared__ FsProducer<CB> pr;  // thread 0's copy-side state, kept out of every thread's registers
  if (tid == 0) {
    pr.coff = coff;
    pr.idw = idw;
    pr.list_e = list_e;
    pr.wg_e = w_gate + (long long)e * f * d;
    pr.wd_e = w_down_t + (long long)e * f * d;
    pr.ring = ring;
    pr.full = full;
    pr.ids = ids;
    pr.g0 = g0;
    pr.g1 = g1;
    pr.nbatch = nbatch;
    pr.nstages = nstages;
    pr.nchunks = nchunks;
    pr.d = d;
    pr.issued = 0;
  }
  __syncthreads();
  if (warp == 0)
    for (int it = 0; it < min(nstages, nitems); ++it) pr.issue(it, lane);
  __syncthreads();

  const int g = lane >> 2, t = lane & 3;
  const int q = lane & 7, j = lane >> 3;  // ldmatrix: this lane names row q of tile j
  const int n16 = (d + 15) / 16;
  const int ub = warp * KT;  // first unit of this warp
  const int k0 = 16 * (ub + (j >> 1)) + 8 * (j & 1);  // this lane's tile column in the first unit pair
  const uint32_t zero_addr = smem_u32(zero_row), ring_addr = smem_u32(ring);
  const uint32_t xs_addr = ring_addr + (uint32_t)nstages * stage_bytes;  // XS: token rows, FR rows pitch apart
  uint32_t xa[XS ? 1 : KT][2];
  float acc[KT][4];
  // u of an item for lane r CB + v < FR CB of warp 1 (row r, channel v); warp 1 loads
  // the next item's while this one runs (its ids are in the ring by then: >= 3 stages)
  auto load_u = [&](int it2, int& idv, float& uv) {
    const int rg2 = r0 + (ga + it2 / nbatch) * FR, nr2 = min(FR, r1 - rg2);
    idv = -1;
    uv = 0.f;
    if (lane < FR * CB) {
      idv = ids[it2 % nstages][lane % CB];
      if (idv >= 0 && lane / CB < nr2) uv = u[(long long)(rg2 + lane / CB) * f + idv];
    }
  };
  int id_cur = -1;
  float u_cur = 0.f;
  if (warp == 1 && nitems > 0) load_u(0, id_cur, u_cur);
  int it = 0;
  bool aborted = false;
  for (int gi = ga; gi < gb && !aborted; ++gi) {  // one pass: FR token rows against the whole channel range
    const int rg = r0 + gi * FR, nr = min(FR, r1 - rg);
    if constexpr (XS) {  // the pass's token rows into shared memory (rows past nr zero)
      const int d8 = d / 8;
      for (int i = tid; i < FR * d8; i += FM_THREADS) {
        const int r = i / d8, c = i - r * d8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < nr) v = reinterpret_cast<const uint4*>(x_perm)[(long long)(rg + r) * d8 + c];
        *reinterpret_cast<uint4*>(ring + (size_t)nstages * stage_bytes + (size_t)r * pitch + (size_t)c * 16) = v;
      }
      __syncthreads();
    } else {
#pragma unroll
      for (int uu = 0; uu < KT; ++uu) {  // the pass's token rows as the gate's A fragments
        const int k = 16 * (ub + uu) + 2 * t;
        uint32_t v0 = 0u, v1 = 0u;
        if (g < nr) {
          const uint32_t* xrow = x_perm + (long long)(rg + g) * (d / 2);
          if (FULL || k < d) v0 = xrow[k / 2];
          if (FULL || k + 8 < d) v1 = xrow[(k + 8) / 2];
        }
        xa[XS ? 0 : uu][0] = v0;
        xa[XS ? 0 : uu][1] = v1;
      }
    }
#pragma unroll
    for (int uu = 0; uu < KT; ++uu)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[uu][i] = 0.f;
    for (int bi = 0; bi < nbatch; ++bi, ++it) {
      const int st = it % nstages;
      const uint32_t par = (uint32_t)(it / nstages) & 1u;
      const uint32_t stage_addr = ring_addr + (uint32_t)st * stage_bytes;
      int id_nx = -1;
      float u_nx = 0.f;
      if (warp == 1 && it + 1 < nitems) load_u(it + 1, id_nx, u_nx);
      const bool ok = mbar_wait(&full[st], par, lim, &abort_s);
      if (!ok) {
        set_status(status, MOE_ERR_TIMEOUT);
        abort_s = 1;
      }
      const int idq = q < CB ? ids[st][q] : -1;  // the channel behind this lane's tile row
      float c[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};  // two chains of dependent MMAs
      if (ok) {
        const uint32_t grow = stage_addr + (uint32_t)q * pitch;
        if constexpr (KT == 1) {
          const int k = 16 * ub + 8 * (j & 1);
          const uint32_t addr = (idq >= 0 && k < d) ? grow + 2u * k : zero_addr;
          uint32_t b0, b1;
          ldsm_x2(addr, b0, b1);
          if (ub < n16) mma_bf16_k16(c, xa[0][0], 0u, xa[0][1], 0u, b0, b1);
        } else {
          // this lane's tile row of the first unit pair, then 64 bytes per pair (0 for the zero row)
          const uint32_t base = idq >= 0 ? grow + 2u * k0 : zero_addr, step = idq >= 0 ? 64u : 0u;
#pragma unroll
          for (int uu = 0; uu < KT; uu += 2) {
            if (!FULL && ub + uu >= n16) break;
            const uint32_t addr = (FULL || k0 + 16 * uu < d) ? base + step * (uu / 2) : zero_addr;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(addr, b0, b1, b2, b3);
            if constexpr (XS) {
              uint32_t x0, x1, x2, x3;  // rows q of the pass, the same tile columns
              const uint32_t xaddr = (FULL || k0 + 16 * uu < d) ? xs_addr + (uint32_t)q * pitch + 2u * k0 + 64u * (uu / 2)
                                                                : zero_addr;
              ldsm_x4(xaddr, x0, x1, x2, x3);
              mma_bf16_k16(c, x0, 0u, x1, 0u, b0, b1);
              mma_bf16_k16(c2, x2, 0u, x3, 0u, b2, b3);
            } else {
              mma_bf16_k16(c, xa[uu][0], 0u, xa[uu][1], 0u, b0, b1);
              mma_bf16_k16(c2, xa[uu + 1][0], 0u, xa[uu + 1][1], 0u, b2, b3);
            }
          }
        }
      }
      if (2 * t < CB) red[warp][g][2 * t] = c[0] + c2[0];
      if (2 * t + 1 < CB) red[warp][g][2 * t + 1] = c[1] + c2[1];
      __syncthreads();
      if (abort_s) {
        aborted = true;
        break;
      }
      if (warp == 0 && it >= 1 && it - 1 + nstages < nitems) pr.issue(it - 1 + nstages, lane);  // the previous stage is free
      if (warp == 1 && lane < FR * CB) {  // off thread 0's warp, which issues copies meanwhile
        const int r = lane / CB, v = lane % CB;
        float gs = 0.f;
#pragma unroll
        for (int w = 0; w < FM_WARPS; ++w) gs += red[w][r][v];
        const float hv = (id_cur >= 0 && r < nr && fabsf(u_cur) >= t_e) ? gs / (1.f + expf(-gs)) * u_cur : 0.f;
        hs[r][v] = __float2bfloat16_rn(hv);
      }
      __syncthreads();
      {
        const uint32_t b = *reinterpret_cast<const uint32_t*>(&hs[g][2 * t]);
        const uint32_t drow = stage_addr + (uint32_t)(CB + q) * pitch;
        if constexpr (KT == 1) {
          const int col = 16 * ub + 8 * (j & 1);
          const uint32_t addr = (idq >= 0 && col < d) ? drow + 2u * col : zero_addr;
          uint32_t a0, a1;
          ldsm_x2_t(addr, a0, a1);
          if (ub < n16) mma_bf16_k8(acc[0], a0, a1, b);
        } else {
          const uint32_t base = idq >= 0 ? drow + 2u * k0 : zero_addr, step = idq >= 0 ? 64u : 0u;
#pragma unroll
          for (int uu = 0; uu < KT; uu += 2) {
            if (!FULL && ub + uu >= n16) break;
            const uint32_t addr = (FULL || k0 + 16 * uu < d) ? base + step * (uu / 2) : zero_addr;
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(addr, a0, a1, a2, a3);
            mma_bf16_k8(acc[uu], a0, a1, b);
            mma_bf16_k8(acc[uu + 1], a2, a3, b);
          }
        }
      }
      id_cur = id_nx;
      u_cur = u_nx;
    }
    if (aborted) break;
    // the pass is complete: w_r acc to this block's slot
    const int ra = 2 * t, rb = 2 * t + 1;
    const float wa = ra < nr ? (row_w ? row_w[rg + ra] : 1.f) : 0.f;
    const float wb = rb < nr ? (row_w ? row_w[rg + rb] : 1.f) : 0.f;
    float* oa = ys + (long long)(rg + ra) * d + 16 * ub + g;
    float* ob = ys + (long long)(rg + rb) * d + 16 * ub + g;
#pragma unroll
    for (int uu = 0; uu < KT; ++uu) {
      const int c0 = 16 * (ub + uu) + g;
      if (ra < nr) {
        if (FULL || c0 < d) oa[16 * uu] = acc[uu][0] * wa;
        if (FULL || c0 + 8 < d) oa[16 * uu + 8] = acc[uu][2] * wa;
      }
      if (rb < nr) {
        if (FULL || c0 < d) ob[16 * uu] = acc[uu][1] * wb;
        if (FULL || c0 + 8 < d) ob[16 * uu + 8] = acc[uu][3] * wb;
      }
    }
    if constexpr (XS) __syncthreads();  // every warp is past its last read of the staged rows
  }
  if (tid == 0) {  // after an abort: let the copies still in flight land before the block exits
    const volatile int never = 0;
    for (int jj = it; jj < pr.issued; ++jj)
      if (!mbar_wait(&full[jj % nstages], (uint32_t)(jj / nstages) & 1u, lim, &never)) break;
  }
  __syncthreads();
}

cudaError_t launch_floe_sparse_ffn(int m, int d, int f, const int32_t* offsets, const void* x_perm,
                                   const void* w_gate, const void* w_down_t, const float* u, const float* thr,
                                   int32_t* list, int32_t* cnt, const float* row_w, float* y, long long y_split,
                                   int max_slots, int32_t* row_splits, int32_t* kept_out, int* status,
                                   unsigned long long lim, cudaStream_t s) {
  const int nchunks = (f + FL_CHUNK - 1) / FL_CHUNK;
  launch_k(floe_keep_kernel, dim3(m, nchunks), FL_KEEP_THREADS, 0, s, m, f, nchunks, offsets, u, thr, list, cnt,
           status);
  count_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int nblk = num_sms();
  const dim3 grid(nblk + m);
#define MOE_FLOE_RING(KERN_, CB_, XS_BYTES_, THREADS_, XTYPE_)                                                  \
  do {                                                                                                          \
    const size_t stage = (size_t)(CB_) * 2 * fs_pitch(d), xs_bytes = (XS_BYTES_);                              \
    const int nst = (int)std::min<size_t>(FS_MAX_STAGES, (FS_DYN_BYTES - xs_bytes) / stage);                   \
    if (nst < 3) return cudaErrorInvalidValue; /* the u prefetch reads ids one item ahead */                   \
    const size_t dyn = std::max<size_t>(FS_PLAN_BYTES, nst * stage + xs_bytes);                                \
    static bool attr = false;                                                                                   \
    if (!attr) {                                                                                                \
      err = cudaFuncSetAttribute(KERN_, cudaFuncAttributeMaxDynamicSharedMemorySize, FS_DYN_BYTES);             \
      if (err != cudaSuccess) return err;                                                                       \
      attr = true;                                                                                              \
    }                                                                                                           \
    err = launch_k(KERN_, grid, THREADS_, dyn, s, m, d, f, nchunks, nst, nblk, max_slots, offsets,             \
                   (const XTYPE_*)x_perm, (const __nv_bfloat16*)w_gate, (const __nv_bfloat16*)w_down_t, u, thr, \
                   (const int32_t*)list, (const int32_t*)cnt, row_w, y, y_split, row_splits, kept_out, status,  \
                   lim);                                                                                        \
  } while (0)
  const int n16 = (d + 15) / 16;
  // token-row fragments in registers up to 4 units per warp (and at d = 2048), else
  // staged in shared memory so the registers can hold the accumulators
  if (d == 4096)
    MOE_FLOE_RING((floe_mma_kernel<16, true, 3, true>), 3, (size_t)FM_ROWS * fs_pitch(d), FM_THREADS, uint32_t);
  else if (d == 2048)
    MOE_FLOE_RING((floe_mma_kernel<8, true, FM_CB, false>), FM_CB, 0, FM_THREADS, uint32_t);
  else if (n16 <= FM_WARPS)
    MOE_FLOE_RING((floe_mma_kernel<1, false, FM_CB, false>), FM_CB, 0, FM_THREADS, uint32_t);
  else if (n16 <= 2 * FM_WARPS)
    MOE_FLOE_RING((floe_mma_kernel<2, false, FM_CB, false>), FM_CB, 0, FM_THREADS, uint32_t);
  else if (n16 <= 4 * FM_WARPS)
    MOE_FLOE_RING((floe_mma_kernel<4, false, FM_CB, false>), FM_CB, 0, FM_THREADS, uint32_t);
  else if (n16 <= 8 * FM_WARPS)
    MOE_FLOE_RING((floe_mma_kernel<8, false, FM_CB, true>), FM_CB, (size_t)FM_ROWS * fs_pitch(d), FM_THREADS,
                  uint32_t);
  else if (d <= FM_MAX_D)  // 2048 < d < 4096: as at 4096, with column checks
    MOE_FLOE_RING((floe_mma_kernel<16, false, 3, true>), 3, (size_t)FM_ROWS * fs_pitch(d), FM_THREADS, uint32_t);
  else
    MOE_FLOE_RING((floe_stream_kernel<4, 2>), 2, 0, FS_THREADS, uint4);
#undef MOE_FLOE_RING
  count_launch();
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// partial-output slots per segment row the workspace holds
int floe_max_slots(long long rows, int d) {
  const long long per = std::max(1ll, rows * d * 4);
  return (int)std::max(1ll, std::min<long long>(64, (long long)FS_SLOT_BUDGET / per));
}
bool floe_shape_ok(int d, int f) { return d <= 4 * 8 * FS_THREADS && f <= 64 * FL_CHUNK; }

int floe_chunks(int f) { return (f + FL_CHUNK - 1) / FL_CHUNK; }
int floe_chunk_size() { return FL_CHUNK; }

}  // namespace moe
