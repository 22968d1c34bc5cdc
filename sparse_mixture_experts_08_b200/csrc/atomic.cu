// Atomic-expert layer (OmniMoE): Cartesian Product Router selection and the
// Dynamic Expert Assembly of atomic experts sigma(x w_in^T) w_out.
//
// Exact top-K over the implicit Nr x Nc grid (OmniMoE App. A), scores
// S(i,j) = fl32(lr_i + lc_j), order (S desc, flat id i*Nc + j asc):
//  1. R = top-K rows by (lr desc, i asc), C = top-K cols by (lc desc, j asc).
//  2. tau = K-th best score inside R x C.
//  3. No pair outside R x C scores ABOVE tau: for i not in R and any j, every
//     (i', j') in R x C' (C' = the K best columns when j not in C, else j itself)
//     has lr_i' >= lr_i and lc_j' >= lc_j, so fl(lr_i' + lc_j') >= fl(lr_i + lc_j)
//     (rounding is monotone); that gives K pairs at least as good, so the pair
//     can only tie tau. Hence the answer = the pairs of R x C above tau, followed
//     by the lowest-id pairs of the WHOLE grid that equal tau. (Selecting inside
//     R x C alone is not exact: rounding can make a pair outside R x C tie tau
//     with a lower flat id.)
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace moe {

namespace {
constexpr unsigned FULL = 0xffffffffu;
constexpr int SEL_THREADS = 1024;
constexpr int SEL_MAX_SIDE = 1024;
constexpr int SEL_MAX_K = 64;
constexpr int SEL_CAND = SEL_MAX_K * SEL_MAX_K;  // 4096

__device__ __forceinline__ uint32_t ordered_bits(float v) {
  if (v == 0.f) v = 0.f;  // -0 and +0 are equal scores
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ uint64_t make_key(float v, uint32_t id) {
  return ((uint64_t)ordered_bits(v) << 32) | (uint64_t)(0xFFFFFFFFu - id);
}
__device__ __forceinline__ uint32_t key_id(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu); }

__device__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = -FLT_MAX;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}
__device__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double r = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r += red[w];
  __syncthreads();
  return r;
}
}  // namespace

__device__ __forceinline__ float ordered_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

constexpr int TIE_CAP = 512;

// One block per token. zr/zc: split-K partial logits [ksplit][T][Nr|Nc].
//  1. log-softmax of the row and column logits (fp32 values; max and
//     log-sum-exp in fp64);
//  2. R, C: top-K rows / columns by (value desc, index asc), each element's rank
//     counted directly (one comparison pass, no sort);
//  3. tau = K-th largest S over R x C: radix select over the order-preserving
//     32-bit image of the fp32 scores (four 8-bit passes);
//  4. the pairs of R x C above tau (fewer than K), and the pairs of the whole grid
//     equal to tau (scanned in parallel, kept when at most TIE_CAP; otherwise the
//     exact flat-id-order block scan runs instead), of which the lowest `need` ids;
//  5. the K winners ordered by (S desc, id asc) by rank counting; g = softmax.
__global__ void __launch_bounds__(SEL_THREADS, 1)
    atomic_select_kernel(int T, int Nr, int Nc, int K, int ksplit, const float* __restrict__ zr, long long zr_split,
                         const float* __restrict__ zc, long long zc_split, float* __restrict__ lr_out,
                         float* __restrict__ lc_out, int32_t* __restrict__ idx_out, float* __restrict__ g_out,
                         int* status) {
  __shared__ float lr[SEL_MAX_SIDE], lc[SEL_MAX_SIDE];
  __shared__ float redf[32];
  __shared__ double redd[32];
  __shared__ int rows_sel[SEL_MAX_K], cols_sel[SEL_MAX_K];
  __shared__ unsigned hist[256];
  __shared__ unsigned whist[SEL_THREADS / 32][257];  // per-warp histograms (+1 bin for non-matching keys)
  __shared__ uint32_t prefix_s, mask_s;
  __shared__ int krem_s;
  __shared__ int n_gt, n_tie, found_s;
  __shared__ uint32_t gt_ids[SEL_MAX_K], tie_ids[TIE_CAP], win_ids[SEL_MAX_K];
  __shared__ int warp_cnt[32];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = blockDim.x;
  pdl_launch_dependents();
  pdl_wait();

  // 1. sum the split-K partials; log-softmax of rows and of columns
  for (int side = 0; side < 2; ++side) {
    const int n = side ? Nc : Nr;
    const float* z = side ? zc : zr;
    const long long sp = side ? zc_split : zr_split;
    float* l = side ? lc : lr;
    float v = -FLT_MAX;
    if (tid < n) {
      float a = 0.f;
      for (int s = 0; s < ksplit; ++s) a += z[s * sp + (long long)t * n + tid];
      l[tid] = a;
      v = a;
    }
    const float mx = block_max(v, redf);
    const double se = block_sum(tid < n ? (double)expf(l[tid] - mx) : 0.0, redd);
    const double lse = (double)mx + log(se);
    if (tid < n) {
      l[tid] = (float)((double)l[tid] - lse);
      float* o = side ? lc_out : lr_out;
      if (o) o[(long long)t * n + tid] = l[tid];
    }
    __syncthreads();
  }
  // 2. top rows / columns, ranked directly
  const int kr = min(K, Nr), kc = min(K, Nc);
  for (int side = 0; side < 2; ++side) {
    const int n = side ? Nc : Nr;
    const float* l = side ? lc : lr;
    for (int i = tid; i < n; i += nthr) {
      const float v = l[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const float u = l[j];
        rank += (u > v) || (u == v && j < i);
      }
      if (rank < (side ? kc : kr)) (side ? cols_sel : rows_sel)[rank] = i;
    }
  }
  if (tid == 0) {
    prefix_s = 0;
    mask_s = 0;
    krem_s = K;
    n_gt = 0;
    n_tie = 0;
  }
  __syncthreads();
  // 3. tau: the K-th largest candidate score (radix select, most significant byte first)
  const int nc = kr * kc;
  auto cand_score = [&](int i) { return lr[rows_sel[i / kc]] + lc[cols_sel[i % kc]]; };
  // (The scores of the candidates share their leading bytes, so one shared histogram
  // would serialise on a few bins: each warp counts into its own histogram, equal
  // bins within a warp combined by __match_any_sync, then the warps are summed.)
  const int nw = nthr >> 5;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < nw * 257; b += nthr) (&whist[0][0])[b] = 0;
    __syncthreads();
    const uint32_t prefix = prefix_s, mask = mask_s;
    for (int i0 = 0; i0 < nc; i0 += nthr) {
      const int i = i0 + tid;
      int bin = 256;
      if (i < nc) {
        const uint32_t key = ordered_bits(cand_score(i));
        if ((key & mask) == prefix) bin = (int)((key >> shift) & 255u);
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (lane == __ffs(peers) - 1) whist[warp][bin] += __popc(peers);
    }
    __syncthreads();
    for (int b = tid; b < 256; b += nthr) {
      unsigned sum = 0;
      for (int w = 0; w < nw; ++w) sum += whist[w][b];
      hist[b] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255 - 8l .. 248 - 8l (descending); find the bin where the
      // running count from the top reaches krem
      unsigned c8[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        c8[u] = hist[255 - 8 * lane - u];
        tot += c8[u];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int krem = krem_s;
      unsigned above = incl - tot;  // count in the bins above this lane's
      const bool here = above < (unsigned)krem && incl >= (unsigned)krem;
      int digit = 0;
      if (here) {
        digit = 255 - 8 * lane;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (above + c8[u] >= (unsigned)krem) {
            digit = 255 - 8 * lane - u;
            break;
          }
          above += c8[u];
        }
      }
      const unsigned who = __ballot_sync(0xffffffffu, here);
      const int src = who ? __ffs(who) - 1 : 31;
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      if (lane == 0) {
        krem_s = krem - (int)above;
        prefix_s = prefix | ((uint32_t)digit << shift);
        mask_s = mask | (255u << shift);
      }
    }
    __syncthreads();
  }
  const uint32_t tau_key = prefix_s;
  const float tau = ordered_to_float(tau_key);
  const int need = krem_s;  // tau-valued pairs to take; K - need candidates score above tau
  // 4. candidates above tau, and every grid pair equal to tau
  for (int i = tid; i < nc; i += nthr)
    if (ordered_bits(cand_score(i)) > tau_key) {
      const int slot = atomicAdd(&n_gt, 1);
      if (slot < SEL_MAX_K) gt_ids[slot] = (uint32_t)(rows_sel[i / kc] * Nc + cols_sel[i % kc]);
    }
  const float lc_max = lc[cols_sel[0]], lr_max = lr[rows_sel[0]];
  for (int j = tid; j < Nc; j += nthr) {
    const float cj = lc[j];
    if (lr_max + cj < tau) continue;  // no row can bring this column up to tau
    for (int i = 0; i < Nr; ++i) {
      const float ri = lr[i];
      if (ri + lc_max < tau) continue;
      if (ri + cj == tau) {
        const int slot = atomicAdd(&n_tie, 1);
        if (slot < TIE_CAP) tie_ids[slot] = (uint32_t)(i * Nc + j);
      }
    }
  }
  __syncthreads();
  if (n_gt != K - need) {  // cannot happen (every pair above tau lies in R x C)
    if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  if (n_tie <= TIE_CAP) {
    // lowest `need` tied ids: rank the ids (they are distinct)
    for (int u = tid; u < n_tie; u += nthr) {
      const uint32_t id = tie_ids[u];
      int rank = 0;
      for (int v = 0; v < n_tie; ++v) rank += tie_ids[v] < id;
      if (rank < need) win_ids[K - need + rank] = id;
    }
  } else {
    // massive ties: walk the grid rows in flat-id order, block-wide, until `need` found
    if (tid == 0) found_s = 0;
    __syncthreads();
    for (int i = 0; i < Nr; ++i) {
      if (found_s >= need) break;
      if (lr[i] + lc_max < tau) continue;  // uniform across the block
      bool eq = false;
      int jj = 0;
      const int per = (Nc + nthr - 1) / nthr;  // Nc <= 1024 = nthr, so per == 1
      for (int r = 0; r < per; ++r) {
        jj = tid * per + r;
        if (jj < Nc && lr[i] + lc[jj] == tau) {
          eq = true;
          break;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      int before = 0, total = 0;
      for (int w = 0; w < (int)(nthr >> 5); ++w) {
        if (w < warp) before += warp_cnt[w];
        total += warp_cnt[w];
      }
      const int base = found_s;
      if (eq) {
        const int p = base + before + __popc(bal & ((1u << lane) - 1u));
        if (p < need) win_ids[K - need + p] = (uint32_t)(i * Nc + jj);
      }
      __syncthreads();
      if (tid == 0) found_s = base + total;
      __syncthreads();
    }
  }
  for (int u = tid; u < K - need; u += nthr) win_ids[u] = gt_ids[u];
  __syncthreads();
  // 5. order the K winners by (S desc, id asc), then the gate weights
  auto score_of = [&](uint32_t id) { return lr[id / Nc] + lc[id % Nc]; };
  uint32_t my_id = 0;
  int my_rank = 0;
  if (tid < K) {
    my_id = win_ids[tid];
    const uint64_t mk = make_key(score_of(my_id), my_id);
    for (int v = 0; v < K; ++v) my_rank += make_key(score_of(win_ids[v]), win_ids[v]) > mk;
  }
  __syncthreads();
  if (tid < K) rows_sel[my_rank] = (int)my_id;  // reuse as the ordered output staging area
  __syncthreads();
  const float smax = score_of((uint32_t)rows_sel[0]);
  double z = 0.0;
  if (tid < K) z = (double)expf(score_of((uint32_t)rows_sel[tid]) - smax);
  const double zs = block_sum(z, redd);
  if (tid < K) {
    idx_out[(long long)t * K + tid] = rows_sel[tid];
    g_out[(long long)t * K + tid] = (float)(z / zs);
  }
}

cudaError_t launch_atomic_select(int T, int Nr, int Nc, int K, int ksplit, const float* zr, long long zr_split,
                                 const float* zc, long long zc_split, float* lr_out, float* lc_out, int32_t* idx,
                                 float* g, int* status, cudaStream_t s) {
  launch_k(atomic_select_kernel, T, SEL_THREADS, 0, s, T, Nr, Nc, K, ksplit, zr, zr_split, zc, zc_split, lr_out,
           lc_out, idx, g, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ assembly
// coef[t, s] = g[t, s] * act(x_t . w_in[idx[t, s]]): one warp per task, 16-byte
// loads of the 2 d-byte expert row issued eight at a time, fp32 dot, shuffle-tree
// reduction.
__global__ void atomic_coef_kernel(int T, int d, int K, int act, const uint4* __restrict__ x,
                                   const uint4* __restrict__ w_in, const int32_t* __restrict__ idx,
                                   const float* __restrict__ g, float* __restrict__ coef, long long n_experts,
                                   int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (task >= (long long)T * K) return;
  const long long t = task / K;
  const long long e = idx[task];
  if (e < 0 || e >= n_experts) {
    if (lane == 0) {
      set_status(status, MOE_ERR_DEVICE_INDEX);
      coef[task] = 0.f;
    }
    return;
  }
  const int chunks = d / 8;
  const uint4* xr = x + t * chunks;
  const uint4* wr = w_in + e * chunks;
  float s = 0.f;
  for (int c0 = lane; c0 < chunks; c0 += 32 * 8) {
    uint4 a[8], b[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 32 * u;
      if (c < chunks) {
        a[u] = xr[c];
        b[u] = wr[c];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (c0 + 32 * u >= chunks) break;
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 fa = __bfloat1622float2(pa[h]), fb = __bfloat1622float2(pb[h]);
        s = fmaf(fa.x, fb.x, s);
        s = fmaf(fa.y, fb.y, s);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
  if (lane == 0) {
    const float sg = 1.f / (1.f + expf(-s));
    coef[task] = g[task] * (act == MOE_ATOMIC_SILU ? s * sg : sg);
  }
}

// out[t, c..c+7] = sum_s coef[t, s] w_out[idx[t, s], c..c+7]. A block handles one
// token and 64 column chunks of 8; its four thread groups take every fourth slot
// (loads issued eight at a time) and their partial sums are added in group order,
// so the result is the same on every run.
constexpr int ASM_GROUPS = 4, ASM_CHUNKS = 64;
__global__ void atomic_assemble_kernel(int T, int d, int K, const uint4* __restrict__ w_out,
                                       const int32_t* __restrict__ idx, const float* __restrict__ coef,
                                       uint4* __restrict__ out, long long n_experts) {
  __shared__ float part[ASM_GROUPS][ASM_CHUNKS][8];
  pdl_launch_dependents();
  pdl_wait();
  const int chunks = d / 8;
  const int cblocks = (chunks + ASM_CHUNKS - 1) / ASM_CHUNKS;
  const long long t = blockIdx.x / cblocks;
  const int cl = threadIdx.x % ASM_CHUNKS, grp = threadIdx.x / ASM_CHUNKS;
  const int c = (blockIdx.x % cblocks) * ASM_CHUNKS + cl;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (c < chunks) {
    for (int s0 = grp; s0 < K; s0 += ASM_GROUPS * 8) {
      uint4 v[8];
      float cf[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int sl = s0 + ASM_GROUPS * u;
        cf[u] = 0.f;
        if (sl < K) {
          const long long e = idx[t * K + sl];
          if (e >= 0 && e < n_experts) {
            cf[u] = coef[t * K + sl];
            v[u] = w_out[e * chunks + c];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (cf[u] == 0.f) continue;
        const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __bfloat1622float2(pv[h]);
          acc[2 * h] = fmaf(cf[u], f.x, acc[2 * h]);
          acc[2 * h + 1] = fmaf(cf[u], f.y, acc[2 * h + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) part[grp][cl][h] = acc[h];
  __syncthreads();
  if (grp == 0 && c < chunks) {
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = ((part[0][cl][h] + part[1][cl][h]) + part[2][cl][h]) + part[3][cl][h];
    uint4 o;
    __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int h = 0; h < 4; ++h) po[h] = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
    out[t * chunks + c] = o;
  }
}

cudaError_t launch_atomic_experts(int T, int d, int K, int act, const void* x, const void* w_in, const void* w_out,
                                  const int32_t* idx, const float* g, float* coef, void* out, long long n_experts,
                                  int* status, cudaStream_t s, bool stage_marks) {
  const long long tasks = (long long)T * K;
  launch_k(atomic_coef_kernel, (unsigned)((tasks + 7) / 8), 256, 0, s, T, d, K, act, (const uint4*)x, (const uint4*)w_in,
                                                                 idx, g, coef, n_experts, status);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (stage_marks && (e = mark_stage_event(3, s)) != cudaSuccess) return e;
  const int cblocks = (d / 8 + ASM_CHUNKS - 1) / ASM_CHUNKS;
  launch_k(atomic_assemble_kernel, (unsigned)(T * cblocks), ASM_GROUPS * ASM_CHUNKS, 0, s, T, d, K,
           (const uint4*)w_out, idx, coef, (uint4*)out, n_experts);
  
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe
