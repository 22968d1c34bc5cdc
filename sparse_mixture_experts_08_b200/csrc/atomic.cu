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
//     with a lower flat id.) Step 3 scans grid rows in id order, skipping any row
//     with fl(lr_i + max lc) < tau, until enough ties are found.
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

// In-place bitonic sort of n (power of two) keys into DESCENDING order.
__device__ void bitonic_desc(uint64_t* key, int n) {
  for (int size = 2; size <= n; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
        const int lo = (i / stride) * (2 * stride) + (i % stride);
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = key[lo], b = key[hi];
        if ((a < b) == desc) {
          key[lo] = b;
          key[hi] = a;
        }
      }
      __syncthreads();
    }
}

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

// One block per token. zr/zc: split-K partial logits [ksplit][T][Nr|Nc].
__global__ void __launch_bounds__(SEL_THREADS, 1)
    atomic_select_kernel(int T, int Nr, int Nc, int K, int ksplit, const float* __restrict__ zr, long long zr_split,
                         const float* __restrict__ zc, long long zc_split, float* __restrict__ lr_out,
                         float* __restrict__ lc_out, int32_t* __restrict__ idx_out, float* __restrict__ g_out,
                         int* status) {
  __shared__ float lr[SEL_MAX_SIDE], lc[SEL_MAX_SIDE];
  __shared__ uint64_t key[SEL_CAND];
  __shared__ float redf[32];
  __shared__ double redd[32];
  __shared__ int rows_sel[SEL_MAX_K], cols_sel[SEL_MAX_K];
  __shared__ uint32_t tied[SEL_MAX_K];
  __shared__ int warp_cnt[32];
  __shared__ int found_s;
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();

  // 1. sum the split-K partials, log-softmax of rows and of columns (fp32 values,
  //    max and log-sum-exp formed in fp64).
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
  // 2. candidate rows and columns: top-kr / top-kc by (value desc, index asc).
  const int kr = min(K, Nr), kc = min(K, Nc);
  for (int side = 0; side < 2; ++side) {
    const int n = side ? Nc : Nr;
    const float* l = side ? lc : lr;
    int np = 1;
    while (np < n) np <<= 1;
    for (int i = tid; i < np; i += blockDim.x) key[i] = i < n ? make_key(l[i], (uint32_t)i) : 0ull;
    __syncthreads();
    bitonic_desc(key, np);
    if (tid < (side ? kc : kr)) (side ? cols_sel : rows_sel)[tid] = (int)key_id(key[tid]);
    __syncthreads();
  }
  // 3. candidate block R x C, sorted by (S desc, id asc).
  const int nc = kr * kc;
  int np = 1;
  while (np < nc) np <<= 1;
  for (int i = tid; i < np; i += blockDim.x) {
    if (i < nc) {
      const int ri = rows_sel[i / kc], cj = cols_sel[i % kc];
      key[i] = make_key(lr[ri] + lc[cj], (uint32_t)(ri * Nc + cj));
    } else {
      key[i] = 0ull;
    }
  }
  __syncthreads();
  bitonic_desc(key, np);
  auto score_of = [&](uint32_t id) { return lr[id / Nc] + lc[id % Nc]; };
  const float tau = score_of(key_id(key[K - 1]));
  int n_above = 0;
  for (int q = 0; q < K; ++q) n_above += score_of(key_id(key[q])) > tau ? 1 : 0;
  const int need = K - n_above;
  // 4. the first `need` pairs of the whole grid (flat-id order) scoring exactly tau.
  if (tid == 0) found_s = 0;
  __syncthreads();
  const float lc_max = lc[cols_sel[0]];
  for (int i = 0; i < Nr; ++i) {
    if (found_s >= need) break;
    if (lr[i] + lc_max < tau) continue;  // uniform across the block
    const bool eq = tid < Nc && (lr[i] + lc[tid] == tau);
    const unsigned bal = __ballot_sync(FULL, eq);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      if (w < warp) before += warp_cnt[w];
      total += warp_cnt[w];
    }
    const int base = found_s;
    if (eq) {
      const int p = base + before + __popc(bal & ((1u << lane) - 1u));
      if (p < need) tied[p] = (uint32_t)(i * Nc + tid);
    }
    __syncthreads();
    if (tid == 0) found_s = base + total;
    __syncthreads();
  }
  if (found_s < need) {  // cannot happen: the K-th candidate itself scores tau
    if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  // 5. selection = candidates above tau (already ordered) then the tied ids in id
  //    order; gate weights = softmax of the selected scores.
  if (tid < K) {
    const uint32_t id = tid < n_above ? key_id(key[tid]) : tied[tid - n_above];
    rows_sel[tid] = (int)id;  // reuse as the output staging area
  }
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
  launch_k(atomic_select_kernel, T, SEL_THREADS, 0, s, T, Nr, Nc, K, ksplit, zr, zr_split, zc, zc_split, lr_out, lc_out, idx,
                                                 g, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ assembly
// coef[t, s] = g[t, s] * act(x_t . w_in[idx[t, s]]): one warp per task, 16-byte
// loads of the 2 d-byte expert row, fp32 dot, shuffle-tree reduction.
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
  for (int c = lane; c < chunks; c += 32) {
    const uint4 a = xr[c], b = wr[c];
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 fa = __bfloat1622float2(pa[h]), fb = __bfloat1622float2(pb[h]);
      s = fmaf(fa.x, fb.x, s);
      s = fmaf(fa.y, fb.y, s);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
  if (lane == 0) {
    const float sg = 1.f / (1.f + expf(-s));
    coef[task] = g[task] * (act == MOE_ATOMIC_SILU ? s * sg : sg);
  }
}

// out[t, c..c+7] = sum_s coef[t, s] w_out[idx[t, s], c..c+7] (fp32, slot order).
__global__ void atomic_assemble_kernel(int T, int d, int K, const uint4* __restrict__ w_out,
                                       const int32_t* __restrict__ idx, const float* __restrict__ coef,
                                       uint4* __restrict__ out, long long n_experts) {
  pdl_launch_dependents();
  pdl_wait();
  const int chunks = d / 8;
  const long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (item >= (long long)T * chunks) return;
  const long long t = item / chunks;
  const int c = (int)(item - t * chunks);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < K; ++s) {
    const long long e = idx[t * K + s];
    if (e < 0 || e >= n_experts) continue;
    const float cf = coef[t * K + s];
    const uint4 v = w_out[e * chunks + c];
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float2 f = __bfloat1622float2(pv[h]);
      acc[2 * h] = fmaf(cf, f.x, acc[2 * h]);
      acc[2 * h + 1] = fmaf(cf, f.y, acc[2 * h + 1]);
    }
  }
  uint4 o;
  __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
  for (int h = 0; h < 4; ++h) po[h] = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
  out[item] = o;
}

cudaError_t launch_atomic_experts(int T, int d, int K, int act, const void* x, const void* w_in, const void* w_out,
                                  const int32_t* idx, const float* g, float* coef, void* out, long long n_experts,
                                  int* status, cudaStream_t s) {
  const long long tasks = (long long)T * K;
  launch_k(atomic_coef_kernel, (unsigned)((tasks + 7) / 8), 256, 0, s, T, d, K, act, (const uint4*)x, (const uint4*)w_in,
                                                                 idx, g, coef, n_experts, status);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long items = (long long)T * (d / 8);
  launch_k(atomic_assemble_kernel, (unsigned)((items + 63) / 64), 64, 0, s, T, d, K, (const uint4*)w_out, idx, coef,
                                                                      (uint4*)out, n_experts);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe
