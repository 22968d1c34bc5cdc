// Router top-k/softmax, per-expert histogram + LIS + stable ranks, row permutation
// and the weighted combine (CUDA cores; these steps are integer work or
// memory-bound streaming, so they stay off the tensor cores).
#include <float.h>

#include <algorithm>

#include "common.cuh"

namespace moe {

namespace {
constexpr unsigned FULL = 0xffffffffu;
constexpr int TOPK_WARPS = 8;
constexpr int RI_THREADS = 1024;
}  // namespace

// ------------------------------------------------------------------ SIMT logits
// logits[t, e] = sum_i x[t,i] w_r[e,i] (fp32 FMA, lane-strided, warp tree) + bias[e].
// Used for fp32 layers; bf16 layers use the tensor-core GEMM.
template <typename TIn>
__device__ __forceinline__ float ld_f32(const TIn* p, long long i);
template <>
__device__ __forceinline__ float ld_f32<float>(const float* p, long long i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}

template <typename TIn>
__global__ void simt_logits_kernel(int T, int d, int m, const TIn* __restrict__ x, const TIn* __restrict__ w,
                                   const float* __restrict__ bias, float* __restrict__ logits) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < (long long)T * m;
       item += warps) {
    const long long t = item / m;
    const int e = (int)(item % m);
    float s = 0.f;
    for (int i = lane; i < d; i += 32) s = fmaf(ld_f32(x, t * d + i), ld_f32(w, (long long)e * d + i), s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
    if (lane == 0) logits[item] = s + (bias ? bias[e] : 0.f);
  }
}

cudaError_t launch_simt_logits(int dtype, int T, int d, int m, const void* x, const void* w_r, const float* bias,
                               float* logits, cudaStream_t s) {
  const long long items = (long long)T * m;
  const int blocks = (int)std::min<long long>((items + 7) / 8, 4LL * num_sms() * 8);
  if (dtype == MOE_F32)
    launch_k(simt_logits_kernel<float>, blocks, 256, 0, s, T, d, m, (const float*)x, (const float*)w_r, bias, logits);
  else
    launch_k(simt_logits_kernel<__nv_bfloat16>, blocks, 256, 0, s, T, d, m, (const __nv_bfloat16*)x,
                                                             (const __nv_bfloat16*)w_r, bias, logits);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ few-expert logits
// logits[t, e] = x_t . W_r[e] + bias[e] for routers with few experts (m <= 32,
// bf16): one block per token, 256 threads; each thread takes d / 8 / 256 16-byte
// chunks of the token and the same chunks of every expert row (all loads
// independent), forms m partial dots in fp32 and the block sums them (warp
// shuffles, then the eight warp results in order).
constexpr int FE_MAX_M = 32;
constexpr int FE_THREADS = 256;

__global__ void __launch_bounds__(FE_THREADS) few_expert_logits_kernel(int d, int m, const uint4* __restrict__ x,
                                                                       const uint4* __restrict__ w,
                                                                       const float* __restrict__ bias,
                                                                       float* __restrict__ logits) {
  __shared__ float part[FE_THREADS / 32][FE_MAX_M];
  pdl_launch_dependents();
  pdl_wait();
  const long long t = blockIdx.x;
  const int chunks = d / 8;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[FE_MAX_M];
#pragma unroll
  for (int e = 0; e < FE_MAX_M; ++e) acc[e] = 0.f;
  for (int c = threadIdx.x; c < chunks; c += FE_THREADS) {
    const uint4 xv = x[t * chunks + c];
    const __nv_bfloat162* px = reinterpret_cast<const __nv_bfloat162*>(&xv);
    float2 xf[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) xf[h] = __bfloat1622float2(px[h]);
#pragma unroll
    for (int e = 0; e < FE_MAX_M; ++e) {
      if (e < m) {
        const uint4 wv = w[(long long)e * chunks + c];
        const __nv_bfloat162* pw = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 wf = __bfloat1622float2(pw[h]);
          acc[e] = fmaf(xf[h].x, wf.x, acc[e]);
          acc[e] = fmaf(xf[h].y, wf.y, acc[e]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < FE_MAX_M; ++e) {
    if (e < m) {
      float v = acc[e];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
      if (lane == 0) part[warp][e] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < m) {
    float v = 0.f;
    for (int w8 = 0; w8 < FE_THREADS / 32; ++w8) v += part[w8][threadIdx.x];
    logits[t * m + threadIdx.x] = v + (bias ? bias[threadIdx.x] : 0.f);
  }
}

bool few_expert_logits_ok(int dtype, int T, int m) { return dtype == MOE_BF16 && T <= 64 && m <= FE_MAX_M; }

cudaError_t launch_few_expert_logits(int T, int d, int m, const void* x, const void* w, const float* bias,
                                     float* logits, cudaStream_t s) {
  launch_k(few_expert_logits_kernel, T, FE_THREADS, 0, s, d, m, (const uint4*)x, (const uint4*)w, bias, logits);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ router for few experts, any batch
// Logits, top-k and gate weights in one launch for bf16 layers with m <= 16 experts
// (R&Q's token-choice routing over a Mixtral-like expert count). One block of
// SR_THREADS per SR_VALUES / M tokens: thread i owns the 16-byte chunks i, i +
// SR_THREADS, ... of the model dimension, loads those chunks of every expert's
// router row once and applies them to each of the block's tokens (fp32 FMAs, chunks
// in ascending order). The SR_VALUES partial sums per thread are reduced by a
// shuffle reduce-scatter in each warp (lane L ends with value L) and
// then over the warps in warp order; the logit gets its bias. Then one thread per
// token takes the top-k by (logit desc, expert asc) and the gate weights as
// topk_softmax_kernel does: exp in fp32 of l - max, sums in fp64, renormalised over
// the k chosen when asked. Every sum has a fixed order: the result does not depend
// on timing.
constexpr int SR_THREADS = 256, SR_VALUES = 32;

// Top-k and gate weights of one token from its m <= M logits (one thread): k passes
// over the experts in ascending order (a tie keeps the lower expert), then the
// softmax over all m in fp64 (exp in fp32 of l - max, summed in expert order),
// renormalised over the k chosen when asked.
template <int M>
__device__ __forceinline__ void small_topk_token(const float* L, int m, int k, int renorm, int32_t* idx_row,
                                                 float* w_row) {
  int sel_e[M];
  float sel_v[M];
#pragma unroll
  for (int s2 = 0; s2 < M; ++s2) {
    if (s2 >= k) break;
    float bv = 0.f;
    int be = -1;
#pragma unroll
    for (int e = 0; e < M; ++e) {
      if (e >= m) break;
      bool taken = false;
#pragma unroll
      for (int j = 0; j < M; ++j)
        if (j < s2) taken |= sel_e[j] == e;
      if (!taken && (be < 0 || L[e] > bv)) {  // ascending e: a tie keeps the lower expert
        bv = L[e];
        be = e;
      }
    }
    sel_e[s2] = be;
    sel_v[s2] = bv;
  }
  const float mx = sel_v[0];
  double z = 0.0;
#pragma unroll
  for (int e = 0; e < M; ++e)
    if (e < m) z += (double)expf(L[e] - mx);
  double sel = 0.0;
#pragma unroll
  for (int s2 = 0; s2 < M; ++s2)
    if (s2 < k) sel += (double)expf(sel_v[s2] - mx) / z;
#pragma unroll
  for (int s2 = 0; s2 < M; ++s2) {
    if (s2 >= k) break;
    double pr = (double)expf(sel_v[s2] - mx) / z;
    if (renorm) pr /= sel;
    idx_row[s2] = sel_e[s2];
    w_row[s2] = (float)pr;
  }
}

template <int M>
__global__ void __launch_bounds__(SR_THREADS)
    small_route_kernel(int T, int d, int m, int k, int renorm, const uint4* __restrict__ x,
                       const uint4* __restrict__ w, const float* __restrict__ bias, float* __restrict__ logits,
                       int32_t* __restrict__ idx, float* __restrict__ wout) {
  constexpr int TB = SR_VALUES / M;  // tokens per block
  __shared__ float red[SR_THREADS / 32][SR_VALUES];
  __shared__ float lg[TB][M];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunks = d / 8;
  const long long t0 = (long long)blockIdx.x * TB;
  pdl_launch_dependents();
  pdl_wait();
  float acc[TB][M];
#pragma unroll
  for (int t = 0; t < TB; ++t)
#pragma unroll
    for (int e = 0; e < M; ++e) acc[t][e] = 0.f;
  for (int c = tid; c < chunks; c += SR_THREADS) {
    // every load of a chunk is independent: all of them (M router rows, TB tokens)
    // are issued before the chunk's FMAs
    uint4 wv[M], xv[TB];
#pragma unroll
    for (int e = 0; e < M; ++e) wv[e] = e < m ? w[(long long)e * chunks + c] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int t = 0; t < TB; ++t) xv[t] = t0 + t < T ? x[(t0 + t) * chunks + c] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv[t]);
#pragma unroll
      for (int e = 0; e < M; ++e) {
        const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wv[e]);
        float a = acc[t][e];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 xf = __bfloat1622float2(xh[u]), wf = __bfloat1622float2(wh[u]);
          a = fmaf(xf.x, wf.x, a);
          a = fmaf(xf.y, wf.y, a);
        }
        acc[t][e] = a;
      }
    }
  }
  // reduce-scatter over the warp: value index v = t M + e; lane L keeps value L
  float* v = &acc[0][0];
#pragma unroll
  for (int half = SR_VALUES / 2, bit = 16; half >= 1; half >>= 1, bit >>= 1) {
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[half + i] : v[i];
      const float send = upper ? v[i] : v[half + i];
      v[i] = keep + __shfl_xor_sync(FULL, send, bit);
    }
  }
  red[warp][lane] = v[0];
  __syncthreads();
  if (tid < SR_VALUES) {
    const int t = tid / M, e = tid % M;
    float sum = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < SR_THREADS / 32; ++w8) sum += red[w8][tid];
    if (e < m) {
      sum += bias ? bias[e] : 0.f;
      lg[t][e] = sum;
      if (logits && t0 + t < T) logits[(t0 + t) * m + e] = sum;
    }
  }
  __syncthreads();
  if (tid < TB && t0 + tid < T) small_topk_token<M>(lg[tid], m, k, renorm, idx + (t0 + tid) * k, wout + (t0 + tid) * k);
}

// Tensor-core form of the small-expert router (d a multiple of 32): a block of
// SRT_WARPS warps takes 16 tokens, warp w the 32-element groups w, w + SRT_WARPS, ...
// of the model dimension, with mma.sync m16n8k16 (bf16 operands, fp32 accumulate) on
// A = the 16 token rows and B = the router rows (M / 8 tiles of 8 experts). Within a
// group each lane loads 16 bytes of each operand (row g = lane / 4, elements
// 8 (lane % 4) .. + 7), and the two k-steps take those elements as the fragment
// positions 2t, 2t + 1, 2t + 8, 2t + 9 (t = lane % 4): the same position -> element
// map for A and B, so every product pairs matching elements. The warps' partial
// logits are added in warp order, then the bias; one thread per token takes the
// top-k and gate weights as small_route_kernel does. The sums have a fixed order.
constexpr int SRT_WARPS = 16, SRT_UNROLL = 4;
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int M>
__global__ void __launch_bounds__(SRT_WARPS * 32)
    small_route_mma_kernel(int T, int d, int m, int k, int renorm, const uint4* __restrict__ x,
                           const uint4* __restrict__ w, const float* __restrict__ bias, float* __restrict__ logits,
                           int32_t* __restrict__ idx, float* __restrict__ wout) {
  constexpr int NT = M / 8;  // expert tiles of 8
  __shared__ float part[SRT_WARPS][16][M + 1];
  __shared__ float lg[16][M];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const long long t0 = (long long)blockIdx.x * 16;
  const int groups = d / 32, chunks = d / 8;  // 32-element groups; 16-byte chunks per row
  const bool ra = t0 + g < T, rb = t0 + g + 8 < T;
  const uint4* xa = x + (t0 + g) * chunks + t4;
  const uint4* xb = x + (t0 + g + 8) * chunks + t4;
  pdl_launch_dependents();
  pdl_wait();
  float c[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int j = 0; j < 4; ++j) c[n][j] = 0.f;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int g0 = warp; g0 < groups; g0 += SRT_WARPS * SRT_UNROLL) {
    uint4 va[SRT_UNROLL], vb[SRT_UNROLL], vw[SRT_UNROLL][NT];
#pragma unroll
    for (int u = 0; u < SRT_UNROLL; ++u) {  // every load of the step before the MMAs
      const int gr = g0 + u * SRT_WARPS;
      const bool ok = gr < groups;
      va[u] = ok && ra ? xa[gr * 4] : zero;
      vb[u] = ok && rb ? xb[gr * 4] : zero;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int e = n * 8 + g;
        vw[u][n] = ok && e < m ? w[(long long)e * chunks + gr * 4 + t4] : zero;
      }
    }
#pragma unroll
    for (int u = 0; u < SRT_UNROLL; ++u) {
      const uint32_t a1[4] = {va[u].x, vb[u].x, va[u].y, vb[u].y};
      const uint32_t a2[4] = {va[u].z, vb[u].z, va[u].w, vb[u].w};
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        mma_bf16_16816(c[n], a1, vw[u][n].x, vw[u][n].y);
        mma_bf16_16816(c[n], a2, vw[u][n].z, vw[u][n].w);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    part[warp][g][n * 8 + 2 * t4] = c[n][0];
    part[warp][g][n * 8 + 2 * t4 + 1] = c[n][1];
    part[warp][g + 8][n * 8 + 2 * t4] = c[n][2];
    part[warp][g + 8][n * 8 + 2 * t4 + 1] = c[n][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * M; i += blockDim.x) {
    const int tt = i / M, e = i % M;
    float sum = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < SRT_WARPS; ++w8) sum += part[w8][tt][e];
    if (e < m) {
      sum += bias ? bias[e] : 0.f;
      lg[tt][e] = sum;
      if (logits && t0 + tt < T) logits[(t0 + tt) * m + e] = sum;
    }
  }
  __syncthreads();
  if (threadIdx.x < 16 && t0 + threadIdx.x < T)
    small_topk_token<M>(lg[threadIdx.x], m, k, renorm, idx + (t0 + threadIdx.x) * k, wout + (t0 + threadIdx.x) * k);
}

bool small_route_ok(int dtype, int m) { return dtype == MOE_BF16 && m <= 16; }

cudaError_t launch_small_route(int T, int d, int m, int k, int renorm, const void* x, const void* w, const float* bias,
                               float* logits, int32_t* idx, float* wout, cudaStream_t s) {
  // tensor-core form (16 tokens per block) from 128 tokens on; below that the
  // CUDA-core form's 4-token blocks give a short batch more SMs (decode: 10.5 µs
  // against 14.4 for the single 16-token block)
  if (d % 32 == 0 && T >= 128) {
    const int blocks = (T + 15) / 16;
    if (m <= 8)
      launch_k(small_route_mma_kernel<8>, blocks, SRT_WARPS * 32, 0, s, T, d, m, k, renorm, (const uint4*)x,
               (const uint4*)w, bias, logits, idx, wout);
    else
      launch_k(small_route_mma_kernel<16>, blocks, SRT_WARPS * 32, 0, s, T, d, m, k, renorm, (const uint4*)x,
               (const uint4*)w, bias, logits, idx, wout);
  } else if (m <= 8) {
    const int tb = SR_VALUES / 8;
    launch_k(small_route_kernel<8>, (T + tb - 1) / tb, SR_THREADS, 0, s, T, d, m, k, renorm, (const uint4*)x,
             (const uint4*)w, bias, logits, idx, wout);
  } else {
    const int tb = SR_VALUES / 16;
    launch_k(small_route_kernel<16>, (T + tb - 1) / tb, SR_THREADS, 0, s, T, d, m, k, renorm, (const uint4*)x,
             (const uint4*)w, bias, logits, idx, wout);
  }
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ top-k + softmax
// One warp per token; lane l holds the logits of experts l, l + 32, ... (NI of
// them, in registers). k rounds of a warp arg-max over the not-yet-chosen experts,
// ordered by (logit desc, expert index asc): each lane's best candidate, then the
// warp's largest logit by one redux on an order-preserving 32-bit code of it, then
// the lowest expert holding that logit by a second redux; the winner's lane marks
// it taken. (A NaN logit codes below -inf, so it is picked only when nothing else
// is left.) Gate weights: softmax over all m logits (exp in fp32 of l - max, the
// per-lane fp64 sums in expert order, then a fixed xor tree), renormalised over the
// k chosen when requested, their sum taken in pick order.
__device__ __forceinline__ uint32_t order_code(float v) {
  const uint32_t b = __float_as_uint(v == 0.f ? 0.f : v);  // -0 and +0 compare equal: one code
  if (v != v) return 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <int NI>
__global__ void topk_softmax_kernel(int T, int m, int k, int renorm, const float* __restrict__ logits,
                                    int32_t* __restrict__ idx, float* __restrict__ w) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int t = blockIdx.x * TOPK_WARPS + wib;
  if (t >= T) return;  // uniform across the warp
  const float* L = logits + (long long)t * m;
  float v[NI];
#pragma unroll
  for (int i = 0; i < NI; ++i) v[i] = lane + 32 * i < m ? L[lane + 32 * i] : 0.f;
  uint32_t taken = 0u;  // bit i: expert lane + 32 i chosen already
  int my_e = -1;        // lane s < k: the s-th pick
  float my_v = 0.f;
  float mx = 0.f;
  for (int s2 = 0; s2 < k; ++s2) {
    uint32_t bc = 0u;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int e = lane + 32 * i;
      const uint32_t cd = order_code(v[i]);
      if (e < m && !((taken >> i) & 1u) && (be == 0x7fffffff || cd > bc)) {  // ascending e: ties keep the lower
        bc = cd;
        be = e;
      }
    }
    const uint32_t wc = __reduce_max_sync(FULL, be == 0x7fffffff ? 0u : bc);
    const int we = (int)__reduce_min_sync(FULL, (be != 0x7fffffff && bc == wc) ? (uint32_t)be : 0x7fffffffu);
    // the winner's logit, from the lane that holds it
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < NI; ++i)
      if (lane + 32 * i == we) mine = v[i];
    const float pick = __shfl_sync(FULL, mine, we & 31);
    if ((we & 31) == lane) taken |= 1u << (we >> 5);
    if (lane == s2) {
      my_e = we;
      my_v = pick;
    }
    if (s2 == 0) mx = pick;
  }
  double z = 0.0;
#pragma unroll
  for (int i = 0; i < NI; ++i)
    if (lane + 32 * i < m) z += (double)expf(v[i] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
  double p = lane < k ? (double)expf(my_v - mx) / z : 0.0;
  double sel = 0.0;
  for (int s2 = 0; s2 < k; ++s2) sel += __shfl_sync(FULL, p, s2);
  if (lane < k) {
    if (renorm) p /= sel;
    idx[(long long)t * k + lane] = my_e;
    w[(long long)t * k + lane] = (float)p;
  }
}

cudaError_t launch_topk_softmax(int T, int m, int k, int renorm, const float* logits, int32_t* idx, float* w,
                                cudaStream_t s) {
  const int blocks = (T + TOPK_WARPS - 1) / TOPK_WARPS, threads = TOPK_WARPS * 32;
  if (m > 1024 || k > 32 || k > m) return cudaErrorInvalidValue;
  if (m <= 64)
    launch_k(topk_softmax_kernel<2>, blocks, threads, 0, s, T, m, k, renorm, logits, idx, w);
  else if (m <= 256)
    launch_k(topk_softmax_kernel<8>, blocks, threads, 0, s, T, m, k, renorm, logits, idx, w);
  else
    launch_k(topk_softmax_kernel<32>, blocks, threads, 0, s, T, m, k, renorm, logits, idx, w);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------ histogram, offsets, LIS, range starts
// The T k tasks (q = t k + s, in increasing order) are cut into R contiguous
// ranges of L tasks; range r holds tasks [r L, min(T k, (r + 1) L)). One block of
// 1024 threads (the routing tables are tiny):
//  pass 1: c[r][e] = tasks of expert e in range r (thread i takes tasks i, i + 1024,
//          ..., eight of its ids loaded together, then shared-memory atomics).
//  scan:   per expert (one warp each, a shuffle scan over its R entries),
//          c[r][e] <- tasks of e in ranges before r; the total is n_e.
//  mode & 1: offsets = exclusive scan of n_e, max / lowest argmax of n_e and
//           LIS = m max / (T k) (R&Q Definition 1); otherwise offsets are given.
//  start[r][e] = offsets[e] + c[r][e]: where range r's first task of expert e
//  goes in the stable counting sort; rank_kernel finishes it with one warp per
//  range.
// Any id outside [0, m) sets MOE_ERR_DEVICE_INDEX and nothing else is written.
__global__ void __launch_bounds__(RI_THREADS, 1)
    route_index_kernel(int mode, int T, int k, int m, int R, int L, const int32_t* __restrict__ idx,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets, moe_lis_t* __restrict__ lis,
                       int32_t* __restrict__ start, int* status) {
  extern __shared__ int sm[];
  const int MS = m + 1;     // padded row stride: the per-expert scan reads a column
  int* c = sm;              // [R][MS]
  int* off = c + R * MS;    // [m + 1]
  __shared__ int bad;
  __shared__ int wsum[32], wmax[32], warg[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int Tk = T * k;
  if (tid == 0) bad = 0;
  for (int i = tid; i < R * MS; i += blockDim.x) c[i] = 0;
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  const int nth = blockDim.x;
  // a thread's tasks are q = tid + n nth; their range q / L is walked by adding
  // (nth / L, nth % L) with one carry instead of a division per task
  const int dq = nth / L, dl = nth - dq * L;
  int rq = tid / L, rl = tid - rq * L;
  for (int q0 = tid; q0 < Tk; q0 += 8 * nth) {
    int ev[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = q0 + u * nth;
      ev[u] = q < Tk ? idx[q] : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = q0 + u * nth;
      if (q >= Tk) break;
      const int e = ev[u];
      if (e < 0 || e >= m)
        bad = 1;
      else
        atomicAdd(&c[rq * MS + e], 1);
      rq += dq;
      rl += dl;
      if (rl >= L) {
        rl -= L;
        ++rq;
      }
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  for (int e = warp; e < m; e += nw) {
    const int per = (R + 31) / 32;
    const int r0 = min(R, lane * per), r1 = min(R, r0 + per);
    int local = 0;
    for (int r = r0; r < r1; ++r) local += c[r * MS + e];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int r = r0; r < r1; ++r) {
      const int t = c[r * MS + e];
      c[r * MS + e] = run;
      run += t;
    }
    if (lane == 31) off[e] = incl;  // n_e for now
  }
  __syncthreads();
  if (mode & 1) {
    const int cn = tid < m ? off[tid] : 0;
    int incl = cn;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    int mv = tid < m ? cn : -1, ma = tid;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const int ov = __shfl_xor_sync(FULL, mv, o), oa = __shfl_xor_sync(FULL, ma, o);
      if (ov > mv || (ov == mv && oa < ma)) {
        mv = ov;
        ma = oa;
      }
    }
    if (lane == 31) wsum[warp] = incl;
    if (lane == 0) {
      wmax[warp] = mv;
      warg[warp] = ma;
    }
    __syncthreads();
    if (warp == 0) {
      const int ws = lane < nw ? wsum[lane] : 0;
      int wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(FULL, wi, o);
        if (lane >= o) wi += v;
      }
      wsum[lane] = wi - ws;
      int bv = lane < nw ? wmax[lane] : -1, ba = lane < nw ? warg[lane] : 0x7fffffff;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const int ov = __shfl_xor_sync(FULL, bv, o), oa = __shfl_xor_sync(FULL, ba, o);
        if (ov > bv || (ov == bv && oa < ba)) {
          bv = ov;
          ba = oa;
        }
      }
      if (lane == 0) {
        wmax[0] = bv;
        warg[0] = ba;
      }
    }
    __syncthreads();
    if (tid < m) {
      const int ex = incl - cn + wsum[warp];
      off[tid] = ex;
      counts[tid] = cn;
      offsets[tid] = ex;
      if (tid == m - 1) {
        off[m] = ex + cn;
        offsets[m] = ex + cn;
      }
    }
    if (tid == 0 && lis) {
      lis->max_count = wmax[0];
      lis->argmax_expert = warg[0];
      lis->lis = (double)((long long)m * wmax[0]) / (double)((long long)T * k);
    }
  } else {
    __syncthreads();
    for (int e = tid; e <= m; e += blockDim.x) off[e] = offsets[e];
  }
  __syncthreads();
  for (int r = warp; r < R; r += nw)  // a warp per range row, lanes along the experts
    for (int e = lane; e < m; e += 32) start[(long long)r * m + e] = off[e] + c[r * MS + e];
}

size_t route_index_smem(int R, int m) { return sizeof(int) * ((size_t)R * (m + 1) + m + 1); }

// Ranges for the stable sort: short enough that one warp ranks each range in a
// few shuffle passes, few enough that the [R][m + 1] count table fits 32 KB.
void route_ranges(int Tk, int m, int* R, int* L) {
  int r = std::min(8192 / (m + 1), (Tk + 31) / 32);
  r = std::max(1, r);
  *L = (Tk + r - 1) / r;
  *R = (Tk + *L - 1) / *L;
}

// ------------------------------------------------ LIS of a given histogram
// R&Q Definition 1 over counts that another step produced (e.g. the histogram of
// every rank's batch, summed across ranks): max_j n_j, the lowest j attaining it,
// and LIS = m max / tasks as one fp64 division. One block; counts are read once.
__global__ void lis_from_counts_kernel(int m, long long tasks, const int32_t* __restrict__ counts,
                                       moe_lis_t* __restrict__ lis) {
  __shared__ int wmax[32], warg[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  int mv = -1, ma = 0x7fffffff;
  for (int e = tid; e < m; e += blockDim.x) {  // ascending e per thread: a strict > keeps the lowest
    const int c = counts[e];
    if (c > mv) {
      mv = c;
      ma = e;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const int ov = __shfl_xor_sync(FULL, mv, o), oa = __shfl_xor_sync(FULL, ma, o);
    if (ov > mv || (ov == mv && oa < ma)) {
      mv = ov;
      ma = oa;
    }
  }
  if (lane == 0) {
    wmax[warp] = mv;
    warg[warp] = ma;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int bv = lane < nw ? wmax[lane] : -1, ba = lane < nw ? warg[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const int ov = __shfl_xor_sync(FULL, bv, o), oa = __shfl_xor_sync(FULL, ba, o);
      if (ov > bv || (ov == bv && oa < ba)) {
        bv = ov;
        ba = oa;
      }
    }
    if (lane == 0) {
      lis->max_count = bv;
      lis->argmax_expert = ba;
      lis->lis = (double)((long long)m * bv) / (double)tasks;
    }
  }
}

cudaError_t launch_lis_from_counts(int m, long long tasks, const int32_t* counts, moe_lis_t* lis, cudaStream_t s) {
  launch_k(lis_from_counts_kernel, 1, 1024, 0, s, m, tasks, counts, lis);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_route_index(int mode, int T, int k, int m, const int32_t* idx, int32_t* counts, int32_t* offsets,
                               moe_lis_t* lis, int32_t* start, int* status, cudaStream_t s) {
  int R, L;
  route_ranges(T * k, m, &R, &L);
  const size_t smem = route_index_smem(R, m);
  static size_t attr = 0;
  if (smem > 48 * 1024 && smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(route_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  launch_k(route_index_kernel, 1, RI_THREADS, smem, s, mode, T, k, m, R, L, idx, counts, offsets, lis, start,
           status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------ ranks
// One warp per task range r walks it 32 tasks at a time in increasing task id (the
// ids of eight such steps loaded together): a task's rank among the lower lanes with
// the same expert (one match over the warp) plus the expert's cursor (started at
// start[r][e]) is its position pos in the stable counting sort; the group's last
// lane advances the cursor. Writes
// inv_perm[q] = pos, perm[pos] = q and, when given, w_perm[pos] = task_w[q] (the
// gate weight in segment order). A position outside its expert's segment
// [offsets[e], offsets[e + 1]) sets MOE_ERR_DEVICE_INDEX and that task is not
// written; after an earlier device error the kernel does nothing.
__global__ void rank_kernel(int Tk, int m, int L, const int32_t* __restrict__ idx, const int32_t* __restrict__ offsets,
                            const int32_t* __restrict__ start, const float* __restrict__ task_w,
                            int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm, float* __restrict__ w_perm,
                            int* status) {
  extern __shared__ int cur[];  // [m] cursors, then [m + 1] offsets
  int* off_s = cur + m;
  const int lane = threadIdx.x;
  const int r = blockIdx.x;
  const int lo = r * L, hi = min(Tk, lo + L);
  pdl_launch_dependents();
  pdl_wait();
  // an earlier device error stops the kernel; its status word is read in the same batch
  // of loads as the first eight steps' ids and gate weights, the cursors and the
  // offsets (one round trip before the first step, none inside it; nothing is stored
  // to global memory before the check)
  const int prior = status ? *reinterpret_cast<volatile int*>(status) : 0;
  int ev[8];
  float wv[8];
  auto load_steps = [&](int base) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int qq = base + 32 * u + lane;
      ev[u] = qq < hi ? idx[qq] : -1;
      wv[u] = (w_perm && qq < hi) ? task_w[qq] : 0.f;
    }
  };
  load_steps(lo);
  for (int e = lane; e < m; e += 32) cur[e] = start[(long long)r * m + e];
  for (int e = lane; e <= m; e += 32) off_s[e] = offsets[e];  // each step validates against them
  __syncwarp();
  if (prior != 0) return;
  for (int base = lo; base < hi; base += 32) {
    const int step = ((base - lo) >> 5) & 7;
    if (step == 0 && base != lo) load_steps(base);  // the ids of the next eight steps
    const int q = base + lane;
    int e = -1;
    float tw = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u == step) {
        e = ev[u];
        tw = wv[u];
      }
    if (e >= m) e = -1;
    // lanes holding the same expert (tasks past the range hold -1 and match only each other)
    const unsigned same = __match_any_sync(FULL, e);
    const int rank = __popc(same & ((1u << lane) - 1u)), cnt = __popc(same);
    const int b = e >= 0 ? cur[e] : 0;
    __syncwarp();
    if (q < hi) {
      const int pos = b + rank;
      const bool ok = e >= 0 && pos >= 0 && pos < Tk && pos >= off_s[e] && pos < off_s[e + 1];
      inv_perm[q] = ok ? pos : -1;
      if (ok) {
        perm[pos] = q;
        if (w_perm) w_perm[pos] = tw;
      } else {
        set_status(status, MOE_ERR_DEVICE_INDEX);
      }
    }
    if (e >= 0 && rank == cnt - 1) cur[e] = b + cnt;
    __syncwarp();
  }
}

cudaError_t launch_rank(int T, int k, int m, const int32_t* idx, const int32_t* offsets, const int32_t* start,
                        const float* task_w, int32_t* perm, int32_t* inv_perm, float* w_perm, int* status,
                        cudaStream_t s) {
  int R, L;
  route_ranges(T * k, m, &R, &L);
  launch_k(rank_kernel, R, 32, sizeof(int) * (2 * (size_t)m + 1), s, T * k, m, L, idx, offsets, start, task_w, perm,
           inv_perm, w_perm, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ permute rows
// One warp per (token t, part of its row): the part's chunks of x[t] are read once, 8
// of each lane's 16-byte chunks in flight, and written to the permuted position of
// each of t's k tasks: x_perm[inv_perm[t k + s], c] = x[t, c] (tasks without a valid
// position are skipped). A row is cut into parts when the batch has too few tokens
// to give every SM a few warps (decode batches).
constexpr int PR_THREADS = 256, PR_BATCH = 8;
__global__ void __launch_bounds__(PR_THREADS)
    permute_rows_kernel(int T, int k, int chunks, int parts, const int4* __restrict__ x,
                        const int32_t* __restrict__ inv_perm, int4* __restrict__ x_perm) {
  __shared__ int dst_s[PR_THREADS / 32][32];  // the warp's token: position of each task (or -1)
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int Tk = T * k;
  const long long nw = (long long)gridDim.x * (PR_THREADS / 32);
  const long long units = (long long)T * parts;
  const int cpp = (chunks + parts - 1) / parts;  // chunks per part
  for (long long un = (long long)blockIdx.x * (PR_THREADS / 32) + wib; un < units; un += nw) {
    const long long t = un / parts;
    const int c_lo = (int)(un % parts) * cpp, c_hi = min(chunks, c_lo + cpp);
    __syncwarp();  // the previous unit's readers of dst_s are done
    if (lane < k) {
      const int pos = inv_perm[t * k + lane];
      dst_s[wib][lane] = (pos >= 0 && pos < Tk) ? pos : -1;
    }
    __syncwarp();
    const int4* src = x + t * chunks;
    for (int c0 = c_lo + lane; c0 < c_hi; c0 += 32 * PR_BATCH) {  // lanes past the part's chunks skip it
      int4 v[PR_BATCH];
#pragma unroll
      for (int u = 0; u < PR_BATCH; ++u)
        if (c0 + 32 * u < c_hi) v[u] = src[c0 + 32 * u];
      for (int sl = 0; sl < k; ++sl) {
        const int dp = dst_s[wib][sl];
        if (dp < 0) continue;
        int4* o = x_perm + (long long)dp * chunks;
#pragma unroll
        for (int u = 0; u < PR_BATCH; ++u)
          if (c0 + 32 * u < c_hi) o[c0 + 32 * u] = v[u];
      }
    }
  }
}

cudaError_t launch_permute_rows(int dtype, int Tk, int k, int d, const void* x, const int32_t* inv_perm, void* x_perm,
                                cudaStream_t s) {
  const int chunks = d * (dtype == MOE_F32 ? 4 : 2) / 16;
  const int T = Tk / k;
  const int wpb = PR_THREADS / 32;
  // parts per row: halve the rows of a short batch until every SM has 4 warps' worth of
  // units, keeping at least a chunk per lane in each part (decode, 16 tokens: 8 parts,
  // 8.4 -> 6.5 µs; at 2048 tokens two parts measured slower than whole rows)
  int parts = 1;
  while ((long long)T * parts < 4LL * num_sms() && chunks / (2 * parts) >= 32) parts *= 2;
  const long long units = (long long)T * parts;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((units + wpb - 1) / wpb, (long long)num_sms() * 16));
  launch_k(permute_rows_kernel, blocks, PR_THREADS, 0, s, T, k, chunks, parts, (const int4*)x, inv_perm,
           (int4*)x_perm);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------ offsets, LIS and the permutation from tile ranks
// The router's epilogue left, per 128-token tile, the tasks of each expert
// (tile_cnt[tile][e]) and each task's rank among its tile's tasks of that expert
// (lrank). In the stable counting sort task q = t k + s of expert e goes to
//   offsets[e] + (tasks of e in earlier tiles) + lrank[q].
// Block (tile, part): every block sums the whole count table (the totals give
// the offsets), places its tile's tasks and copies its share of their rows (the
// 16-byte columns are split over the parts). Part 0 writes inv_perm, perm and
// w_perm; block (0, 0) writes counts, offsets and the LIS (R&Q Definition 1).
// The block's row chunks are loaded in the same batch as the tables, so the copy
// costs one store pass at the end.
constexpr int RS_THREADS = 512;
constexpr int RS_PRE = 8;  // row chunks per thread loaded ahead
__global__ void __launch_bounds__(RS_THREADS)
    route_scatter_kernel(int T, int k, int m, int ntiles, int parts, int chunks, const int32_t* __restrict__ tile_cnt,
                         const int32_t* __restrict__ idx, const int32_t* __restrict__ lrank,
                         const float* __restrict__ task_w, const int4* __restrict__ x, int32_t* __restrict__ counts,
                         int32_t* __restrict__ offsets, moe_lis_t* __restrict__ lis, int32_t* __restrict__ perm,
                         int32_t* __restrict__ inv_perm, float* __restrict__ w_perm, int4* __restrict__ x_perm,
                         int* status) {
  __shared__ int part_t[RS_THREADS], part_b[RS_THREADS];
  __shared__ int tot[ROUTE_MAX_M], base[ROUTE_MAX_M], off[ROUTE_MAX_M + 1];
  __shared__ int dest[128 * ROUTE_MAX_K];
  __shared__ int wsum[RS_THREADS / 32], wmax[RS_THREADS / 32], warg[RS_THREADS / 32];
  __shared__ int prior_s;
  const int tile = blockIdx.x, part = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long Tk = (long long)T * k;
  const long long q0 = (long long)tile * 128 * k;
  const int nitems = (int)min((long long)128 * k, Tk - q0);
  const int c_lo = (int)((long long)chunks * part / parts), c_hi = (int)((long long)chunks * (part + 1) / parts);
  const int pc = c_hi - c_lo, total = nitems * pc;
  pdl_launch_dependents();
  // (nothing is read before the wait: a kernel launched early may run beside an
  // earlier kernel of the stream that is still writing x)
  pdl_wait();
  // Item j of the block's copy is task i = j / pc of the tile (token tile * 128 + i / k)
  // and column chunk c_lo + j % pc. A thread's items are j = tid + n * RS_THREADS, so
  // (i, j % pc) is walked by adding (RS_THREADS / pc, RS_THREADS % pc) with one carry:
  // no division per item (divisions were most of the kernel's instructions).
  const unsigned upc = (unsigned)pc, uk = (unsigned)k;  // pc >= 1: parts <= chunks
  const unsigned di = RS_THREADS / upc, dr = RS_THREADS - di * upc;
  const unsigned wi0 = (unsigned)tid / upc, wr0 = (unsigned)tid - wi0 * upc;
  const long long tok0 = (long long)tile * 128;
  auto advance = [&](unsigned& i, unsigned& r) {
    i += di;
    r += dr;
    if (r >= upc) {
      r -= upc;
      ++i;
    }
  };
  auto src_row = [&](unsigned i) { return (tok0 + (uk == 1u ? i : i / uk)) * chunks; };
  int4 pre[RS_PRE];  // the row chunks, loaded together with the tables below
  unsigned wi = wi0, wr = wr0;
#pragma unroll
  for (int u = 0; u < RS_PRE; ++u) {
    if (tid + u * RS_THREADS < total) pre[u] = x[src_row(wi) + c_lo + wr];
    advance(wi, wr);
  }
  if (tid == 0) prior_s = *reinterpret_cast<volatile int*>(status);
  // 1. per (group g, expert e): tasks of e in tiles g, g + G, ..., all and before this tile
  const int G = RS_THREADS / m;  // >= 2 for m <= 256
  int pt = 0, pb = 0;
  if (tid < G * m) {
    const int g = tid / m, e = tid - g * m;
    for (int tl0 = g; tl0 < ntiles; tl0 += 16 * G) {
      int v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int tl = tl0 + u * G;
        v[u] = tl < ntiles ? tile_cnt[(long long)tl * m + e] : 0;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        pt += v[u];
        pb += tl0 + u * G < tile ? v[u] : 0;
      }
    }
  }
  int ie[2], ir[2];  // this tile's tasks (at most 128 k <= 2 per thread)
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = tid + u * RS_THREADS;
    ie[u] = i < nitems ? idx[q0 + i] : -1;
    ir[u] = i < nitems ? lrank[q0 + i] : 0;
  }
  if (tid < G * m) {
    part_t[tid] = pt;
    part_b[tid] = pb;
  }
  __syncthreads();
  if (prior_s != 0) return;  // an earlier kernel flagged an error (uniform: read once)
  // 2. totals, exclusive scan over experts, this tile's bases; LIS in block (0, 0)
  int n = 0, b = 0;
  if (tid < m)
    for (int g = 0; g < G; ++g) {
      n += part_t[g * m + tid];
      b += part_b[g * m + tid];
    }
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += v;
  }
  int mv = tid < m ? n : -1, ma = tid;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const int ov = __shfl_xor_sync(FULL, mv, o), oa = __shfl_xor_sync(FULL, ma, o);
    if (ov > mv || (ov == mv && oa < ma)) {
      mv = ov;
      ma = oa;
    }
  }
  if (lane == 31) wsum[warp] = incl;
  if (lane == 0) {
    wmax[warp] = mv;
    warg[warp] = ma;
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = RS_THREADS / 32;
    const int ws = lane < nw ? wsum[lane] : 0;
    int wi = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < nw) wsum[lane] = wi - ws;
    int bv = lane < nw ? wmax[lane] : -1, ba = lane < nw ? warg[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const int ov = __shfl_xor_sync(FULL, bv, o), oa = __shfl_xor_sync(FULL, ba, o);
      if (ov > bv || (ov == bv && oa < ba)) {
        bv = ov;
        ba = oa;
      }
    }
    if (lane == 0) {
      wmax[0] = bv;
      warg[0] = ba;
    }
  }
  __syncthreads();
  if (tid < m) {
    const int ex = incl - n + wsum[warp];
    tot[tid] = n;
    off[tid] = ex;
    base[tid] = ex + b;
    if (tid == m - 1) off[m] = ex + n;
    if (tile == 0 && part == 0) {
      counts[tid] = n;
      offsets[tid] = ex;
      if (tid == m - 1) offsets[m] = ex + n;
    }
  }
  if (tile == 0 && part == 0 && tid == 0 && lis) {
    lis->max_count = wmax[0];
    lis->argmax_expert = warg[0];
    lis->lis = (double)((long long)m * wmax[0]) / (double)((long long)T * k);
  }
  __syncthreads();
  // 3. this tile's tasks
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int i = tid + u * RS_THREADS;
    if (i >= nitems) continue;
    const long long q = q0 + i;
    const int e = ie[u];
    int d = -1;
    if (e >= 0 && e < m) {
      d = base[e] + ir[u];
      if (d < off[e] || d >= off[e] + tot[e]) d = -1;
    }
    if (d < 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    dest[i] = d;
    if (part == 0) {
      inv_perm[q] = d;
      if (d >= 0) {
        perm[d] = (int32_t)q;
        if (w_perm) w_perm[d] = task_w[q];
      }
    }
  }
  __syncthreads();
  // 4. rows: x_perm[dest, c] = x[q / k, c] for this part's columns
  {
    unsigned si = wi0, sr = wr0;
#pragma unroll
    for (int u = 0; u < RS_PRE; ++u) {
      if (tid + u * RS_THREADS < total) {
        const int d = dest[si];
        if (d >= 0) x_perm[(long long)d * chunks + c_lo + sr] = pre[u];
      }
      advance(si, sr);
    }
  }
  for (int j0 = tid + RS_PRE * RS_THREADS; j0 < total; j0 += RS_PRE * RS_THREADS) {  // beyond the first batch
    int4 v[RS_PRE];
    long long o[RS_PRE];
#pragma unroll
    for (int u = 0; u < RS_PRE; ++u) {
      o[u] = -1;
      if (j0 + u * RS_THREADS < total) {
        const int d = dest[wi];
        if (d >= 0) {
          v[u] = x[src_row(wi) + c_lo + wr];
          o[u] = (long long)d * chunks + c_lo + wr;
        }
      }
      advance(wi, wr);
    }
#pragma unroll
    for (int u = 0; u < RS_PRE; ++u)
      if (o[u] >= 0) x_perm[o[u]] = v[u];
  }
}

cudaError_t launch_route_scatter(int dtype, int T, int k, int m, int d, const int32_t* tile_cnt, const int32_t* idx,
                                 const int32_t* lrank, const float* task_w, const void* x, int32_t* counts,
                                 int32_t* offsets, moe_lis_t* lis, int32_t* perm, int32_t* inv_perm, float* w_perm,
                                 void* x_perm, int* status, cudaStream_t s) {
  const int ntiles = (T + 127) / 128;
  const int chunks = d * (dtype == MOE_F32 ? 4 : 2) / 16;
  // about one wave of blocks (one 512-thread block fits an SM's registers); the
  // rows beyond a block's first batch of loads go through the unrolled loop
  const int parts = std::max(1, std::min({(num_sms() + ntiles / 2) / ntiles, chunks, 65535}));
  launch_k(route_scatter_kernel, dim3(ntiles, parts), RS_THREADS, 0, s, T, k, m, ntiles, parts, chunks, tile_cnt, idx,
           lrank, task_w, (const int4*)x, counts, offsets, lis, perm, inv_perm, w_perm, (int4*)x_perm, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ R&Q replica dispatch
// The heavy-hitter h is the device LIS record's argmax (most tasks, lowest index).
// A task's rank in h's segment of the stable sort is inv_perm[q] - offsets[h]; the
// odd ranks go to the replica, expert m (every second task of h in task order).
// Block 0 also writes the group -> weight map (g, and h for the replica) and, when
// given, the counts and the LIS (R&Q Definition 1) over the m + 1 experts.
__global__ void replica_split_kernel(int T, int k, int m, const int32_t* __restrict__ idx,
                                     const int32_t* __restrict__ offsets, const int32_t* __restrict__ inv_perm,
                                     const moe_lis_t* __restrict__ lis_in, int32_t* __restrict__ idx_out,
                                     int32_t* __restrict__ gmap, int32_t* __restrict__ counts_out,
                                     moe_lis_t* __restrict__ lis_out, int* status) {
  __shared__ int prior_s;
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) prior_s = *reinterpret_cast<volatile int*>(status);
  __syncthreads();
  if (prior_s != 0) return;  // uniform across the block
  const long long Tk = (long long)T * k;
  const int h = lis_in->argmax_expert;
  if (h < 0 || h >= m) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  const int n_h = offsets[h + 1] - offsets[h];
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < Tk; q += (long long)gridDim.x * blockDim.x) {
    const int e = idx[q];
    int o = e;
    if (e < 0 || e >= m) {
      set_status(status, MOE_ERR_DEVICE_INDEX);
    } else if (e == h) {
      const int r = inv_perm[q] - offsets[h];
      if (r < 0 || r >= n_h) set_status(status, MOE_ERR_DEVICE_INDEX);
      o = (r & 1) ? m : h;
    }
    idx_out[q] = o;
  }
  if (blockIdx.x != 0) return;
  for (int g = threadIdx.x; g <= m; g += blockDim.x) gmap[g] = g < m ? g : h;
  auto count_after = [&](int j) {
    if (j == m) return n_h / 2;
    const int n = offsets[j + 1] - offsets[j];
    return j == h ? n - n_h / 2 : n;
  };
  if (counts_out)
    for (int j = threadIdx.x; j <= m; j += blockDim.x) counts_out[j] = count_after(j);
  if (lis_out && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int bv = -1, ba = 0x7fffffff;
    for (int j = lane; j <= m; j += 32) {
      const int v = count_after(j);
      if (v > bv) {  // ascending j per lane: an equal count keeps the lower expert
        bv = v;
        ba = j;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const int ov = __shfl_xor_sync(FULL, bv, o), oa = __shfl_xor_sync(FULL, ba, o);
      if (ov > bv || (ov == bv && oa < ba)) {
        bv = ov;
        ba = oa;
      }
    }
    if (lane == 0) {
      lis_out->max_count = bv;
      lis_out->argmax_expert = ba;
      lis_out->lis = (double)((long long)(m + 1) * bv) / (double)((long long)T * k);
    }
  }
}

cudaError_t launch_replica_split(int T, int k, int m, const int32_t* idx, const int32_t* offsets,
                                 const int32_t* inv_perm, const moe_lis_t* lis_in, int32_t* idx_out, int32_t* gmap,
                                 int32_t* counts_out, moe_lis_t* lis_out, int* status, cudaStream_t s) {
  const long long Tk = (long long)T * k;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((Tk + 255) / 256, (long long)num_sms() * 4));
  launch_k(replica_split_kernel, blocks, 256, 0, s, T, k, m, idx, offsets, inv_perm, lis_in, idx_out, gmap, counts_out,
           lis_out, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ combine
// out[t, c] = sum_s sum_split y[split][inv_perm[t k + s], c]
//           + sum_sh sum_split ysh[split][sh T + t, c], fp32, in that order. With
// row_splits the routed rows have their own split counts (row_splits[pos] <= ksplit
// partials for permuted row pos).
template <typename OutT>
__device__ __forceinline__ void store4(OutT* out, long long i4, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* out, long long i4, float4 v) {
  reinterpret_cast<float4*>(out)[i4] = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* out, long long i4, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  reinterpret_cast<uint2*>(out)[i4] = u;
}

// Block (token t, column block): the token's partial rows are listed first — the
// (slot, split) rows of its routed tasks, then the (shared expert, split) rows — as
// float4 offsets in shared memory, built in parallel (one thread per slot); then
// each thread owns CPT 16-byte column chunks and loads U listed rows' chunks at once
// (U CPT = 8 float4 in flight), adding them in list order, so every output is the
// same sum in the same order as one thread walking the list. Few tokens (decode)
// take narrow column blocks so the grid still covers the SMs.
constexpr int CB_THREADS = 256;
constexpr int CB_MAX_ROWS = 32 * 64 + 8 * 64;  // k <= 32 slots, n_shared <= 8, <= 64 splits each
template <typename OutT, int CPT>
__global__ void __launch_bounds__(CB_THREADS, 4)
    combine_kernel(int T, int d4, int k, int ksplit, const float4* __restrict__ y, long long ysplit4,
                   const int32_t* __restrict__ inv_perm, int n_sh, const float4* __restrict__ ysh,
                   long long yshsplit4, OutT* __restrict__ out, const int32_t* __restrict__ row_splits, int ncb) {
  constexpr int U = 8 / CPT > 1 ? 8 / CPT : 2;
  __shared__ long long rows_s[CB_MAX_ROWS];
  __shared__ int cnt_s[33];
  pdl_launch_dependents();
  pdl_wait();
  const int Tk = T * k;
  const int tid = threadIdx.x, lane = tid & 31;
  for (long long tb = blockIdx.x; tb < (long long)T * ncb; tb += gridDim.x) {
    const long long t = tb / ncb;
    const int cb = (int)(tb - t * ncb) * CB_THREADS * CPT;
    __syncthreads();  // the previous token's readers of rows_s are done
    if (tid < 32) {  // warp 0: rows per slot, their prefix, then each slot's rows
      long long base = -1;
      int ns = 0;
      if (lane < k) {
        const int pos = inv_perm[t * k + lane];
        if (pos >= 0 && pos < Tk) {
          base = (long long)pos * d4;
          ns = row_splits ? min(ksplit, row_splits[pos]) : ksplit;
        }
      }
      int incl = ns;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      for (int sp = 0; sp < ns; ++sp) rows_s[incl - ns + sp] = base + sp * ysplit4;
      if (lane == 31) cnt_s[0] = incl;
    }
    __syncthreads();
    const int nr = cnt_s[0];
    for (int i = tid; i < n_sh * ksplit; i += CB_THREADS) {  // shared-expert rows after the routed ones
      const int sh = i / ksplit, sp = i - sh * ksplit;
      rows_s[nr + i] = -1 - (sp * yshsplit4 + ((long long)sh * T + t) * d4);  // tagged: from ysh
    }
    __syncthreads();
    const int P = nr + n_sh * ksplit;
    float4 a[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) a[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < P; i0 += U) {
      float4 v[U][CPT];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (i0 + u < P) {
          const long long r = rows_s[i0 + u];
          const float4* src = r >= 0 ? y + r : ysh + (-1 - r);
#pragma unroll
          for (int j = 0; j < CPT; ++j) {
            const int c = cb + tid + CB_THREADS * j;
            if (c < d4) v[u][j] = src[c];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + u < P)
#pragma unroll
          for (int j = 0; j < CPT; ++j) {
            a[j].x += v[u][j].x; a[j].y += v[u][j].y; a[j].z += v[u][j].z; a[j].w += v[u][j].w;
          }
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = cb + tid + CB_THREADS * j;
      if (c < d4) store4<OutT>(out, t * d4 + c, a[j]);
    }
  }
}

cudaError_t launch_combine(int dtype, int T, int d, int k, int ksplit, const float* y_perm, long long y_split_stride,
                           const int32_t* inv_perm, int n_shared, const float* y_shared, long long ysh_split_stride,
                           void* out, cudaStream_t s, const int32_t* row_splits) {
  const int d4 = d / 4;
  const int nsh = y_shared ? n_shared : 0;
  if (k > 32 || nsh > 8 || ksplit > 64) return cudaErrorInvalidValue;
  // widest column blocks that leave no thread without columns (a 512-float4 row keeps
  // every thread of a 2-per-thread block busy, where 4 per thread idled half of them)
  // and still give the grid two blocks per SM
  int cpt = 4;
  while (cpt > 1 && (CB_THREADS * cpt > d4 ||
                     (long long)T * ((d4 + CB_THREADS * cpt - 1) / (CB_THREADS * cpt)) < 2LL * num_sms()))
    cpt >>= 1;
  const int ncb = (d4 + CB_THREADS * cpt - 1) / (CB_THREADS * cpt);
  const int blocks = (int)std::max<long long>(1, std::min<long long>((long long)T * ncb, (long long)num_sms() * 8));
#define MOE_COMBINE(CPT_)                                                                                          \
  do {                                                                                                           \
    if (dtype == MOE_F32)                                                                                        \
      launch_k(combine_kernel<float, CPT_>, blocks, CB_THREADS, 0, s, T, d4, k, ksplit, (const float4*)y_perm,   \
               y_split_stride / 4, inv_perm, nsh, (const float4*)y_shared, ysh_split_stride / 4, (float*)out,      \
               row_splits, ncb);                                                                                 \
    else                                                                                                         \
      launch_k(combine_kernel<__nv_bfloat16, CPT_>, blocks, CB_THREADS, 0, s, T, d4, k, ksplit,                  \
               (const float4*)y_perm, y_split_stride / 4, inv_perm, nsh, (const float4*)y_shared,                  \
               ysh_split_stride / 4, (__nv_bfloat16*)out, row_splits, ncb);                                      \
  } while (0)
  if (cpt == 1)
    MOE_COMBINE(1);
  else if (cpt == 2)
    MOE_COMBINE(2);
  else
    MOE_COMBINE(4);
#undef MOE_COMBINE
  count_launch();
  return cudaGetLastError();
}

__global__ void reduce_splits_kernel(long long n4, int ksplit, const float4* __restrict__ in, long long split4,
                                     float4* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    float4 a = in[i];
    for (int sp = 1; sp < ksplit; ++sp) {
      const float4 v = in[sp * split4 + i];
      a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
    }
    out[i] = a;
  }
}

cudaError_t launch_reduce_splits(long long n, int ksplit, const float* in, long long split_stride, float* out,
                                 cudaStream_t s) {
  const long long n4 = n / 4;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((n4 + 255) / 256, (long long)num_sms() * 16));
  launch_k(reduce_splits_kernel, blocks, 256, 0, s, n4, ksplit, (const float4*)in, split_stride / 4, (float4*)out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe
