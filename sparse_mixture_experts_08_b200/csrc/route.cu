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
    simt_logits_kernel<float><<<blocks, 256, 0, s>>>(T, d, m, (const float*)x, (const float*)w_r, bias, logits);
  else
    simt_logits_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(T, d, m, (const __nv_bfloat16*)x,
                                                             (const __nv_bfloat16*)w_r, bias, logits);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ top-k + softmax
// One warp per token. k rounds of a warp arg-max over the not-yet-chosen
// experts, ordered by (logit desc, expert index asc). Gate weights: softmax over
// all m logits (exp in fp32 of l - max, sum in fp64), renormalised over the k
// chosen when requested.
__global__ void topk_softmax_kernel(int T, int m, int k, int renorm, const float* __restrict__ logits,
                                    int32_t* __restrict__ idx, float* __restrict__ w) {
  __shared__ int s_sel[TOPK_WARPS][32];
  __shared__ float s_val[TOPK_WARPS][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int t = blockIdx.x * TOPK_WARPS + wib;
  if (t >= T) return;
  const float* L = logits + (long long)t * m;
  for (int s = 0; s < k; ++s) {
    float bv = -FLT_MAX;
    int be = 0x7fffffff;
    for (int e = lane; e < m; e += 32) {
      bool taken = false;
      for (int j = 0; j < s; ++j) taken |= (s_sel[wib][j] == e);
      if (taken) continue;
      const float v = L[e];
      if (be == 0x7fffffff || v > bv || (v == bv && e < be)) {
        bv = v;
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(FULL, bv, o);
      const int oe = __shfl_xor_sync(FULL, be, o);
      if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
        bv = ov;
        be = oe;
      }
    }
    if (lane == 0) {
      s_sel[wib][s] = be;
      s_val[wib][s] = bv;
    }
    __syncwarp();
  }
  const float mx = s_val[wib][0];
  double z = 0.0;
  for (int e = lane; e < m; e += 32) z += (double)expf(L[e] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
  double sel = 0.0;
  for (int s = 0; s < k; ++s) sel += (double)expf(s_val[wib][s] - mx) / z;
  if (lane < k) {
    double p = (double)expf(s_val[wib][lane] - mx) / z;
    if (renorm) p /= sel;
    idx[(long long)t * k + lane] = s_sel[wib][lane];
    w[(long long)t * k + lane] = (float)p;
  }
}

cudaError_t launch_topk_softmax(int T, int m, int k, int renorm, const float* logits, int32_t* idx, float* w,
                                cudaStream_t s) {
  topk_softmax_kernel<<<(T + TOPK_WARPS - 1) / TOPK_WARPS, TOPK_WARPS * 32, 0, s>>>(T, m, k, renorm, logits, idx, w);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------ histogram, offsets, LIS, ranks
// One block of 1024 threads (the routing tables are tiny: T k ids). Warp w owns
// the contiguous task range [w L, (w + 1) L), L = ceil(T k / 32), walked 32 tasks
// at a time in increasing task id.
//  pass 1: per-warp counts wc[w][e] (peer groups from __match_any_sync; each warp
//          writes only its own row, so no atomics).
//  scan:   per expert, exclusive prefix over warps -> wc[w][e] = tasks of e in
//          warps before w; the total is n_e.
// mode & 1: offsets = exclusive scan of n_e, max / lowest argmax, and
//           LIS = m max / (T k) (R&Q Definition 1).
// mode & 2: pass 2 re-walks each warp's range in the same order:
//           pos = offsets[e] + wc[w][e] + (rank among the sub-chunk's peers), then
//           wc[w][e] += peers: the stable counting-sort position, inv_perm[q] = pos
//           (its inverse perm[pos] = q is scattered by the many-block row copy, so
//           this one-SM kernel issues only coalesced stores).
// Any id outside [0, m) (or, with given offsets, a position outside its segment)
// sets MOE_ERR_DEVICE_INDEX and nothing further is written.
constexpr int RI_MAX_REG = 16;  // sub-chunks per warp kept in registers between the passes

__global__ void __launch_bounds__(RI_THREADS, 1)
    route_index_kernel(int mode, int T, int k, int m, const int32_t* __restrict__ idx, int32_t* __restrict__ counts,
                       int32_t* __restrict__ offsets, moe_lis_t* __restrict__ lis, int32_t* __restrict__ inv_perm,
                       int* status) {
  extern __shared__ int sm[];
  int* wc = sm;             // [32][m]
  int* off = wc + 32 * m;   // [m + 1]
  __shared__ int bad;
  __shared__ int wsum[32], wmax[32], warg[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = blockDim.x >> 5;
  const int Tk = T * k;
  const int L = (Tk + nw - 1) / nw;
  const int lo = min(Tk, warp * L), hi = min(Tk, lo + L);
  const unsigned lt = (1u << lane) - 1u;
  if (tid == 0) bad = 0;
  for (int i = tid; i < nw * m; i += blockDim.x) wc[i] = 0;
  __syncthreads();
  // All of this warp's ids (up to RI_MAX_REG sub-chunks) are loaded up front so the
  // loads overlap; longer ranges reload the rest in the loops below.
  int ev[RI_MAX_REG];
#pragma unroll
  for (int r = 0; r < RI_MAX_REG; ++r) {
    const int q = lo + r * 32 + lane;
    ev[r] = q < hi ? idx[q] : -1;
  }
  for (int base = lo, r = 0; base < hi; base += 32, ++r) {
    const int q = base + lane;
    int e = -1;
    if (r < RI_MAX_REG) {
#pragma unroll
      for (int rr = 0; rr < RI_MAX_REG; ++rr)
        if (rr == r) e = ev[rr];
    } else {
      e = q < hi ? idx[q] : -1;
    }
    if (q < hi && (e < 0 || e >= m)) {
      bad = 1;
      e = -2;
    }
    const unsigned peers = __match_any_sync(FULL, e);
    if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * m + e] += __popc(peers);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
    return;
  }
  for (int e = tid; e < m; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < nw; ++w) {
      const int t = wc[w * m + e];
      wc[w * m + e] = run;
      run += t;
    }
    off[e] = run;  // n_e for now
  }
  __syncthreads();
  if (mode & 1) {
    const int c = tid < m ? off[tid] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += v;
    }
    int mv = tid < m ? c : -1, ma = tid;
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
      const int ex = incl - c + wsum[warp];
      off[tid] = ex;
      counts[tid] = c;
      offsets[tid] = ex;
      if (tid == m - 1) {
        off[m] = ex + c;
        offsets[m] = ex + c;
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
  if (!(mode & 2)) return;
  for (int base = lo, r = 0; base < hi; base += 32, ++r) {
    const int q = base + lane;
    int e = -1;
    if (r < RI_MAX_REG) {
#pragma unroll
      for (int rr = 0; rr < RI_MAX_REG; ++rr)
        if (rr == r) e = ev[rr];
    } else {
      e = q < hi ? idx[q] : -1;
    }
    const unsigned peers = __match_any_sync(FULL, e);
    const int leader = __ffs(peers) - 1;
    const int b = e >= 0 ? wc[warp * m + e] : 0;
    __syncwarp();
    if (e >= 0) {
      const int pos = off[e] + b + __popc(peers & lt);
      if (pos >= 0 && pos >= off[e] && pos < off[e + 1] && pos < Tk) {
        inv_perm[q] = pos;  // coalesced; the scattered perm[pos] is written by the row copy
      } else {
        set_status(status, MOE_ERR_DEVICE_INDEX);
      }
      if (lane == leader) wc[warp * m + e] = b + __popc(peers);
    }
    __syncwarp();
  }
}

size_t route_index_smem(int m) { return sizeof(int) * ((size_t)33 * m + 1); }

cudaError_t launch_route_index(int mode, int T, int k, int m, const int32_t* idx, int32_t* counts, int32_t* offsets,
                               moe_lis_t* lis, int32_t* inv_perm, int* status, cudaStream_t s) {
  const size_t smem = route_index_smem(m);
  static size_t attr = 0;
  if (smem > 48 * 1024 && smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(route_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  route_index_kernel<<<1, RI_THREADS, smem, s>>>(mode, T, k, m, idx, counts, offsets, lis, inv_perm, status);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ permute rows
// Walks the tasks q in order (one warp each): pos = inv_perm[q];
// x_perm[pos, :] = x[q / k, :] with 16-byte vectors; perm[pos] = q; and, when
// given, w_perm[pos] = task_w[q] (the gate weight in segment order, read by the
// down-projection epilogue).
__global__ void permute_rows_kernel(int Tk, int k, int chunks, const int4* __restrict__ x,
                                    const int32_t* __restrict__ inv_perm, const float* __restrict__ task_w,
                                    int32_t* __restrict__ perm, float* __restrict__ w_perm, int4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long q = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); q < Tk; q += warps) {
    const int pos = inv_perm[q];
    if (pos < 0 || pos >= Tk) continue;
    if (lane == 0) {
      perm[pos] = (int32_t)q;
      if (w_perm) w_perm[pos] = task_w[q];
    }
    const int4* src = x + (q / k) * chunks;
    int4* dst = x_perm + (long long)pos * chunks;
    for (int c = lane; c < chunks; c += 32) dst[c] = src[c];
  }
}

cudaError_t launch_permute_rows(int dtype, int Tk, int k, int d, const void* x, const int32_t* inv_perm,
                                const float* task_w, int32_t* perm, float* w_perm, void* x_perm, cudaStream_t s) {
  const int chunks = d * (dtype == MOE_F32 ? 4 : 2) / 16;
  const int blocks = std::max(1, std::min((Tk + 7) / 8, num_sms() * 8));
  permute_rows_kernel<<<blocks, 256, 0, s>>>(Tk, k, chunks, (const int4*)x, inv_perm, task_w, perm, w_perm,
                                             (int4*)x_perm);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ combine
// out[t, c] = sum_s sum_split y[split][inv_perm[t k + s], c]
//           + sum_sh sum_split ysh[split][sh T + t, c], fp32, slot order; 4 columns
// per thread (16-byte loads).
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

template <typename OutT>
__global__ void combine_kernel(int T, int d4, int k, int ksplit, const float4* __restrict__ y, long long ysplit4,
                               const int32_t* __restrict__ inv_perm, int n_sh, const float4* __restrict__ ysh,
                               long long yshsplit4, OutT* __restrict__ out) {
  const long long n = (long long)T * d4;
  const int Tk = T * k;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / d4;
    const int c = (int)(i - t * d4);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < k; ++s) {
      const int pos = inv_perm[t * k + s];
      if (pos < 0 || pos >= Tk) continue;
      for (int sp = 0; sp < ksplit; ++sp) {
        const float4 v = y[sp * ysplit4 + (long long)pos * d4 + c];
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
      }
    }
    for (int sh = 0; sh < n_sh; ++sh)
      for (int sp = 0; sp < ksplit; ++sp) {
        const float4 v = ysh[sp * yshsplit4 + ((long long)sh * T + t) * d4 + c];
        a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
      }
    store4<OutT>(out, i, a);
  }
}

cudaError_t launch_combine(int dtype, int T, int d, int k, int ksplit, const float* y_perm, long long y_split_stride,
                           const int32_t* inv_perm, int n_shared, const float* y_shared, long long ysh_split_stride,
                           void* out, cudaStream_t s) {
  const int d4 = d / 4;
  const long long n = (long long)T * d4;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((n + 255) / 256, (long long)num_sms() * 16));
  if (dtype == MOE_F32)
    combine_kernel<float><<<blocks, 256, 0, s>>>(T, d4, k, ksplit, (const float4*)y_perm, y_split_stride / 4, inv_perm,
                                                 y_shared ? n_shared : 0, (const float4*)y_shared,
                                                 ysh_split_stride / 4, (float*)out);
  else
    combine_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(T, d4, k, ksplit, (const float4*)y_perm, y_split_stride / 4,
                                                         inv_perm, y_shared ? n_shared : 0, (const float4*)y_shared,
                                                         ysh_split_stride / 4, (__nv_bfloat16*)out);
  count_launch();
  return cudaGetLastError();
}

__global__ void reduce_splits_kernel(long long n4, int ksplit, const float4* __restrict__ in, long long split4,
                                     float4* __restrict__ out) {
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
  reduce_splits_kernel<<<blocks, 256, 0, s>>>(n4, ksplit, (const float4*)in, split_stride / 4, (float4*)out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe
