// Grouped expert FFN on the CUDA cores in fp32 (for fp32 layers, whose 1e-5
// tolerance rules out tf32/bf16 tensor-core inputs). Same problem description as
// the tensor-core path (GemmParams): out = epi(A_g . B_row^T) per segment row.
// One warp per (row, 32 output features); lanes stride over K with fp32 FMA and
// reduce with a shuffle tree.
#include <algorithm>

#include "common.cuh"

namespace moe {

namespace {
constexpr unsigned FULL = 0xffffffffu;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, long long i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, long long i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void stf(T* p, long long i, float v);
template <>
__device__ __forceinline__ void stf<float>(float* p, long long i, float v) { p[i] = v; }
template <>
__device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, long long i, float v) {
  p[i] = __float2bfloat16_rn(v);
}
}  // namespace

template <typename TIn, int EPI>
__global__ void simt_gemm_kernel(const __grid_constant__ GemmParams p, long long max_rows) {
  const GemmClass& c = p.cls[blockIdx.y];
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  pdl_wait();
  if (p.status && *reinterpret_cast<volatile int*>(p.status) != 0) return;  // earlier device error
  const int fblocks = (c.R + 31) / 32;
  const long long nrows = c.seg_off ? max_rows : (long long)c.n_groups * c.const_rows;
  const long long items = nrows * fblocks;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const TIn* A0 = (const TIn*)c.a0;
  const TIn* A1 = (const TIn*)c.a1;
  const TIn* B = (const TIn*)c.b;
  for (long long it = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items; it += warps) {
    const long long i = it / fblocks;
    const int fb = (int)(it - i * fblocks);
    int g;
    long long brow, orow;
    if (c.seg_off) {
      if (i >= c.seg_off[c.n_groups] || i >= c.max_row) continue;
      int lo = 0, hi = c.n_groups - 1;  // largest g with seg_off[g] <= i
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c.seg_off[mid] <= i) lo = mid; else hi = mid - 1;
      }
      g = lo;
      brow = orow = i;
    } else {
      g = (int)(i / c.const_rows);
      const long long r = i - (long long)g * c.const_rows;
      brow = (long long)g * c.b_group_stride + r;
      orow = (long long)g * c.out_group_stride + r;
    }
    const int f_end = min(c.R, fb * 32 + 32);
    float keep0 = 0.f, keep1 = 0.f;
    for (int j = fb * 32; j < f_end; ++j) {
      const long long arow = (long long)g * c.R + j;
      float s0 = 0.f, s1 = 0.f;
      for (int q = lane; q < c.K; q += 32) {
        const float bv = ldf(B, brow * c.b_ld + q);
        s0 = fmaf(ldf(A0, arow * c.a_ld + q), bv, s0);
        if (EPI == EPI_SWIGLU) s1 = fmaf(ldf(A1, arow * c.a_ld + q), bv, s1);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        s0 += __shfl_xor_sync(FULL, s0, o);
        if (EPI == EPI_SWIGLU) s1 += __shfl_xor_sync(FULL, s1, o);
      }
      if (lane == j - fb * 32) {
        keep0 = s0;
        keep1 = s1;
      }
    }
    const int j = fb * 32 + lane;
    if (j < f_end) {
      if (EPI == EPI_SWIGLU) {
        stf((TIn*)c.out, orow * c.out_ld + j, keep0 / (1.f + expf(-keep0)) * keep1);
      } else if (EPI == EPI_RELU) {
        stf((TIn*)c.out, orow * c.out_ld + j, fmaxf(keep0, 0.f));
      } else {  // EPI_DOWN
        float wgt = 1.f;
        if (c.task_w) {
          const int qq = c.perm[orow];
          wgt = (qq >= 0 && qq < c.max_row) ? c.task_w[qq] : 0.f;
        }
        ((float*)c.out)[orow * c.out_ld + j] = keep0 * wgt;
      }
    }
  }
}

cudaError_t launch_simt_gemm(int epi, int dtype, const GemmParams& p, int max_rows_per_class, cudaStream_t s) {
  dim3 grid(std::max(1, num_sms() * 4), p.n_classes);
#define MOE_SIMT_CASE(EPI_)                                                                          \
  if (epi == EPI_) {                                                                                 \
    if (dtype == MOE_F32)                                                                            \
      launch_k(simt_gemm_kernel<float, EPI_>, grid, 256, 0, s, p, max_rows_per_class);                     \
    else                                                                                             \
      launch_k(simt_gemm_kernel<__nv_bfloat16, EPI_>, grid, 256, 0, s, p, max_rows_per_class);             \
    count_launch();                                                                                  \
    return cudaGetLastError();                                                                       \
  }
  MOE_SIMT_CASE(EPI_SWIGLU)
  MOE_SIMT_CASE(EPI_RELU)
  MOE_SIMT_CASE(EPI_DOWN)
#undef MOE_SIMT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
