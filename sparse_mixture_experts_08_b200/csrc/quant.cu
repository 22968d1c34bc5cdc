// Per-row E4M3 quantization of bf16 rows (8-bit expert weights, R&Q "Free
// parameters": 8-bit expert copies). For each row: scale = max |v| / 448 in IEEE
// fp32 (1 when the row is all zero); code_j = E4M3(v_j / scale), round to nearest
// even, saturating at +-448. Used once on the expert weights (per output channel)
// and on every projection's input rows (x per token, h per task) in the 8-bit layer.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

namespace {

constexpr int QZ_WARPS = 8;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t e4m3(float v, float sc) {
  return (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v, sc), __NV_SATFINITE, __NV_E4M3);
}

// One warp per row; 16-byte loads (8 bf16), 8-byte stores (8 codes).
__global__ void __launch_bounds__(QZ_WARPS * 32) quantize_e4m3_rows_kernel(long long rows, int cols,
                                                                            const uint4* __restrict__ src,
                                                                            long long src_ld8, uint2* __restrict__ dst,
                                                                            long long dst_ld8, float* __restrict__ scale) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * QZ_WARPS + warp;
  if (row >= rows) return;
  const uint4* s = src + row * src_ld8;
  const int n8 = cols >> 3;
  float amax = 0.f;
  for (int i = lane; i < n8; i += 32) {
    const uint4 v = s[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  if (lane == 0) scale[row] = sc;
  uint2* d = dst + row * dst_ld8;
  for (int i = lane; i < n8; i += 32) {
    const uint4 v = s[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      out[h] = e4m3(bf16_lo(w[2 * h]), sc) | (e4m3(bf16_hi(w[2 * h]), sc) << 8) |
               (e4m3(bf16_lo(w[2 * h + 1]), sc) << 16) | (e4m3(bf16_hi(w[2 * h + 1]), sc) << 24);
    d[i] = make_uint2(out[0], out[1]);
  }
}

}  // namespace

cudaError_t launch_quantize_e4m3(long long rows, int cols, const void* src, long long src_ld, uint8_t* dst,
                                 long long dst_ld, float* scale, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (cols <= 0 || cols % 8 || src_ld % 8 || dst_ld % 8 || ((uintptr_t)src & 15) || ((uintptr_t)dst & 7))
    return cudaErrorInvalidValue;
  const long long blocks = (rows + QZ_WARPS - 1) / QZ_WARPS;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  cudaError_t e = launch_k(quantize_e4m3_rows_kernel, dim3((unsigned)blocks), dim3(QZ_WARPS * 32), 0, s, rows, cols,
                           reinterpret_cast<const uint4*>(src), src_ld / 8, reinterpret_cast<uint2*>(dst), dst_ld / 8,
                           scale);
  count_launch();
  return e;
}

}  // namespace moe
