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
constexpr int FL_GATE_MAXQ = 32;    // 16-byte chunks of a gate row per lane held at once (d <= 8192)
constexpr int FL_DOWN_THREADS = 128;  // 8 output columns per thread
constexpr int FL_SPLITS = 16;       // kept-channel ranges per expert in the down kernel (partial outputs)
constexpr int FL_RANGE_MAX = 64 * FL_CHUNK / FL_SPLITS;  // channels in one range (f <= 64 FL_CHUNK)
constexpr int FL_DOWN_BATCH = 8;    // kept channels whose rows are loaded together
constexpr int FL_DOWN_ROWS = 4;     // segment rows per pass of the down kernel
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

// ------------------------------------------------------------------ gate
// Block (expert e, chunk c, part; parts fill one wave), one warp per kept channel j: the whole gate row
// W_gate[e][j] is loaded into registers at once (one HBM round trip), then dotted
// with each segment row's x (L1-resident), h[r][j] = g sigma(g) u[r][j] when
// |u[r][j]| >= t_e, else 0, stored at column c FL_CHUNK + i (i = the channel's
// place in the chunk's list).
template <int Q>  // 16-byte chunks of the gate row per lane: d <= 256 Q
__global__ void __launch_bounds__(256)
    floe_gate_kernel(int m, int d, int f, int nchunks, const int32_t* __restrict__ offsets,
                     const uint4* __restrict__ x_perm, const uint4* __restrict__ w_gate, const float* __restrict__ u,
                     const float* __restrict__ thr, const int32_t* __restrict__ list, const int32_t* __restrict__ cnt,
                     float* __restrict__ hc) {
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.x, c = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.z * (blockDim.x >> 5) + (threadIdx.x >> 5), nw = gridDim.z * (blockDim.x >> 5);
  const int r0 = offsets[e], r1 = offsets[e + 1];
  const float t = thr[e];
  const int n = cnt[e * nchunks + c];
  const int32_t* lst = list + ((long long)e * nchunks + c) * FL_CHUNK;
  const int chunks16 = d / 8;
  int jn = gw < n ? lst[gw] : 0;  // the next channel's id, loaded a step ahead
  for (int i = gw; i < n; i += nw) {
    const int j = jn;
    if (i + nw < n) jn = lst[i + nw];
    const uint4* wr = w_gate + ((long long)e * f + j) * chunks16;
    uint4 a[Q];
#pragma unroll
    for (int v = 0; v < Q; ++v)
      if (lane + 32 * v < chunks16) a[v] = wr[lane + 32 * v];
    for (int r = r0; r < r1; ++r) {
      const uint4* xr = x_perm + (long long)r * chunks16;
      const float uv = lane == 0 ? u[(long long)r * f + j] : 0.f;  // issued before the dot product
      float acc = 0.f;
#pragma unroll
      for (int v = 0; v < Q; ++v) {
        if (lane + 32 * v >= chunks16) break;
        const uint4 b = xr[lane + 32 * v];
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[v]);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const float2 fa = __bfloat1622float2(pa[hh]), fb = __bfloat1622float2(pb[hh]);
          acc = fmaf(fa.x, fb.x, acc);
          acc = fmaf(fa.y, fb.y, acc);
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
      if (lane == 0)
        hc[(long long)r * f + (long long)c * FL_CHUNK + i] = fabsf(uv) >= t ? acc / (1.f + expf(-acc)) * uv : 0.f;
    }
  }
}

// ------------------------------------------------------------------ down
// Block (expert e, kept-channel range sp, column slice): the partial
// y[sp][r][cols] = w_r sum over the range's kept channels of h[r][j] W_down_t[e][j][cols],
// 8 columns per thread (16-byte loads), 8 channels in flight, 4 segment rows at a time. The combine adds the FL_SPLITS partials in range order (as split-K).
__global__ void __launch_bounds__(FL_DOWN_THREADS)
    floe_down_kernel(int m, int d, int f, int nchunks, const int32_t* __restrict__ offsets,
                     const uint4* __restrict__ w_dt, const float* __restrict__ hc,
                     const int32_t* __restrict__ list, const int32_t* __restrict__ cnt,
                     const float* __restrict__ row_w, float* __restrict__ y, long long y_split,
                     int32_t* __restrict__ kept_out) {
  __shared__ int coff[64 + 1];  // kept channels before each chunk (f <= 64 FL_CHUNK)
  __shared__ int rj[FL_RANGE_MAX], rcol[FL_RANGE_MAX];  // the range's channel ids and compact h columns
  pdl_launch_dependents();
  pdl_wait();
  const int e = blockIdx.x, sp = blockIdx.y;
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int c = 0; c < nchunks; ++c) {
      coff[c] = tot;
      tot += cnt[e * nchunks + c];
    }
    coff[nchunks] = tot;
    if (kept_out && sp == 0 && blockIdx.z == 0) kept_out[e] = tot;
  }
  __syncthreads();
  const int total = coff[nchunks];
  const int g0 = (int)((long long)total * sp / FL_SPLITS), g1 = (int)((long long)total * (sp + 1) / FL_SPLITS);
  for (int gg = g0 + threadIdx.x; gg < g1; gg += blockDim.x) {  // g1 - g0 <= FL_RANGE_MAX
    int c = 0;
    while (coff[c + 1] <= gg) ++c;
    const int i = gg - coff[c];
    rj[gg - g0] = list[((long long)e * nchunks + c) * FL_CHUNK + i];
    rcol[gg - g0] = c * FL_CHUNK + i;
  }
  __syncthreads();
  const int col8 = blockIdx.z * FL_DOWN_THREADS + threadIdx.x;  // 8-column group
  const int d8 = d / 8;
  const bool cv = col8 < d8;
  const int r0 = offsets[e], r1 = offsets[e + 1];
  float* ys = y + (long long)sp * y_split;
  for (int rb = r0; rb < r1; rb += FL_DOWN_ROWS) {
    const int nr = min(FL_DOWN_ROWS, r1 - rb);
    float acc[FL_DOWN_ROWS][8];
#pragma unroll
    for (int q = 0; q < FL_DOWN_ROWS; ++q)
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[q][v] = 0.f;
    for (int g = 0; g < g1 - g0; g += FL_DOWN_BATCH) {
      uint4 wv[FL_DOWN_BATCH];
      int col[FL_DOWN_BATCH];  // compact h column of each channel
#pragma unroll
      for (int v = 0; v < FL_DOWN_BATCH; ++v) {
        col[v] = -1;
        if (g + v < g1 - g0) {
          col[v] = rcol[g + v];
          if (cv) wv[v] = w_dt[((long long)e * f + rj[g + v]) * d8 + col8];
        }
      }
#pragma unroll
      for (int v = 0; v < FL_DOWN_BATCH; ++v) {
        if (col[v] < 0 || !cv) continue;
        const __nv_bfloat162* pw = reinterpret_cast<const __nv_bfloat162*>(&wv[v]);
        float2 wf[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) wf[hh] = __bfloat1622float2(pw[hh]);
#pragma unroll
        for (int q = 0; q < FL_DOWN_ROWS; ++q) {
          if (q >= nr) break;
          const float h = hc[(long long)(rb + q) * f + col[v]];
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            acc[q][2 * hh] = fmaf(h, wf[hh].x, acc[q][2 * hh]);
            acc[q][2 * hh + 1] = fmaf(h, wf[hh].y, acc[q][2 * hh + 1]);
          }
        }
      }
    }
    if (cv)
#pragma unroll
      for (int q = 0; q < FL_DOWN_ROWS; ++q) {
        if (q >= nr) break;
        const float wr = row_w ? row_w[rb + q] : 1.f;
        float4* o = reinterpret_cast<float4*>(ys + (long long)(rb + q) * d) + 2 * col8;
        o[0] = make_float4(acc[q][0] * wr, acc[q][1] * wr, acc[q][2] * wr, acc[q][3] * wr);
        o[1] = make_float4(acc[q][4] * wr, acc[q][5] * wr, acc[q][6] * wr, acc[q][7] * wr);
      }
  }
}

cudaError_t launch_floe_sparse_ffn(int m, int d, int f, const int32_t* offsets, const void* x_perm,
                                   const void* w_gate, const void* w_down_t, const float* u, const float* thr,
                                   int32_t* list, int32_t* cnt, float* hc, const float* row_w, float* y,
                                   long long y_split, int32_t* kept_out, int* status, cudaStream_t s) {
  const int nchunks = (f + FL_CHUNK - 1) / FL_CHUNK;
  launch_k(floe_keep_kernel, dim3(m, nchunks), FL_KEEP_THREADS, 0, s, m, f, nchunks, offsets, u, thr, list, cnt,
           status);
  count_launch();
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int q = (d / 8 + 31) / 32;
  // blocks per (expert, chunk): as many as fill one wave (two 256-thread blocks per SM)
  const int parts = std::max(1, (2 * num_sms()) / std::max(1, m * nchunks));
  const dim3 gg(m, nchunks, parts);
#define MOE_FLOE_GATE(Q_)                                                                                          \
  launch_k(floe_gate_kernel<Q_>, gg, 256, 0, s, m, d, f, nchunks, offsets, (const uint4*)x_perm,                  \
           (const uint4*)w_gate, u, thr, (const int32_t*)list, (const int32_t*)cnt, hc)
  if (q <= 1)
    MOE_FLOE_GATE(1);
  else if (q <= 4)
    MOE_FLOE_GATE(4);
  else if (q <= 8)
    MOE_FLOE_GATE(8);
  else if (q <= 16)
    MOE_FLOE_GATE(16);
  else
    MOE_FLOE_GATE(FL_GATE_MAXQ);
#undef MOE_FLOE_GATE
  count_launch();
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  launch_k(floe_down_kernel, dim3(m, FL_SPLITS, (d / 8 + FL_DOWN_THREADS - 1) / FL_DOWN_THREADS), FL_DOWN_THREADS, 0,
           s, m, d, f, nchunks, offsets, (const uint4*)w_down_t, (const float*)hc, (const int32_t*)list,
           (const int32_t*)cnt, row_w, y, y_split, kept_out);
  count_launch();
  return cudaGetLastError();
}

int floe_splits() { return FL_SPLITS; }
bool floe_shape_ok(int d, int f) { return d <= 32 * 8 * FL_GATE_MAXQ && f <= 64 * FL_CHUNK; }

int floe_chunks(int f) { return (f + FL_CHUNK - 1) / FL_CHUNK; }
int floe_chunk_size() { return FL_CHUNK; }

}  // namespace moe
