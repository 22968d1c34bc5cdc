// Atomic-expert layer (OmniMoE): Cartesian Product Router selection and the
// Dynamic Expert Assembly of atomic experts sigma(x w_in^T) w_out.
//
// Exact top-K over the implicit Nr x Nc grid (OmniMoE App. A), scores
// S(i,j) = fl32(lr_i + lc_j), order (S desc, flat id i*Nc + j asc).
// With rows and columns sorted by (value desc, index asc), write (a, b) for the
// pair of the a-th row and the b-th column. Its (a+1)(b+1) dominators (a' <= a,
// b' <= b) all score at least as much (fp32 rounding is monotone), so
//  * tau, the K-th best score of the grid, is also the K-th best over the
//    staircase set {(a, b) : (a+1)(b+1) <= K} (about K ln K pairs): ordering by
//    (S desc, a asc, b asc) puts every dominator of a pair ahead of it, so the
//    first K pairs of that order lie in the staircase;
//  * every pair scoring ABOVE tau lies in the staircase (fewer than K pairs do);
//  * the pairs equal to tau may lie anywhere: the lowest flat ids among them are
//    found row by row (row i first holds flat ids i*Nc .. i*Nc + Nc - 1), each
//    row's tied columns being one contiguous run of the sorted columns.
#include <float.h>

#include <algorithm>

#include "atomic.cuh"

namespace moe {

namespace {
constexpr unsigned FULL = 0xffffffffu;
constexpr int SEL_THREADS = 1024;
constexpr int SEL_MAX_SIDE = 1024;
constexpr int SEL_MAX_K = 64;
constexpr int WIDE_MAX_K = 4096;  // the wide selection (K > SEL_MAX_K)

__device__ __forceinline__ uint32_t ordered_bits(float v) {
  if (v == 0.f) v = 0.f;  // -0 and +0 are equal scores
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ uint64_t make_key(float v, uint32_t id) {
  return ((uint64_t)ordered_bits(v) << 32) | (uint64_t)(0xFFFFFFFFu - id);
}
__device__ __forceinline__ uint32_t key_id(uint64_t key) { return 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu); }

// Log-sum-exp state (m, s): the values seen are s * e^m in total. Merging two
// states rescales both sums to the larger maximum (fp32 exponentials, fp64 sums).
struct Lse {
  float m;
  double s;
};
__device__ __forceinline__ Lse lse_merge(Lse a, Lse b) {
  const float m = fmaxf(a.m, b.m);
  return {m, a.s * (double)expf(a.m - m) + b.s * (double)expf(b.m - m)};
}
__device__ __forceinline__ Lse lse_shfl_xor(Lse a, int o) {
  return {__shfl_xor_sync(FULL, a.m, o), __shfl_xor_sync(FULL, a.s, o)};
}
}  // namespace

__device__ __forceinline__ float ordered_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// ---- top 64 of a list of distinct 64-bit keys, descending
// A warp holds 64 keys: element `lane` in k0, element `lane + 32` in k1.
__device__ __forceinline__ uint64_t kmax(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t kmin(uint64_t a, uint64_t b) { return a > b ? b : a; }

// Bitonic sort of the warp's 64 keys, descending. For the pair (e, e ^ j) of
// stage k the lower index keeps the larger key when (e & k) == 0.
__device__ __forceinline__ void warp_sort64_desc(uint64_t& k0, uint64_t& k1) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {  // k == 64: elements lane and lane + 32 of one thread
        const uint64_t hi = kmax(k0, k1), lo = kmin(k0, k1);
        k0 = hi;
        k1 = lo;
      } else {
        const bool lower = (lane & j) == 0;
        const bool desc0 = (lane & k) == 0;  // element lane (k <= 64)
        const bool desc1 = k == 64 ? true : (k == 32 ? false : (lane & k) == 0);  // element lane + 32
        const uint64_t o0 = __shfl_xor_sync(FULL, k0, j), o1 = __shfl_xor_sync(FULL, k1, j);
        k0 = (lower == desc0) ? kmax(k0, o0) : kmin(k0, o0);
        k1 = (lower == desc1) ? kmax(k1, o1) : kmin(k1, o1);
      }
    }
  }
}

// Sorts a bitonic 64-key sequence descending (the merge half of the sort).
__device__ __forceinline__ void warp_merge64_desc(uint64_t& k0, uint64_t& k1) {
  const int lane = threadIdx.x & 31;
  const uint64_t hi = kmax(k0, k1), lo = kmin(k0, k1);
  k0 = hi;
  k1 = lo;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const bool lower = (lane & j) == 0;
    const uint64_t o0 = __shfl_xor_sync(FULL, k0, j), o1 = __shfl_xor_sync(FULL, k1, j);
    k0 = lower ? kmax(k0, o0) : kmin(k0, o0);
    k1 = lower ? kmax(k1, o1) : kmin(k1, o1);
  }
}

// Top 64 (descending) of `nchunks` chunks of 64 keys, one chunk per warp
// base_warp .. base_warp + nchunks - 1, each warp's keys already in (k0, k1).
// buf: nchunks x 64 keys of shared memory owned by these warps; on return
// buf[0..63] holds the result. Called by every thread of the block (it syncs),
// with max_chunks >= nchunks the same in every thread.
__device__ void block_top64(uint64_t k0, uint64_t k1, bool mine, int lw, int nchunks, int max_chunks,
                            uint64_t* buf) {
  const int lane = threadIdx.x & 31;
  if (mine) {
    warp_sort64_desc(k0, k1);
    buf[lw * 64 + lane] = k0;
    buf[lw * 64 + lane + 32] = k1;
  }
  for (int stride = 1; stride < max_chunks; stride <<= 1) {  // max_chunks: the same in every thread
    __syncthreads();
    if (mine && (lw % (2 * stride)) == 0 && lw + stride < nchunks) {
      const uint64_t* b = buf + (lw + stride) * 64;  // both lists descending: A[i] vs B[63 - i]
      k0 = kmax(k0, b[63 - lane]);
      k1 = kmax(k1, b[31 - lane]);
      warp_merge64_desc(k0, k1);
      buf[lw * 64 + lane] = k0;
      buf[lw * 64 + lane + 32] = k1;
    }
  }
  __syncthreads();
}

// Row and column log-probabilities of token t into shared lr[Nr], lc[Nc] (and
// lr_out / lc_out when given): the split-K partials summed in split order (up to 16
// loads of each side in flight together), then log-softmax with a block-wide
// log-sum-exp (a fixed shuffle tree per warp, then warp 0 over the warps: the same
// result on every run). One thread per row and per column (blockDim = SEL_THREADS
// >= Nr, Nc); ends with a block barrier.
__device__ void block_logprobs(int t, int Nr, int Nc, int ksplit, const float* __restrict__ zr, long long zr_split,
                               const float* __restrict__ zc, long long zc_split, float* lr, float* lc,
                               float* __restrict__ lr_out, float* __restrict__ lc_out) {
  __shared__ Lse red_r[32], red_c[32];
  __shared__ double lse_s[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool hr = tid < Nr, hc = tid < Nc;
  float ar = 0.f, ac = 0.f;
  for (int s0 = 0; s0 < ksplit; s0 += 16) {
    float vr[16], vc[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int s = s0 + u;
      vr[u] = (s < ksplit && hr) ? zr[s * zr_split + (long long)t * Nr + tid] : 0.f;
      vc[u] = (s < ksplit && hc) ? zc[s * zc_split + (long long)t * Nc + tid] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (s0 + u < ksplit) {
        ar += vr[u];
        ac += vc[u];
      }
    }
  }
  Lse er = {hr ? ar : -FLT_MAX, hr ? 1.0 : 0.0}, ec = {hc ? ac : -FLT_MAX, hc ? 1.0 : 0.0};
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    er = lse_merge(er, lse_shfl_xor(er, o));
    ec = lse_merge(ec, lse_shfl_xor(ec, o));
  }
  if (lane == 0) {
    red_r[warp] = er;
    red_c[warp] = ec;
  }
  __syncthreads();
  if (warp == 0) {
    Lse r = lane < SEL_THREADS / 32 ? red_r[lane] : Lse{-FLT_MAX, 0.0};
    Lse q = lane < SEL_THREADS / 32 ? red_c[lane] : Lse{-FLT_MAX, 0.0};
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      r = lse_merge(r, lse_shfl_xor(r, o));
      q = lse_merge(q, lse_shfl_xor(q, o));
    }
    if (lane == 0) lse_s[0] = (double)r.m + log(r.s);
    if (lane == 1) lse_s[1] = (double)q.m + log(q.s);
  }
  __syncthreads();
  if (hr) {
    lr[tid] = (float)((double)ar - lse_s[0]);
    if (lr_out) lr_out[(long long)t * Nr + tid] = lr[tid];
  }
  if (hc) {
    lc[tid] = (float)((double)ac - lse_s[1]);
    if (lc_out) lc_out[(long long)t * Nc + tid] = lc[tid];
  }
  __syncthreads();
}

// One block (1024 threads) per token. zr/zc: split-K partial logits [ksplit][T][Nr|Nc].
//  1. log-softmax of the row and column logits (fp32 values; log-sum-exp with
//     fp64 sums);
//  2. the top 64 rows and the top 64 columns by (value desc, index asc): warps
//     0-15 hold the rows, 16-31 the columns, 64 per warp; warp sorts, then a
//     merge tree;
//  3. the staircase pairs (a, b), (a+1)(b+1) <= K, keyed by (score, flat id); their
//     top 64 give tau (the K-th score) and, in final order, the pairs above tau;
//  4. the lowest flat ids scoring exactly tau: when three counts show that every
//     pair scoring >= tau is a staircase pair (the usual case), the first K sorted
//     candidates; otherwise the rows that can reach tau, in index order, one warp
//     per row scanning its columns (tied ids come out in ascending order), 32 rows
//     per wave, until `need` are found;
//  5. g = softmax of the K scores (one warp).
__global__ void __launch_bounds__(SEL_THREADS, 1)
    atomic_select_kernel(int T, int Nr, int Nc, int K, int ksplit, const float* __restrict__ zr, long long zr_split,
                         const float* __restrict__ zc, long long zc_split, float* __restrict__ lr_out,
                         float* __restrict__ lc_out, int32_t* __restrict__ idx_out, float* __restrict__ g_out,
                         int* status, unsigned* bar_reset) {
  __shared__ float lr[SEL_MAX_SIDE], lc[SEL_MAX_SIDE];
  // the next kernel's grid barrier counts from zero: it passes griddepcontrol.wait
  // only after this grid has completed, so clearing the word here is enough
  if (bar_reset && blockIdx.x == 0 && threadIdx.x == 0) *bar_reset = 0u;
  __shared__ uint64_t buf[2][16 * 64];  // merge buffers: rows, columns (candidates reuse rows')
  __shared__ int stair_off[SEL_MAX_K], top_rows[SEL_MAX_K];
  __shared__ uint32_t win_ids[SEL_MAX_K];
  __shared__ int row_list[SEL_MAX_SIDE];
  __shared__ int warp_cnt[32];
  __shared__ int n_cand, n_rows, found_s;
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();

  // 1. log-softmax of rows and columns (from the split-K partials)
  block_logprobs(t, Nr, Nc, ksplit, zr, zr_split, zc, zc_split, lr, lc, lr_out, lc_out);
  if (warp == 1) {  // staircase row offsets (K <= 64 rows: two per lane)
    const int kr = min(K, Nr), kc = min(K, Nc);
    const int c0 = lane < kr ? min(K / (lane + 1), kc) : 0;
    const int c1 = lane + 32 < kr ? min(K / (lane + 33), kc) : 0;
    int s0 = c0;  // rows 0 .. 31, then rows 32 .. 63
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, s0, o);
      if (lane >= o) s0 += u;
    }
    const int tot0 = __shfl_sync(FULL, s0, 31);  // rows 0 .. 31
    int s1 = c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(FULL, s1, o);
      if (lane >= o) s1 += u;
    }
    stair_off[lane] = s0 - c0;
    stair_off[lane + 32] = tot0 + s1 - c1;
    if (lane == 31) n_cand = tot0 + s1;
  }
  if (tid == 64) {
    n_rows = 0;
    found_s = 0;
  }
  __syncthreads();
  // 2. top 64 rows and columns
  {
    const int side = warp >> 4, lw = warp & 15;
    const int n = side ? Nc : Nr;
    const float* l = side ? lc : lr;
    const int e0 = lw * 64 + lane, e1 = e0 + 32;
    const uint64_t k0 = e0 < n ? make_key(l[e0], (uint32_t)e0) : 0ull;
    const uint64_t k1 = e1 < n ? make_key(l[e1], (uint32_t)e1) : 0ull;
    const int nchunks = (n + 63) / 64, max_chunks = (max(Nr, Nc) + 63) / 64;
    // both sides merge in the same barrier steps: block_top64 syncs the whole block
    block_top64(k0, k1, lw < nchunks, lw, nchunks, max_chunks, buf[side]);
  }
  // 3. staircase candidates and tau: row a of the staircase holds the pairs
  //    (a, 0 .. cnt_a - 1), cnt_a = min(K / (a + 1), kc), at slots off_a .. off_a + cnt_a - 1
  const int kr = min(K, Nr), kc = min(K, Nc);
  const float lc_max = lc[key_id(buf[1][0])];
  {
    const int nc = n_cand, nchunks = (nc + 63) / 64;  // nc <= 280 for K <= 64
    uint64_t kk[2] = {0ull, 0ull};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = warp * 64 + lane + 32 * h;
      if (warp < nchunks && c < nc) {
        int lo = 0, hi = kr - 1;  // last a with off_a <= c
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (stair_off[mid] <= c) lo = mid; else hi = mid - 1;
        }
        const uint32_t ri = key_id(buf[0][lo]), cj = key_id(buf[1][c - stair_off[lo]]);
        kk[h] = make_key(lr[ri] + lc[cj], ri * (uint32_t)Nc + cj);
      }
    }
    if (tid < kr) top_rows[tid] = (int)key_id(buf[0][tid]);
    __syncthreads();  // every read of the rows' list is done: its buffer is reused below
    block_top64(kk[0], kk[1], warp < nchunks, warp, nchunks, nchunks, buf[0]);
  }
  const uint32_t tau_key = (uint32_t)(buf[0][K - 1] >> 32);
  const float tau = ordered_to_float(tau_key);
  int n_above = 0;  // the sorted prefix scoring above tau
  {
    const bool a0 = lane < K && (uint32_t)(buf[0][lane] >> 32) > tau_key;
    const bool a1 = lane + 32 < K && (uint32_t)(buf[0][lane + 32] >> 32) > tau_key;
    n_above = __popc(__ballot_sync(FULL, a0)) + __popc(__ballot_sync(FULL, a1));
    if (warp == 0) {
      if (a0) win_ids[lane] = key_id(buf[0][lane]);
      if (a1) win_ids[lane + 32] = key_id(buf[0][lane + 32]);
    }
  }
  const int need = K - n_above;
  // 4. ties at tau. Every pair scoring >= tau is a staircase pair when (i) at most
  //    kr rows reach tau with the best column, (ii) at most kc columns reach tau
  //    with the best row and (iii) the first pair past each staircase row, (a, cnt_a)
  //    with cnt_a < kc, scores below tau: by (i) and (ii) such a pair has row rank
  //    a < kr and column rank b < kc, and outside the staircase b >= cnt_a, so
  //    (a, cnt_a) dominates it. Then the winners are the first K sorted candidates.
  const float lr_max = lr[top_rows[0]];
  const int reach_r = __syncthreads_count(tid < Nr && lr[tid] + lc_max >= tau);
  const int reach_c = __syncthreads_count(tid < Nc && lr_max + lc[tid] >= tau);
  bool past = false;
  if (tid < kr) {
    const int ca = min(K / (tid + 1), kc);
    past = ca < kc && lr[top_rows[tid]] + lc[key_id(buf[1][ca])] >= tau;
  }
  const int any_past = __syncthreads_or(past);
  const bool fast = reach_r <= kr && reach_c <= kc && !any_past;
  if (fast) {
    if (tid >= n_above && tid < K) win_ids[tid] = key_id(buf[0][tid]);
    __syncthreads();
  } else {  // rows able to reach tau, in index order, scanned for tied pairs
    {
      const bool cand_row = tid < Nr && lr[tid] + lc_max >= tau;
      const unsigned bal = __ballot_sync(FULL, cand_row);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w];
      if (cand_row) row_list[before + __popc(bal & ((1u << lane) - 1u))] = tid;
      if (tid == SEL_THREADS - 1) n_rows = before + __popc(bal);
      __syncthreads();
    }
    const int nrows = n_rows;
    uint32_t* tied = reinterpret_cast<uint32_t*>(buf[1]) + warp * SEL_MAX_K;  // first tied columns of this warp's row
    for (int w0 = 0; w0 < nrows; w0 += SEL_THREADS / 32) {
      if (found_s >= need) break;  // uniform: read after a barrier
      const int ri = w0 + warp;
      const int r = ri < nrows ? row_list[ri] : -1;
      int cnt = 0;
      if (r >= 0) {
        const float lrr = lr[r];
        for (int j0 = 0; j0 < Nc; j0 += 32) {
          const int j = j0 + lane;
          const bool eq = j < Nc && lrr + lc[j] == tau;
          const unsigned bal = __ballot_sync(FULL, eq);
          const int q = cnt + __popc(bal & ((1u << lane) - 1u));
          if (eq && q < SEL_MAX_K) tied[q] = (uint32_t)j;
          cnt += __popc(bal);
        }
      }
      if (lane == 0) warp_cnt[warp] = cnt;
      __syncthreads();
      int before = found_s, wave = 0;
      for (int w = 0; w < SEL_THREADS / 32; ++w) {
        const int c = warp_cnt[w];
        if (w < warp) before += c;
        wave += c;
      }
      if (r >= 0 && cnt > 0 && before < need) {  // this row's lowest tied ids (ascending)
        const int take = min(cnt, need - before);  // <= need <= SEL_MAX_K
        for (int q = lane; q < take; q += 32) win_ids[n_above + before + q] = (uint32_t)r * (uint32_t)Nc + tied[q];
      }
      __syncthreads();
      if (tid == 0) found_s += wave;
      __syncthreads();
    }
    if (found_s < need) {  // cannot happen: tau is the score of a grid pair
      if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
      return;
    }
  }
  // 5. the gate weights (winners are already ordered by (score desc, id asc))
  if (warp == 0) {
    float sc0 = 0.f, sc1 = 0.f;
    uint32_t id0 = 0, id1 = 0;
    if (lane < K) {
      id0 = win_ids[lane];
      sc0 = lr[id0 / Nc] + lc[id0 % Nc];
    }
    if (lane + 32 < K) {
      id1 = win_ids[lane + 32];
      sc1 = lr[id1 / Nc] + lc[id1 % Nc];
    }
    const float smax = __shfl_sync(FULL, sc0, 0);
    const double z0 = lane < K ? (double)expf(sc0 - smax) : 0.0;
    const double z1 = lane + 32 < K ? (double)expf(sc1 - smax) : 0.0;
    double zs = z0 + z1;
#pragma unroll
    for (int o = 16; o; o >>= 1) zs += __shfl_xor_sync(FULL, zs, o);
    if (lane < K) {
      idx_out[(long long)t * K + lane] = (int32_t)id0;
      g_out[(long long)t * K + lane] = (float)(z0 / zs);
    }
    if (lane + 32 < K) {
      idx_out[(long long)t * K + lane + 32] = (int32_t)id1;
      g_out[(long long)t * K + lane + 32] = (float)(z1 / zs);
    }
  }
}

// Exact top-K for K > 64 (prefill budgets, OmniMoE "Top-K budget K = 512-4096"),
// one block (1024 threads) per token:
//  1. log-softmax of rows and columns (block_logprobs);
//  2. rows and columns sorted by (value desc, index asc) (bitonic, in shared memory);
//  3. tau, the K-th best score, by a radix select over the staircase pairs
//     {(a, b) : (a+1)(b+1) <= K} of sorted row a and sorted column b (about K ln K
//     of them; the file header shows tau and every pair above it lie there), on
//     the scores' order-preserving 32-bit codes: digits of 11, 11 and 10 bits from
//     the top, each pass a histogram (warp-aggregated shared atomics) of the pairs
//     that match the digits fixed so far; it also gives n_gt, the pairs above tau;
//  4. the winners. When the first pair past the staircase in every staircase row,
//     and the best pair of the first row left out, all score below tau (the usual
//     case), no pair outside the staircase reaches tau: the staircase pairs scoring
//     >= tau (above tau, plus every tied pair) are sorted and the first K kept.
//     Otherwise one pass over the whole grid takes the pairs above tau and those
//     scoring exactly tau; when these number more than need = K - n_gt, the grid is
//     walked in flat-id order, 1024 ids per step, a block-wide count ranking the
//     tied pairs, until the need lowest ids are found;
//  5. a bitonic sort of the winners' keys (score desc, flat id asc);
//  6. g = softmax of the K scores (fp32 exponentials, fp64 sum in a fixed tree).
__global__ void __launch_bounds__(SEL_THREADS, 1)
    atomic_select_wide_kernel(int T, int Nr, int Nc, int K, int ksplit, const float* __restrict__ zr,
                              long long zr_split, const float* __restrict__ zc, long long zc_split,
                              float* __restrict__ lr_out, float* __restrict__ lc_out, int32_t* __restrict__ idx_out,
                              float* __restrict__ g_out, int* status, unsigned* bar_reset) {
  __shared__ float lr[SEL_MAX_SIDE], lc[SEL_MAX_SIDE];
  __shared__ uint16_t row_ord[SEL_MAX_SIDE], col_ord[SEL_MAX_SIDE];
  // winners' keys; before them the row / column sort and the radix histograms
  __shared__ uint64_t sel[WIDE_MAX_K];
  __shared__ int warp_cnt[32];
  __shared__ double warp_z[32];
  __shared__ uint32_t digit_s;
  __shared__ int above_s, bin_s, n_sel, n_tie, found_s, stop_s, outside_s;
  if (bar_reset && blockIdx.x == 0 && threadIdx.x == 0) *bar_reset = 0u;  // as atomic_select_kernel
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  block_logprobs(t, Nr, Nc, ksplit, zr, zr_split, zc, zc_split, lr, lc, lr_out, lc_out);

  // 2. sorted rows (sel[0, 1024)) and columns (sel[1024, 2048)); padding keys 0 sink
  sel[tid] = tid < Nr ? make_key(lr[tid], (uint32_t)tid) : 0ull;
  sel[SEL_MAX_SIDE + tid] = tid < Nc ? make_key(lc[tid], (uint32_t)tid) : 0ull;
  __syncthreads();
  for (int k = 2; k <= SEL_MAX_SIDE; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int q = tid; q < 2 * SEL_MAX_SIDE; q += SEL_THREADS) {  // both lists in the same steps
        const int e = q & (SEL_MAX_SIDE - 1), base = q - e, r = e ^ jj;
        if (r > e) {
          const uint64_t va = sel[base + e], vb = sel[base + r];
          if ((e & k) == 0 ? va < vb : va > vb) {
            sel[base + e] = vb;
            sel[base + r] = va;
          }
        }
      }
      __syncthreads();
    }
  }
  if (tid < Nr) row_ord[tid] = (uint16_t)key_id(sel[tid]);
  if (tid < Nc) col_ord[tid] = (uint16_t)key_id(sel[SEL_MAX_SIDE + tid]);
  __syncthreads();

  // 3. radix select of the K-th largest code over the staircase
  uint32_t* hist = reinterpret_cast<uint32_t*>(sel);  // 2048 bins = 8 KB of the 32 KB
  const int kr = min(Nr, K);
  uint32_t prefix = 0, pmask = 0;
  int krem = K, n_gt = 0;
  const int bits[3] = {11, 11, 10};
  int shift = 32;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int nb = 1 << bits[pass];
    shift -= bits[pass];
    for (int b = tid; b < nb; b += SEL_THREADS) hist[b] = 0u;
    __syncthreads();
    for (int a = warp; a < kr; a += SEL_THREADS / 32) {  // one sorted row per warp
      const int cnt = min(Nc, K / (a + 1));
      const float la = lr[row_ord[a]];
      for (int b = lane; b < cnt; b += 32) {
        const uint32_t u = ordered_bits(la + lc[col_ord[b]]);
        if ((u & pmask) == prefix) {
          const uint32_t dg = (u >> shift) & (uint32_t)(nb - 1);
          const unsigned same = __match_any_sync(__activemask(), dg);
          if (lane == __ffs(same) - 1) atomicAdd(&hist[dg], (uint32_t)__popc(same));
        }
      }
    }
    __syncthreads();
    if (warp == 0) {  // the bin holding the krem-th largest: scan bins from the top
      const int per = nb / 32;  // bins per lane, lane 0 holding the highest
      int sum = 0;
      for (int b = 0; b < per; ++b) sum += (int)hist[nb - 1 - (lane * per + b)];
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - sum;  // pairs in the bins above this lane's
      const unsigned hit = __ballot_sync(FULL, excl < krem && incl >= krem);
      if (lane == 0 && !hit) digit_s = 0xFFFFFFFFu;  // (cannot happen: the staircase holds K pairs)
      if (hit && lane == __ffs(hit) - 1) {
        int above = excl;
        for (int b = 0; b < per; ++b) {
          const int bin = nb - 1 - (lane * per + b);
          const int c = (int)hist[bin];
          if (above + c >= krem) {
            digit_s = (uint32_t)bin;
            above_s = above;
            bin_s = c;
            break;
          }
          above += c;
        }
      }
    }
    __syncthreads();
    if (digit_s == 0xFFFFFFFFu) {
      if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
      return;
    }
    prefix |= digit_s << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    krem -= above_s;
    n_gt += above_s;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need = krem;         // >= 1: tau is the code of the K-th pair
  const int n_stair = n_gt + bin_s;  // staircase pairs scoring >= tau
  // 4. the winners
  if (tid == 0) {
    n_sel = 0;
    n_tie = 0;
    found_s = 0;
    stop_s = 0;
    outside_s = 0;
  }
  __syncthreads();
  // can a pair outside the staircase reach tau? (columns and rows are sorted, so
  // each row's first pair past the staircase, and the first row left out, bound them)
  for (int a = tid; a <= kr; a += SEL_THREADS) {
    if (a < kr) {
      const int cnt = min(Nc, K / (a + 1));
      if (cnt < Nc && ordered_bits(lr[row_ord[a]] + lc[col_ord[cnt]]) >= tau) outside_s = 1;
    } else if (kr < Nr && ordered_bits(lr[row_ord[kr]] + lc[col_ord[0]]) >= tau) {
      outside_s = 1;
    }
  }
  __syncthreads();
  int n_win = K;
  if (!outside_s && n_stair <= WIDE_MAX_K) {
    // every pair >= tau is a staircase pair: all of them, sorted below, the first K kept
    for (int a = warp; a < kr; a += SEL_THREADS / 32) {
      const int cnt = min(Nc, K / (a + 1));
      const int ri = row_ord[a];
      const float la = lr[ri];
      for (int b = lane; b < cnt; b += 32) {
        const int cj = col_ord[b];
        const float sc = la + lc[cj];
        if (ordered_bits(sc) >= tau) {
          const unsigned grp = __activemask();
          const int leader = __ffs(grp) - 1;
          int base = 0;
          if (lane == leader) base = atomicAdd(&n_sel, __popc(grp));
          base = __shfl_sync(grp, base, leader);
          const int pos = base + __popc(grp & ((1u << lane) - 1u));
          if (pos < n_stair) sel[pos] = make_key(sc, (uint32_t)(ri * Nc + cj));
        }
      }
    }
    __syncthreads();
    if (n_sel != n_stair) {  // cannot happen: the same codes were counted in the radix passes
      if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
      return;
    }
    n_win = n_stair;
  } else {
    const int N = Nr * Nc;
    const int di = SEL_THREADS / Nc, dj = SEL_THREADS % Nc;  // (i, j) step of a thread's walk
    int i = tid / Nc, j = tid % Nc;
    for (int p = tid; p < N; p += SEL_THREADS) {
      const float sc = lr[i] + lc[j];
      const uint32_t u = ordered_bits(sc);
      if (u >= tau) {
        const unsigned grp = __match_any_sync(__activemask(), u > tau ? 1u : 0u);
        const int leader = __ffs(grp) - 1;
        int base = 0;
        if (lane == leader) base = atomicAdd(u > tau ? &n_sel : &n_tie, __popc(grp));
        base = __shfl_sync(grp, base, leader);
        const int pos = (u > tau ? 0 : n_gt) + base + __popc(grp & ((1u << lane) - 1u));
        if (pos < (u > tau ? n_gt : K)) sel[pos] = make_key(sc, (uint32_t)p);
      }
      i += di;
      j += dj;
      if (j >= Nc) {
        j -= Nc;
        ++i;
      }
    }
    __syncthreads();
    if (n_sel != n_gt || n_tie < need) {  // cannot happen: the counts come from the same codes
      if (tid == 0) set_status(status, MOE_ERR_DEVICE_INDEX);
      return;
    }
    if (n_tie > need) {  // a real tie at the threshold: the lowest flat ids, 1024 ids at a time
      const int N = Nr * Nc;
      for (int p0 = 0; p0 < N; p0 += SEL_THREADS) {
        const int p = p0 + tid;
        const bool eq = p < N && ordered_bits(lr[p / Nc] + lc[p % Nc]) == tau;
        const unsigned bal = __ballot_sync(FULL, eq);
        if (lane == 0) warp_cnt[warp] = __popc(bal);
        __syncthreads();
        int before = found_s;
        for (int w = 0; w < warp; ++w) before += warp_cnt[w];
        const int rank = before + __popc(bal & ((1u << lane) - 1u));
        if (eq && rank < need) sel[n_gt + rank] = make_key(lr[p / Nc] + lc[p % Nc], (uint32_t)p);
        __syncthreads();
        if (tid == 0) {
          int tot = 0;
          for (int w = 0; w < SEL_THREADS / 32; ++w) tot += warp_cnt[w];
          found_s += tot;
          stop_s = found_s >= need;
        }
        __syncthreads();
        if (stop_s) break;
      }
    }
  }
  // 5. bitonic sort, descending, over the next power of two (padding keys are 0)
  int n2 = 1;
  while (n2 < n_win) n2 <<= 1;
  for (int q = n_win + tid; q < n2; q += SEL_THREADS) sel[q] = 0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int q = tid; q < n2; q += SEL_THREADS) {
        const int r = q ^ jj;
        if (r > q) {
          const uint64_t va = sel[q], vb = sel[r];
          if ((q & k) == 0 ? va < vb : va > vb) {
            sel[q] = vb;
            sel[r] = va;
          }
        }
      }
      __syncthreads();
    }
  }
  // 6. gate weights
  const float smax = ordered_to_float((uint32_t)(sel[0] >> 32));
  double z = 0.0;
  for (int q = tid; q < K; q += SEL_THREADS) z += (double)expf(ordered_to_float((uint32_t)(sel[q] >> 32)) - smax);
#pragma unroll
  for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
  if (lane == 0) warp_z[warp] = z;
  __syncthreads();
  if (warp == 0) {
    double zz = warp_z[lane];
#pragma unroll
    for (int o = 16; o; o >>= 1) zz += __shfl_xor_sync(FULL, zz, o);
    if (lane == 0) warp_z[0] = zz;
  }
  __syncthreads();
  const double zs = warp_z[0];
  for (int q = tid; q < K; q += SEL_THREADS) {
    const uint64_t key = sel[q];
    idx_out[(long long)t * K + q] = (int32_t)key_id(key);
    g_out[(long long)t * K + q] = (float)((double)expf(ordered_to_float((uint32_t)(key >> 32)) - smax) / zs);
  }
}

cudaError_t launch_atomic_select(int T, int Nr, int Nc, int K, int ksplit, const float* zr, long long zr_split,
                                 const float* zc, long long zc_split, float* lr_out, float* lc_out, int32_t* idx,
                                 float* g, int* status, unsigned* bar_reset, cudaStream_t s) {
  if (K > WIDE_MAX_K) return cudaErrorInvalidValue;
  if (K > SEL_MAX_K)
    launch_k(atomic_select_wide_kernel, T, SEL_THREADS, 0, s, T, Nr, Nc, K, ksplit, zr, zr_split, zc, zc_split,
             lr_out, lc_out, idx, g, status, bar_reset);
  else
    launch_k(atomic_select_kernel, T, SEL_THREADS, 0, s, T, Nr, Nc, K, ksplit, zr, zr_split, zc, zc_split, lr_out,
             lc_out, idx, g, status, bar_reset);
  count_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ assembly
constexpr int ASM_GROUPS = 16, ASM_BATCH = 4;  // phase 2: slot groups per 8 columns, loads per batch

// The atomic-expert FFN (OmniMoE Eq. 4) in one cooperative launch, one 1024-thread
// block per SM (all of them resident, as the grid barrier needs):
//  phase 1, AX_PARTS warps per task (t, s), each over its quarter of d:
//    coef[t, s] = g[t, s] act(x_t . w_in[idx[t, s]]), fp32 FMAs over each lane's
//    16-byte chunks in ascending order, a shuffle tree per warp, and the parts added
//    in part order; when all gathered w_out rows fit comfortably in L2 (decode
//    budgets) each warp also prefetches its part of the task's w_out row for phase 2;
//  a grid-wide barrier (bounded: on expiry the block records MOE_ERR_TIMEOUT and
//    returns without phase 2, whose coefficients other blocks may not have written);
//  phase 2, sixteen lanes per 8 output columns: lane group j sums slots j, j + 16,
//    ... in order, the groups are added by a fixed xor tree, and out[t, c..c+7] is
//    rounded to bf16, so the result is the same on every run.
// Splitting each dot product over four warps and each output chunk over sixteen
// lanes keeps every SM's 32 warps busy at decode budgets (16 tokens x 64 slots).
constexpr int AX_THREADS = 1024;
constexpr int AX_WARPS = AX_THREADS / 32;
constexpr int AX_PARTS = 4;                   // warps per task in phase 1
constexpr int AX_TPB = AX_WARPS / AX_PARTS;   // tasks per block per round
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// x . w over the 16-byte chunks [c_lo, c_hi) of bf16 by one warp: fp32 FMAs over
// each lane's chunks in ascending order (4 chunks of each operand in flight), then a
// shuffle tree; every lane returns the sum.
__device__ __forceinline__ float warp_dot_bf16(const uint4* __restrict__ xr, const uint4* __restrict__ wr, int c_lo,
                                               int c_hi, int lane) {
  float sacc = 0.f;
  for (int c0 = c_lo + lane; c0 < c_hi; c0 += 32 * 4) {
    uint4 av[4], bv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u;
      if (c < c_hi) {
        av[u] = xr[c];
        bv[u] = wr[c];
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (c0 + 32 * u >= c_hi) break;
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&av[u]);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&bv[u]);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 fa = __bfloat1622float2(pa[h]), fb = __bfloat1622float2(pb[h]);
        sacc = fmaf(fa.x, fb.x, sacc);
        sacc = fmaf(fa.y, fb.y, sacc);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
  return sacc;
}

__device__ __forceinline__ float atomic_act(float z, int act) {
  const float sg = 1.f / (1.f + expf(-z));
  return act == MOE_ATOMIC_SILU ? z * sg : sg;
}

__global__ void __launch_bounds__(AX_THREADS)
    atomic_experts_kernel(int T, int d, int K, int act, const uint4* __restrict__ x, const uint4* __restrict__ w_in,
                          const uint4* __restrict__ w_out, const int32_t* __restrict__ idx,
                          const float* __restrict__ g, float* __restrict__ coef, uint4* __restrict__ out,
                          long long n_experts, int prefetch_out, unsigned* bar, unsigned bar_extra,
                          unsigned long long limit_ns, int* status) {
  __shared__ float part_s[AX_TPB][AX_PARTS];
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const long long gwarp = ((long long)blockIdx.x * AX_THREADS + threadIdx.x) >> 5;
  const long long nwarps = (long long)gridDim.x * AX_WARPS;
  const int chunks = d / 8;
  const long long tasks = (long long)T * K;
  // ---- phase 1: coef[t, s] = g[t, s] act(x_t . w_in[idx[t, s]]); warp wib takes part
  // wib % AX_PARTS of task slot wib / AX_PARTS (rounds are uniform per block)
  {
    const int tslot = wib / AX_PARTS, part = wib % AX_PARTS;
    const int pc = (chunks + AX_PARTS - 1) / AX_PARTS;
    const int c_lo = min(chunks, part * pc), c_hi = min(chunks, c_lo + pc);
    for (long long base = (long long)blockIdx.x * AX_TPB; base < tasks; base += (long long)gridDim.x * AX_TPB) {
      const long long task = base + tslot;
      float z = 0.f;
      if (task < tasks) {
        const long long e = idx[task];
        if (e >= 0 && e < n_experts) {
          if (prefetch_out) {  // this part's bytes of the task's w_out row, one 128-byte line per lane
            const char* po = reinterpret_cast<const char*>(w_out + e * chunks);
            for (int b = c_lo * 16 + lane * 128; b < c_hi * 16; b += 32 * 128) prefetch_l2(po + b);
          }
          z = warp_dot_bf16(x + (task / K) * chunks, w_in + e * chunks, c_lo, c_hi, lane);
        }
      }
      if (lane == 0) part_s[tslot][part] = z;
      __syncthreads();
      if (threadIdx.x < AX_TPB) {
        const long long tk = base + threadIdx.x;
        if (tk < tasks) {
          const long long e = idx[tk];
          if (e < 0 || e >= n_experts) {
            set_status(status, MOE_ERR_DEVICE_INDEX);
            coef[tk] = 0.f;
          } else {
            float zz = part_s[threadIdx.x][0];
#pragma unroll
            for (int q = 1; q < AX_PARTS; ++q) zz += part_s[threadIdx.x][q];
            coef[tk] = g[tk] * atomic_act(zz, act);
          }
        }
      }
      __syncthreads();
    }
  }
  // ---- grid-wide barrier (every block is resident: cooperative launch, one per SM).
  // It waits for gridDim.x + bar_extra arrivals; bar_extra is 0 except under the
  // fault-injection hook, where the wait can only end at its time limit.
  __shared__ int bar_failed;
  __syncthreads();
  if (threadIdx.x == 0) {
    bar_failed = 0;
    __threadfence();
    atomicAdd(bar, 1u);
    const unsigned target = gridDim.x + bar_extra;
    const unsigned long long t0 = globaltimer_ns();
    while (*reinterpret_cast<volatile unsigned*>(bar) < target) {
      if (globaltimer_ns() - t0 > limit_ns) {
        set_status(status, MOE_ERR_TIMEOUT);
        bar_failed = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  if (bar_failed) return;
  // ---- phase 2: out[t, c..c+7] = sum_s coef[t, s] w_out[idx[t, s], c..c+7]; a warp
  // covers two output chunks, sixteen lanes (slot groups) each
  const long long unitsG = (long long)T * chunks * ASM_GROUPS;
  for (long long qb = gwarp * 32; qb < unitsG; qb += nwarps * 32) {  // warp-aligned: shuffles see all lanes
    const long long q = qb + lane;
    const bool valid = q < unitsG;
    const int grp = (int)(q & (ASM_GROUPS - 1));
    const long long unit = q / ASM_GROUPS;
    const long long t = unit / chunks;
    const int c = (int)(unit - t * chunks);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (valid) {
      for (int s0 = grp; s0 < K; s0 += ASM_GROUPS * ASM_BATCH) {
        uint4 v[ASM_BATCH];
        float cf[ASM_BATCH];
#pragma unroll
        for (int u = 0; u < ASM_BATCH; ++u) {
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
        for (int u = 0; u < ASM_BATCH; ++u) {
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
    for (int o = 1; o < ASM_GROUPS; o <<= 1)  // the sixteen groups by a fixed xor tree (a + b = b + a)
#pragma unroll
      for (int h = 0; h < 8; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
    if (valid && grp == 0) {
      uint4 o;
      __nv_bfloat162* po2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int h = 0; h < 4; ++h) po2[h] = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
      out[t * chunks + c] = o;
    }
  }
}

// Prefill budgets (many tasks): the two phases as separate, fully occupied kernels.
// Coefficients: one warp per task, as phase 1 above, with the tasks taken in
// expert order (OmniMoE's expert-centric scheduling: a counting sort of the tasks
// by expert), so each w_in row is read from HBM once and its other tasks hit L2
// while the token rows (T x d) stay in L2 too.
constexpr int AW_THREADS = 256;
constexpr long long AW_MIN_TASKS = ATOMIC_WIDE_MIN_TASKS;  // below this the single cooperative launch wins

// counts[e] = tasks of expert e (counts zeroed by the caller); a task whose expert
// index is out of range is counted nowhere and flagged
__global__ void __launch_bounds__(AW_THREADS)
    atomic_count_kernel(long long tasks, const int32_t* __restrict__ idx, int32_t* __restrict__ counts,
                        long long n_experts, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long q = (long long)blockIdx.x * AW_THREADS + threadIdx.x; q < tasks; q += (long long)gridDim.x * AW_THREADS) {
    const long long e = idx[q];
    if (e >= 0 && e < n_experts) atomicAdd(&counts[e], 1);
    else set_status(status, MOE_ERR_DEVICE_INDEX);
  }
}

// counts -> exclusive prefix sums in place (one block): thread i scans a contiguous
// run of counters (a multiple of 4, read and written as int4: the array is 16-byte
// aligned), the runs' totals are scanned across the block.
__global__ void __launch_bounds__(1024) atomic_scan_kernel(long long n, int32_t* __restrict__ counts) {
  __shared__ int warp_tot[32];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long per = (((n + 1023) / 1024) + 3) & ~3LL;
  const long long lo = min(n, (long long)tid * per), hi = min(n, lo + per);
  const long long hi4 = lo + ((hi - lo) & ~3LL);  // end of the whole int4s of the run
  int sum = 0;
#pragma unroll 8
  for (long long i = lo; i < hi4; i += 4) {
    const int4 v = *reinterpret_cast<const int4*>(counts + i);
    sum += (v.x + v.y) + (v.z + v.w);
  }
  for (long long i = hi4; i < hi; ++i) sum += counts[i];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(FULL, w, o);
      if (lane >= o) w += v;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - sum + (warp ? warp_tot[warp - 1] : 0);
#pragma unroll 8
  for (long long i = lo; i < hi4; i += 4) {
    int4 v = *reinterpret_cast<const int4*>(counts + i);
    const int4 c = v;
    v.x = run;
    v.y = run + c.x;
    v.z = v.y + c.y;
    v.w = v.z + c.z;
    run = v.w + c.w;
    *reinterpret_cast<int4*>(counts + i) = v;
  }
  for (long long i = hi4; i < hi; ++i) {
    const int c = counts[i];
    counts[i] = run;
    run += c;
  }
}

// order[cursor[e]++] = task: afterwards cursor[e] is the end of expert e's run (the
// order inside a run is arbitrary; every coefficient is computed on its own)
__global__ void __launch_bounds__(AW_THREADS)
    atomic_scatter_kernel(long long tasks, const int32_t* __restrict__ idx, int32_t* __restrict__ cursor,
                          int32_t* __restrict__ order, long long n_experts) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long q = (long long)blockIdx.x * AW_THREADS + threadIdx.x; q < tasks; q += (long long)gridDim.x * AW_THREADS) {
    const long long e = idx[q];
    if (e >= 0 && e < n_experts) {
      const int pos = atomicAdd(&cursor[e], 1);
      if (pos >= 0 && pos < tasks) order[pos] = (int32_t)q;
    }
  }
}

__global__ void __launch_bounds__(AW_THREADS)
    atomic_coef_kernel(int T, int d, int K, int act, const uint4* __restrict__ x, const uint4* __restrict__ w_in,
                       const int32_t* __restrict__ idx, const float* __restrict__ g, float* __restrict__ coef,
                       const int32_t* __restrict__ order, const int32_t* __restrict__ n_ordered, long long n_experts,
                       int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long gwarp = ((long long)blockIdx.x * AW_THREADS + threadIdx.x) >> 5;
  const long long nwarps = (long long)gridDim.x * (AW_THREADS / 32);
  const int chunks = d / 8;
  const long long tasks = (long long)T * K;
  if (order) {  // expert order: valid tasks only (a task with a bad index never entered it)
    const long long n_valid = min((long long)*n_ordered, tasks);  // end of the last expert's run
    for (long long pos = gwarp; pos < n_valid; pos += nwarps) {
      const long long task = order[pos];
      if (task < 0 || task >= tasks) continue;
      const long long e = idx[task];
      const float z = warp_dot_bf16(x + (task / K) * chunks, w_in + e * chunks, 0, chunks, lane);
      if (lane == 0) coef[task] = g[task] * atomic_act(z, act);
    }
    return;
  }
  for (long long task = gwarp; task < tasks; task += nwarps) {
    const long long e = idx[task];
    if (e < 0 || e >= n_experts) {
      if (lane == 0) {
        set_status(status, MOE_ERR_DEVICE_INDEX);
        coef[task] = 0.f;
      }
      continue;
    }
    const float z = warp_dot_bf16(x + (task / K) * chunks, w_in + e * chunks, 0, chunks, lane);
    if (lane == 0) coef[task] = g[task] * atomic_act(z, act);
  }
}

// Assembly: out[t, cols] = sum over s (ascending) of coef[t, s] w_out[idx[t, s], cols].
// A half-warp owns one token and 128 columns (8 per lane, one 16-byte load per
// slot); units run column block by column block over all tokens, so the slice of
// W_out being gathered (N rows x 256 B) stays in L2 while every token reads it.
__global__ void __launch_bounds__(AW_THREADS)
    atomic_assemble_kernel(int T, int d, int K, const uint4* __restrict__ w_out, const int32_t* __restrict__ idx,
                           const float* __restrict__ coef, uint4* __restrict__ out, long long n_experts) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, hl = lane & 15;
  const long long gwarp = ((long long)blockIdx.x * AW_THREADS + threadIdx.x) >> 5;
  const long long nwarps = (long long)gridDim.x * (AW_THREADS / 32);
  const int chunks = d / 8;
  const int blocks = (chunks + 15) / 16;
  const long long pairs = ((long long)T + 1) / 2;
  const long long units = (long long)blocks * pairs;
  for (long long u = gwarp; u < units; u += nwarps) {
    const int cb = (int)(u / pairs);
    const long long t = (u - (long long)cb * pairs) * 2 + (lane >> 4);
    const int c = cb * 16 + hl;
    if (t >= T || c >= chunks) continue;
    const int32_t* ir = idx + t * K;
    const float* cr = coef + t * K;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < K; s0 += 8) {
      uint4 v[8];
      float cf[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int sl = s0 + q;
        cf[q] = 0.f;
        if (sl < K) {
          const long long e = ir[sl];
          if (e >= 0 && e < n_experts) {  // (phase 1 flagged any bad index)
            cf[q] = cr[sl];
            v[q] = w_out[e * chunks + c];
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (cf[q] == 0.f) continue;
        const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v[q]);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float2 f = __bfloat1622float2(pv[h]);
          acc[2 * h] = fmaf(cf[q], f.x, acc[2 * h]);
          acc[2 * h + 1] = fmaf(cf[q], f.y, acc[2 * h + 1]);
        }
      }
    }
    uint4 o;
    __nv_bfloat162* po2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int h = 0; h < 4; ++h) po2[h] = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
    out[t * chunks + c] = o;
  }
}

static unsigned g_barrier_extra = 0;
void set_grid_barrier_extra(unsigned n) { g_barrier_extra = n; }

cudaError_t launch_atomic_experts(int T, int d, int K, int act, const void* x, const void* w_in, const void* w_out,
                                  const int32_t* idx, const float* g, float* coef, void* out, long long n_experts,
                                  unsigned* bar, bool bar_zeroed, unsigned long long limit_ns, int* status,
                                  cudaStream_t s) {
  return launch_atomic_experts_sorted(T, d, K, act, x, w_in, w_out, idx, g, coef, out, n_experts, bar, bar_zeroed,
                                      limit_ns, status, nullptr, s);
}

cudaError_t launch_atomic_experts_sorted(int T, int d, int K, int act, const void* x, const void* w_in,
                                         const void* w_out, const int32_t* idx, const float* g, float* coef, void* out,
                                         long long n_experts, unsigned* bar, bool bar_zeroed,
                                         unsigned long long limit_ns, int* status, int32_t* sort_ws, cudaStream_t s) {
  if ((long long)T * K >= AW_MIN_TASKS) {
    const long long tasks = (long long)T * K;
    const long long cap = (long long)num_sms() * 8;  // 8 blocks of 8 warps per SM
    const int gc = (int)std::min<long long>(cap, (tasks + AW_THREADS / 32 - 1) / (AW_THREADS / 32));
    cudaError_t e = cudaSuccess;
    const int32_t* order = nullptr;
    const int32_t* n_ordered = nullptr;
    if (sort_ws) {  // counting sort of the tasks by expert
      int32_t* cursor = sort_ws;
      int32_t* ord = sort_ws + n_experts;
      // tasks with a bad index are left out of the order: zero their coefficients first
      if ((e = cudaMemsetAsync(coef, 0, (size_t)tasks * sizeof(float), s)) != cudaSuccess) return e;
      if ((e = cudaMemsetAsync(cursor, 0, (size_t)n_experts * sizeof(int32_t), s)) != cudaSuccess) return e;
      const int gs = (int)std::min<long long>((long long)num_sms() * 8, (tasks + AW_THREADS - 1) / AW_THREADS);
      e = launch_k(atomic_count_kernel, gs, AW_THREADS, 0, s, tasks, idx, cursor, n_experts, status);
      count_launch();
      if (e != cudaSuccess) return e;
      e = launch_k(atomic_scan_kernel, 1, 1024, 0, s, n_experts, cursor);
      count_launch();
      if (e != cudaSuccess) return e;
      e = launch_k(atomic_scatter_kernel, gs, AW_THREADS, 0, s, tasks, idx, cursor, ord, n_experts);
      count_launch();
      if (e != cudaSuccess) return e;
      order = ord;
      n_ordered = cursor + (n_experts - 1);  // after the scatter: the end of the last run
    }
    e = launch_k(atomic_coef_kernel, gc, AW_THREADS, 0, s, T, d, K, act, (const uint4*)x, (const uint4*)w_in, idx,
                 g, coef, order, n_ordered, n_experts, status);
    count_launch();
    if (e != cudaSuccess) return e;
    const long long units = (long long)((d / 8 + 15) / 16) * (((long long)T + 1) / 2);
    const int ga = (int)std::min<long long>(cap, (units + AW_THREADS / 32 - 1) / (AW_THREADS / 32));
    e = launch_k(atomic_assemble_kernel, ga, AW_THREADS, 0, s, T, d, K, (const uint4*)w_out, idx, coef, (uint4*)out,
                 n_experts);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (!bar_zeroed) {
    cudaError_t e = cudaMemsetAsync(bar, 0, sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());  // one block per SM: all resident, as the grid barrier needs
  cfg.blockDim = dim3(AX_THREADS);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // rows gathered for phase 2 prefetched in phase 1 only while they stay well inside L2
  const int prefetch_out = (double)T * K * d * 2 <= 32.0 * (1 << 20) ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, atomic_experts_kernel, T, d, K, act, (const uint4*)x, (const uint4*)w_in,
                                     (const uint4*)w_out, idx, g, coef, (uint4*)out, n_experts, prefetch_out, bar,
                                     g_barrier_extra, limit_ns, status);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
