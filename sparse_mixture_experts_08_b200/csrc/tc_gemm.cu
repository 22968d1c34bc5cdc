// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Expert-centric scheduling (OmniMoE, "What carries the argument" and Fig. 3):
// once the (token, expert) tasks sit in one contiguous segment per expert, every
// expert's work is a dense GEMM over its segment, and all experts run in ONE
// persistent launch. The segment boundaries live only in device memory (the
// offsets written by the histogram kernel), so the tile schedule is built on the
// device: each CTA reads the per-group row counts, forms the tile prefix sum in
// shared memory and walks tiles blockIdx.x, blockIdx.x + gridDim.x, ...
//
// Orientation ("swap-AB"): the weight matrix is the MMA's A operand (M = 128
// output features per tile) and the segment's activation rows are the B operand
// (N = BN rows, 16..256), so short segments (decode: a few tokens per expert;
// Switch: ~64) waste no 128-row M tile. The MMA's N is chosen per tile as the
// segment rows left, rounded up to 16. Both operands are K-major (nn.Linear
// weights [out, in] and row-major activations), staged by TMA with the 128-byte
// swizzle. One tile = the full K loop (or one of `ksplit` K ranges).
//
// 8-bit variant (F8): both operands are E4M3 codes with one fp32 scale per row
// (weight output channel, activation row); the MMA is kind::f8f6f4 and the
// epilogue multiplies each accumulator by its two scales. A 128-byte swizzle row
// then holds 128 elements, so stages, boxes and descriptors keep their byte sizes
// and only the K elements per k-block double.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM
// owner), warps 2..5 = epilogue (TMEM -> registers -> activation -> global); pair
// SwiGLU tiles use 320 threads, warps 2..9 = epilogue, two per TMEM lane quarter.
// The accumulator is double-buffered in TMEM when it fits (2 x mats x BN <= 512
// columns) so the epilogue of tile i overlaps the MMAs of tile i + 1.
//
// Every wait on an mbarrier is bounded in time (globaltimer); on expiry the kernel
// records MOE_ERR_TIMEOUT in the status word, the other roles stop, outstanding
// TMA copies and MMAs are drained (again with a bound) and TMEM is freed.
//
// Pair variant (PAIR, large segments): a cluster of two CTAs on two SMs runs one
// tcgen05.mma.cta_group::2 per K step with M = 256 weight rows, 128 in each CTA's
// shared memory, and N = up to 256 token rows, half of them in each CTA; each CTA's
// TMEM holds its own 128 features x N tokens, so the epilogue stays local. Per SM
// the MMA then reads half the operand bytes from shared memory that a one-SM tile
// of the same N reads, which is what bounds the one-SM kernel on the prefill
// shapes. The leader CTA (rank 0) issues the MMAs; both CTAs' TMA copies complete
// on the leader's stage barrier; the leader's commits arrive on both CTAs' barriers;
// both CTAs' epilogues release the accumulator on the leader's barrier. Both CTAs
// meet at a cluster barrier before TMEM is freed and the CTAs exit.
#include <algorithm>
#include <cstring>
#include <cstdio>

#include "common.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;  // bf16 elements of one 128-byte swizzle row
constexpr int TC_BK8 = 128;  // E4M3 elements of one 128-byte swizzle row
// Epilogue warps of a kernel instance. Pair SwiGLU tiles and pair down tiles with two
// feature blocks hold one accumulator (2 x 256 TMEM columns), so the MMAs of the next
// tile wait for the epilogue: SwiGLU gives each TMEM lane quarter three warps that
// share its chunks (12 warps), the down tiles two warps that take one feature block
// each (8). The router uses 8, the rest 4.
template <int EPI, bool PAIR, bool F8, int MATS>
constexpr int tc_epi_warps() {
  return (PAIR && EPI == EPI_SWIGLU && !F8) ? 12 : (PAIR && EPI == EPI_DOWN && MATS == 2) || EPI == EPI_ROUTE ? 8 : 4;
}
template <int EPI, bool PAIR, bool F8, int MATS>
constexpr int tc_threads() { return 64 + 32 * tc_epi_warps<EPI, PAIR, F8, MATS>(); }
constexpr int TC_MAX_GROUPS = 1040;
constexpr int TC_SMEM_BUDGET = 200 * 1024;
constexpr unsigned long long TC_DRAIN_LIMIT_NS = 200ull * 1000 * 1000;

int tc_max_groups() { return TC_MAX_GROUPS; }

template <int BN, int MATS, bool PAIR = false>
struct TcShape {
  static constexpr int TILE_M = PAIR ? 2 * TC_BM : TC_BM;  // weight rows per tile (both CTAs)
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;        // token rows per CTA
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;    // 16 KB
  static constexpr int B_BYTES = B_ROWS * TC_BK * 2;   // B_ROWS * 128 B
  static constexpr int STAGE_BYTES = MATS * A_BYTES + B_BYTES;
  static constexpr int STAGES_RAW = TC_SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = MATS * BN;
  static constexpr int NUM_ACC = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int TMEM_NEED = NUM_ACC * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int DYN_SMEM = STAGES * STAGE_BYTES + 1024;  // + alignment slack
  static_assert(STAGES >= 2, "pipeline needs at least two stages");
  static_assert(TMEM_NEED <= 512, "accumulators exceed TMEM");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N range");
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- two-CTA (cluster pair) forms
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `addr` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Every thread of both CTAs arrives, then waits (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on an
// mbarrier that may sit in the peer CTA of the pair (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster, void* dst, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// Relaxed arrivals: they order no memory operation of the arriving thread, so they do
// not wait for its global stores to be performed. Used where the waiter only reuses
// TMEM whose reads (tcgen05.wait::ld) the arriving warp has already completed.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t* bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// SiLU(g) * u for the gated epilogue with one special-function op per element (e^-g):
// 1 / (1 + e^-g) comes from an integer seed (relative error at most 5.1% over any
// binade; the constant minimises that maximum) and two Newton steps r += r (1 - d r)
// on the FMA pipe (relative error below 7e-6, far under the bf16 rounding of h). The
// exponent is clamped at 44 so that d stays below 2^64 and the seed stays normal;
// for g < -44 the sigmoid below e^-44 is then taken as e^-44.
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float d = 1.f + __expf(fminf(-g, 44.f));
  float r = __int_as_float(0x7EF311C2 - __float_as_int(d));
  r = fmaf(r, fmaf(-d, r, 1.f), r);
  r = fmaf(r, fmaf(-d, r, 1.f), r);
  return g * r * u;
}

template <bool PAIR>
__device__ __forceinline__ void tmem_alloc_g(uint32_t* dst, uint32_t ncols) {
  if (PAIR)
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tmem_relinquish_g() {
  if (PAIR)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
template <bool PAIR>
__device__ __forceinline__ void tmem_dealloc_g(uint32_t taddr, uint32_t ncols) {
  if (PAIR)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T over the pair: M = 256 (128 rows of A in each CTA), N token rows
// (N / 2 in each CTA), kind::f16 (bf16 operands, fp32 accumulator)
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the mbarrier at shared::cluster address `bar_cluster` (this CTA's or the
// peer's) once every pair MMA this thread issued so far completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, kind::f16 (bf16 operands, fp32 accumulator)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A * B^T, kind::f8f6f4 with both operands E4M3 (fp32 accumulator)
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Waits for this thread's TMEM loads, naming the registers they fill as read-write
// operands: the compiler then reads them only after the wait, even when other loads
// were issued in between (the epilogue keeps the next chunk's load in flight).
__device__ __forceinline__ void tmem_ld_wait_keep(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait_keep(uint32_t (&r)[16], uint32_t (&u)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]),
                 "+r"(u[7]), "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]), "+r"(u[12]), "+r"(u[13]),
                 "+r"(u[14]), "+r"(u[15])
               :
               : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 B, 8-row core groups 1024 B apart (SBO), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)(16 >> 4) << 16;    // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset
  d |= (uint64_t)1 << 46;            // version
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::f8f6f4: D fp32, A and B E4M3 (format code 0), both K-major.
__device__ __forceinline__ uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Two floats -> bf16 pair (round to nearest even), the first in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Barrier of the two epilogue warps of TMEM lane quarter q (named barriers 2..5),
// reached by both with the warp converged.
__device__ __forceinline__ void quarter_bar(int q) {
  __syncwarp();
  asm volatile("barrier.sync %0, 64;" ::"r"(2 + q) : "memory");
}

// Barrier of the router's eight epilogue warps only (named barrier 1; 0 is
// __syncthreads), in its non-aligned form and after reconverging the warp, so lanes
// that took different branches before it are all counted.
__device__ __forceinline__ void epi_bar() {
  __syncwarp();
  asm volatile("barrier.sync 1, 256;" ::: "memory");
}

// One pass of the router epilogue over a token's m logits (TMEM columns, 32 per
// step): the largest logit strictly after (pv, pe) in the order (logit desc,
// expert asc). Per 32 columns a pairwise max tree gives the largest remaining
// logit and a bitmask of the columns equal to it gives the lowest expert holding
// it (a tree carrying (logit, expert) pairs through conditional swaps cost about
// three times as much). With EXP (the first pass: nothing picked yet, so "after"
// means "not NaN") it also writes the logits (lg, when given) and folds the
// softmax denominator: per 32 columns a pairwise fp32 sum of exp(logit - running
// max), added to an fp64 sum rescaled whenever the running maximum grows; that
// maximum is the pick's (the max tree ignores NaN just as fmaxf does). A pass
// covers the columns [c_lo, c_hi) (multiples of 32); the two threads of a token
// take the lower and the upper half of the experts.
template <bool EXP>
__device__ __forceinline__ void route_pass(uint32_t t_row, int c_lo, int c_hi, int m, const float* rbias, float pv,
                                           int pe, float& bv, int& be, float& mrun, double& z, float* lg) {
  bv = -INFINITY;
  be = -1;
#pragma unroll 1
  for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
    uint32_t r[32];
    tmem_ld_x16(t_row + c0, r);
    if (c0 + 16 < m) {
      tmem_ld_x16(t_row + c0 + 16, r + 16);
    } else {
#pragma unroll
      for (int j = 16; j < 32; ++j) r[j] = 0u;
    }
    float v[32];
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // c0 + 32 <= ROUTE_MAX_M
      const float4 bb = reinterpret_cast<const float4*>(rbias + c0)[u];
      v[4 * u] = bb.x;
      v[4 * u + 1] = bb.y;
      v[4 * u + 2] = bb.z;
      v[4 * u + 3] = bb.w;
    }
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = c0 + j < m ? __uint_as_float(r[j]) + v[j] : -INFINITY;
    if (EXP && lg)
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < m) lg[c0 + j] = v[j];
    float cv[32], mt[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool after = EXP ? v[j] == v[j] : (v[j] < pv || (v[j] == pv && c0 + j > pe));
      cv[j] = after ? v[j] : -INFINITY;
      mt[j] = cv[j];
    }
#pragma unroll
    for (int st = 1; st < 32; st <<= 1)
#pragma unroll
      for (int j = 0; j < 32; j += 2 * st) mt[j] = fmaxf(mt[j], mt[j + st]);
    const float mx = mt[0];
    uint32_t tie = 0u;
#pragma unroll
    for (int j = 0; j < 32; ++j) tie |= (cv[j] == mx ? 1u : 0u) << j;
    if (mx > bv) {  // earlier steps hold lower experts; an all -inf step changes nothing
      bv = mx;
      be = c0 + __ffs(tie) - 1;
    }
    if (EXP) {
      float mxs[32];
      if (mx > mrun) {
        z *= (double)expf(mrun - mx);
        mrun = mx;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) mxs[j] = c0 + j < m ? expf(v[j] - mrun) : 0.f;
#pragma unroll
      for (int st = 1; st < 32; st <<= 1)
#pragma unroll
        for (int j = 0; j < 32; j += 2 * st) mxs[j] += mxs[j + st];
      z += (double)mxs[0];
    }
  }
}

// ------------------------------------------------------------------ tile schedule
struct TileInfo {
  int cls, g, mt, ks, nt, rows_in_tile, b_row, out_row, a_row, kb0, kb1;
};

// Groups in walk order: gid[pos] is the group at position pos and tile_start[pos] its
// first tile (tile_start[G] = all tiles); rows and brow are indexed by group.
struct SchedSmem {
  int tile_start[TC_MAX_GROUPS + 1];
  int gid[TC_MAX_GROUPS];
  int rows[TC_MAX_GROUPS];
  int brow[TC_MAX_GROUPS];
};

// Height of the tiles a group of `rows` rows splits into: NT = ceil(rows / BN) tiles of
// equal height (a multiple of 16, at most BN) rather than full tiles and a ragged last
// one: a tile streams the whole weight panel whatever its height, so a short last tile
// costs nearly a full one, while NT tiles of height rows / NT keep every tile near the
// MMA-bound rate. (NT - 1) * height < rows, as height <= BN and (NT - 1) * BN < rows.
template <int BN>
__device__ __forceinline__ int tile_height(int rows) {
  const int NT = (rows + BN - 1) / BN;
  return NT > 0 ? min(BN, (((rows + NT - 1) / NT) + 15) & ~15) : 0;
}

// The r-th tile of walker `walker`: rounds of `walkers` consecutive tiles, taken in
// alternating direction, so that with the groups ordered tallest tiles first every
// walker draws from each height band.
__device__ __forceinline__ int walk_tile(int r, int walker, int walkers) {
  return r * walkers + ((r & 1) ? walkers - 1 - walker : walker);
}

template <int BN, int BKE, int TILE_M = TC_BM>
__device__ __forceinline__ void decode_tile(const GemmParams& p, const SchedSmem& s, int G, int w, TileInfo& ti) {
  int lo = 0, hi = G - 1;  // largest position with tile_start[pos] <= w
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (s.tile_start[mid] <= w) lo = mid; else hi = mid - 1;
  }
  const int pos = lo;
  const int gi = s.gid[pos];
  const int G0 = p.cls[0].n_groups;
  ti.cls = gi < G0 ? 0 : 1;
  ti.g = gi - (ti.cls ? G0 : 0);
  const GemmClass& c = p.cls[ti.cls];
  const int rows = s.rows[gi];
  const int NT = (rows + BN - 1) / BN;
  const int tsz = tile_height<BN>(rows);
  const int local = w - s.tile_start[pos];
  ti.nt = local % NT;
  const int rest = local / NT;
  ti.ks = rest % c.ksplit;
  ti.mt = rest / c.ksplit;
  ti.rows_in_tile = min(tsz, rows - ti.nt * tsz);
  ti.b_row = s.brow[gi] + ti.nt * tsz;
  ti.out_row = (c.seg_off ? s.brow[gi] : ti.g * c.out_group_stride) + ti.nt * tsz;
  // the weight matrix of the group (a replica group reads another group's weights)
  int wg = ti.g;
  if (c.group_map) {
    wg = c.group_map[ti.g];
    if (wg < 0 || wg >= c.n_wgroups) wg = 0;  // (validated where the map is written)
  }
  ti.a_row = wg * c.R + ti.mt * TILE_M;
  const int KB = (c.K + BKE - 1) / BKE;
  ti.kb0 = ti.ks * c.kb_per_split;
  ti.kb1 = min(KB, ti.kb0 + c.kb_per_split);
}

// Per-row epilogue data of the down projection, fetched for the whole tile into the
// warp's shared-memory slice: the gate weight of the row's task and, for the fused
// top-1 combine, the destination token.
struct RowAux {
  float w;
  int dst;
};

template <int EPI>
__device__ __forceinline__ RowAux load_row_aux(const GemmClass& c, const TileInfo& ti, int j) {
  RowAux a{1.f, -1};
  if (EPI != EPI_DOWN || j >= ti.rows_in_tile) return a;
  const long long row = (long long)ti.out_row + j;
  if (c.row_w) a.w = c.row_w[row];
  if ((c.task_w && !c.row_w) || c.scatter_k1) {
    const int q = c.perm[row];
    const bool ok = q >= 0 && q < c.max_row;
    if (c.task_w && !c.row_w) a.w = ok ? c.task_w[q] : 0.f;
    a.dst = ok ? q : -1;
  }
  return a;
}

// LOGITS: one fp32 logit (its row pitch, the expert count, need not keep 16-byte
// alignment, so these rows stay scalar; the expert epilogues store vectors)
__device__ __forceinline__ void store_logit(const GemmClass& c, const TileInfo& ti, int feature, int j, float v) {
  float* o = reinterpret_cast<float*>(c.out) + (long long)ti.ks * c.out_split_stride;
  o[((long long)ti.out_row + j) * c.out_ld + feature] = v;
}

template <int BN, int MATS, int EPI, bool F8, bool PAIR>
__global__ void __launch_bounds__(tc_threads<EPI, PAIR, F8, MATS>(), 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tA0_0, const __grid_constant__ CUtensorMap tA1_0,
                           const __grid_constant__ CUtensorMap tB_0, const __grid_constant__ CUtensorMap tA0_1,
                           const __grid_constant__ CUtensorMap tA1_1, const __grid_constant__ CUtensorMap tB_1,
                           const __grid_constant__ GemmParams p) {
  using S = TcShape<BN, MATS, PAIR>;
  constexpr int STAGES = S::STAGES;
  constexpr int BKE = F8 ? TC_BK8 : TC_BK;  // K elements per k-block (one 128-byte row)
  // DUAL (the down projection with MATS = 2): two consecutive blocks of S::TILE_M
  // output features of the same weight matrix share each token tile, so the token
  // rows are staged once for twice the MMA work (less shared-memory traffic per flop)
  constexpr bool DUAL = EPI == EPI_DOWN && MATS == 2;
  constexpr int TILE_M = S::TILE_M * (DUAL ? 2 : 1);
  static_assert(!F8 || EPI == EPI_SWIGLU || EPI == EPI_RELU || EPI == EPI_DOWN, "8-bit operands: expert GEMMs only");
  static_assert(!DUAL || !F8, "two feature blocks: bf16 only");
  static_assert(!PAIR || (!F8 && (EPI == EPI_SWIGLU || EPI == EPI_RELU || EPI == EPI_DOWN)),
                "pair tiles: bf16 expert GEMMs only");

  __shared__ SchedSmem sched;
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES], accf_bar[2], acce_bar[2], drain_bar;
  __shared__ float aux_w[4][EPI == EPI_DOWN ? BN : 1];  // per epilogue warp: row weights of the tile
  __shared__ int aux_d[4][EPI == EPI_DOWN ? BN : 1];    // and destination tokens (fused top-1 combine)
  __shared__ float aux_s[4][F8 && EPI != EPI_DOWN ? BN : 1];  // F8: activation-row scales of the tile
  // SWIGLU / RELU / DOWN into bf16 rows: per epilogue warp, 16 output rows x its 32
  // features, so the global writes leave as 16-byte vectors along the feature axis.
  // DOWN stages fp32, 8 rows at a time (rows padded to 36 floats: 16-byte aligned, and
  // the column-wise writes hit 32 distinct banks); SWIGLU and RELU stage the rounded
  // bf16 values of all 16 rows (rows of 64 bytes: a row's column-wise writes fill 16
  // distinct banks, and the two rows a quarter-warp reads back as 16-byte vectors
  // cover all 32).
  constexpr bool VEC = EPI == EPI_SWIGLU || EPI == EPI_RELU || EPI == EPI_DOWN;
  constexpr bool STG16 = EPI == EPI_SWIGLU || EPI == EPI_RELU;
  constexpr int NEPI = tc_epi_warps<EPI, PAIR, F8, MATS>();
  __shared__ __align__(16) float stg[VEC && !STG16 ? NEPI : 1][8][36];  // 8 rows per pass
  __shared__ __align__(16) __nv_bfloat16 stg16[STG16 ? NEPI : 1][16][32];
  constexpr int RMASK_M = EPI == EPI_ROUTE ? ROUTE_MAX_M : 1;
  __shared__ __align__(16) float rbias[RMASK_M];  // ROUTE: router bias (zeros when absent)
  __shared__ uint32_t rmask[EPI == EPI_ROUTE ? 2 : 1][4][RMASK_M];  // ROUTE: expert -> lanes holding it
  constexpr int RX = EPI == EPI_ROUTE ? 4 : 1;  // ROUTE: the upper-half thread's pick and sums, per token
  __shared__ float rx_v[RX][32], rx_m[RX][32];
  __shared__ int rx_e[RX][32];
  __shared__ double rx_z[RX][32];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, epi_fail_s, qfail_s[4];
  __shared__ int total_tiles_s;
  extern __shared__ uint8_t dyn_smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // PAIR: rank 0 of the cluster pair is the leader (it issues the MMAs); both CTAs
  // walk the same tiles, indexed by cluster. Otherwise one CTA is one walker.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int walker = PAIR ? (int)cluster_id_x() : (int)blockIdx.x;
  const int walkers = PAIR ? (int)nclusters_x() : (int)gridDim.x;
  const uint32_t smem_base = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  uint8_t* smem_gen = dyn_smem + (smem_base - smem_u32(dyn_smem));
  const int G0 = p.cls[0].n_groups;
  const int G = G0 + (p.n_classes > 1 ? p.cls[1].n_groups : 0);
  volatile int* abort_flag = &abort_s;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accf_bar[i], 1);
      mbar_init(&acce_bar[i], (PAIR ? 2 : 1) * NEPI);  // PAIR: the epilogue warps of both CTAs release the leader's
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    epi_fail_s = 0;
    for (int i = 0; i < 4; ++i) qfail_s[i] = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tA0_0);
    tma_prefetch_desc(&tB_0);
  }
  if (warp == 1) {
    tmem_alloc_g<PAIR>(&tmem_base_s, S::TMEM_COLS);
    tmem_relinquish_g<PAIR>();
  }
  // PAIR: the peer's barriers must be initialised before either CTA signals them
  __syncwarp();
  if (PAIR) cluster_sync_all();
  // Everything above overlaps the previous kernel; the segment offsets, the token
  // rows (TMA) and the row data read below are its outputs.
  pdl_launch_dependents();
  pdl_wait();
  // Tile schedule from the device-resident segment sizes. Groups are walked tallest
  // tiles first (a tile's height sets its MMA work and so its time): a counting sort
  // over the heights 16, 32, ..., BN, stable in group order.
  if (warp == 0) {
    constexpr int NB = BN / 16 + 1;  // bucket = tile height / 16 (0: a group without rows)
    const int per = (G + 31) / 32;
    const int lo = lane * per, hi = min(G, lo + per);
    auto group_tiles = [&](const int gi, const int rows) {
      const GemmClass& c = p.cls[gi < G0 ? 0 : 1];
      return ((c.R + TILE_M - 1) / TILE_M) * c.ksplit * ((rows + BN - 1) / BN);
    };
    int cnt[NB], tl[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) cnt[b] = tl[b] = 0;
    for (int gi = lo; gi < hi; ++gi) {
      const int cl = gi < G0 ? 0 : 1;
      const int g = gi - (cl ? G0 : 0);
      const GemmClass& c = p.cls[cl];
      int rows, brow;
      if (c.seg_off) {
        const int a = c.seg_off[g], b = c.seg_off[g + 1];
        rows = b - a;
        brow = a;
        if (a < 0 || b < a || b > c.max_row) {
          set_status(p.status, MOE_ERR_DEVICE_INDEX);
          rows = 0;
          brow = 0;
        }
      } else {
        rows = c.const_rows;
        brow = g * c.b_group_stride;
      }
      sched.rows[gi] = rows;
      sched.brow[gi] = brow;
      const int key = tile_height<BN>(rows) / 16, tiles = group_tiles(gi, rows);
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b == key) {
          ++cnt[b];
          tl[b] += tiles;
        }
    }
    // first position and first tile of this lane's groups in each bucket: the buckets
    // above it, then the lanes below in this bucket
    int base_c = 0, base_t = 0;
#pragma unroll
    for (int b = NB - 1; b >= 0; --b) {
      int ic = cnt[b], it = tl[b];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int vc = __shfl_up_sync(0xffffffffu, ic, off), vt = __shfl_up_sync(0xffffffffu, it, off);
        if (lane >= off) {
          ic += vc;
          it += vt;
        }
      }
      const int sum_c = __shfl_sync(0xffffffffu, ic, 31), sum_t = __shfl_sync(0xffffffffu, it, 31);
      cnt[b] = base_c + ic - cnt[b];
      tl[b] = base_t + it - tl[b];
      base_c += sum_c;
      base_t += sum_t;
    }
    for (int gi = lo; gi < hi; ++gi) {
      const int rows = sched.rows[gi];
      const int key = tile_height<BN>(rows) / 16, tiles = group_tiles(gi, rows);
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b == key) {
          sched.gid[cnt[b]] = gi;
          sched.tile_start[cnt[b]] = tl[b];
          ++cnt[b];
          tl[b] += tiles;
        }
    }
    const int incl = base_t;  // every tile
    if (lane == 0) sched.tile_start[G] = incl;
    // An earlier kernel of this layer flagged a device error: its index tables
    // cannot be trusted, so this launch does no work.
    const int prior = p.status ? *reinterpret_cast<volatile int*>(p.status) : 0;
    if (lane == 31) total_tiles_s = prior ? 0 : incl;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total = total_tiles_s;
  const unsigned long long lim = p.wait_limit_ns;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    int stage = 0;
    uint32_t phase = 0;
    int last_parity[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) last_parity[i] = -1;
    bool ok = true;
    for (int r = 0, w = walker; w < total && ok; ++r, w = walk_tile(r, walker, walkers)) {
      TileInfo ti;
      decode_tile<BN, BKE, TILE_M>(p, sched, G, w, ti);
      const CUtensorMap* mA0 = ti.cls ? &tA0_1 : &tA0_0;
      const CUtensorMap* mA1 = ti.cls ? &tA1_1 : &tA1_0;
      const CUtensorMap* mB = ti.cls ? &tB_1 : &tB_0;
      // PAIR: this CTA's 128 weight rows and its half of the tile's token rows
      const int n_inst = max(16, (ti.rows_in_tile + 15) & ~15);
      const int a_row = ti.a_row + (int)rank * TC_BM;
      const int b_row = ti.b_row + (int)rank * (n_inst / 2);
      // PAIR: a CTA's 128 weight rows of a block that lie wholly past the group's rows
      // (the last feature tile when R is not a multiple of 256) are not loaded: they
      // belong to the next group, and the stale stage bytes left in their place feed
      // only accumulator rows that the epilogue skips (feature >= R). The leader arms
      // the stage barrier with the bytes both CTAs do load.
      const int a_loc = ti.mt * TILE_M;  // the tile's first weight row within its group
      const int a_rows = p.cls[ti.cls].R;
      auto a_live = [&](int cta, int blk) { return a_loc + blk * S::TILE_M + cta * TC_BM < a_rows; };
      const bool live0 = a_live((int)rank, 0), live1 = a_live((int)rank, DUAL ? 1 : 0);
      uint32_t pair_bytes = 2 * S::B_BYTES;
      if (PAIR)
        for (int cta = 0; cta < 2; ++cta)
          pair_bytes += (a_live(cta, 0) ? S::A_BYTES : 0) + (MATS == 2 && a_live(cta, DUAL ? 1 : 0) ? S::A_BYTES : 0);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, lim, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* st = smem_gen + stage * S::STAGE_BYTES;
        if (PAIR) {
          // both CTAs' copies complete on the leader's barrier, which expects them all
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], pair_bytes);
          if (live0) tma_load_2d_pair(mA0, fb, st, kb * BKE, a_row);
          if (MATS == 2 && live1)
            tma_load_2d_pair(DUAL ? mA0 : mA1, fb, st + S::A_BYTES, kb * BKE, a_row + (DUAL ? S::TILE_M : 0));
          tma_load_2d_pair(mB, fb, st + MATS * S::A_BYTES, kb * BKE, b_row);
          if (leader) last_parity[stage] = (int)phase;
        } else {
          mbar_arrive_expect_tx(&full_bar[stage], S::STAGE_BYTES);
          tma_load_2d(mA0, &full_bar[stage], st, kb * BKE, ti.a_row);
          if (MATS == 2)
            tma_load_2d(DUAL ? mA0 : mA1, &full_bar[stage], st + S::A_BYTES, kb * BKE,
                        ti.a_row + (DUAL ? S::TILE_M : 0));
          tma_load_2d(mB, &full_bar[stage], st + MATS * S::A_BYTES, kb * BKE, ti.b_row);
          last_parity[stage] = (int)phase;
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok) {
      set_status(p.status, MOE_ERR_TIMEOUT);
      abort_s = 1;
    }
    // Drain: every issued copy must land before the CTA may exit. (PAIR: the leader's
    // barriers count both CTAs' copies, and the peer waits for the leader at the
    // final cluster barrier.)
    for (int i = 0; i < STAGES; ++i)
      if (last_parity[i] >= 0) {
        const volatile int never = 0;
        if (!mbar_wait(&full_bar[i], (uint32_t)last_parity[i], TC_DRAIN_LIMIT_NS, &never))
          set_status(p.status, MOE_ERR_TIMEOUT);
      }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int r = 0, w = walker; w < total && ok; ++r, w = walk_tile(r, walker, walkers)) {
      TileInfo ti;
      decode_tile<BN, BKE, TILE_M>(p, sched, G, w, ti);
      if (!mbar_wait(&acce_bar[acc], acc_phase ^ 1u, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S::ACC_COLS);
      const int n_inst = max(16, (ti.rows_in_tile + 15) & ~15);
      // one MMA covers S::TILE_M weight rows (DUAL tiles issue two of them per K step)
      const uint32_t idesc = F8 ? idesc_e4m3(S::TILE_M, n_inst) : idesc_bf16(S::TILE_M, n_inst);
      for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_base + stage * S::STAGE_BYTES;
        const uint64_t da0 = sdesc_sw128(st);
        const uint64_t da1 = sdesc_sw128(st + S::A_BYTES);
        const uint64_t db = sdesc_sw128(st + MATS * S::A_BYTES);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t accum = (kb > ti.kb0 || kk > 0) ? 1u : 0u;
          // one MMA takes 32 B of K (16 bf16 or 32 E4M3): +2 in the >>4 address field
          if (PAIR) {
            umma_bf16_pair(d_tmem, da0 + 2 * kk, db + 2 * kk, idesc, accum);
            if (MATS == 2) umma_bf16_pair(d_tmem + BN, da1 + 2 * kk, db + 2 * kk, idesc, accum);
          } else if (F8) {
            umma_e4m3(d_tmem, da0 + 2 * kk, db + 2 * kk, idesc, accum);
            if (MATS == 2) umma_e4m3(d_tmem + BN, da1 + 2 * kk, db + 2 * kk, idesc, accum);
          } else {
            umma_bf16(d_tmem, da0 + 2 * kk, db + 2 * kk, idesc, accum);
            if (MATS == 2) umma_bf16(d_tmem + BN, da1 + 2 * kk, db + 2 * kk, idesc, accum);
          }
        }
        if (PAIR) {  // the stage is free in both CTAs
          umma_commit_pair(smem_u32(&empty_bar[stage]));
          umma_commit_pair(mapa_shared(smem_u32(&empty_bar[stage]), 1));
        } else {
          umma_commit(&empty_bar[stage]);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (PAIR) {  // both CTAs' accumulators are ready
        umma_commit_pair(smem_u32(&accf_bar[acc]));
        umma_commit_pair(mapa_shared(smem_u32(&accf_bar[acc]), 1));
      } else {
        umma_commit(&accf_bar[acc]);
      }
      if (++acc == S::NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (!ok) {
      set_status(p.status, MOE_ERR_TIMEOUT);
      abort_s = 1;
    }
    if (PAIR)
      umma_commit_pair(smem_u32(&drain_bar));
    else
      umma_commit(&drain_bar);
    const volatile int never = 0;
    if (!mbar_wait(&drain_bar, 0, TC_DRAIN_LIMIT_NS, &never)) set_status(p.status, MOE_ERR_TIMEOUT);
  } else if (EPI == EPI_ROUTE && warp >= 2) {
    // ---------------------------------------------------------------- router epilogue
    // TMEM lane = token (quarter q of the 128-token tile), column = expert. Two warps
    // per lane quarter: half 0 takes the lower half of the expert columns, half 1 the
    // upper, and each pass merges them through shared memory (half 1's pick wins only
    // when strictly larger, as a walk over all columns in order would have it; the
    // softmax sums are rescaled to the larger maximum). Every epilogue warp reaches
    // every epilogue barrier of every tile; a failed wait is published through
    // epi_fail_s before the barrier, so all eight leave together.
    const int q = warp & 3, half = (warp - 2) >> 2;
    const int et = (warp - 2) * 32 + lane;  // 0..255
    {
      const GemmClass& c = p.cls[0];
      for (int e = et; e < ROUTE_MAX_M; e += 256) rbias[e] = (c.bias && e < c.const_rows) ? c.bias[e] : 0.f;
      epi_bar();
    }
    int acc = 0, iter = 0;
    uint32_t acc_phase = 0;
    for (int r = 0, w = walker; w < total; ++r, w = walk_tile(r, walker, walkers), ++iter) {
      TileInfo ti;
      decode_tile<BN, BKE>(p, sched, G, w, ti);
      const GemmClass& c = p.cls[0];
      const int t = ti.mt * TC_BM + q * 32 + lane;  // token
      const bool tv_ok = t < c.R;
      const int m = ti.rows_in_tile, k = c.k_sel;
      const int nch = (m + 31) / 32, hch = (nch + 1) / 2;
      const int c_lo = half ? 32 * hch : 0, c_hi = half ? 32 * nch : 32 * hch;
      const bool got = mbar_wait(&accf_bar[acc], acc_phase, lim, abort_flag);
      if (!got) {
        set_status(p.status, MOE_ERR_TIMEOUT);
        abort_s = 1;
        epi_fail_s = 1;
      }
      epi_bar();
      if (epi_fail_s) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * S::ACC_COLS);
      // Pass s picks the largest logit strictly after pick s - 1 in the order
      // (logit desc, expert asc), reading the accumulator again from TMEM; pass 0
      // also writes the logits (when asked) and the softmax denominator. Each pass
      // stores its expert and, for now, its logit in the outputs (half 0).
      float mrun = -INFINITY, mx = -INFINITY;
      double z = 0.0;
      float* lg = c.out && tv_ok ? reinterpret_cast<float*>(c.out) + (long long)t * m : nullptr;
      int32_t* oi = c.sel_idx + (long long)t * k;
      float* ow = c.sel_w + (long long)t * k;
      float pv = INFINITY;
      int pe = -1;
      bool bad = false;
#pragma unroll 1
      for (int s2 = 0; s2 < k; ++s2) {
        float bv;
        int be;
        if (s2 == 0) {
          route_pass<true>(t_row, c_lo, c_hi, m, rbias, pv, pe, bv, be, mrun, z, lg);
        } else {
          float dm = 0.f;
          double dz = 0.0;
          route_pass<false>(t_row, c_lo, c_hi, m, rbias, pv, pe, bv, be, dm, dz, nullptr);
        }
        if (half) {
          rx_v[q][lane] = bv;
          rx_e[q][lane] = be;
          if (s2 == 0) {
            rx_m[q][lane] = mrun;
            rx_z[q][lane] = z;
          }
        }
        epi_bar();
        if (!half) {
          const float ov = rx_v[q][lane];
          const int oe = rx_e[q][lane];
          if (ov > bv) {  // the upper half holds higher experts: it wins only when strictly larger
            bv = ov;
            be = oe;
          }
          if (s2 == 0) {
            const float om = rx_m[q][lane], mm = fmaxf(mrun, om);
            z = z * (double)expf(mrun - mm) + rx_z[q][lane] * (double)expf(om - mm);
            mrun = mm;
            mx = bv;
            z *= (double)expf(mrun - mx);  // the running maximum is the top logit
          }
          rx_v[q][lane] = bv;  // the merged pick, for the upper half's next pass
          rx_e[q][lane] = be;
          if (tv_ok) {
            oi[s2] = be;
            ow[s2] = bv;
          }
          bad |= be < 0;  // NaN logits
        }
        epi_bar();
        if (half) {
          bv = rx_v[q][lane];
          be = rx_e[q][lane];
        }
        pv = bv;
        pe = be;
      }
      // the accumulator is free for the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce_bar[acc]);
      if (++acc == S::NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (tv_ok && !half) {  // gate weights: softmax over all m, renormalised over the k chosen when asked
        double sel = 0.0;
#pragma unroll 1
        for (int s2 = 0; s2 < k; ++s2) sel += (double)expf(ow[s2] - mx) / z;
#pragma unroll 1
        for (int s2 = 0; s2 < k; ++s2) {
          double pr = (double)expf(ow[s2] - mx) / z;
          if (c.renorm) pr /= sel;
          ow[s2] = (float)pr;
        }
        if (bad) set_status(p.status, MOE_ERR_DEVICE_INDEX);
      }
      if (c.lrank) {
        // rank of each task among the tile's tasks of its expert, in (token, slot)
        // order: lanes below in this quarter plus all tasks of the quarters before
        // (the lower-half warps build the masks; every epilogue warp passes the barrier)
        uint32_t(*mk)[RMASK_M] = rmask[EPI == EPI_ROUTE ? (iter & 1) : 0];
        if (!half) {
          for (int e = lane; e < m; e += 32) mk[q][e] = 0u;
          __syncwarp();
          if (tv_ok)
#pragma unroll 1
            for (int s2 = 0; s2 < k; ++s2) {
              const int e = oi[s2];
              if (e >= 0) atomicOr(&mk[q][e], 1u << lane);
            }
        }
        epi_bar();
        if (tv_ok && !half)
#pragma unroll 1
          for (int s2 = 0; s2 < k; ++s2) {
            const int e = oi[s2];
            if (e < 0) continue;
            int rk = __popc(mk[q][e] & ((1u << lane) - 1u));
            for (int q2 = 0; q2 < q; ++q2) rk += __popc(mk[q2][e]);
            c.lrank[(long long)t * k + s2] = rk;
          }
        for (int e = et; e < m; e += 256)
          c.tile_cnt[(long long)ti.mt * m + e] =
              __popc(mk[0][e]) + __popc(mk[1][e]) + __popc(mk[2][e]) + __popc(mk[3][e]);
        // (the masks are double-buffered: the next tile writes the other set, and the
        // one after that passes an epilogue barrier every warp reaches only after
        // finishing the reads above)
      }
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - 2;  // epilogue warp index (its staging tile)
    // SPLITB (down tiles with two feature blocks, 8 warps): the two warps of a quarter
    // take one feature block each over all chunks, and share the quarter's row data.
    // Otherwise the NEPI / 4 warps of a quarter take alternate 16-row chunks.
    constexpr bool SPLITB = DUAL && NEPI == 8;
    const int blk = SPLITB ? (ew >> 2) : 0;
    const int cfirst = SPLITB ? 0 : 16 * (ew >> 2), cstep = SPLITB ? 16 : 16 * (NEPI / 4);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int r = 0, w = walker; w < total; ++r, w = walk_tile(r, walker, walkers)) {
      TileInfo ti;
      decode_tile<BN, BKE, TILE_M>(p, sched, G, w, ti);
      const GemmClass& c = p.cls[ti.cls];
      const int fcta = ti.mt * TILE_M + (int)rank * TC_BM;  // first feature of this CTA's TMEM lanes
      const int feature = fcta + q * 32 + lane;
      const bool fvalid = feature < c.R;
      const bool has_k = ti.kb1 > ti.kb0;  // an empty K range leaves the accumulator unwritten
      const float bias = (EPI == EPI_LOGITS && c.bias && fvalid) ? c.bias[feature] : 0.f;
      // F8: scale of this lane's weight row (index = weight-matrix row of the feature)
      const float sa0 = (F8 && fvalid) ? c.a0_scale[ti.a_row + (int)rank * TC_BM + q * 32 + lane] : 1.f;
      const float sa1 = (F8 && MATS == 2 && fvalid) ? c.a1_scale[ti.a_row + (int)rank * TC_BM + q * 32 + lane] : 1.f;
      // Row data of the whole tile (gate weight, destination token), fetched into this
      // quarter's shared-memory slice before waiting for the accumulator so the loads
      // overlap the MMAs; the chunk loop below then reads it with broadcasts. SPLITB:
      // both warps of the quarter write the same values, after both finished reading
      // the previous tile's.
      if (SPLITB) quarter_bar(q);
      if (EPI == EPI_DOWN) {
        for (int j = lane; j < BN; j += 32) {
          const RowAux a = load_row_aux<EPI>(c, ti, j);
          // F8: the activation row's scale folds into the row weight
          aux_w[q][j] = (F8 && j < ti.rows_in_tile) ? a.w * c.b_scale[ti.b_row + j] : a.w;
          aux_d[q][j] = a.dst;
        }
        __syncwarp();
      } else if (F8) {
        for (int j = lane; j < BN; j += 32) aux_s[q][j] = j < ti.rows_in_tile ? c.b_scale[ti.b_row + j] : 0.f;
        __syncwarp();
      }
      const bool got = mbar_wait(&accf_bar[acc], acc_phase, lim, abort_flag);
      if (!got) {
        set_status(p.status, MOE_ERR_TIMEOUT);
        abort_s = 1;
        if (!SPLITB) break;
        qfail_s[q] = 1;
      }
      if (SPLITB) {  // both warps of the quarter leave together or go on together
        quarter_bar(q);
        if (qfail_s[q]) break;
      }
      tc_fence_after();
      // (SPLITB: the columns of this warp's feature block)
      const uint32_t t_row =
          tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * S::ACC_COLS + (SPLITB ? blk * BN : 0));
      // One 16-row chunk of accumulator columns (r0: gate or the single matrix, r1: up).
      auto chunk = [&](const int c0, const uint32_t (&r0)[16], const uint32_t (&r1)[16]) {
        const int jn = min(16, ti.rows_in_tile - c0);
        // DOWN: the chunk's 16 row weights, read once for both feature blocks
        float wrow[16];
        if constexpr (EPI == EPI_DOWN) {
#pragma unroll
          for (int j = 0; j < 16; ++j) wrow[j] = aux_w[q][c0 + j];
        }
        // activation of 16 rows x this warp's 32 features, staged, then stored as
        // 16-byte vectors along the feature axis from feature fbase on
        auto emit = [&](const uint32_t (&ra)[16], const uint32_t (&rb)[16], const int fbase) {
          if constexpr (STG16) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              float v0 = has_k ? __uint_as_float(ra[j]) : 0.f;
              float v1 = (MATS == 2 && has_k) ? __uint_as_float(rb[j]) : 0.f;
              if (F8) {
                const float sb = aux_s[q][c0 + j];
                v0 = v0 * sa0 * sb;
                v1 = v1 * sa1 * sb;
              }
              stg16[ew][j][lane] = __float2bfloat16_rn(EPI == EPI_SWIGLU ? silu_mul(v0, v1) : fmaxf(v0, 0.f));
            }
            __syncwarp();
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(c.out) + fbase;  // bf16 rows of h: 4 x 8 per row
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int idx = lane + 32 * i, jj = idx >> 2, part = idx & 3;
              if (jj < jn && fbase + part * 8 < c.R)
                *reinterpret_cast<uint4*>(o + ((long long)ti.out_row + c0 + jj) * c.out_ld + part * 8) =
                    *reinterpret_cast<const uint4*>(&stg16[ew][jj][part * 8]);
            }
            __syncwarp();
          } else if constexpr (EPI == EPI_DOWN) {
            // rows weighted by their task's gate weight, in two passes of 8 rows
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float v0 = has_k ? __uint_as_float(ra[8 * h + j]) * (F8 ? sa0 : 1.f) : 0.f;
                stg[ew][j][lane] = v0 * wrow[8 * h + j];
              }
              __syncwarp();
              if (!c.scatter_k1) {  // fp32 partial rows: 8 float4 per row
                float* o = reinterpret_cast<float*>(c.out) + (long long)ti.ks * c.out_split_stride + fbase;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                  const int idx = lane + 32 * i, jj = idx >> 3, part = idx & 7;
                  if (8 * h + jj < jn && fbase + part * 4 < c.R)
                    *reinterpret_cast<float4*>(o + (long long)(ti.out_row + c0 + 8 * h + jj) * c.out_ld + part * 4) =
                        *reinterpret_cast<const float4*>(&stg[ew][jj][part * 4]);
                }
              } else {  // bf16 rows of the layer output with the top-1 combine fused: 4 x 8 per row
                __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(c.out) + fbase;
                const int jj = lane >> 2, part = lane & 3;
                const long long orow = (long long)aux_d[q][c0 + 8 * h + jj];
                if (8 * h + jj < jn && fbase + part * 8 < c.R && orow >= 0) {
                  const float* v = &stg[ew][jj][part * 8];
                  uint4 pk;
                  pk.x = pack_bf16x2(v[0], v[1]);
                  pk.y = pack_bf16x2(v[2], v[3]);
                  pk.z = pack_bf16x2(v[4], v[5]);
                  pk.w = pack_bf16x2(v[6], v[7]);
                  *reinterpret_cast<uint4*>(o + orow * c.out_ld + part * 8) = pk;
                }
              }
              __syncwarp();
            }
          }
        };
        if (VEC) {
          const int fbase = fcta + q * 32;  // first feature of this warp (R is a multiple of 8)
          if (SPLITB) {
            emit(r0, r0, fbase + blk * S::TILE_M);  // this warp's feature block
          } else {
            emit(r0, r1, fbase);
            if (DUAL) emit(r1, r1, fbase + S::TILE_M);  // the second feature block
          }
        } else if (fvalid) {  // LOGITS
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (j < jn) store_logit(c, ti, feature, c0 + j, (has_k ? __uint_as_float(r0[j]) : 0.f) + bias);
        }
        __syncwarp();
      };
      // The accumulator goes back to the MMA issuer as soon as this warp's last TMEM
      // load has landed in registers: its last chunk is computed and stored while the
      // next tile's MMAs already run (with one accumulator, as for the SwiGLU pair
      // tiles, this is the only overlap of epilogue and MMAs). Called exactly once per
      // tile by every epilogue warp.
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR && !leader)  // the leader's MMA waits for both CTAs' epilogues
            mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&acce_bar[acc]), 0));
          else
            mbar_arrive_relaxed(&acce_bar[acc]);
        }
      };
      // The loads of chunk i + 1 are in flight while chunk i is computed and stored
      // (two register buffers; the loop body takes the even chunk, then the odd one).
      const int rows = ti.rows_in_tile;
      constexpr bool LD2 = MATS == 2 && !SPLITB;  // both matrices' (or blocks') columns
      uint32_t ra0[16], ra1[16], rb0[16], rb1[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) ra1[j] = rb1[j] = 0u;
      if (cfirst < rows) {
        tmem_ld_x16(t_row + cfirst, ra0);
        if (LD2) tmem_ld_x16(t_row + BN + cfirst, ra1);
      } else {
        release_acc();
      }
#pragma unroll 1
      for (int c0 = cfirst; c0 < rows; c0 += 2 * cstep) {
        if (LD2) tmem_ld_wait_keep(ra0, ra1); else tmem_ld_wait_keep(ra0);
        if (c0 + cstep < rows) {
          tmem_ld_x16(t_row + c0 + cstep, rb0);
          if (LD2) tmem_ld_x16(t_row + BN + c0 + cstep, rb1);
        } else {
          release_acc();
        }
        chunk(c0, ra0, ra1);
        if (c0 + cstep >= rows) break;
        if (LD2) tmem_ld_wait_keep(rb0, rb1); else tmem_ld_wait_keep(rb0);
        if (c0 + 2 * cstep < rows) {
          tmem_ld_x16(t_row + c0 + 2 * cstep, ra0);
          if (LD2) tmem_ld_x16(t_row + BN + c0 + 2 * cstep, ra1);
        } else {
          release_acc();
        }
        chunk(c0 + cstep, rb0, rb1);
      }
      if (++acc == S::NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }
  // Warps 0 and 1 ran their roles on lane 0 alone: reconverge each warp before the
  // block barrier (an aligned barrier reached by part of a warp does not wait for
  // the rest of the block), so TMEM is freed only after every epilogue read.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // PAIR: neither CTA frees TMEM or exits while the other may still signal its
  // barriers or (leader) have MMAs writing the peer's accumulators
  if (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_g<PAIR>(tmem_base, S::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [rows, K] row-major, bf16 or (u8) E4M3 codes; box = one 128-byte row of K x
// box_rows, 128-byte swizzle; out-of-range elements read as zero.
static bool make_map(CUtensorMap* m, const TcOperand& op, int box_rows, bool u8) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !op.ptr || op.rows <= 0 || op.K <= 0) return false;
  const int es_bytes = u8 ? 1 : 2;
  if ((op.K * es_bytes) % 16) return false;  // row pitch must be a multiple of 16 bytes
  cuuint64_t dims[2] = {(cuuint64_t)op.K, (cuuint64_t)op.rows};
  cuuint64_t strides[1] = {(cuuint64_t)op.K * es_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(u8 ? TC_BK8 : TC_BK), (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(op.ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int MATS, int EPI, bool F8, bool PAIR = false>
static cudaError_t launch_impl(const TcMaps& maps, const GemmParams& p, int num_ctas, cudaStream_t s) {
  using S = TcShape<BN, MATS, PAIR>;
  CUtensorMap m[6];
  const int nc = p.n_classes;
  for (int c = 0; c < 2; ++c) {
    const int src = c < nc ? c : 0;
    if (!make_map(&m[3 * c + 0], maps.a0[src], TC_BM, F8)) return cudaErrorInvalidValue;
    const TcOperand& a1 = MATS == 2 ? maps.a1[src] : maps.a0[src];
    if (!make_map(&m[3 * c + 1], a1, TC_BM, F8)) return cudaErrorInvalidValue;
    if (!make_map(&m[3 * c + 2], maps.b[src], S::B_ROWS, F8)) return cudaErrorInvalidValue;
  }
  auto kern = tc_grouped_gemm_kernel<BN, MATS, EPI, F8, PAIR>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::DYN_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (PAIR) {
    // clusters of two CTAs on two SMs (persistent): as many pairs as can be resident
    // at once, so no pair waits for another to finish (a GPC with an odd number of
    // free SMs leaves one SM out)
    static int max_pairs = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(tc_threads<EPI, PAIR, F8, MATS>());
    cfg.dynamicSmemBytes = S::DYN_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    if (!max_pairs) {  // the occupancy query takes the cluster shape alone
      cfg.gridDim = dim3(std::max(2, num_ctas & ~1));
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      const cudaError_t eo = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (eo != cudaSuccess) return eo;
      max_pairs = std::max(1, n);
    }
    cfg.gridDim = dim3(2 * std::min(max_pairs, std::max(1, num_ctas / 2)));
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], p);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  launch_k(kern, num_ctas, tc_threads<EPI, PAIR, F8, MATS>(), S::DYN_SMEM, s, m[0], m[1], m[2], m[3], m[4], m[5], p);
  count_launch();
  return cudaGetLastError();
}

// Token rows per tile: about twice the mean segment, so most experts' segments fit
// one tile and each weight tile is streamed once (every extra row tile of a segment
// re-reads the expert's weights), capped by TMEM (two SwiGLU accumulators of BN
// columns, double-buffered, must fit 512 columns). The down projection takes 256-row
// tiles only when the mean segment fills them: a 256-row tile leaves room for four
// pipeline stages, too few to cover the loads of a 1408-deep K loop over short
// segments (measured: dsv2lite down 283 -> 242 us with 128; mixtral, 1024-row
// segments, 853 us with 256 against 1228 with 128).
int tc_pick_bn(int epi, double avg) {
  int cap = (epi == EPI_SWIGLU || epi == EPI_LOGITS) ? 128 : 256;
  if (epi == EPI_DOWN && avg < 256.0) cap = 128;
  int bn = 16;
  while (bn < cap && bn < 2.0 * avg) bn <<= 1;
  return bn;
}

// Pair tiles (256 weight rows over two SMs, up to 256 token rows) when the mean
// segment is longer than the 128 token rows a one-SM tile takes. A one-SM tile then
// needs two or more token tiles per expert, each streaming the expert's weights again,
// where a pair tile covers up to 256 rows with one pass; and for long segments each
// SM reads half the operand bytes per MMA, so shared-memory bandwidth stops bounding
// the tensor pipe (Mixtral-shaped prefill: 1024 rows per expert on average;
// DeepSeek-V2-Lite-shaped: 192).
bool tc_pick_pair(double avg) { return avg > 128.0; }

cudaError_t launch_tc_gemm(int epi, int bn, const TcMaps& maps, const GemmParams& p, int num_ctas,
                           cudaStream_t s, bool f8, bool pair) {
  if (pair) {  // two-CTA tiles: bf16 expert GEMMs with 256-row token tiles, no K split
    if (f8 || bn != 256) return cudaErrorInvalidValue;
    for (int c = 0; c < p.n_classes; ++c)
      if (p.cls[c].ksplit != 1) return cudaErrorInvalidValue;
    if (epi == EPI_SWIGLU) return launch_impl<256, 2, EPI_SWIGLU, false, true>(maps, p, num_ctas, s);
    if (epi == EPI_RELU) return launch_impl<256, 1, EPI_RELU, false, true>(maps, p, num_ctas, s);
    if (epi == EPI_DOWN) return launch_impl<256, 1, EPI_DOWN, false, true>(maps, p, num_ctas, s);
    if (epi == EPI_DOWN_DUAL) return launch_impl<256, 2, EPI_DOWN, false, true>(maps, p, num_ctas, s);
    return cudaErrorInvalidValue;
  }
  if (f8) {
    if (epi != EPI_SWIGLU && epi != EPI_RELU && epi != EPI_DOWN) return cudaErrorInvalidValue;
    for (int c = 0; c < p.n_classes; ++c)
      if (!p.cls[c].a0_scale || !p.cls[c].b_scale || (epi == EPI_SWIGLU && !p.cls[c].a1_scale))
        return cudaErrorInvalidValue;
  }
#define MOE_TC_CASE(EPI_, MATS_, BN_) \
  if (epi == EPI_ && bn == BN_ && !f8) return launch_impl<BN_, MATS_, EPI_, false>(maps, p, num_ctas, s);
#define MOE_TC_CASE8(EPI_, MATS_, BN_) \
  if (epi == EPI_ && bn == BN_ && f8) return launch_impl<BN_, MATS_, EPI_, true>(maps, p, num_ctas, s);
  MOE_TC_CASE(EPI_LOGITS, 1, 16)
  MOE_TC_CASE(EPI_LOGITS, 1, 32)
  MOE_TC_CASE(EPI_LOGITS, 1, 64)
  MOE_TC_CASE(EPI_LOGITS, 1, 128)
  MOE_TC_CASE(EPI_SWIGLU, 2, 16)
  MOE_TC_CASE(EPI_SWIGLU, 2, 32)
  MOE_TC_CASE(EPI_SWIGLU, 2, 64)
  MOE_TC_CASE(EPI_SWIGLU, 2, 128)
  MOE_TC_CASE(EPI_RELU, 1, 16)
  MOE_TC_CASE(EPI_RELU, 1, 32)
  MOE_TC_CASE(EPI_RELU, 1, 64)
  MOE_TC_CASE(EPI_RELU, 1, 128)
  MOE_TC_CASE(EPI_RELU, 1, 256)
  MOE_TC_CASE(EPI_DOWN, 1, 16)
  MOE_TC_CASE(EPI_DOWN, 1, 32)
  MOE_TC_CASE(EPI_DOWN, 1, 64)
  MOE_TC_CASE(EPI_DOWN, 1, 128)
  MOE_TC_CASE(EPI_DOWN, 1, 256)
  MOE_TC_CASE(EPI_ROUTE, 1, 16)
  MOE_TC_CASE(EPI_ROUTE, 1, 32)
  MOE_TC_CASE(EPI_ROUTE, 1, 64)
  MOE_TC_CASE(EPI_ROUTE, 1, 128)
  MOE_TC_CASE(EPI_ROUTE, 1, 256)
  MOE_TC_CASE8(EPI_SWIGLU, 2, 16)
  MOE_TC_CASE8(EPI_SWIGLU, 2, 32)
  MOE_TC_CASE8(EPI_SWIGLU, 2, 64)
  MOE_TC_CASE8(EPI_SWIGLU, 2, 128)
  MOE_TC_CASE8(EPI_RELU, 1, 16)
  MOE_TC_CASE8(EPI_RELU, 1, 32)
  MOE_TC_CASE8(EPI_RELU, 1, 64)
  MOE_TC_CASE8(EPI_RELU, 1, 128)
  MOE_TC_CASE8(EPI_RELU, 1, 256)
  MOE_TC_CASE8(EPI_DOWN, 1, 16)
  MOE_TC_CASE8(EPI_DOWN, 1, 32)
  MOE_TC_CASE8(EPI_DOWN, 1, 64)
  MOE_TC_CASE8(EPI_DOWN, 1, 128)
  MOE_TC_CASE8(EPI_DOWN, 1, 256)
#undef MOE_TC_CASE
#undef MOE_TC_CASE8
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_topk(const moe_config_t& c, const void* x, const void* w_r, const float* bias, float* logits,
                              int32_t* idx, float* w, int32_t* lrank, int32_t* tile_cnt, int* status,
                              unsigned long long wait_limit_ns, cudaStream_t s) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  GemmClass& g = p.cls[0];
  g.n_groups = 1;
  g.R = c.T;  // A = x: tokens are the MMA's rows
  g.K = c.d;
  g.ksplit = 1;
  g.kb_per_split = (c.d + TC_BK - 1) / TC_BK;
  g.const_rows = c.m;  // B = W_r: every expert in one N tile
  g.out = logits;
  g.out_ld = c.m;
  g.bias = bias;
  g.k_sel = c.k;
  g.renorm = c.renormalize;
  g.sel_idx = idx;
  g.sel_w = w;
  g.lrank = lrank;
  g.tile_cnt = tile_cnt;
  p.n_classes = 1;
  p.status = status;
  p.wait_limit_ns = wait_limit_ns;
  int bn = 16;
  while (bn < c.m) bn <<= 1;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  maps.a0[0] = {x, c.T, c.d};
  maps.a1[0] = maps.a0[0];
  maps.b[0] = {w_r, c.m, c.d};
  const int tiles = (c.T + TC_BM - 1) / TC_BM;
  return launch_tc_gemm(EPI_ROUTE, bn, maps, p, std::min(tiles, num_sms()), s);
}

}  // namespace moe
