// libmoe C ABI: argument checks, workspace layout and launch orchestration.
// Every entry point validates on the host before launching anything, launches
// asynchronously on the caller's stream, allocates nothing and never blocks the
// host (except moe_read_device_status, which exists to do exactly that).
#include <algorithm>
#include <atomic>
#include <cstring>
#include <initializer_list>

#include "atomic.cuh"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches += (uint64_t)n; }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static unsigned long long g_wait_limit_ns = 2000ull * 1000 * 1000;
static cudaEvent_t g_stage_events[8];
static int g_n_stage_events = 0;

// Inside a stream capture the record becomes an event-record node of the graph
// (external), so replays of the graph time their stages too.
cudaError_t mark_stage_event(int i, cudaStream_t s) {
  if (i >= g_n_stage_events || !g_stage_events[i]) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(g_stage_events[i], s, cudaEventRecordExternal);
  return cudaEventRecord(g_stage_events[i], s);
}

static moe_status_t mark_stage(int i, cudaStream_t s) {
  return mark_stage_event(i, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
constexpr int PLAN_SMS = 148;
  // B200 SM count used for static planning (split-K, tile sizes)

static moe_status_t check_device() {
  static int ok_cache[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  if (!ok_cache[dev]) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    ok_cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return ok_cache[dev] == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// ------------------------------------------------------------------ planning
struct Plan {
  int es;          // element size of x / weights
  int bn_up, bn_down;
  int ksplit;      // down-projection K split (1 when shared experts are present)
  int kbps;        // k-blocks per split of the routed down projection
  bool pair;       // bf16 expert GEMMs as two-CTA tiles (256 token rows, no K split)
};

static int kblocks(int K) { return (K + 63) / 64; }

static Plan make_plan(const moe_config_t& c) {
  Plan p;
  p.es = c.dtype == MOE_F32 ? 4 : 2;
  const double avg = (double)c.T * c.k / c.m;
  p.bn_up = tc_pick_bn(c.act == MOE_SWIGLU ? EPI_SWIGLU : EPI_RELU, avg);
  p.bn_down = tc_pick_bn(EPI_DOWN, avg);
  p.ksplit = 1;
  p.kbps = kblocks(c.f);
  p.pair = c.dtype == MOE_BF16 && tc_pick_pair(avg);
  if (c.dtype == MOE_BF16 && c.n_shared == 0 && !p.pair) {
    const long long active = std::min<long long>(c.m, (long long)c.T * c.k);
    const long long nt = std::max<long long>(1, (long long)((avg + p.bn_down - 1) / p.bn_down));
    const long long tiles = active * ((c.d + 127) / 128) * nt;
    const long long want = 4LL * PLAN_SMS;
    if (tiles < want) {
      int ks = (int)std::min<long long>((want + tiles - 1) / tiles, 16);
      ks = std::min(ks, kblocks(c.f));
      const int kbps = (kblocks(c.f) + ks - 1) / ks;
      p.ksplit = (kblocks(c.f) + kbps - 1) / kbps;  // no empty split
      p.kbps = kbps;
    }
  }
  return p;
}

struct Layout {
  size_t status, logits, idx, w, counts, offsets, lis, perm, inv_perm, w_perm, start, x_perm, h, h_sh, y, y_sh;
  size_t lrank, tile_cnt, idx2, gmap, lis2, total;
};

static Layout make_layout(const moe_config_t& c, const Plan& p) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t Tk = (size_t)c.T * c.k;
  const size_t T = (size_t)c.T;
  L.status = take(256);
  L.logits = take(T * c.m * 4);
  L.idx = take(Tk * 4);
  L.w = take(Tk * 4);
  L.counts = take((size_t)c.m * 4);
  L.offsets = take((size_t)(c.m + 1) * 4);
  L.lis = take(sizeof(moe_lis_t));
  L.perm = take(Tk * 4);
  L.inv_perm = take(Tk * 4);
  L.w_perm = take(Tk * 4);
  L.start = take((size_t)8192 * 4);  // [R][m] range starts of the stable sort, R * (m + 1) <= 8192
  L.x_perm = take(Tk * c.d * p.es);
  L.h = take(Tk * c.f * p.es);
  L.h_sh = take((size_t)c.n_shared * T * std::max(c.f_shared, 0) * p.es);
  L.y = take((size_t)p.ksplit * Tk * c.d * 4);
  L.y_sh = take((size_t)p.ksplit * c.n_shared * T * c.d * 4);
  L.lrank = take(Tk * 4);                          // fused router: task ranks within their tile
  L.tile_cnt = take((T + 127) / 128 * c.m * 4);    // and tasks per expert per 128-token tile
  L.idx2 = take(Tk * 4);                           // replica dispatch: experts after the split
  L.gmap = take((size_t)(c.m + 1) * 4);            // and the group -> weight matrix map
  L.lis2 = take(sizeof(moe_lis_t));
  L.total = off;
  return L;
}

template <typename Tp>
static Tp* at(void* ws, size_t off) {
  return reinterpret_cast<Tp*>(reinterpret_cast<char*>(ws) + off);
}

static moe_status_t check_cfg(const moe_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->d < 8 || c->f < 8 || c->m < 1 || c->k < 1) return MOE_ERR_INVALID_ARG;
  if (c->k > c->m) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_SWIGLU && c->act != MOE_RELU) return MOE_ERR_INVALID_ARG;
  if (c->renormalize != 0 && c->renormalize != 1) return MOE_ERR_INVALID_ARG;
  if (c->n_shared < 0 || (c->n_shared > 0 && c->f_shared < 8)) return MOE_ERR_INVALID_ARG;
  if (c->d % 8 || c->f % 8 || (c->n_shared && c->f_shared % 8)) return MOE_ERR_UNSUPPORTED;
  if (c->m > 1024 || c->k > 32 || c->n_shared > 8) return MOE_ERR_UNSUPPORTED;
  if ((long long)c->T * c->k >= (1LL << 31) / 2) return MOE_ERR_UNSUPPORTED;
  if (c->m + c->n_shared > tc_max_groups()) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

static moe_status_t check_ws(const moe_config_t& c, void* ws, size_t ws_bytes, size_t need) {
  (void)c;
  if (!ws || ((uintptr_t)ws & 255u)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

static moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                          \
  do {                                         \
    const moe_status_t st_ = (expr);           \
    if (st_ != MOE_OK) return st_;             \
  } while (0)
#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

// ------------------------------------------------------------------ building blocks

unsigned long long wait_limit_ns() { return g_wait_limit_ns; }

// Router logits (x W_r^T + bias, fp32) into `logits`, by the kernel that suits the
// batch; shared by the workspace entry points and moe_route_static.
cudaError_t launch_router_logits(const moe_config_t& c, const void* x, const void* w_r, const float* bias,
                                 float* logits, int* status, cudaStream_t s) {
  // Batches too small to fill the tensor cores (decode) and fp32 layers use CUDA cores.
  if (few_expert_logits_ok(c.dtype, c.T, c.m)) return launch_few_expert_logits(c.T, c.d, c.m, x, w_r, bias, logits, s);
  if (c.dtype == MOE_F32 || c.T <= 64) return launch_simt_logits(c.dtype, c.T, c.d, c.m, x, w_r, bias, logits, s);
  // logits^T = W_r . x^T on the tensor cores: one group, features = experts.
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  GemmClass& g = p.cls[0];
  g.n_groups = 1;
  g.R = c.m;
  g.K = c.d;
  g.ksplit = 1;
  g.kb_per_split = kblocks(c.d);
  g.const_rows = c.T;
  g.out = logits;
  g.out_ld = c.m;
  g.bias = bias;
  p.n_classes = 1;
  p.status = status;
  p.wait_limit_ns = g_wait_limit_ns;
  // Smallest token tile that still covers the batch in one wave of CTAs (each tile
  // re-reads all of W_r from L2, so fewer, larger tiles are cheaper).
  const long long mt = (c.m + 127) / 128;
  int bn = 16;
  while (bn < 128 && mt * ((c.T + bn - 1) / bn) > PLAN_SMS) bn <<= 1;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  maps.a0[0] = {w_r, c.m, c.d};
  maps.a1[0] = maps.a0[0];
  maps.b[0] = {x, c.T, c.d};
  const long long tiles = mt * ((c.T + bn - 1) / bn);
  const int ctas = (int)std::min<long long>(tiles, num_sms());
  return launch_tc_gemm(EPI_LOGITS, bn, maps, p, ctas, s);
}

// Everything moe_route computes on the device: logits (from x, or logits_in
// verbatim), top-k ids and gate weights, by the kernels that suit the batch.
// logits_out receives the logits when given; otherwise logits_scratch holds them
// where a kernel needs them in memory. With stage_marks, stage events 1 (logits)
// and 2 (top-k) are recorded (together when one kernel does both).
cudaError_t launch_route(const moe_config_t& c, const void* x, const void* w_r, const float* bias,
                         const float* logits_in, float* logits_out, float* logits_scratch, int32_t* idx, float* w,
                         int* status, cudaStream_t s, bool stage_marks) {
  cudaError_t e = cudaSuccess;
  const float* lg = logits_in;
  if (!lg && fused_route_ok(c)) {  // logits and top-k in one tensor-core launch
    e = launch_route_topk(c, x, w_r, bias, logits_out, idx, w, nullptr, nullptr, status, g_wait_limit_ns, s);
    if (e == cudaSuccess && stage_marks) e = mark_stage_event(1, s);
    if (e == cudaSuccess && stage_marks) e = mark_stage_event(2, s);
    return e;
  }
  if (!lg && small_route_ok(c.dtype, c.m)) {  // few experts: logits and top-k in one CUDA-core launch
    e = launch_small_route(c.T, c.d, c.m, c.k, c.renormalize, x, w_r, bias, logits_out, idx, w, s);
    if (e == cudaSuccess && stage_marks) e = mark_stage_event(1, s);
    if (e == cudaSuccess && stage_marks) e = mark_stage_event(2, s);
    return e;
  }
  if (!lg) {
    float* dst = logits_out ? logits_out : logits_scratch;
    if ((e = launch_router_logits(c, x, w_r, bias, dst, status, s)) != cudaSuccess) return e;
    lg = dst;
  } else if (logits_out && logits_out != logits_in) {
    if ((e = cudaMemcpyAsync(logits_out, logits_in, (size_t)c.T * c.m * 4, cudaMemcpyDeviceToDevice, s)) !=
        cudaSuccess)
      return e;
  }
  if (stage_marks && (e = mark_stage_event(1, s)) != cudaSuccess) return e;
  if ((e = launch_topk_softmax(c.T, c.m, c.k, c.renormalize, lg, idx, w, s)) != cudaSuccess) return e;
  if (stage_marks) e = mark_stage_event(2, s);
  return e;
}

// 8-bit expert path: the quantized weights and the per-row codes and scales of
// each projection's input (x_perm rows, h rows, and for shared experts x and h_sh).
struct Fp8Io {
  const moe_fp8_experts_t* w;
  uint8_t* xq;     // [T k, d]
  float* sx;       // [T k]
  uint8_t* hq;     // [T k, f]
  float* sh;       // [T k]
  uint8_t* xq_sh;  // [T, d]
  float* sx_sh;    // [T]
  uint8_t* hq_sh;  // [n_shared T, f_shared]
  float* sh_sh;    // [n_shared T]
};

static int kblocks8(int K) { return (K + 127) / 128; }

struct FfnIo {
  // routed class (may be absent: n_routed_groups == 0)
  int n_routed;           // groups (experts) of the routed class
  const int32_t* offsets; // device
  const void* x_perm;     // [rows, d]
  long long routed_rows;  // rows of x_perm / h / y (T k)
  const void *w_gate, *w_up, *w_down;
  void* h;
  float* y;
  const float* task_w;
  const int32_t* perm;
  const float* row_w;     // task_w already gathered into segment order (nullable)
  void* out_k1;           // top-1 layers: the down projection writes the layer output directly
  const int* group_map;   // device [n_routed]: weight matrix of each routed group (nullable = identity)
  int n_wgroups;          // routed weight matrices (== n_routed without a map)
  // shared class
  int n_shared;
  const void* x;          // [T, d]
  const void *ws_gate, *ws_up, *ws_down;
  void* h_sh;             // [n_shared T, f_shared]
  float* y_sh;            // [n_shared T, d]
  const Fp8Io* q8;        // 8-bit experts (nullable)
};

static void fill_common(GemmParams& p, int* status) {
  p.status = status;
  p.wait_limit_ns = g_wait_limit_ns;
}

static moe_status_t run_ffn(const moe_config_t& c, const Plan& pl, const FfnIo& io, int ksplit, int kbps, int* status,
                            cudaStream_t s, bool stage_marks = false) {
  const bool swiglu = c.act == MOE_SWIGLU;
  const bool tc = c.dtype == MOE_BF16;
  const Fp8Io* q8 = io.q8;
  auto kbl = [&](int K) { return q8 ? kblocks8(K) : kblocks(K); };
  if (q8) {  // E4M3 rows of the up projection's inputs
    MOE_CUDA(launch_quantize_e4m3(io.routed_rows, c.d, io.x_perm, c.d, q8->xq, c.d, q8->sx, s));
    if (io.n_shared > 0) MOE_CUDA(launch_quantize_e4m3(c.T, c.d, io.x, c.d, q8->xq_sh, c.d, q8->sx_sh, s));
  }
  // ---- up projection (+ activation): h = act(x W_gate^T [, x W_up^T])
  GemmParams up;
  std::memset(&up, 0, sizeof(up));
  fill_common(up, status);
  TcMaps mu;
  std::memset(&mu, 0, sizeof(mu));
  int ncls = 0;
  if (io.n_routed > 0) {
    GemmClass& g = up.cls[ncls];
    g.n_groups = io.n_routed;
    g.R = c.f;
    g.K = c.d;
    g.ksplit = 1;
    g.kb_per_split = kbl(c.d);
    g.seg_off = io.offsets;
    g.max_row = (int)io.routed_rows;
    g.out = io.h;
    g.out_ld = c.f;
    g.a0 = io.w_gate;
    g.a1 = swiglu ? io.w_up : nullptr;
    g.b = io.x_perm;
    g.a_ld = c.d;
    g.b_ld = c.d;
    g.group_map = io.group_map;
    g.n_wgroups = io.group_map ? io.n_wgroups : io.n_routed;
    mu.a0[ncls] = {io.w_gate, (long long)g.n_wgroups * c.f, c.d};
    mu.a1[ncls] = {swiglu ? io.w_up : io.w_gate, (long long)g.n_wgroups * c.f, c.d};
    mu.b[ncls] = {io.x_perm, io.routed_rows, c.d};
    if (q8) {
      mu.a0[ncls].ptr = q8->w->gate;
      mu.a1[ncls].ptr = swiglu ? q8->w->up : q8->w->gate;
      mu.b[ncls].ptr = q8->xq;
      g.a0_scale = q8->w->gate_scale;
      g.a1_scale = swiglu ? q8->w->up_scale : nullptr;
      g.b_scale = q8->sx;
    }
    ++ncls;
  }
  if (io.n_shared > 0) {
    GemmClass& g = up.cls[ncls];
    g.n_groups = io.n_shared;
    g.R = c.f_shared;
    g.K = c.d;
    g.ksplit = 1;
    g.kb_per_split = kbl(c.d);
    g.const_rows = c.T;
    g.b_group_stride = 0;
    g.out_group_stride = c.T;
    g.out = io.h_sh;
    g.out_ld = c.f_shared;
    g.a0 = io.ws_gate;
    g.a1 = swiglu ? io.ws_up : nullptr;
    g.b = io.x;
    g.a_ld = c.d;
    g.b_ld = c.d;
    mu.a0[ncls] = {io.ws_gate, (long long)io.n_shared * c.f_shared, c.d};
    mu.a1[ncls] = {swiglu ? io.ws_up : io.ws_gate, (long long)io.n_shared * c.f_shared, c.d};
    mu.b[ncls] = {io.x, c.T, c.d};
    if (q8) {
      mu.a0[ncls].ptr = q8->w->sh_gate;
      mu.a1[ncls].ptr = swiglu ? q8->w->sh_up : q8->w->sh_gate;
      mu.b[ncls].ptr = q8->xq_sh;
      g.a0_scale = q8->w->sh_gate_scale;
      g.a1_scale = swiglu ? q8->w->sh_up_scale : nullptr;
      g.b_scale = q8->sx_sh;
    }
    ++ncls;
  }
  if (ncls == 0) return MOE_OK;
  up.n_classes = ncls;
  const int epi_up = swiglu ? EPI_SWIGLU : EPI_RELU;
  const bool pair = tc && pl.pair && !q8 && ksplit == 1;  // two-CTA tiles: bf16 operands only
  if (tc)
    MOE_CUDA(launch_tc_gemm(epi_up, pair ? 256 : pl.bn_up, mu, up, num_sms(), s, q8 != nullptr, pair));
  else
    MOE_CUDA(launch_simt_gemm(epi_up, c.dtype, up, (int)std::min<long long>(io.routed_rows, 1LL << 30), s));
  if (stage_marks) MOE_TRY(mark_stage(5, s));
  if (q8) {  // E4M3 rows of the stored bf16 h
    MOE_CUDA(launch_quantize_e4m3(io.routed_rows, c.f, io.h, c.f, q8->hq, c.f, q8->sh, s));
    if (io.n_shared > 0)
      MOE_CUDA(launch_quantize_e4m3((long long)io.n_shared * c.T, c.f_shared, io.h_sh, c.f_shared, q8->hq_sh,
                                    c.f_shared, q8->sh_sh, s));
  }

  // ---- down projection: y = w * (h W_down^T), K split into `ksplit` partial outputs
  GemmParams dn;
  std::memset(&dn, 0, sizeof(dn));
  fill_common(dn, status);
  TcMaps md;
  std::memset(&md, 0, sizeof(md));
  ncls = 0;
  if (io.n_routed > 0) {
    GemmClass& g = dn.cls[ncls];
    g.n_groups = io.n_routed;
    g.R = c.d;
    g.K = c.f;
    g.ksplit = ksplit;
    g.kb_per_split = kbps;
    g.seg_off = io.offsets;
    g.max_row = (int)io.routed_rows;
    g.out = io.out_k1 ? io.out_k1 : io.y;
    g.scatter_k1 = io.out_k1 ? 1 : 0;
    g.out_ld = c.d;
    g.out_split_stride = io.routed_rows * c.d;
    g.task_w = io.task_w;
    g.row_w = io.row_w;
    g.perm = io.perm;
    g.a0 = io.w_down;
    g.b = io.h;
    g.a_ld = c.f;
    g.b_ld = c.f;
    g.group_map = io.group_map;
    g.n_wgroups = io.group_map ? io.n_wgroups : io.n_routed;
    md.a0[ncls] = {io.w_down, (long long)g.n_wgroups * c.d, c.f};
    md.b[ncls] = {io.h, io.routed_rows, c.f};
    if (q8) {
      md.a0[ncls].ptr = q8->w->down;
      md.b[ncls].ptr = q8->hq;
      g.a0_scale = q8->w->down_scale;
      g.b_scale = q8->sh;
    }
    md.a1[ncls] = md.a0[ncls];
    ++ncls;
  }
  if (io.n_shared > 0) {
    GemmClass& g = dn.cls[ncls];
    g.n_groups = io.n_shared;
    g.R = c.d;
    g.K = c.f_shared;
    g.ksplit = 1;
    g.kb_per_split = kbl(c.f_shared);
    g.const_rows = c.T;
    g.b_group_stride = c.T;
    g.out_group_stride = c.T;
    g.out = io.y_sh;
    g.out_ld = c.d;
    g.a0 = io.ws_down;
    g.b = io.h_sh;
    g.a_ld = c.f_shared;
    g.b_ld = c.f_shared;
    md.a0[ncls] = {io.ws_down, (long long)io.n_shared * c.d, c.f_shared};
    md.b[ncls] = {io.h_sh, (long long)io.n_shared * c.T, c.f_shared};
    if (q8) {
      md.a0[ncls].ptr = q8->w->sh_down;
      md.b[ncls].ptr = q8->hq_sh;
      g.a0_scale = q8->w->sh_down_scale;
      g.b_scale = q8->sh_sh;
    }
    md.a1[ncls] = md.a0[ncls];
    ++ncls;
  }
  dn.n_classes = ncls;
  // pair tiles of the down projection take two 256-row feature blocks per token tile
  // when d covers them and segments average 256+ rows (long K loops per tile, where
  // staging the token rows once for twice the MMA work keeps shared memory below its
  // limit); shorter segments keep one block per tile: twice the tiles to spread over
  // the pairs, and two accumulators, so the epilogue overlaps the next tile
  const bool long_segments = (double)c.T * c.k / c.m >= 256.0;
  const int epi_dn = pair && c.d >= 512 && long_segments ? EPI_DOWN_DUAL : EPI_DOWN;
  if (tc)
    return cuda_status(launch_tc_gemm(epi_dn, pair ? 256 : pl.bn_down, md, dn, num_sms(), s, q8 != nullptr, pair));
  return cuda_status(launch_simt_gemm(EPI_DOWN, c.dtype, dn, (int)std::min<long long>(io.routed_rows, 1LL << 30), s));
}

}  // namespace moe

using namespace moe;

// ====================================================================== C ABI
extern "C" {

moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  MOE_TRY(check_cfg(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_layout(*cfg, make_plan(*cfg)).total;
  return MOE_OK;
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                       const float* logits_in, float* logits_out, int32_t* topk_idx, float* topk_w, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  const Layout L = make_layout(c, make_plan(c));
  if (!topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!logits_in && (!x || !w_router)) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_router, (const void*)bias, (const void*)logits_in, (const void*)logits_out,
                        (const void*)topk_idx, (const void*)topk_w})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(c, ws, ws_bytes, L.logits + align256((size_t)c.T * c.m * 4)));
  MOE_TRY(check_device());
  return cuda_status(launch_route(c, x, w_router, bias, logits_in, logits_out, at<float>(ws, L.logits), topk_idx,
                                  topk_w, at<int>(ws, L.status), (cudaStream_t)stream, false));
}

moe_status_t moe_histogram_lis(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                               moe_lis_t* lis, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!topk_idx || !counts || !offsets) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{(const void*)topk_idx, (const void*)counts, (const void*)offsets, (const void*)lis})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(c, make_plan(c));
  MOE_TRY(check_ws(c, ws, ws_bytes, L.start + (size_t)8192 * 4));
  MOE_TRY(check_device());
  return cuda_status(launch_route_index(1, c.T, c.k, c.m, topk_idx, counts, offsets, lis, at<int32_t>(ws, L.start),
                                        at<int>(ws, L.status), (cudaStream_t)stream));
}

moe_status_t moe_lis_from_counts(int32_t m, int64_t tasks, const int32_t* counts, moe_lis_t* lis,
                                 moe_stream_t stream) {
  if (m < 1 || tasks < 1 || !counts || !lis) return MOE_ERR_INVALID_ARG;
  if (m > 1024) return MOE_ERR_UNSUPPORTED;
  if (((uintptr_t)counts & 3u) || !aligned16(lis)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_lis_from_counts(m, (long long)tasks, counts, lis, (cudaStream_t)stream));
}

moe_status_t moe_permute(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, const int32_t* offsets,
                         void* x_perm, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!x || !topk_idx || !offsets || !x_perm || !perm || !inv_perm) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, (const void*)topk_idx, (const void*)offsets, (const void*)x_perm, (const void*)perm,
                        (const void*)inv_perm})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(c, make_plan(c));
  MOE_TRY(check_ws(c, ws, ws_bytes, L.start + (size_t)8192 * 4));
  MOE_TRY(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  const long long Tk = (long long)c.T * c.k;
  // Tasks that get no valid position keep inv_perm = -1, so the row copy skips them.
  MOE_CUDA(cudaMemsetAsync(inv_perm, 0xFF, (size_t)Tk * 4, s));
  int32_t* start = at<int32_t>(ws, L.start);
  int* status = at<int>(ws, L.status);
  MOE_CUDA(launch_route_index(2, c.T, c.k, c.m, topk_idx, nullptr, const_cast<int32_t*>(offsets), nullptr, start,
                              status, s));
  MOE_CUDA(launch_rank(c.T, c.k, c.m, topk_idx, offsets, start, nullptr, perm, inv_perm, nullptr, status, s));
  return cuda_status(launch_permute_rows(c.dtype, (int)Tk, c.k, c.d, x, inv_perm, x_perm, s));
}

moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets, const void* w_gate,
                             const void* w_up, const void* w_down, const float* task_w, const int32_t* perm,
                             float* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!x_perm || !offsets || !w_gate || !w_down || !y_perm) return MOE_ERR_INVALID_ARG;
  if (c.act == MOE_SWIGLU && !w_up) return MOE_ERR_INVALID_ARG;
  if (task_w && !perm) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x_perm, (const void*)offsets, w_gate, w_up, w_down, (const void*)task_w, (const void*)perm,
                        (const void*)y_perm})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Plan pl = make_plan(c);
  const Layout L = make_layout(c, pl);
  MOE_TRY(check_ws(c, ws, ws_bytes, L.h + align256((size_t)c.T * c.k * c.f * pl.es)));
  MOE_TRY(check_device());
  FfnIo io;
  std::memset(&io, 0, sizeof(io));
  io.n_routed = c.m;
  io.offsets = offsets;
  io.x_perm = x_perm;
  io.routed_rows = (long long)c.T * c.k;
  io.w_gate = w_gate;
  io.w_up = w_up;
  io.w_down = w_down;
  io.h = at<void>(ws, L.h);
  io.y = y_perm;
  io.task_w = task_w;
  io.perm = perm;
  return run_ffn(c, pl, io, 1, kblocks(c.f), at<int>(ws, L.status), (cudaStream_t)stream);
}

moe_status_t moe_shared_ffn(const moe_config_t* cfg, const void* x, const void* ws_gate, const void* ws_up,
                            const void* ws_down, float* y_shared, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (c.n_shared == 0) return MOE_OK;
  if (!x || !ws_gate || !ws_down || !y_shared) return MOE_ERR_INVALID_ARG;
  if (c.act == MOE_SWIGLU && !ws_up) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, ws_gate, ws_up, ws_down, (const void*)y_shared})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Plan pl = make_plan(c);
  const Layout L = make_layout(c, pl);
  MOE_TRY(check_ws(c, ws, ws_bytes, L.h_sh + align256((size_t)c.n_shared * c.T * c.f_shared * pl.es)));
  MOE_TRY(check_device());
  FfnIo io;
  std::memset(&io, 0, sizeof(io));
  io.n_shared = c.n_shared;
  io.x = x;
  io.ws_gate = ws_gate;
  io.ws_up = ws_up;
  io.ws_down = ws_down;
  io.h_sh = at<void>(ws, L.h_sh);
  io.y_sh = y_shared;
  return run_ffn(c, pl, io, 1, kblocks(c.f), at<int>(ws, L.status), (cudaStream_t)stream);
}

moe_status_t moe_combine(const moe_config_t* cfg, const float* y_perm, const int32_t* inv_perm, const float* y_shared,
                         void* out, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!y_perm || !inv_perm || !out) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{(const void*)y_perm, (const void*)inv_perm, (const void*)y_shared, (const void*)out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_combine(c.dtype, c.T, c.d, c.k, 1, y_perm, 0, inv_perm, c.n_shared, y_shared, 0, out,
                                    (cudaStream_t)stream));
}

}  // extern "C"

// The 8-bit path's buffers, after the bf16 layer's workspace.
struct Fp8Layout {
  size_t xq, sx, hq, sh, xq_sh, sx_sh, hq_sh, sh_sh, total;
};

static Fp8Layout make_fp8_layout(const moe_config_t& c, size_t base) {
  Fp8Layout F;
  size_t off = base;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t Tk = (size_t)c.T * c.k;
  const size_t nsT = (size_t)c.n_shared * c.T;
  F.xq = take(Tk * c.d);
  F.sx = take(Tk * 4);
  F.hq = take(Tk * c.f);
  F.sh = take(Tk * 4);
  F.xq_sh = take(c.n_shared ? (size_t)c.T * c.d : 0);
  F.sx_sh = take(c.n_shared ? (size_t)c.T * 4 : 0);
  F.hq_sh = take(nsT * std::max(c.f_shared, 0));
  F.sh_sh = take(nsT * 4);
  F.total = off;
  return F;
}

// Route -> histogram/LIS -> permute -> expert FFN -> combine; the expert weights
// are bf16 (w_gate ...) or, with wq, E4M3 codes and scales.
static moe_status_t layer_forward_impl(const moe_config_t& c, const void* x, const void* w_router, const float* bias,
                                       const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                                       const void* ws_up, const void* ws_down, const moe_fp8_experts_t* wq, void* out,
                                       float* logits_out, int32_t* topk_idx_out, float* topk_w_out,
                                       int32_t* counts_out, moe_lis_t* lis_out, void* h_out, void* h_shared_out,
                                       int32_t* perm_out, int32_t* offsets_out, int32_t* inv_perm_out,
                                       void* x_perm_out, void* ws, cudaStream_t s) {
  const Plan pl = make_plan(c);
  const Layout L = make_layout(c, pl);
  int* status = at<int>(ws, L.status);
  float* logits = logits_out ? logits_out : at<float>(ws, L.logits);
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  float* w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  moe_lis_t* lis = lis_out ? lis_out : at<moe_lis_t>(ws, L.lis);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  const long long Tk = (long long)c.T * c.k;

  float* w_perm = at<float>(ws, L.w_perm);
  MOE_TRY(mark_stage(0, s));
  if (fused_route_ok(c)) {
    // router + top-k + per-tile counts and ranks in the GEMM epilogue, then one
    // kernel for offsets / LIS / permutation / row copy (stages 1-3 coincide)
    int32_t* lrank = at<int32_t>(ws, L.lrank);
    int32_t* tile_cnt = at<int32_t>(ws, L.tile_cnt);
    MOE_CUDA(launch_route_topk(c, x, w_router, bias, logits_out, idx, w, lrank, tile_cnt, status, g_wait_limit_ns, s));
    MOE_TRY(mark_stage(1, s));
    MOE_TRY(mark_stage(2, s));
    MOE_TRY(mark_stage(3, s));
    MOE_CUDA(launch_route_scatter(c.dtype, c.T, c.k, c.m, c.d, tile_cnt, idx, lrank, w, x, counts, offsets, lis, perm,
                                  inv_perm, w_perm, at<void>(ws, L.x_perm), status, s));
  } else {
    MOE_CUDA(launch_route(c, x, w_router, bias, nullptr, logits_out, logits, idx, w, status, s, true));
    int32_t* start = at<int32_t>(ws, L.start);
    MOE_CUDA(launch_route_index(1, c.T, c.k, c.m, idx, counts, offsets, lis, start, status, s));
    MOE_CUDA(launch_rank(c.T, c.k, c.m, idx, offsets, start, w, perm, inv_perm, w_perm, status, s));
    MOE_TRY(mark_stage(3, s));
    MOE_CUDA(launch_permute_rows(c.dtype, (int)Tk, c.k, c.d, x, inv_perm, at<void>(ws, L.x_perm), s));
  }
  MOE_TRY(mark_stage(4, s));
  FfnIo io;
  std::memset(&io, 0, sizeof(io));
  io.n_routed = c.m;
  io.offsets = offsets;
  io.x_perm = at<void>(ws, L.x_perm);
  io.routed_rows = Tk;
  io.w_gate = w_gate;
  io.w_up = w_up;
  io.w_down = w_down;
  io.h = at<void>(ws, L.h);
  io.y = at<float>(ws, L.y);
  io.task_w = w;
  io.row_w = w_perm;
  io.perm = perm;
  io.n_shared = c.n_shared;
  io.x = x;
  io.ws_gate = ws_gate;
  io.ws_up = ws_up;
  io.ws_down = ws_down;
  io.h_sh = at<void>(ws, L.h_sh);
  io.y_sh = at<float>(ws, L.y_sh);
  // K split of the down projection: the plan's, re-cut into 128-element k-blocks
  // for 8-bit operands (never more splits than the plan sized y for)
  int ksplit = pl.ksplit, kbps = pl.kbps;
  Fp8Io q8;
  if (wq) {
    const Fp8Layout F = make_fp8_layout(c, L.total);
    q8 = {wq,
          at<uint8_t>(ws, F.xq), at<float>(ws, F.sx), at<uint8_t>(ws, F.hq), at<float>(ws, F.sh),
          at<uint8_t>(ws, F.xq_sh), at<float>(ws, F.sx_sh), at<uint8_t>(ws, F.hq_sh), at<float>(ws, F.sh_sh)};
    io.q8 = &q8;
    const int kb = kblocks8(c.f);
    const int ks = std::min(pl.ksplit, kb);
    kbps = (kb + ks - 1) / ks;
    ksplit = (kb + kbps - 1) / kbps;
  }
  // Top-1 routing without shared experts: each token has exactly one weighted
  // expert output, so the down projection's epilogue scatters it straight into
  // `out` and the combine kernel (and the fp32 y_perm round trip) disappears.
  const bool fuse_combine = c.k == 1 && c.n_shared == 0 && ksplit == 1 && c.dtype == MOE_BF16;
  io.out_k1 = fuse_combine ? out : nullptr;
  MOE_TRY(run_ffn(c, pl, io, ksplit, kbps, status, s, true));
  MOE_TRY(mark_stage(6, s));
  // inspection copies (the stored h rows and the task of each segment row)
  if (h_out) MOE_CUDA(cudaMemcpyAsync(h_out, io.h, (size_t)Tk * c.f * 2, cudaMemcpyDeviceToDevice, s));
  if (h_shared_out && c.n_shared > 0)
    MOE_CUDA(cudaMemcpyAsync(h_shared_out, io.h_sh, (size_t)c.n_shared * c.T * c.f_shared * 2,
                             cudaMemcpyDeviceToDevice, s));
  if (perm_out) MOE_CUDA(cudaMemcpyAsync(perm_out, perm, (size_t)Tk * 4, cudaMemcpyDeviceToDevice, s));
  if (inv_perm_out) MOE_CUDA(cudaMemcpyAsync(inv_perm_out, inv_perm, (size_t)Tk * 4, cudaMemcpyDeviceToDevice, s));
  if (offsets_out)
    MOE_CUDA(cudaMemcpyAsync(offsets_out, offsets, (size_t)(c.m + 1) * 4, cudaMemcpyDeviceToDevice, s));
  if (x_perm_out)
    MOE_CUDA(cudaMemcpyAsync(x_perm_out, io.x_perm, (size_t)Tk * c.d * pl.es, cudaMemcpyDeviceToDevice, s));
  if (!fuse_combine)
    MOE_CUDA(launch_combine(c.dtype, c.T, c.d, c.k, ksplit, io.y, Tk * c.d, inv_perm, c.n_shared, io.y_sh,
                            (long long)c.n_shared * c.T * c.d, out, s));
  return mark_stage(7, s);
}

extern "C" {

moe_status_t moe_layer_forward(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                               const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                               const void* ws_up, const void* ws_down, void* out, float* logits_out,
                               int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, moe_lis_t* lis_out,
                               int32_t* offsets_out, int32_t* perm_out, int32_t* inv_perm_out, void* x_perm_out,
                               void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!x || !w_router || !w_gate || !w_down || !out) return MOE_ERR_INVALID_ARG;
  if (c.act == MOE_SWIGLU && !w_up) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!ws_gate || !ws_down || (c.act == MOE_SWIGLU && !ws_up))) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_router, (const void*)bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out,
                        (const void*)logits_out, (const void*)topk_idx_out, (const void*)topk_w_out,
                        (const void*)counts_out, (const void*)lis_out, (const void*)offsets_out,
                        (const void*)perm_out, (const void*)inv_perm_out, x_perm_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_ws(c, ws, ws_bytes, make_layout(c, make_plan(c)).total));
  MOE_TRY(check_device());
  return layer_forward_impl(c, x, w_router, bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, nullptr, out,
                            logits_out, topk_idx_out, topk_w_out, counts_out, lis_out, nullptr, nullptr, perm_out,
                            offsets_out, inv_perm_out, x_perm_out, ws, (cudaStream_t)stream);
}

static moe_status_t check_fp8_cfg(const moe_config_t* cfg) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (c.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c.d % 16 || c.f % 16 || (c.n_shared && c.f_shared % 16)) return MOE_ERR_UNSUPPORTED;  // 16-byte code rows
  return MOE_OK;
}

moe_status_t moe_fp8_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  MOE_TRY(check_fp8_cfg(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_fp8_layout(*cfg, make_layout(*cfg, make_plan(*cfg)).total).total;
  return MOE_OK;
}

moe_status_t moe_quantize_e4m3(int64_t rows, int64_t cols, const void* src, uint8_t* codes, float* scales,
                               moe_stream_t stream) {
  if (rows < 0 || cols < 8 || cols % 16 || cols > (1LL << 30)) return rows < 0 || cols < 8 ? MOE_ERR_INVALID_ARG
                                                                                          : MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!src || !codes || !scales || !aligned16(src) || !aligned16(codes) || ((uintptr_t)scales & 3u))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_quantize_e4m3(rows, (int)cols, src, cols, codes, cols, scales, (cudaStream_t)stream));
}

moe_status_t moe_layer_forward_fp8(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                                   const moe_fp8_experts_t* wq, void* out, float* logits_out, int32_t* topk_idx_out,
                                   float* topk_w_out, int32_t* counts_out, moe_lis_t* lis_out, void* h_out,
                                   void* h_shared_out, int32_t* perm_out, void* ws, size_t ws_bytes,
                                   moe_stream_t stream) {
  MOE_TRY(check_fp8_cfg(cfg));
  const moe_config_t& c = *cfg;
  const bool swiglu = c.act == MOE_SWIGLU;
  if (!x || !w_router || !wq || !out) return MOE_ERR_INVALID_ARG;
  if (!wq->gate || !wq->gate_scale || !wq->down || !wq->down_scale) return MOE_ERR_INVALID_ARG;
  if (swiglu && (!wq->up || !wq->up_scale)) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!wq->sh_gate || !wq->sh_gate_scale || !wq->sh_down || !wq->sh_down_scale ||
                         (swiglu && (!wq->sh_up || !wq->sh_up_scale))))
    return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_router, (const void*)bias, out, (const void*)logits_out,
                        (const void*)topk_idx_out, (const void*)topk_w_out, (const void*)counts_out,
                        (const void*)lis_out, wq->gate, wq->up, wq->down, wq->sh_gate, wq->sh_up, wq->sh_down,
                        h_out, h_shared_out, (const void*)perm_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  for (const float* p : {wq->gate_scale, wq->up_scale, wq->down_scale, wq->sh_gate_scale, wq->sh_up_scale,
                         wq->sh_down_scale})
    if (p && ((uintptr_t)p & 3u)) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  MOE_TRY(moe_fp8_workspace_size(cfg, &need));
  MOE_TRY(check_ws(c, ws, ws_bytes, need));
  MOE_TRY(check_device());
  return layer_forward_impl(c, x, w_router, bias, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, wq, out,
                            logits_out, topk_idx_out, topk_w_out, counts_out, lis_out, h_out, h_shared_out, perm_out,
                            nullptr, nullptr, nullptr, ws, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ atomic experts
static moe_status_t check_atomic_cfg(const moe_atomic_config_t* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->d < 8 || c->Nr < 1 || c->Nc < 1 || c->K < 1) return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_ATOMIC_SILU && c->act != MOE_ATOMIC_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if ((long long)c->K > (long long)c->Nr * c->Nc) return MOE_ERR_INVALID_ARG;
  if (c->d % 8 || c->Nr % 8 || c->Nc % 8 || c->Nr < 64 || c->Nc < 64 || c->Nr > 1024 || c->Nc > 1024 || c->K > 4096)
    return MOE_ERR_UNSUPPORTED;
  if (c->T > 65535) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct AtomicPlan {
  int ksplit, kbps;
  size_t status, zr, zc, idx, g, coef, bar, sort, total;
};

static AtomicPlan make_atomic_plan(const moe_atomic_config_t& c) {
  AtomicPlan p;
  const long long tiles = (long long)((c.Nr + 127) / 128 + (c.Nc + 127) / 128) * ((c.T + 15) / 16);
  int ks = (int)std::min<long long>(16, std::max<long long>(1, (PLAN_SMS + tiles - 1) / tiles));
  ks = std::min(ks, kblocks(c.d));
  p.kbps = (kblocks(c.d) + ks - 1) / ks;
  p.ksplit = (kblocks(c.d) + p.kbps - 1) / p.kbps;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  p.status = take(256);
  p.zr = take((size_t)p.ksplit * c.T * c.Nr * 4);
  p.zc = take((size_t)p.ksplit * c.T * c.Nc * 4);
  p.idx = take((size_t)c.T * c.K * 4);
  p.g = take((size_t)c.T * c.K * 4);
  p.coef = take((size_t)c.T * c.K * 4);
  p.bar = take(256);  // grid-barrier word of the experts kernel
  const long long tasks = (long long)c.T * c.K;
  // prefill budgets: the counting sort of the tasks by expert (run ends, then the order)
  p.sort = tasks >= ATOMIC_WIDE_MIN_TASKS ? take(((size_t)c.Nr * c.Nc + (size_t)tasks) * 4) : 0;
  p.total = off;
  return p;
}

moe_status_t moe_atomic_workspace_size(const moe_atomic_config_t* cfg, size_t* bytes) {
  MOE_TRY(check_atomic_cfg(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = make_atomic_plan(*cfg).total;
  return MOE_OK;
}

static moe_status_t atomic_route_impl(const moe_atomic_config_t& c, const AtomicPlan& P, const void* x,
                                      const void* w_row, const void* w_col, float* lr_out, float* lc_out,
                                      int32_t* idx, float* g, void* ws, cudaStream_t s, bool stage_marks = false) {
  int* status = at<int>(ws, P.status);
  float* zr = at<float>(ws, P.zr);
  float* zc = at<float>(ws, P.zc);
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, status);
  p.n_classes = 2;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  for (int side = 0; side < 2; ++side) {
    GemmClass& gc = p.cls[side];
    const int n = side ? c.Nc : c.Nr;
    gc.n_groups = 1;
    gc.R = n;
    gc.K = c.d;
    gc.ksplit = P.ksplit;
    gc.kb_per_split = P.kbps;
    gc.const_rows = c.T;
    gc.out = side ? zc : zr;
    gc.out_ld = n;
    gc.out_split_stride = (long long)c.T * n;
    maps.a0[side] = {side ? w_col : w_row, n, c.d};
    maps.a1[side] = maps.a0[side];
    maps.b[side] = {x, c.T, c.d};
  }
  const int bn = c.T <= 16 ? 16 : c.T <= 32 ? 32 : c.T <= 64 ? 64 : 128;
  MOE_CUDA(launch_tc_gemm(EPI_LOGITS, bn, maps, p, num_sms(), s));
  if (stage_marks) MOE_TRY(mark_stage(1, s));
  MOE_CUDA(launch_atomic_select(c.T, c.Nr, c.Nc, c.K, P.ksplit, zr, (long long)c.T * c.Nr, zc, (long long)c.T * c.Nc,
                                lr_out, lc_out, idx, g, status, at<unsigned>(ws, P.bar), s));
  if (stage_marks) MOE_TRY(mark_stage(2, s));
  return MOE_OK;
}

moe_status_t moe_atomic_route(const moe_atomic_config_t* cfg, const void* x, const void* w_row, const void* w_col,
                              float* row_logp_out, float* col_logp_out, int32_t* idx_out, float* g_out, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_atomic_cfg(cfg));
  const moe_atomic_config_t& c = *cfg;
  if (!x || !w_row || !w_col || !idx_out || !g_out) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_row, w_col, (const void*)row_logp_out, (const void*)col_logp_out, (const void*)idx_out,
                        (const void*)g_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const AtomicPlan P = make_atomic_plan(c);
  if (!ws || ((uintptr_t)ws & 255u)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < P.total) return MOE_ERR_WORKSPACE;
  MOE_TRY(check_device());
  return atomic_route_impl(c, P, x, w_row, w_col, row_logp_out, col_logp_out, idx_out, g_out, ws,
                           (cudaStream_t)stream);
}

moe_status_t moe_atomic_experts(const moe_atomic_config_t* cfg, const void* x, const void* w_in, const void* w_out,
                                const int32_t* idx, const float* g, void* out, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  MOE_TRY(check_atomic_cfg(cfg));
  const moe_atomic_config_t& c = *cfg;
  if (!x || !w_in || !w_out || !idx || !g || !out) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_in, w_out, (const void*)idx, (const void*)g, out})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  const AtomicPlan P = make_atomic_plan(c);
  if (!ws || ((uintptr_t)ws & 255u)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < P.total) return MOE_ERR_WORKSPACE;
  MOE_TRY(check_device());
  return cuda_status(launch_atomic_experts_sorted(c.T, c.d, c.K, c.act, x, w_in, w_out, idx, g, at<float>(ws, P.coef), out,
                                           (long long)c.Nr * c.Nc, at<unsigned>(ws, P.bar), false, g_wait_limit_ns,
                                           at<int>(ws, P.status), P.sort ? at<int32_t>(ws, P.sort) : nullptr,
                                           (cudaStream_t)stream));
}

moe_status_t moe_atomic_forward(const moe_atomic_config_t* cfg, const void* x, const void* w_row, const void* w_col,
                                const void* w_in, const void* w_out, void* out, int32_t* idx_out, float* g_out,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_atomic_cfg(cfg));
  const moe_atomic_config_t& c = *cfg;
  if (!x || !w_row || !w_col || !w_in || !w_out || !out) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_row, w_col, w_in, w_out, out, (const void*)idx_out, (const void*)g_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const AtomicPlan P = make_atomic_plan(c);
  if (!ws || ((uintptr_t)ws & 255u)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < P.total) return MOE_ERR_WORKSPACE;
  MOE_TRY(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, P.idx);
  float* g = g_out ? g_out : at<float>(ws, P.g);
  MOE_TRY(mark_stage(0, s));
  MOE_TRY(atomic_route_impl(c, P, x, w_row, w_col, nullptr, nullptr, idx, g, ws, s, true));
  // the select kernel cleared the barrier word; the experts kernel is one launch
  MOE_CUDA(launch_atomic_experts_sorted(c.T, c.d, c.K, c.act, x, w_in, w_out, idx, g, at<float>(ws, P.coef), out,
                                 (long long)c.Nr * c.Nc, at<unsigned>(ws, P.bar), true, g_wait_limit_ns,
                                 at<int>(ws, P.status), P.sort ? at<int32_t>(ws, P.sort) : nullptr, s));
  MOE_TRY(mark_stage(3, s));
  return mark_stage(4, s);
}

// ------------------------------------------------------------------ R&Q replica dispatch
moe_status_t moe_replica_split(const moe_config_t* cfg, const int32_t* topk_idx, const int32_t* offsets,
                               const int32_t* inv_perm, const moe_lis_t* lis, int32_t* idx_out, int32_t* counts_out,
                               moe_lis_t* lis_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!topk_idx || !offsets || !inv_perm || !lis || !idx_out) return MOE_ERR_INVALID_ARG;
  if (c.m + 1 > 1024) return MOE_ERR_UNSUPPORTED;  // the replica is expert m
  for (const void* p : std::initializer_list<const void*>{(const void*)topk_idx, (const void*)offsets,
                                                          (const void*)inv_perm, (const void*)lis, (const void*)idx_out,
                                                          (const void*)counts_out, (const void*)lis_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(c, make_plan(c));
  MOE_TRY(check_ws(c, ws, ws_bytes, L.total));
  MOE_TRY(check_device());
  return cuda_status(launch_replica_split(c.T, c.k, c.m, topk_idx, offsets, inv_perm, lis, idx_out,
                                          at<int32_t>(ws, L.gmap), counts_out, lis_out, at<int>(ws, L.status),
                                          (cudaStream_t)stream));
}

moe_status_t moe_layer_forward_replicated(const moe_config_t* cfg, const void* x, const void* w_router,
                                          const float* bias, const void* w_gate, const void* w_up, const void* w_down,
                                          const void* ws_gate, const void* ws_up, const void* ws_down, void* out,
                                          float* logits_out, int32_t* topk_idx_out, float* topk_w_out,
                                          int32_t* dispatch_idx_out, int32_t* counts_out, moe_lis_t* lis_before_out,
                                          moe_lis_t* lis_after_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(check_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (c.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  moe_config_t c1 = c;  // the layer after the split: m + 1 routed groups
  c1.m = c.m + 1;
  MOE_TRY(check_cfg(&c1));
  if (!x || !w_router || !w_gate || !w_down || !out) return MOE_ERR_INVALID_ARG;
  if (c.act == MOE_SWIGLU && !w_up) return MOE_ERR_INVALID_ARG;
  if (c.n_shared > 0 && (!ws_gate || !ws_down || (c.act == MOE_SWIGLU && !ws_up))) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{
           x, w_router, (const void*)bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, out, (const void*)logits_out,
           (const void*)topk_idx_out, (const void*)topk_w_out, (const void*)dispatch_idx_out, (const void*)counts_out,
           (const void*)lis_before_out, (const void*)lis_after_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Plan pl = make_plan(c1);
  const Layout L = make_layout(c1, pl);
  MOE_TRY(check_ws(c1, ws, ws_bytes, L.total));
  MOE_TRY(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  int* status = at<int>(ws, L.status);
  float* logits = logits_out ? logits_out : at<float>(ws, L.logits);
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  float* w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  moe_lis_t* lis0 = lis_before_out ? lis_before_out : at<moe_lis_t>(ws, L.lis);
  moe_lis_t* lis1 = lis_after_out ? lis_after_out : at<moe_lis_t>(ws, L.lis2);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  float* w_perm = at<float>(ws, L.w_perm);
  int32_t* start = at<int32_t>(ws, L.start);
  int32_t* idx2 = dispatch_idx_out ? dispatch_idx_out : at<int32_t>(ws, L.idx2);
  int32_t* gmap = at<int32_t>(ws, L.gmap);
  const long long Tk = (long long)c.T * c.k;

  // 1. router and top-k over the m experts (stage events as in moe_layer_forward)
  MOE_TRY(mark_stage(0, s));
  MOE_CUDA(launch_route(c, x, w_router, bias, nullptr, logits_out, logits, idx, w, status, s, true));
  // 2. histogram / LIS and the stable ranks over the m experts (the heavy-hitter's
  //    segment order is the split order)
  MOE_CUDA(launch_route_index(1, c.T, c.k, c.m, idx, counts, offsets, lis0, start, status, s));
  MOE_CUDA(launch_rank(c.T, c.k, c.m, idx, offsets, start, nullptr, perm, inv_perm, nullptr, status, s));
  // 3. every second task of the heavy-hitter to the replica, expert m
  MOE_CUDA(launch_replica_split(c.T, c.k, c.m, idx, offsets, inv_perm, lis0, idx2, gmap, nullptr, nullptr, status, s));
  // 4. histogram / LIS, ranks and rows over the m + 1 experts
  int32_t* counts1 = counts_out ? counts_out : counts;
  MOE_CUDA(launch_route_index(1, c.T, c.k, c1.m, idx2, counts1, offsets, lis1, start, status, s));
  MOE_CUDA(launch_rank(c.T, c.k, c1.m, idx2, offsets, start, w, perm, inv_perm, w_perm, status, s));
  MOE_TRY(mark_stage(3, s));
  MOE_CUDA(launch_permute_rows(c.dtype, (int)Tk, c.k, c.d, x, inv_perm, at<void>(ws, L.x_perm), s));
  MOE_TRY(mark_stage(4, s));
  // 5. the grouped FFN over m + 1 groups; group m reads the heavy-hitter's weights
  FfnIo io;
  std::memset(&io, 0, sizeof(io));
  io.n_routed = c1.m;
  io.offsets = offsets;
  io.x_perm = at<void>(ws, L.x_perm);
  io.routed_rows = Tk;
  io.w_gate = w_gate;
  io.w_up = w_up;
  io.w_down = w_down;
  io.h = at<void>(ws, L.h);
  io.y = at<float>(ws, L.y);
  io.task_w = w;
  io.row_w = w_perm;
  io.perm = perm;
  io.group_map = gmap;
  io.n_wgroups = c.m;
  io.n_shared = c.n_shared;
  io.x = x;
  io.ws_gate = ws_gate;
  io.ws_up = ws_up;
  io.ws_down = ws_down;
  io.h_sh = at<void>(ws, L.h_sh);
  io.y_sh = at<float>(ws, L.y_sh);
  const bool fuse_combine = c.k == 1 && c.n_shared == 0 && pl.ksplit == 1;
  io.out_k1 = fuse_combine ? out : nullptr;
  MOE_TRY(run_ffn(c1, pl, io, pl.ksplit, pl.kbps, status, s, true));
  MOE_TRY(mark_stage(6, s));
  if (!fuse_combine)
    MOE_CUDA(launch_combine(c.dtype, c.T, c.d, c.k, pl.ksplit, io.y, Tk * c.d, inv_perm, c.n_shared, io.y_sh,
                            (long long)c.n_shared * c.T * c.d, out, s));
  return mark_stage(7, s);
}

// ------------------------------------------------------------------ FloE contextual sparsity
struct FloeLayout {
  size_t u, list, cnt, rsplit, y, total;
  int slots;
};

static FloeLayout make_floe_layout(const moe_config_t& c, size_t base) {
  FloeLayout F;
  size_t off = base;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t Tk = (size_t)c.T * c.k;
  const size_t nch = (size_t)floe_chunks(c.f);
  F.u = take(Tk * c.f * 4);
  F.list = take((size_t)c.m * nch * floe_chunk_size() * 4);
  F.cnt = take((size_t)c.m * nch * 4);
  F.rsplit = take(Tk * 4);
  F.slots = floe_max_slots((long long)Tk, c.d);
  F.y = take((size_t)F.slots * Tk * c.d * 4);  // partial outputs of the kept-channel ranges
  F.total = off;
  return F;
}

static moe_status_t check_floe_cfg(const moe_config_t* cfg) {
  MOE_TRY(check_cfg(cfg));
  if (cfg->dtype != MOE_BF16 || cfg->act != MOE_SWIGLU || cfg->n_shared != 0) return MOE_ERR_UNSUPPORTED;
  if (!floe_shape_ok(cfg->d, cfg->f)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t moe_floe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
  MOE_TRY(check_floe_cfg(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(*cfg, make_plan(*cfg));
  *bytes = make_floe_layout(*cfg, L.total).total;
  return MOE_OK;
}

moe_status_t moe_floe_pack_down(const moe_config_t* cfg, const void* w_down, void* w_down_t, moe_stream_t stream) {
  MOE_TRY(check_floe_cfg(cfg));
  if (!w_down || !w_down_t || !aligned16(w_down) || !aligned16(w_down_t)) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_floe_pack(cfg->m, cfg->d, cfg->f, w_down, w_down_t, (cudaStream_t)stream));
}

moe_status_t moe_floe_calibrate(const moe_config_t* cfg, const void* x_calib, int32_t T_calib, const void* w_up,
                                double sparsity, float* u_scratch, float* thresholds_out, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  MOE_TRY(check_floe_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!x_calib || !w_up || !u_scratch || !thresholds_out || T_calib < 1) return MOE_ERR_INVALID_ARG;
  if (!(sparsity >= 0.0 && sparsity <= 1.0)) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x_calib, w_up, (const void*)u_scratch,
                                                          (const void*)thresholds_out})
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  if ((long long)c.m * c.f > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  const Layout L = make_layout(c, make_plan(c));
  MOE_TRY(check_ws(c, ws, ws_bytes, L.total));
  MOE_TRY(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  // u[t][e f + j] = x_calib[t] . W_up[e][j] for every expert: one tensor-core group
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, at<int>(ws, L.status));
  GemmClass& g = p.cls[0];
  g.n_groups = 1;
  g.R = c.m * c.f;
  g.K = c.d;
  g.ksplit = 1;
  g.kb_per_split = kblocks(c.d);
  g.const_rows = T_calib;
  g.out = u_scratch;
  g.out_ld = (long long)c.m * c.f;
  p.n_classes = 1;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  maps.a0[0] = {w_up, (long long)c.m * c.f, c.d};
  maps.a1[0] = maps.a0[0];
  maps.b[0] = {x_calib, T_calib, c.d};
  int bn = 16;
  while (bn < 128 && bn < T_calib) bn <<= 1;
  MOE_CUDA(launch_tc_gemm(EPI_LOGITS, bn, maps, p, num_sms(), s));
  return cuda_status(launch_floe_calib(T_calib, c.m, c.f, u_scratch, sparsity, thresholds_out, s));
}

moe_status_t moe_layer_forward_floe(const moe_config_t* cfg, const void* x, const void* w_router, const float* bias,
                                    const void* w_gate, const void* w_up, const void* w_down_t,
                                    const float* thresholds, void* out, int32_t* topk_idx_out, float* topk_w_out,
                                    int32_t* kept_out, float* u_out, int32_t* perm_out, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  MOE_TRY(check_floe_cfg(cfg));
  const moe_config_t& c = *cfg;
  if (!x || !w_router || !w_gate || !w_up || !w_down_t || !thresholds || !out) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{
           x, w_router, (const void*)bias, w_gate, w_up, w_down_t, (const void*)thresholds, out,
           (const void*)topk_idx_out, (const void*)topk_w_out, (const void*)kept_out, (const void*)u_out,
           (const void*)perm_out})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Plan pl = make_plan(c);
  const Layout L = make_layout(c, pl);
  const FloeLayout F = make_floe_layout(c, L.total);
  MOE_TRY(check_ws(c, ws, ws_bytes, F.total));
  MOE_TRY(check_device());
  cudaStream_t s = (cudaStream_t)stream;
  int* status = at<int>(ws, L.status);
  float* logits = at<float>(ws, L.logits);
  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  float* w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv_perm = at<int32_t>(ws, L.inv_perm);
  float* w_perm = at<float>(ws, L.w_perm);
  int32_t* start = at<int32_t>(ws, L.start);
  void* x_perm = at<void>(ws, L.x_perm);
  float* u = at<float>(ws, F.u);
  float* y = at<float>(ws, F.y);
  const long long Tk = (long long)c.T * c.k;
  // route and sort as in moe_layer_forward (stages 0-4)
  MOE_TRY(mark_stage(0, s));
  MOE_CUDA(launch_route(c, x, w_router, bias, nullptr, nullptr, logits, idx, w, status, s, true));
  MOE_CUDA(launch_route_index(1, c.T, c.k, c.m, idx, at<int32_t>(ws, L.counts), offsets, at<moe_lis_t>(ws, L.lis),
                              start, status, s));
  MOE_CUDA(launch_rank(c.T, c.k, c.m, idx, offsets, start, w, perm, inv_perm, w_perm, status, s));
  MOE_TRY(mark_stage(3, s));
  MOE_CUDA(launch_permute_rows(c.dtype, (int)Tk, c.k, c.d, x, inv_perm, x_perm, s));
  MOE_TRY(mark_stage(4, s));
  // dense up projection u = x W_up^T per segment (fp32, tensor cores)
  GemmParams up;
  std::memset(&up, 0, sizeof(up));
  fill_common(up, status);
  GemmClass& g = up.cls[0];
  g.n_groups = c.m;
  g.R = c.f;
  g.K = c.d;
  g.ksplit = 1;
  g.kb_per_split = kblocks(c.d);
  g.seg_off = offsets;
  g.max_row = (int)Tk;
  g.out = u;
  g.out_ld = c.f;
  up.n_classes = 1;
  TcMaps mu;
  std::memset(&mu, 0, sizeof(mu));
  mu.a0[0] = {w_up, (long long)c.m * c.f, c.d};
  mu.a1[0] = mu.a0[0];
  mu.b[0] = {x_perm, Tk, c.d};
  MOE_CUDA(launch_tc_gemm(EPI_LOGITS, tc_pick_bn(EPI_LOGITS, (double)Tk / c.m), mu, up, num_sms(), s));
  MOE_TRY(mark_stage(5, s));
  // kept channels, gate rows and down rows of the kept channels only
  int32_t* rsplit = at<int32_t>(ws, F.rsplit);
  MOE_CUDA(launch_floe_sparse_ffn(c.m, c.d, c.f, offsets, x_perm, w_gate, w_down_t, u, thresholds,
                                  at<int32_t>(ws, F.list), at<int32_t>(ws, F.cnt), w_perm, y, Tk * c.d, F.slots,
                                  rsplit, kept_out, status, g_wait_limit_ns, s));
  MOE_TRY(mark_stage(6, s));
  MOE_CUDA(launch_combine(c.dtype, c.T, c.d, c.k, F.slots, y, Tk * c.d, inv_perm, 0, nullptr, 0, out, s, rsplit));
  if (u_out) MOE_CUDA(cudaMemcpyAsync(u_out, u, (size_t)Tk * c.f * 4, cudaMemcpyDeviceToDevice, s));
  if (perm_out) MOE_CUDA(cudaMemcpyAsync(perm_out, perm, (size_t)Tk * 4, cudaMemcpyDeviceToDevice, s));
  return mark_stage(7, s);
}

// ------------------------------------------------------------------ status helpers
moe_status_t moe_read_device_status(void* ws, moe_stream_t stream, moe_status_t* out) {
  if (!ws || !out) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  *out = (moe_status_t)v;
  return MOE_OK;
}

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_INDEX: return "expert index or position out of range (device)";
  }
  return "unknown status";
}

moe_status_t moe_debug_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns ? (unsigned long long)ns : 2000ull * 1000 * 1000;
  return MOE_OK;
}

moe_status_t moe_debug_set_barrier_extra(uint32_t n) {
  set_grid_barrier_extra(n);
  return MOE_OK;
}

moe_status_t moe_set_stage_events(void* const* events, int n) {
  if (n < 0 || (n > 0 && !events)) return MOE_ERR_INVALID_ARG;
  g_n_stage_events = std::min(n, 8);
  for (int i = 0; i < g_n_stage_events; ++i) g_stage_events[i] = (cudaEvent_t)events[i];
  return MOE_OK;
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

}  // extern "C"
