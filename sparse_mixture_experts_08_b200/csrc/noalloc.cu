// moe_route_static: the router (logits -> top-k -> gate weights) for callers that
// cannot hand the library a workspace.
//
// Some callers have no way to obtain device memory for scratch: plugins that only
// ever see the tensors a host framework gives them (the framework owns the
// allocator and hands out no extra buffers), and serving loops that forbid
// allocation on the request path (an allocation can block, fragment the pool or
// fail under memory pressure at the worst moment). moe_route needs scratch for the
// intermediate router logits (when the caller does not want them) and for the
// device status word; this entry point keeps both in a fixed array compiled into
// the library instead, and allocates nothing.
//
// Limits and sharing:
//  - The array holds MOE_STATIC_SCRATCH_BYTES (8 MiB) on every GPU that loads the
//    library, for the life of the process: the status word plus at most
//    (8 MiB - 256 B) / 4 router logits, i.e. T * m <= 2,097,088 when neither
//    logits_in nor logits_out is given. Larger calls are rejected with
//    MOE_ERR_WORKSPACE before anything is launched.
//  - All calls on a device share the one array and it keeps whatever the last
//    call left in it; the status word is cleared at the start of every call.
//    Calls whose work overlaps on the GPU (different streams without ordering
//    between them) race on the array: order them on one stream.
//  - The first call on each device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current); make that first call
//    before starting any stream capture.
//  - The device work is moe_route's (one shared launcher: the same choice of
//    router kernels, the same bounded-wait limit), so both give identical results.
#include <initializer_list>

#include "common.cuh"

namespace moe {

constexpr size_t MOE_STATIC_SCRATCH_BYTES = 8u << 20;
constexpr size_t STATIC_STATUS_BYTES = 256;  // status word, padded so the logits stay 256-byte aligned

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int MAX_DEVICES = 64;
unsigned char* g_scratch_ptr[MAX_DEVICES] = {nullptr};

// Device address of g_static_scratch on the current device (looked up once per
// device). In host code the array's name is only a host-side handle.
moe_status_t scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return MOE_ERR_CUDA;
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<unsigned char*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

moe_status_t device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  return (major == 10 && minor == 0) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API moe_status_t moe_route_static(const moe_config_t* cfg, const void* x, const void* w_router,
                                                 const float* bias, const float* logits_in, float* logits_out,
                                                 int32_t* topk_idx, float* topk_w, int32_t* device_status_out,
                                                 moe_stream_t stream) {
  size_t unused = 0;
  const moe_status_t cfg_ok = moe_workspace_size(cfg, &unused);  // full config validation
  if (cfg_ok != MOE_OK) return cfg_ok;
  const moe_config_t& c = *cfg;
  if (!topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!logits_in && (!x || !w_router)) return MOE_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{x, w_router, bias, logits_in, logits_out, topk_idx, topk_w})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (device_status_out && ((uintptr_t)device_status_out & 3u)) return MOE_ERR_INVALID_ARG;
  const size_t logits_bytes = (size_t)c.T * c.m * sizeof(float);
  const bool need_logits_scratch = !logits_in && !logits_out;
  if (need_logits_scratch && logits_bytes > MOE_STATIC_SCRATCH_BYTES - STATIC_STATUS_BYTES) return MOE_ERR_WORKSPACE;
  moe_status_t st = device_is_sm100();
  if (st != MOE_OK) return st;
  unsigned char* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != MOE_OK) return st;

  cudaStream_t s = (cudaStream_t)stream;
  int* status = reinterpret_cast<int*>(scratch);
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_route(c, x, w_router, bias, logits_in, logits_out,
                   reinterpret_cast<float*>(scratch + STATIC_STATUS_BYTES), topk_idx, topk_w, status, s,
                   false) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (device_status_out &&
      cudaMemcpyAsync(device_status_out, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
