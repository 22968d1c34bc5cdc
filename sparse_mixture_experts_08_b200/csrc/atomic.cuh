// Atomic-expert launchers shared by atomic.cu and the C ABI (api.cu).
#pragma once

#include "common.cuh"

namespace moe {

// From this many (token, slot) tasks on, the expert phases run as separate fully
// occupied kernels (coefficients, then assembly) instead of one cooperative launch.
constexpr long long ATOMIC_WIDE_MIN_TASKS = 16384;

// launch_atomic_experts with the scratch of the counting sort of the tasks by
// expert (sort_ws: n_experts + T K int32, nullable: tasks then go in token order).
cudaError_t launch_atomic_experts_sorted(int T, int d, int K, int act, const void* x, const void* w_in,
                                         const void* w_out, const int32_t* idx, const float* g, float* coef, void* out,
                                         long long n_experts, unsigned* bar, bool bar_zeroed,
                                         unsigned long long limit_ns, int* status, int32_t* sort_ws, cudaStream_t s);

// Fault-injection hook: the decode-budget atomic-expert kernel's grid barrier waits
// for n arrivals more than its grid has, so it ends only at its time limit.
void set_grid_barrier_extra(unsigned n);

}  // namespace moe
