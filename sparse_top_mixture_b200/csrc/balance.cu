// Aux-loss-free load balancing: the deferred sign-controller update of the
// fp32 selection bias ("Sparse MoE FFN for DFlash-family drafters", What's
// here: MoEGate's bias is moved by a sign controller from all-reduced expert
// loads, never by gradients; a forward stashes its routing counts and the
// update is applied before the next forward; a second apply is a no-op).
//
// moe_bias_stash adds one forward's per-expert counts (written by the
// dispatch) to an int64 stash. moe_bias_update, with L = the stash (summed
// over data-parallel ranks by the caller first) and m = sum(L) / E, adds
// +rate to bias[e] when L[e] < m, -rate when L[e] > m, nothing when equal,
// as one fp32 add, then zeroes the stash. The comparison with the mean is
// done exactly, as sum(L) against E * L[e] in 64-bit integers.
#include <cuda_runtime.h>

#include <cmath>

#include "common.cuh"
#include "moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int BTHREADS = kMaxExperts;  // one thread per expert

__global__ void __launch_bounds__(BTHREADS) bias_stash_kernel(const int32_t* __restrict__ counts,
                                                              int64_t* __restrict__ stash, int E) {
  const int e = threadIdx.x;
  if (e < E) stash[e] += counts[e];
}

__global__ void __launch_bounds__(BTHREADS) bias_update_kernel(int64_t* __restrict__ stash, float* __restrict__ bias,
                                                               int E, float rate) {
  __shared__ long long part[BTHREADS / 32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const long long L = e < E ? stash[e] : 0;
  long long s = L;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) part[warp] = s;
  __syncthreads();
  long long total = 0;
#pragma unroll
  for (int w = 0; w < BTHREADS / 32; ++w) total += part[w];
  if (e < E) {
    const long long under = total - (long long)E * L;  // > 0: below the mean load
    if (under > 0) bias[e] = bias[e] + rate;
    else if (under < 0) bias[e] = bias[e] - rate;
    stash[e] = 0;
  }
}

bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_e(const moe_problem* p) { return p != nullptr && p->E >= 1 && p->E <= kMaxExperts; }

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_bias_stash(const moe_problem* p, const int32_t* counts, int64_t* load_stash,
                                  moe_stream_t stream) {
  if (!valid_e(p) || !aligned(counts, 4) || !aligned(load_stash, 8)) return MOE_ERR_INVALID_ARGUMENT;
  bias_stash_kernel<<<1, BTHREADS, 0, reinterpret_cast<cudaStream_t>(stream)>>>(counts, load_stash, (int)p->E);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status moe_bias_update(const moe_problem* p, int64_t* load_stash, float* bias, float rate,
                                   moe_stream_t stream) {
  if (!valid_e(p) || !aligned(load_stash, 8) || !aligned(bias, 4) || !std::isfinite(rate))
    return MOE_ERR_INVALID_ARGUMENT;
  bias_update_kernel<<<1, BTHREADS, 0, reinterpret_cast<cudaStream_t>(stream)>>>(load_stash, bias, (int)p->E, rate);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
