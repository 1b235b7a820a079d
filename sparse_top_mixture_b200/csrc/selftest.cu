// Self-test of the bounded pipeline waits.
//
// Every mbarrier wait in the tensor-core GEMMs gives up after a fixed budget
// of SM clocks, records MOE_DEVERR_WAIT_TIMEOUT (and the wait site) in the
// workspace header and lets the kernel drain and return, so a stalled
// pipeline is reported instead of hanging the GPU. This kernel exercises that
// path on purpose and safely: one thread waits, with the same wait routine
// and a ~10 ms budget, on an mbarrier that nothing ever arrives on.
#include <cuda_runtime.h>

#include "common.cuh"
#include "moe.h"
#include "tc_ptx.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int kSelftestSite = 99;
constexpr long long kSelftestLimitCycles = 20000000LL;  // about 10 ms of SM clocks

__global__ void wait_timeout_kernel(int32_t* err) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  tc::mbar_init(&bar, 1);
  abort = 0;
  tc::fence_mbar_init();
  // Nothing arrives on `bar`: the bounded wait must give up and report.
  tc::mbar_wait_slow(&bar, 0, &abort, err, kSelftestSite, false, kSelftestLimitCycles);
}

}  // namespace
}  // namespace stm

MOE_API moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 15u) != 0 || ws_bytes < sizeof(stm::WsHeader))
    return MOE_ERR_INVALID_ARGUMENT;
  stm::wait_timeout_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<int32_t*>(ws));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
