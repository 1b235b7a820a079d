// Device helpers of the peer-memory exchanges (expert and tensor
// parallelism): release / acquire flag accesses at system scope, the
// last-block epoch publication, and the bounded flag wait.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace stm {

__device__ __forceinline__ void st_release_sys(uint64_t* p, uint64_t v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ uint64_t ld_acquire_sys(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Called by every block of the grid (1-D or 2-D) after its stores: the last
// block to finish (its
// stores and every other block's fenced at system scope) takes this rank's
// epoch (advanced by one first when `advance`), publishes it into flag slot
// `slot` of every rank's arena (flags at byte offset flag_off), then re-arms
// the counter.
__device__ __forceinline__ void publish_when_done(uint32_t* done, uint64_t* epoch_ctr, bool advance,
                                                  uint8_t* const* arenas, int G, size_t flag_off, int slot) {
  __shared__ bool last;
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1;
  __syncthreads();
  if (!last) return;
  __threadfence_system();
  const uint64_t epoch = *epoch_ctr + (advance ? 1u : 0u);
  __syncthreads();
  if (advance && threadIdx.x == 0) *epoch_ctr = epoch;
  for (int q = threadIdx.x; q < G; q += blockDim.x)
    st_release_sys(reinterpret_cast<uint64_t*>(arenas[q] + flag_off) + slot, epoch);
  if (threadIdx.x == 0) *done = 0u;
}

// Wait until every one of the G flags at `flags` holds at least this rank's
// epoch (acquire), polling each at most max_polls times (about 256 ns
// apart); on giving up, raise MOE_DEVERR_WAIT_TIMEOUT in *err and return.
// (static: each source file that launches it has its own copy)
static __global__ void peer_wait_kernel(const uint64_t* flags, const uint64_t* epoch_ctr, int G, int64_t max_polls,
                                        int32_t* err) {
  const uint64_t epoch = *epoch_ctr;
  for (int s = threadIdx.x; s < G; s += blockDim.x) {
    int64_t n = 0;
    while (ld_acquire_sys(flags + s) < epoch) {
      if (++n >= max_polls) {
        raise_error(err, MOE_DEVERR_WAIT_TIMEOUT);
        break;
      }
      __nanosleep(256);
    }
  }
}

}  // namespace stm
