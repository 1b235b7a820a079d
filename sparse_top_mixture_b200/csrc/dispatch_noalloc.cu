// moe_dispatch_noalloc: sorted-segment dispatch for callers that cannot
// allocate device memory.
//
// Some callers cannot hand this library a workspace: code that runs while
// another thread captures a CUDA graph in global capture mode (cudaMalloc is
// an error there), plug-ins inside a host framework whose memory pool owns
// the whole GPU, and latency-critical paths that must never wait on an
// allocator. For them the dispatch's only scratch -- the [blocks x experts]
// matrix of per-block counts that the histogram, scan and permute kernels
// pass to each other -- lives in a fixed array in device memory that is part
// of this library's image, so the call allocates nothing. The caller still
// passes every input and output.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

// 1 MiB: (T / max(1, 256 / k)) * E count entries fit for, e.g., T = 65536
// tokens at k = 8 and E = 128, or T = 32768 at k = 8 and E = 256.
constexpr int64_t kStaticCountEntries = int64_t(1) << 18;

static __device__ __align__(256) int32_t g_dispatch_counts[kStaticCountEntries];
// The histogram's completion ticket (CTAs done so far; zero between calls).
static __device__ __align__(256) uint32_t g_dispatch_ticket;

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_counts_addr[kMaxDevices] = {};
uint32_t* g_ticket_addr[kMaxDevices] = {};

// Device addresses of the static arrays on the current device. In host code
// their names only stand in for them, so the addresses are looked up per
// device, with that device current, and kept once a lookup has succeeded (a
// failed lookup, e.g. one made while a graph is being captured, is retried by
// the next call).
moe_status static_scratch(int32_t** counts, uint32_t** ticket) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_counts_addr[dev] == nullptr || g_ticket_addr[dev] == nullptr) {
    void* a = nullptr;
    void* b = nullptr;
    if (cudaGetSymbolAddress(&a, g_dispatch_counts) != cudaSuccess || a == nullptr) return MOE_ERR_CUDA;
    if (cudaGetSymbolAddress(&b, g_dispatch_ticket) != cudaSuccess || b == nullptr) return MOE_ERR_CUDA;
    g_counts_addr[dev] = static_cast<int32_t*>(a);
    g_ticket_addr[dev] = static_cast<uint32_t*>(b);
  }
  *counts = g_counts_addr[dev];
  *ticket = g_ticket_addr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_dispatch_noalloc(const moe_problem* p, const int64_t* selected_experts, const void* x,
                                        int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                                        int32_t* pair_pos, void* x_perm, moe_stream_t stream) {
  size_t ws_probe = 0;
  const moe_status vs = moe_workspace_size(p, &ws_probe);  // validates the problem; allocates nothing
  if (vs != MOE_OK) return vs;
  if (counts == nullptr || offsets == nullptr || !aligned16(counts) || !aligned16(offsets))
    return MOE_ERR_INVALID_ARGUMENT;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->T == 0) {
    if (cudaMemsetAsync(counts, 0, (size_t)p->E * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(offsets, 0, (size_t)(p->E + 1) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (selected_experts == nullptr || sorted_pairs == nullptr || pair_pos == nullptr ||
      !aligned16(selected_experts) || !aligned16(sorted_pairs) || !aligned16(pair_pos))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((x == nullptr) != (x_perm == nullptr) || !aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARGUMENT;
  if (dispatch_num_blocks(p->T, p->k) * p->E > kStaticCountEntries) return MOE_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  uint32_t* ticket = nullptr;
  const moe_status ss = static_scratch(&scratch, &ticket);
  if (ss != MOE_OK) return ss;
  // Every count entry the scan reads is written by the histogram first, so
  // nothing carried over from an earlier call is read; the ticket must start
  // at zero (each dispatch leaves it there; it is cleared here as well). The
  // error flag is not kept: a pair with an expert id outside [0, E) is
  // skipped (pair_pos -1) exactly as in moe_dispatch, without a flag to read
  // back.
  if (cudaMemsetAsync(ticket, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = launch_dispatch(p->dtype, selected_experts, x, p->T, p->H, p->E, p->k, scratch, counts,
                                        offsets, sorted_pairs, pair_pos, x_perm, nullptr, ticket, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
