// Tensor-parallel reduction over peer memory, fused with the combine.
//
// Every expert's intermediate dimension I is split over G ranks (the
// tensor-parallel MoE block of "mstar.model.components.moe"): each rank's
// slice of I gives partial routed rows y (fp32) and a partial shared-expert
// output whose sums over ranks are the whole ones; the top-k sum is linear, so
// each rank can combine its own partial rows first. Here that combine is
// fused with the reduction: rank r sums its token's k partial rows in slot
// order (plus its shared part) in fp32, exactly as the library's combine,
// and stores each 1/G column slice straight into that slice's owner's arena
// (a reduce-scatter by plain 16-byte peer stores); the owner adds the G
// slices in rank order, rounds once to the output type, and stores its
// columns into every rank's output (the all-gather). Two launches and two
// bounded waits; nothing is read on the host. Flags, epochs and waits are
// those of the expert-parallel exchange (peer.cuh).
//
// Reuse from one forward to the next: a rank stores its next partials into
// an owner's arena only after its own previous forward ended (it waited for
// every owner's gather, published after the owner had read the partials),
// and owners store into a rank's output only after that rank's next
// partials arrived, which it sends after copying out its previous output.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "peer.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int TP_THREADS = 256;

// Arena of one rank, for G ranks, T tokens, H columns (Hs = H / G each) and
// output element size es (regions 256-byte aligned):
//   part_flag u64[G]  epoch at which source s's partial slice is in place
//   out_flag  u64[G]  epoch at which owner o's output columns are in place
//   done      u32[2]  completed-block counters of the scatter / gather
//   epoch     u64     this rank's forward count (advanced by the scatter)
//   part      f32[G][T][Hs]  partial sums of this rank's columns, by source
//   out       [T][H]  the finished output (problem dtype)
struct TpArena {
  size_t part_flag, out_flag, done, epoch, part, out, total;
};

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

TpArena tp_arena(int64_t G, int64_t T, int64_t H, size_t es) {
  TpArena a;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = al256(off + bytes);
    return at;
  };
  a.part_flag = take((size_t)G * 8);
  a.out_flag = take((size_t)G * 8);
  a.done = take(8);
  a.epoch = take(8);
  a.part = take((size_t)(T * H) * 4);
  a.out = take((size_t)(T * H) * es);
  a.total = off;
  return a;
}

// Scatter: for token t and 4-column vector v, acc = sum over slots j in
// order of y[pair_pos[t*k + j]][v] (slots with pair_pos < 0 skipped), plus
// shared[t][v]; stored to the owner o of column 4v, part[rank][t][4v - o*Hs].
__global__ void __launch_bounds__(TP_THREADS) tp_scatter_kernel(uint8_t* const* __restrict__ arenas, int G, int rank,
                                                                int64_t T, int H, int k, TpArena a,
                                                                const float* __restrict__ y,
                                                                const int32_t* __restrict__ pair_pos,
                                                                const float* __restrict__ shared, uint32_t* done,
                                                                uint64_t* epoch_ctr) {
  const int hv = H / 4, Hs = H / G;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < T * hv; u += stride) {
    const int64_t t = u / hv;
    const int v = (int)(u - t * hv);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int p = pair_pos[t * k + j];
      if (p < 0) continue;
      const float4 r = reinterpret_cast<const float4*>(y + (int64_t)p * H)[v];
      acc.x += r.x;
      acc.y += r.y;
      acc.z += r.z;
      acc.w += r.w;
    }
    if (shared != nullptr) {
      const float4 r = reinterpret_cast<const float4*>(shared + t * H)[v];
      acc.x += r.x;
      acc.y += r.y;
      acc.z += r.z;
      acc.w += r.w;
    }
    const int c = 4 * v, o = c / Hs;
    float* dst = reinterpret_cast<float*>(arenas[o] + a.part) + ((int64_t)rank * T + t) * Hs + (c - o * Hs);
    *reinterpret_cast<float4*>(dst) = acc;
  }
  publish_when_done(done, epoch_ctr, true, arenas, G, a.part_flag, rank);
}

// Gather: for token t and this rank's column c (8 at a time), the sum over
// sources s in order of part[s][t][c], rounded once, into every rank's
// out[t][rank*Hs + c].
template <typename TO>
__global__ void __launch_bounds__(TP_THREADS) tp_gather_kernel(uint8_t* const* __restrict__ arenas, int G, int rank,
                                                               int64_t T, int H, TpArena a, uint32_t* done,
                                                               uint64_t* epoch_ctr) {
  const int Hs = H / G, hv = Hs / 8;
  const float* part = reinterpret_cast<const float*>(arenas[rank] + a.part);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < T * hv; u += stride) {
    const int64_t t = u / hv;
    const int c = (int)(u - t * hv) * 8;
    float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < G; ++s) {
      const float4* src = reinterpret_cast<const float4*>(part + ((int64_t)s * T + t) * Hs + c);
      const float4 lo = src[0], hi = src[1];
      s8[0] += lo.x;
      s8[1] += lo.y;
      s8[2] += lo.z;
      s8[3] += lo.w;
      s8[4] += hi.x;
      s8[5] += hi.y;
      s8[6] += hi.z;
      s8[7] += hi.w;
    }
    const int64_t off = t * H + (int64_t)rank * Hs + c;
    if constexpr (sizeof(TO) == 2) {
      const uint4 w = make_uint4(pack_bf16x2(s8[0], s8[1]), pack_bf16x2(s8[2], s8[3]), pack_bf16x2(s8[4], s8[5]),
                                 pack_bf16x2(s8[6], s8[7]));
      for (int q = 0; q < G; ++q) *reinterpret_cast<uint4*>(reinterpret_cast<TO*>(arenas[q] + a.out) + off) = w;
    } else {
      const float4 lo = make_float4(s8[0], s8[1], s8[2], s8[3]), hi = make_float4(s8[4], s8[5], s8[6], s8[7]);
      for (int q = 0; q < G; ++q) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<TO*>(arenas[q] + a.out) + off);
        dst[0] = lo;
        dst[1] = hi;
      }
    }
  }
  publish_when_done(done + 1, epoch_ctr, false, arenas, G, a.out_flag, rank);
}

int tp_grid(int64_t units) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(units, TP_THREADS), 148 * 8));
}

moe_status tp_check(const moe_problem* p, int32_t G, int32_t rank) {
  if (p == nullptr || G < 1 || G > 64 || rank < 0 || rank >= G) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T < 0 || p->H <= 0 || p->k < 1 || p->H % (8 * G) != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARGUMENT;
  return MOE_OK;
}

bool al16(const void* q) { return q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

TpArena arena_of(const moe_problem* p, int32_t G) {
  return tp_arena(G, p->T, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2);
}

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_tp_arena_size(const moe_problem* p, int32_t G, size_t* bytes) {
  const moe_status st = tp_check(p, G, 0);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = arena_of(p, G).total;
  return MOE_OK;
}

MOE_API moe_status moe_tp_arena_offsets(const moe_problem* p, int32_t G, size_t* part_flag, size_t* out_flag,
                                        size_t* epoch, size_t* part, size_t* out) {
  const moe_status st = tp_check(p, G, 0);
  if (st != MOE_OK) return st;
  const TpArena a = arena_of(p, G);
  if (part_flag) *part_flag = a.part_flag;
  if (out_flag) *out_flag = a.out_flag;
  if (epoch) *epoch = a.epoch;
  if (part) *part = a.part;
  if (out) *out = a.out;
  return MOE_OK;
}

MOE_API moe_status moe_tp_scatter(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas, void* own_arena,
                                  const float* y_perm, const int32_t* pair_pos, const float* shared_out,
                                  moe_stream_t stream) {
  const moe_status st = tp_check(p, G, rank);
  if (st != MOE_OK) return st;
  if (!al16(arenas) || !al16(own_arena)) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T > 0 && (!al16(y_perm) || !al16(pair_pos))) return MOE_ERR_INVALID_ARGUMENT;
  if (shared_out != nullptr && !al16(shared_out)) return MOE_ERR_INVALID_ARGUMENT;
  const TpArena a = arena_of(p, G);
  uint8_t* own = static_cast<uint8_t*>(own_arena);
  tp_scatter_kernel<<<tp_grid(p->T * (p->H / 4)), TP_THREADS, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<uint8_t* const*>(arenas), G, rank, p->T, (int)p->H, (int)p->k, a, y_perm, pair_pos,
      shared_out, reinterpret_cast<uint32_t*>(own + a.done), reinterpret_cast<uint64_t*>(own + a.epoch));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status moe_tp_gather(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas, void* own_arena,
                                 moe_stream_t stream) {
  const moe_status st = tp_check(p, G, rank);
  if (st != MOE_OK) return st;
  if (!al16(arenas) || !al16(own_arena)) return MOE_ERR_INVALID_ARGUMENT;
  const TpArena a = arena_of(p, G);
  uint8_t* own = static_cast<uint8_t*>(own_arena);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* const* ar = reinterpret_cast<uint8_t* const*>(arenas);
  const int grid = tp_grid(p->T * (p->H / G / 8));
  uint32_t* done = reinterpret_cast<uint32_t*>(own + a.done);
  uint64_t* epoch = reinterpret_cast<uint64_t*>(own + a.epoch);
  if (p->dtype == MOE_DTYPE_F32)
    tp_gather_kernel<float><<<grid, TP_THREADS, 0, s>>>(ar, G, rank, p->T, (int)p->H, a, done, epoch);
  else
    tp_gather_kernel<__nv_bfloat16><<<grid, TP_THREADS, 0, s>>>(ar, G, rank, p->T, (int)p->H, a, done, epoch);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status moe_tp_wait(const moe_problem* p, int32_t G, void* own_arena, int32_t which, int64_t max_polls,
                               int32_t* err, moe_stream_t stream) {
  const moe_status st = tp_check(p, G, 0);
  if (st != MOE_OK) return st;
  if (!al16(own_arena) || (which != 0 && which != 1) || max_polls < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (err != nullptr && (reinterpret_cast<uintptr_t>(err) & 3u) != 0) return MOE_ERR_INVALID_ARGUMENT;
  const TpArena a = arena_of(p, G);
  const uint8_t* own = static_cast<const uint8_t*>(own_arena);
  peer_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint64_t*>(own + (which == 0 ? a.part_flag : a.out_flag)),
      reinterpret_cast<const uint64_t*>(own + a.epoch), G, max_polls, err);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
