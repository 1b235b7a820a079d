// Expert-parallel exchange over peer memory, with no host round trip.
//
// The experts of one MoE layer split over G ranks (rank r owns experts
// [r E/G, (r+1) E/G), "mstar.model.components.moe", SparseMoeBlock fused
// layout, the experts being independent segments of one weight): each rank
// routes and dispatches its own T tokens over all E experts, and the rows for
// the experts of rank q -- one contiguous run of its sorted rows -- are stored
// straight into an arena that q owns and every rank can address (NVLink peer
// memory, opened once at set-up). q runs them through its experts with the
// library's grouped GEMM and stores each weighted fp32 row back into the
// sender's arena, at the sender's sorted position, so that the sender finishes
// the layer with its usual combine. Counts never go to the host: each sender
// writes its rows into a fixed region of the receiver's arena (capacity T*k
// rows per source) and marks the slots it leaves empty, and the receiver's
// counting-sort dispatch regroups the occupied slots by local expert on the
// device. Every transfer is a plain 16-byte store to peer memory (no TMA, no
// multicast, no library kernel on peer memory).
//
// Ordering: a launch's last block publishes an epoch number to each peer's
// flag once every block's stores are fenced at system scope (release), and a
// waiter polls its own flags with acquire loads, up to a caller-given number
// of polls, after which it raises MOE_DEVERR_WAIT_TIMEOUT and returns.
// Reuse from one forward to the next needs no further handshake: a sender
// overwrites an owner's region (forward n+1) only after its own forward n
// ended, which waited for that owner's returns, published after the owner's
// GEMM had read the rows; owners store into a sender's y (and sources into
// an owner's y-offset mailbox) only after the rows of forward n+1 arrived,
// which the sender sends after its forward-n combine read y.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "peer.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int EP_THREADS = 256;

// Arena of one rank (byte offsets, regions 256-byte aligned), for G ranks,
// C = T*k slots per source and H columns of element size es:
//   rows_flag u64[G]  epoch at which source s's rows (and its empty-slot
//                     marks and y offset) are in place
//   ret_flag  u64[G]  epoch at which owner q has returned this rank's rows
//   done      u32[2]  completed-block counters of this rank's send / return
//   epoch     u64     this rank's forward count: the send's last block
//                     advances it and publishes the new value; the waits
//                     and the return read it on the device
//   yoff      i32[G]  source s's sorted position of its first row for us
//   x         [G*C][H] rows received, source s in slots [s*C, (s+1)*C)
//   w         f32[G*C] their routing weights
//   id        i64[G*C] their local expert ids, -1 for an empty slot
//   y         f32[C][H] this rank's own sorted rows, weighted, returned
struct EpArena {
  size_t rows_flag, ret_flag, done, epoch, yoff, x, w, id, y, total;
};

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

EpArena ep_arena(int64_t G, int64_t C, int64_t H, size_t es) {
  EpArena a;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = al256(off + bytes);
    return at;
  };
  a.rows_flag = take((size_t)G * 8);
  a.ret_flag = take((size_t)G * 8);
  a.done = take(8);
  a.epoch = take(8);
  a.yoff = take((size_t)G * 4);
  a.x = take((size_t)(G * C * H) * es);
  a.w = take((size_t)(G * C) * 4);
  a.id = take((size_t)(G * C) * 8);
  a.y = take((size_t)(C * H) * 4);
  a.total = off;
  return a;
}

// Send: sorted row p (< offsets[E], the rows the dispatch kept) of expert e
// goes to owner q = e / El, slot rank*C + i, i = p - offsets[q*El]: its
// row of x_perm, its routing weight and local id e - q*El. Slots i >= n_q of
// each owner get id -1; each owner learns where its rows sit in our sorted
// order (yoff). Then the last block publishes rows_flag[rank] = epoch.
template <typename T>
__global__ void __launch_bounds__(EP_THREADS) ep_send_kernel(uint8_t* const* __restrict__ arenas, int G, int rank,
                                                             int64_t C, int H, int El, EpArena a,
                                                             const T* __restrict__ x_perm,
                                                             const int32_t* __restrict__ offsets,
                                                             const int32_t* __restrict__ sorted_pairs,
                                                             const float* __restrict__ rw,
                                                             const int64_t* __restrict__ sel, uint32_t* done,
                                                             uint64_t* epoch_ctr) {
  constexpr int V = Elem<T>::kPerVec;
  const int hv = H / V;
  const int64_t used = offsets[(int64_t)G * El];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t u = t0; u < used * hv; u += stride) {
    const int64_t p = u / hv;
    const int v = (int)(u - p * hv);
    const int32_t q_pair = sorted_pairs[p];
    const int e = (int)sel[q_pair];
    const int q = e / El;
    const int64_t slot = (int64_t)rank * C + (p - offsets[q * El]);
    uint8_t* arena = arenas[q];
    reinterpret_cast<uint4*>(reinterpret_cast<T*>(arena + a.x) + slot * H)[v] =
        reinterpret_cast<const uint4*>(x_perm + p * H)[v];
    if (v == 0) {
      reinterpret_cast<float*>(arena + a.w)[slot] = rw[q_pair];
      reinterpret_cast<int64_t*>(arena + a.id)[slot] = e - q * El;
    }
  }
  for (int64_t j = t0; j < (int64_t)G * C; j += stride) {
    const int q = (int)(j / C);
    const int64_t i = j - (int64_t)q * C;
    const int64_t n_q = offsets[(q + 1) * El] - offsets[q * El];
    if (i >= n_q) reinterpret_cast<int64_t*>(arenas[q] + a.id)[(int64_t)rank * C + i] = -1;
    if (i == 0) reinterpret_cast<int32_t*>(arenas[q] + a.yoff)[rank] = offsets[q * El];
  }
  publish_when_done(done, epoch_ctr, true, arenas, G, a.rows_flag, rank);
}

// Return: sorted row p1 < offsets1[El] of the receiver's regroup came from
// slot j = sorted_pairs1[p1] = s*C + i; its weighted fp32 row goes to source
// s's y at row yoff[s] + i. Then the last block publishes ret_flag[rank].
__global__ void __launch_bounds__(EP_THREADS) ep_return_kernel(uint8_t* const* __restrict__ arenas, int G, int rank,
                                                               int64_t C, int H, int El, EpArena a,
                                                               const float* __restrict__ y_sorted,
                                                               const int32_t* __restrict__ offsets1,
                                                               const int32_t* __restrict__ sorted_pairs1,
                                                               uint32_t* done, uint64_t* epoch_ctr) {
  const int hv = H / 4;
  const int64_t used = offsets1[El];
  const int32_t* yoff = reinterpret_cast<const int32_t*>(arenas[rank] + a.yoff);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < used * hv; u += stride) {
    const int64_t p1 = u / hv;
    const int v = (int)(u - p1 * hv);
    const int64_t j = sorted_pairs1[p1];
    const int s = (int)(j / C);
    const int64_t i = j - (int64_t)s * C;
    float* dst = reinterpret_cast<float*>(arenas[s] + a.y) + (yoff[s] + i) * H;
    reinterpret_cast<float4*>(dst)[v] = reinterpret_cast<const float4*>(y_sorted + p1 * H)[v];
  }
  publish_when_done(done + 1, epoch_ctr, false, arenas, G, a.ret_flag, rank);
}

int ep_grid(int64_t units) {
  return (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(units, EP_THREADS), 148 * 8));
}

moe_status ep_check(const moe_problem* p, int32_t G, int32_t rank) {
  if (p == nullptr || G < 1 || G > 64 || rank < 0 || rank >= G) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T < 0 || p->H <= 0 || p->H % 8 != 0 || p->E < 1 || p->E > kMaxExperts || p->k < 1 || p->k > p->E)
    return MOE_ERR_INVALID_ARGUMENT;
  if (p->E % G != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARGUMENT;
  return MOE_OK;
}

bool al16(const void* q) { return q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

__global__ void ep_publish_kernel(uint8_t* const* arenas, int G, int rank, size_t flag_off, const uint64_t* epoch) {
  __threadfence_system();
  const uint64_t e = *epoch;
  for (int q = threadIdx.x; q < G; q += blockDim.x)
    st_release_sys(reinterpret_cast<uint64_t*>(arenas[q] + flag_off) + rank, e);
}

}  // namespace

bool ep_views(const moe_problem& p, int G, void* own_arena, EpViews* v) {
  if (ep_check(&p, G, 0) != MOE_OK || !al16(own_arena)) return false;
  const int64_t C = p.T * p.k;
  const EpArena a = ep_arena(G, C, p.H, p.dtype == MOE_DTYPE_F32 ? 4 : 2);
  uint8_t* own = static_cast<uint8_t*>(own_arena);
  v->x = own + a.x;
  v->w = reinterpret_cast<float*>(own + a.w);
  v->id = reinterpret_cast<int64_t*>(own + a.id);
  v->yoff = reinterpret_cast<int32_t*>(own + a.yoff);
  v->y_off = a.y;
  v->ret_flag_off = a.ret_flag;
  v->epoch = reinterpret_cast<uint64_t*>(own + a.epoch);
  v->C = C;
  return true;
}

cudaError_t launch_ep_publish(uint8_t* const* arenas, int G, int rank, size_t flag_off, const uint64_t* epoch,
                              cudaStream_t s) {
  ep_publish_kernel<<<1, 64, 0, s>>>(arenas, G, rank, flag_off, epoch);
  return cudaGetLastError();
}

bool ep_dest(const moe_problem& p, int G, int rank, void* const* arenas, void* own_arena, const float* rw,
             EpDest* d) {
  if (ep_check(&p, G, rank) != MOE_OK) return false;
  if (!al16(arenas) || !al16(own_arena) || (p.T > 0 && !al16(rw))) return false;
  const int64_t C = p.T * p.k;
  const EpArena a = ep_arena(G, C, p.H, p.dtype == MOE_DTYPE_F32 ? 4 : 2);
  uint8_t* own = static_cast<uint8_t*>(own_arena);
  d->arenas = reinterpret_cast<uint8_t* const*>(arenas);
  d->G = G;
  d->rank = rank;
  d->El = (int)(p.E / G);
  d->C = C;
  d->x_off = a.x;
  d->w_off = a.w;
  d->id_off = a.id;
  d->yoff_off = a.yoff;
  d->flag_off = a.rows_flag;
  d->rw = rw;
  d->done = reinterpret_cast<uint32_t*>(own + a.done);
  d->epoch = reinterpret_cast<uint64_t*>(own + a.epoch);
  return true;
}

}  // namespace stm

using namespace stm;

MOE_API moe_status moe_ep_arena_size(const moe_problem* p, int32_t G, size_t* bytes) {
  const moe_status st = ep_check(p, G, 0);
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = ep_arena(G, p->T * p->k, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2).total;
  return MOE_OK;
}

MOE_API moe_status moe_ep_arena_offsets(const moe_problem* p, int32_t G, size_t* rows_flag, size_t* ret_flag,
                                        size_t* epoch, size_t* x, size_t* w, size_t* id, size_t* y) {
  const moe_status st = ep_check(p, G, 0);
  if (st != MOE_OK) return st;
  const EpArena a = ep_arena(G, p->T * p->k, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2);
  if (rows_flag) *rows_flag = a.rows_flag;
  if (ret_flag) *ret_flag = a.ret_flag;
  if (epoch) *epoch = a.epoch;
  if (x) *x = a.x;
  if (w) *w = a.w;
  if (id) *id = a.id;
  if (y) *y = a.y;
  return MOE_OK;
}

MOE_API moe_status moe_ep_send(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas, void* own_arena,
                               const void* x_perm, const int32_t* offsets, const int32_t* sorted_pairs,
                               const float* routing_weights, const int64_t* selected_experts, moe_stream_t stream) {
  moe_status st = ep_check(p, G, rank);
  if (st != MOE_OK) return st;
  const int64_t C = p->T * p->k;
  if (!al16(arenas) || !al16(own_arena) || !al16(offsets)) return MOE_ERR_INVALID_ARGUMENT;
  if (C > 0 && (!al16(x_perm) || !al16(sorted_pairs) || !al16(routing_weights) || !al16(selected_experts)))
    return MOE_ERR_INVALID_ARGUMENT;
  const EpArena a = ep_arena(G, C, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* const* ar = reinterpret_cast<uint8_t* const*>(arenas);
  uint32_t* done = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(own_arena) + a.done);
  uint64_t* epoch = reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(own_arena) + a.epoch);
  const int E_l = (int)(p->E / G);
  const int grid = ep_grid(std::max<int64_t>((int64_t)G * C, C * (p->H / 4)));
  if (p->dtype == MOE_DTYPE_F32)
    ep_send_kernel<float><<<grid, EP_THREADS, 0, s>>>(ar, G, rank, C, (int)p->H, E_l, a,
                                                       static_cast<const float*>(x_perm), offsets, sorted_pairs,
                                                       routing_weights, selected_experts, done, epoch);
  else
    ep_send_kernel<__nv_bfloat16><<<grid, EP_THREADS, 0, s>>>(ar, G, rank, C, (int)p->H, E_l, a,
                                                               static_cast<const __nv_bfloat16*>(x_perm), offsets,
                                                               sorted_pairs, routing_weights, selected_experts, done,
                                                               epoch);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status moe_ep_wait(const moe_problem* p, int32_t G, void* own_arena, int32_t which, int64_t max_polls,
                               int32_t* err, moe_stream_t stream) {
  moe_status st = ep_check(p, G, 0);
  if (st != MOE_OK) return st;
  if (!al16(own_arena) || (which != 0 && which != 1) || max_polls < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (err != nullptr && (reinterpret_cast<uintptr_t>(err) & 3u) != 0) return MOE_ERR_INVALID_ARGUMENT;
  const EpArena a = ep_arena(G, p->T * p->k, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2);
  const uint64_t* flags =
      reinterpret_cast<const uint64_t*>(static_cast<uint8_t*>(own_arena) + (which == 0 ? a.rows_flag : a.ret_flag));
  const uint64_t* epoch = reinterpret_cast<const uint64_t*>(static_cast<uint8_t*>(own_arena) + a.epoch);
  peer_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(flags, epoch, G, max_polls, err);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API moe_status moe_ep_return(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas, void* own_arena,
                                 const float* y_sorted, const int32_t* offsets1,
                                 const int32_t* sorted_pairs1, moe_stream_t stream) {
  moe_status st = ep_check(p, G, rank);
  if (st != MOE_OK) return st;
  const int64_t C = p->T * p->k;
  if (!al16(arenas) || !al16(own_arena) || !al16(offsets1)) return MOE_ERR_INVALID_ARGUMENT;
  if (C > 0 && (!al16(y_sorted) || !al16(sorted_pairs1))) return MOE_ERR_INVALID_ARGUMENT;
  const EpArena a = ep_arena(G, C, p->H, p->dtype == MOE_DTYPE_F32 ? 4 : 2);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* done = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(own_arena) + a.done);
  uint64_t* epoch = reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(own_arena) + a.epoch);
  const int grid = ep_grid((int64_t)G * C * (p->H / 4));
  ep_return_kernel<<<grid, EP_THREADS, 0, s>>>(reinterpret_cast<uint8_t* const*>(arenas), G, rank, C, (int)p->H,
                                                (int)(p->E / G), a, y_sorted, offsets1, sorted_pairs1, done, epoch);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
