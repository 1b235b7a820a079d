// C ABI of the sparse top-k MoE FFN forward: argument validation, workspace
// layout and the launch sequence. Declarations and per-call contracts are in
// include/moe.h.
#include <cuda_runtime.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

// ---- workspace layout --------------------------------------------------------
struct Layout {
  size_t header, logits, gamma, local, counts, offsets, sorted_pairs, pair_pos, x_perm, h, y_perm, h_shared,
      shared_out, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

Layout make_layout(const moe_problem& p) {
  Layout L;
  const size_t es = p.dtype == MOE_DTYPE_F32 ? 4 : 2;
  const int64_t P = p.T * p.k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.header = take(sizeof(WsHeader));
  L.logits = take(router_partial_bytes(p.dtype, p.T, p.H, p.E));
  L.gamma = take((size_t)p.T * 4);
  L.local = take((size_t)dispatch_num_blocks(p.T, p.k) * p.E * 4);
  L.counts = take((size_t)p.E * 4);
  L.offsets = take((size_t)(p.E + 1) * 4);
  L.sorted_pairs = take((size_t)P * 4);
  L.pair_pos = take((size_t)P * 4);
  L.x_perm = take((size_t)P * p.H * es);
  L.h = take((size_t)P * p.I * es);
  L.y_perm = take((size_t)P * p.H * 4);  // fp32
  const bool sh = p.shared != MOE_SHARED_NONE;
  L.h_shared = take(sh ? (size_t)p.T * p.I_shared * es : 0);
  L.shared_out = take(sh ? (size_t)p.T * p.H * 4 : 0);  // fp32
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ---- validation ---------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

moe_status validate_problem(const moe_problem* p) {
  if (p == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T < 0 || p->H <= 0 || p->I <= 0 || p->E < 1 || p->k < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (p->E > kMaxExperts || p->k > p->E) return MOE_ERR_INVALID_ARGUMENT;
  if (p->H % 8 != 0 || p->I % 8 != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARGUMENT;
  if (p->score < 0 || p->score > 2 || p->bias_mode < 0 || p->bias_mode > 2) return MOE_ERR_INVALID_ARGUMENT;
  if (p->shared < 0 || p->shared > 2 || p->reserved != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (p->shared != MOE_SHARED_NONE && (p->I_shared <= 0 || p->I_shared % 8 != 0)) return MOE_ERR_INVALID_ARGUMENT;
  // 32-bit pair indices and TMA coordinates.
  if (p->T * p->k >= (int64_t(1) << 31) || p->H >= (int64_t(1) << 31) || p->I >= (int64_t(1) << 31))
    return MOE_ERR_INVALID_ARGUMENT;
  return MOE_OK;
}

moe_status check_ws(const moe_problem& p, const void* ws, size_t ws_bytes, Layout* L) {
  *L = make_layout(p);
  if (!ok_ptr(ws)) return MOE_ERR_INVALID_ARGUMENT;
  if (ws_bytes < L->total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  return MOE_OK;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                         \
  do {                                        \
    const moe_status _st = (expr);            \
    if (_st != MOE_OK) return _st;            \
  } while (0)

#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

// ---- stage implementations (arguments already validated) ----------------------
moe_status do_route(const moe_problem& p, const Layout& L, const void* x, const void* gate_w, const float* bias,
                    const void* shared_gate, float* weights, int64_t* selected, float* gamma, void* ws,
                    cudaStream_t s) {
  MOE_CUDA(launch_route(p.dtype, x, gate_w, shared_gate, bias, p.T, p.H, p.E, p.k, p.score, p.bias_mode,
                        p.renormalize ? 1 : 0, at<float>(ws, L.logits), weights, selected, gamma,
                        at<int32_t>(ws, L.header), s));
  return MOE_OK;
}

moe_status do_dispatch(const moe_problem& p, const Layout& L, const int64_t* selected, const void* x,
                       int32_t* counts, int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos, void* x_perm,
                       void* ws, cudaStream_t s) {
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  MOE_CUDA(launch_dispatch(p.dtype, selected, x, p.T, p.H, p.E, p.k, at<int32_t>(ws, L.local), counts, offsets,
                           sorted_pairs, pair_pos, x_perm, &hdr->error_bits, &hdr->dispatch_ticket, s));
  return MOE_OK;
}

moe_status do_grouped_gate_up(const moe_problem& p, const Layout& L, const void* x_perm, const int32_t* offsets,
                              const void* gate_up, void* ws, cudaStream_t s) {
  Segments sg{offsets, (int32_t)p.E, 0, p.T * p.k};
  void* h = at<void>(ws, L.h);
  if (p.dtype == MOE_DTYPE_F32)
    MOE_CUDA(launch_simt_gate_up(sg, (const float*)x_perm, (const float*)gate_up, (float*)h, p.I, p.H,
                                 at<int32_t>(ws, L.header), s));
  else
    MOE_CUDA(launch_tc_gate_up(sg, x_perm, gate_up, p.E, h, p.I, p.H, at<int32_t>(ws, L.header), s));
  return MOE_OK;
}

moe_status do_grouped_down(const moe_problem& p, const Layout& L, const int32_t* offsets, const void* down,
                           const float* weights, const int32_t* sorted_pairs, void* y_perm, void* ws,
                           cudaStream_t s) {
  Segments sg{offsets, (int32_t)p.E, 0, p.T * p.k};
  const void* h = at<void>(ws, L.h);
  if (p.dtype == MOE_DTYPE_F32)
    MOE_CUDA(launch_simt_down(sg, (const float*)h, (const float*)down, (float*)y_perm, weights, sorted_pairs, p.H,
                              p.I, at<int32_t>(ws, L.header), s));
  else
    MOE_CUDA(launch_tc_down(sg, h, down, p.E, y_perm, weights, sorted_pairs, p.H, p.I, at<int32_t>(ws, L.header),
                            s));
  return MOE_OK;
}

moe_status do_shared(const moe_problem& p, const Layout& L, const void* x, const void* sgu, const void* sdn,
                     const float* gamma, void* shared_out, void* ws, cudaStream_t s) {
  Segments sg{nullptr, 1, (int32_t)p.T, p.T};
  void* hs = at<void>(ws, L.h_shared);
  if (p.dtype == MOE_DTYPE_F32) {
    int32_t* err = at<int32_t>(ws, L.header);
    MOE_CUDA(launch_simt_gate_up(sg, (const float*)x, (const float*)sgu, (float*)hs, p.I_shared, p.H, err, s));
    MOE_CUDA(launch_simt_down(sg, (const float*)hs, (const float*)sdn, (float*)shared_out, gamma, nullptr, p.H,
                              p.I_shared, err, s));
  } else {
    int32_t* err = at<int32_t>(ws, L.header);
    MOE_CUDA(launch_tc_gate_up(sg, x, sgu, 1, hs, p.I_shared, p.H, err, s));
    MOE_CUDA(launch_tc_down(sg, hs, sdn, 1, shared_out, gamma, nullptr, p.H, p.I_shared, err, s));
  }
  return MOE_OK;
}

moe_status validate_weights(const moe_problem& p, const moe_weights* w) {
  if (w == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (!ok_ptr(w->gate_w) || !ok_ptr(w->gate_up) || !ok_ptr(w->down)) return MOE_ERR_INVALID_ARGUMENT;
  if ((p.bias_mode != MOE_BIAS_NONE) != (w->bias != nullptr) || !ok_opt(w->bias)) return MOE_ERR_INVALID_ARGUMENT;
  if (p.shared != MOE_SHARED_NONE) {
    if (!ok_ptr(w->shared_gate_up) || !ok_ptr(w->shared_down)) return MOE_ERR_INVALID_ARGUMENT;
  }
  if ((p.shared == MOE_SHARED_SIGMOID_GATED) != (w->shared_gate != nullptr) || !ok_opt(w->shared_gate))
    return MOE_ERR_INVALID_ARGUMENT;
  return MOE_OK;
}

// Whether moe_forward_ex runs the shared expert on its aux stream: its
// gate_up GEMM must have at most half as many tiles as a B200 has SMs.
bool shared_overlaps(const moe_problem& p) {
  if (p.shared == MOE_SHARED_NONE) return false;
  const int64_t tiles = ceil_div(p.T, 128) * ceil_div(p.I_shared, 128);
  return tiles <= 74;
}

// RAII pair of fork / join events for the two-stream forward.
struct EventPair {
  cudaEvent_t fork = nullptr, join = nullptr;
  ~EventPair() {
    if (fork) cudaEventDestroy(fork);  // safe while pending: released on completion
    if (join) cudaEventDestroy(join);
  }
};

moe_status forward_impl(const moe_problem* p, const moe_weights* w, const void* x, void* out, float* weights,
                        int64_t* selected, void* ws, size_t ws_bytes, cudaStream_t s, cudaStream_t aux,
                        cudaEvent_t* ev) {
  MOE_TRY(validate_problem(p));
  MOE_TRY(validate_weights(*p, w));
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(x) || !ok_ptr(out) || !ok_ptr(weights) || !ok_ptr(selected)) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  // While `s` is being captured into a CUDA graph the events become event
  // record nodes of the graph (recorded at every replay).
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (ev != nullptr) MOE_CUDA(cudaStreamIsCapturing(s, &capture));
  static const char* const kStageNames[MOE_NUM_STAGES] = {"route", "dispatch", "gate_up",
                                                          "down",  "shared",   "combine"};
  NvtxRange range("moe_forward");
  NvtxStages stage;
  auto mark = [&](int i) -> moe_status {
    if (i < MOE_NUM_STAGES) stage.next(kStageNames[i]);
    else stage.close();
    if (ev == nullptr || ev[i] == nullptr) return MOE_OK;
    if (capture == cudaStreamCaptureStatusActive)
      return cuda_status(cudaEventRecordWithFlags(ev[i], s, cudaEventRecordExternal));
    return cuda_status(cudaEventRecord(ev[i], s));
  };
  const bool has_shared = p->shared != MOE_SHARED_NONE;
  const bool gated = p->shared == MOE_SHARED_SIGMOID_GATED;
  // Schedules with an aux stream:
  //  - a small shared expert (too few row tiles to fill the GPU, as in
  //    decode) runs on `aux` beside the whole routed path, joined before the
  //    combine; its sigmoid gate comes from its own small kernel;
  //  - a large one occupies every SM while it runs, so it cannot overlap the
  //    routed GEMMs; it runs on `aux` after the route (whose top-k kernel
  //    already computed the gate) beside the dispatch (the permutation
  //    kernel's CTAs fit next to its persistent CTAs; the histogram's
  //    1024-thread CTAs wait for free SMs), and `s` waits for it before the
  //    routed gate_up.
  const bool use_aux = has_shared && aux != nullptr && aux != s;
  const bool small_shared = use_aux && shared_overlaps(*p);
  const bool large_shared = use_aux && !small_shared;
  float* gamma = at<float>(ws, L.gamma);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* sorted_pairs = at<int32_t>(ws, L.sorted_pairs);
  int32_t* pair_pos = at<int32_t>(ws, L.pair_pos);
  void* x_perm = at<void>(ws, L.x_perm);
  void* y_perm = at<void>(ws, L.y_perm);
  void* shared_out = has_shared ? at<void>(ws, L.shared_out) : nullptr;
  const float* shared_gamma = gated ? gamma : nullptr;

  EventPair evp;
  if (use_aux) {
    MOE_CUDA(cudaEventCreateWithFlags(&evp.fork, cudaEventDisableTiming));
    MOE_CUDA(cudaEventCreateWithFlags(&evp.join, cudaEventDisableTiming));
  }
  if (small_shared) {
    // The shared expert needs only x (and its own gate): run it on `aux`
    // while the routed path runs on `s`; join before the combine.
    MOE_CUDA(cudaEventRecord(evp.fork, s));
    MOE_CUDA(cudaStreamWaitEvent(aux, evp.fork, 0));
    if (gated) MOE_CUDA(launch_shared_gate(p->dtype, x, w->shared_gate, p->T, p->H, gamma, aux));
    MOE_TRY(do_shared(*p, L, x, w->shared_gate_up, w->shared_down, shared_gamma, shared_out, ws, aux));
    MOE_CUDA(cudaEventRecord(evp.join, aux));
  }

  MOE_TRY(mark(MOE_STAGE_ROUTE));
  MOE_TRY(do_route(*p, L, x, w->gate_w, w->bias, (gated && !small_shared) ? w->shared_gate : nullptr, weights,
                   selected, gamma, ws, s));
  if (large_shared) {
    MOE_CUDA(cudaEventRecord(evp.fork, s));
    MOE_CUDA(cudaStreamWaitEvent(aux, evp.fork, 0));
    MOE_TRY(do_shared(*p, L, x, w->shared_gate_up, w->shared_down, shared_gamma, shared_out, ws, aux));
    MOE_CUDA(cudaEventRecord(evp.join, aux));
  }
  // With a large shared expert on `aux`, the dispatch stage's interval ends
  // when both the dispatch and the shared expert are done, and the shared
  // stage is empty.
  MOE_TRY(mark(MOE_STAGE_DISPATCH));
  MOE_TRY(do_dispatch(*p, L, selected, x, counts, offsets, sorted_pairs, pair_pos, x_perm, ws, s));
  if (large_shared) MOE_CUDA(cudaStreamWaitEvent(s, evp.join, 0));
  MOE_TRY(mark(MOE_STAGE_GATE_UP));
  MOE_TRY(do_grouped_gate_up(*p, L, x_perm, offsets, w->gate_up, ws, s));
  MOE_TRY(mark(MOE_STAGE_DOWN));
  MOE_TRY(do_grouped_down(*p, L, offsets, w->down, weights, sorted_pairs, y_perm, ws, s));
  MOE_TRY(mark(MOE_STAGE_SHARED));
  if (has_shared && !use_aux)
    MOE_TRY(do_shared(*p, L, x, w->shared_gate_up, w->shared_down, shared_gamma, shared_out, ws, s));
  if (small_shared) MOE_CUDA(cudaStreamWaitEvent(s, evp.join, 0));
  MOE_TRY(mark(MOE_STAGE_COMBINE));
  MOE_CUDA(launch_combine(p->dtype, (const float*)y_perm, pair_pos, (const float*)shared_out, out, p->T, p->H,
                          p->k, s));
  MOE_TRY(mark(MOE_NUM_STAGES));
  return MOE_OK;
}

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_workspace_size(const moe_problem* p, size_t* bytes) {
  MOE_TRY(validate_problem(p));
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = make_layout(*p).total;
  return MOE_OK;
}

MOE_API moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ok_ptr(ws) || ws_bytes < sizeof(WsHeader)) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream));
}

MOE_API moe_status moe_route(const moe_problem* p, const void* x, const void* gate_w, const float* bias,
                             const void* shared_gate, float* routing_weights, int64_t* selected_experts,
                             float* shared_gamma, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(x) || !ok_ptr(gate_w) || !ok_ptr(routing_weights) || !ok_ptr(selected_experts))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((p->bias_mode != MOE_BIAS_NONE) != (bias != nullptr) || !ok_opt(bias)) return MOE_ERR_INVALID_ARGUMENT;
  if ((shared_gate != nullptr) != (shared_gamma != nullptr) || !ok_opt(shared_gate) || !ok_opt(shared_gamma))
    return MOE_ERR_INVALID_ARGUMENT;
  if (shared_gate != nullptr && p->shared != MOE_SHARED_SIGMOID_GATED) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  return do_route(*p, L, x, gate_w, bias, shared_gate, routing_weights, selected_experts, shared_gamma, ws,
                  (cudaStream_t)stream);
}

MOE_API moe_status moe_topk_from_logits(const moe_problem* p, const float* logits, const float* bias,
                                        float* routing_weights, int64_t* selected_experts, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(logits) || !ok_ptr(routing_weights) || !ok_ptr(selected_experts)) return MOE_ERR_INVALID_ARGUMENT;
  if ((p->bias_mode != MOE_BIAS_NONE) != (bias != nullptr) || !ok_opt(bias)) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_topk(logits, 1, p->E, p->T, p->E, p->k, p->score, p->bias_mode, p->renormalize ? 1 : 0,
                                 bias, routing_weights, selected_experts, nullptr, nullptr, p->H, p->dtype, nullptr,
                                 (cudaStream_t)stream));
}

MOE_API moe_status moe_dispatch(const moe_problem* p, const int64_t* selected_experts, const void* x,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos,
                                void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T == 0) {
    // Empty batch: every segment is empty.
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)p->E * 4, (cudaStream_t)stream));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(p->E + 1) * 4, (cudaStream_t)stream));
    return MOE_OK;
  }
  if (!ok_ptr(selected_experts) || !ok_ptr(sorted_pairs) || !ok_ptr(pair_pos)) return MOE_ERR_INVALID_ARGUMENT;
  if ((x == nullptr) != (x_perm == nullptr) || !ok_opt(x) || !ok_opt(x_perm)) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  return do_dispatch(*p, L, selected_experts, x, counts, offsets, sorted_pairs, pair_pos, x_perm, ws,
                     (cudaStream_t)stream);
}

MOE_API moe_status moe_dispatch_slots(const moe_problem* p, const int64_t* selected_experts, const void* x,
                                      int32_t* counts, int32_t* offsets, int32_t* sorted_pairs, int32_t* pair_pos,
                                      void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)p->E * 4, (cudaStream_t)stream));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(p->E + 1) * 4, (cudaStream_t)stream));
    return MOE_OK;
  }
  if (!ok_ptr(selected_experts) || !ok_ptr(sorted_pairs) || !ok_ptr(pair_pos)) return MOE_ERR_INVALID_ARGUMENT;
  if ((x == nullptr) != (x_perm == nullptr) || !ok_opt(x) || !ok_opt(x_perm)) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  // ids outside [0, E) are empty slots: skipped, no flag raised
  MOE_CUDA(launch_dispatch(p->dtype, selected_experts, x, p->T, p->H, p->E, p->k, at<int32_t>(ws, L.local), counts,
                           offsets, sorted_pairs, pair_pos, x_perm, nullptr, &hdr->dispatch_ticket,
                           (cudaStream_t)stream));
  return MOE_OK;
}

MOE_API moe_status moe_ep_dispatch_send(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas,
                                        void* own_arena, const int64_t* selected_experts, const void* x,
                                        const float* routing_weights, int32_t* counts, int32_t* offsets,
                                        int32_t* sorted_pairs, int32_t* pair_pos, void* ws, size_t ws_bytes,
                                        moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->T == 0) return MOE_ERR_UNSUPPORTED;  // an empty batch sends through moe_ep_send
  if (!ok_ptr(counts) || !ok_ptr(offsets) || !ok_ptr(selected_experts) || !ok_ptr(x) || !ok_ptr(sorted_pairs) ||
      !ok_ptr(pair_pos))
    return MOE_ERR_INVALID_ARGUMENT;
  EpDest ep;
  if (!ep_dest(*p, G, rank, arenas, own_arena, routing_weights, &ep)) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  MOE_CUDA(launch_dispatch_ep(p->dtype, selected_experts, x, p->T, p->H, p->E, p->k, at<int32_t>(ws, L.local),
                              counts, offsets, sorted_pairs, pair_pos, &hdr->error_bits, &hdr->dispatch_ticket, ep,
                              (cudaStream_t)stream));
  return MOE_OK;
}

MOE_API moe_status moe_ep_experts(const moe_problem* p, int32_t G, int32_t rank, void* const* arenas,
                                  void* own_arena, const void* gate_up, const void* down, void* ws, size_t ws_bytes,
                                  moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;  // the tensor-core GEMMs only
  if (G < 1 || rank < 0 || rank >= G || p->E % G != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (!ok_ptr(arenas) || !ok_ptr(gate_up) || !ok_ptr(down)) return MOE_ERR_INVALID_ARGUMENT;
  EpViews v;
  if (!ep_views(*p, G, own_arena, &v)) return MOE_ERR_INVALID_ARGUMENT;
  // the owner's problem: G*T*k one-slot rows over its E/G experts
  moe_problem p1 = *p;
  p1.T = G * v.C;
  p1.k = 1;
  p1.E = p->E / G;
  p1.I_shared = 0;
  p1.shared = MOE_SHARED_NONE;
  p1.bias_mode = MOE_BIAS_NONE;
  MOE_TRY(validate_problem(&p1));
  Layout L;
  MOE_TRY(check_ws(p1, ws, ws_bytes, &L));
  const cudaStream_t s = (cudaStream_t)stream;
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* sorted_pairs = at<int32_t>(ws, L.sorted_pairs);
  uint8_t* const* ar = reinterpret_cast<uint8_t* const*>(arenas);
  if (p1.T > 0) {
    // regroup the occupied slots by local expert (empty slots skipped, no flag)
    MOE_CUDA(launch_dispatch(p1.dtype, v.id, v.x, p1.T, p1.H, p1.E, 1, at<int32_t>(ws, L.local),
                             at<int32_t>(ws, L.counts), offsets, sorted_pairs, at<int32_t>(ws, L.pair_pos),
                             at<void>(ws, L.x_perm), nullptr, &hdr->dispatch_ticket, s));
    MOE_TRY(do_grouped_gate_up(p1, L, at<void>(ws, L.x_perm), offsets, gate_up, ws, s));
    // down with each weighted row stored into its source's y (peer stores)
    const Segments sg{offsets, (int32_t)p1.E, 0, p1.T};
    MOE_CUDA(launch_tc_down_ep(sg, at<void>(ws, L.h), down, p1.E, v.w, sorted_pairs, p1.H, p1.I,
                               EpRet{ar, v.C, v.y_off, v.yoff}, &hdr->error_bits, s));
  }
  MOE_CUDA(launch_ep_publish(ar, G, rank, v.ret_flag_off, v.epoch, s));
  return MOE_OK;
}

MOE_API moe_status moe_grouped_swiglu(const moe_problem* p, const void* x_perm, const int32_t* offsets,
                                      const void* gate_up, const void* down, const float* routing_weights,
                                      const int32_t* sorted_pairs, void* y_perm, void* ws, size_t ws_bytes,
                                      moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(x_perm) || !ok_ptr(offsets) || !ok_ptr(gate_up) || !ok_ptr(down) || !ok_ptr(y_perm))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((routing_weights == nullptr) != (sorted_pairs == nullptr) || !ok_opt(routing_weights) || !ok_opt(sorted_pairs))
    return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  const cudaStream_t s = (cudaStream_t)stream;
  MOE_TRY(do_grouped_gate_up(*p, L, x_perm, offsets, gate_up, ws, s));
  return do_grouped_down(*p, L, offsets, down, routing_weights, sorted_pairs, y_perm, ws, s);
}

MOE_API moe_status moe_shared_expert(const moe_problem* p, const void* x, const void* shared_gate_up,
                                     const void* shared_down, const float* shared_gamma, void* shared_out, void* ws,
                                     size_t ws_bytes, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->shared == MOE_SHARED_NONE) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(x) || !ok_ptr(shared_gate_up) || !ok_ptr(shared_down) || !ok_ptr(shared_out) || !ok_opt(shared_gamma))
    return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  return do_shared(*p, L, x, shared_gate_up, shared_down, shared_gamma, shared_out, ws, (cudaStream_t)stream);
}

MOE_API moe_status moe_combine(const moe_problem* p, const void* y_perm, const int32_t* pair_pos,
                               const void* shared_out, void* out, moe_stream_t stream) {
  MOE_TRY(validate_problem(p));
  if (p->T == 0) return MOE_OK;
  if (!ok_ptr(y_perm) || !ok_ptr(pair_pos) || !ok_opt(shared_out) || !ok_ptr(out)) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_combine(p->dtype, (const float*)y_perm, pair_pos, (const float*)shared_out, out, p->T,
                                    p->H, p->k, (cudaStream_t)stream));
}

MOE_API moe_status moe_forward(const moe_problem* p, const moe_weights* w, const void* x, void* out,
                               float* routing_weights, int64_t* selected_experts, void* ws, size_t ws_bytes,
                               moe_stream_t stream) {
  return forward_impl(p, w, x, out, routing_weights, selected_experts, ws, ws_bytes, (cudaStream_t)stream, nullptr,
                      nullptr);
}

MOE_API moe_status moe_forward_ex(const moe_problem* p, const moe_weights* w, const void* x, void* out,
                                  float* routing_weights, int64_t* selected_experts, void* ws, size_t ws_bytes,
                                  moe_stream_t stream, moe_stream_t aux_stream, moe_event_t* stage_events) {
  return forward_impl(p, w, x, out, routing_weights, selected_experts, ws, ws_bytes, (cudaStream_t)stream,
                      (cudaStream_t)aux_stream, reinterpret_cast<cudaEvent_t*>(stage_events));
}

MOE_API moe_status moe_gemm_path(const moe_problem* p, int32_t* path) {
  MOE_TRY(validate_problem(p));
  if (path == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (p->dtype != MOE_DTYPE_BF16) {
    *path = 0;
  } else {
    Segments sg{nullptr, (int32_t)p->E, 0, p->T * p->k};
    sg.offsets = reinterpret_cast<const int32_t*>(16);  // any non-null: routed segments
    *path = tc_gemm_variant(sg, false);
  }
  return MOE_OK;
}

MOE_API moe_status moe_launches_per_forward(const moe_problem* p, int32_t two_streams, int32_t* n) {
  MOE_TRY(validate_problem(p));
  if (n == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  if (p->T == 0) {
    *n = 0;
    return MOE_OK;
  }
  int count = 2 + 2 + 1;  // router logits + top-k; histogram + scan, permute + gather; combine
  if (p->dtype == MOE_DTYPE_BF16) {
    Segments routed{reinterpret_cast<const int32_t*>(16), (int32_t)p->E, 0, p->T * p->k};
    count += 2 * tc_gemm_launches(routed);
    if (p->shared != MOE_SHARED_NONE) {
      Segments sh{nullptr, 1, (int32_t)p->T, p->T};
      count += 2 * tc_gemm_launches(sh);
    }
  } else {
    count += 2 + (p->shared != MOE_SHARED_NONE ? 2 : 0);
  }
  // the small shared expert's own gate kernel
  if (two_streams && p->shared == MOE_SHARED_SIGMOID_GATED && shared_overlaps(*p)) count += 1;
  *n = count;
  return MOE_OK;
}

MOE_API moe_status moe_forward_counts(const moe_problem* p, const void* ws, size_t ws_bytes, const int32_t** counts) {
  MOE_TRY(validate_problem(p));
  if (counts == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  Layout L;
  MOE_TRY(check_ws(*p, ws, ws_bytes, &L));
  *counts = reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + L.counts);
  return MOE_OK;
}

MOE_API moe_status moe_read_device_error(void* ws, int32_t* code, moe_stream_t stream) {
  if (!ok_ptr(ws) || code == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  const cudaStream_t s = (cudaStream_t)stream;
  WsHeader h;
  MOE_CUDA(cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaStreamSynchronize(s));
  *code = h.error_bits;
  if (h.error_bits != 0) {
    MOE_CUDA(cudaMemsetAsync(ws, 0, sizeof(WsHeader), s));
    MOE_CUDA(cudaStreamSynchronize(s));
    return MOE_ERR_DEVICE_FLAG;
  }
  return MOE_OK;
}

MOE_API moe_status moe_check_device_error(void* ws, moe_stream_t stream, int32_t* code) {
  return moe_read_device_error(ws, code, stream);
}

MOE_API const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported combination";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_FLAG: return "device-side error flag set";
  }
  return "unknown status";
}
