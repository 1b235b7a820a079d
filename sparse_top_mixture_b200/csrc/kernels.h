// Internal launch wrappers (host side). Not part of the public C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <mutex>

namespace stm {

// Host-side NVTX ranges naming the launch sequence (a profiler can select
// "moe_forward/" or "moe_backward/" launches). Header-only NVTX: without an
// attached tool each call is a no-op. A range is closed on every return path.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Consecutive stages inside one range: next() closes the previous stage's
// range and opens the next one; the last one closes with the object.
class NvtxStages {
 public:
  void next(const char* name) {
    close();
    nvtxRangePushA(name);
    open_ = true;
  }
  void close() {
    if (open_) nvtxRangePop();
    open_ = false;
  }
  ~NvtxStages() { close(); }

 private:
  bool open_ = false;
};

// Raise a kernel's dynamic shared memory limit to `bytes` once per device
// (the attribute belongs to the kernel's module in each device context).
// Each kernel passes its own flag and status arrays of kSmemAttrDevices.
constexpr int kSmemAttrDevices = 64;
inline cudaError_t set_max_dynamic_smem_once(const void* kernel, int bytes, std::once_flag* once, cudaError_t* err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSmemAttrDevices) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    err[dev] = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return err[dev];
}

// ---- router -----------------------------------------------------------
// Logits are computed as `splits` fp32 partial sums along H, each [T, ldo]
// (row pitch ldo >= E); the top-k kernel adds them in split order.
struct RouterPlan {
  bool tensor_cores;  // bf16: tcgen05 GEMM; fp32: SIMT GEMM
  int splits;
  int k_per_split;    // SIMT only: H elements per split
  int64_t ldo;
};
RouterPlan router_plan(int dtype, int64_t T, int64_t H, int64_t E);
size_t router_partial_bytes(int dtype, int64_t T, int64_t H, int64_t E);

// logits partials, then scores / top-k / weights (+ shared gate when
// shared_gate != nullptr: gamma[t] = sigmoid(x[t] . shared_gate)).
cudaError_t launch_route(int dtype, const void* x, const void* gate_w, const void* shared_gate, const float* bias,
                         int64_t T, int64_t H, int64_t E, int64_t k, int score, int bias_mode, int renorm,
                         float* partial, float* weights, int64_t* selected, float* gamma, int32_t* err,
                         cudaStream_t s);
// gamma[t] = sigmoid(x[t] . g) on its own (used when the shared expert runs
// on a second stream, independent of the router).
cudaError_t launch_shared_gate(int dtype, const void* x, const void* g, int64_t T, int64_t H, float* gamma,
                               cudaStream_t s);
cudaError_t launch_topk(const float* partial, int splits, int64_t ldo, int64_t T, int64_t E, int64_t k, int score,
                        int bias_mode, int renorm, const float* bias, float* weights, int64_t* selected,
                        const void* x, const void* shared_gate, int64_t H, int dtype, float* gamma, cudaStream_t s);

// ---- dispatch ---------------------------------------------------------
int64_t dispatch_tokens_per_block(int64_t k);
int64_t dispatch_num_blocks(int64_t T, int64_t k);
cudaError_t launch_dispatch(int dtype, const int64_t* selected, const void* x, int64_t T, int64_t H, int64_t E,
                            int64_t k, int32_t* local, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                            int32_t* pair_pos, void* x_perm, int32_t* err, uint32_t* ticket, cudaStream_t s);

// ---- combine ----------------------------------------------------------
// y_perm [T*k, H] and shared_out [T, H] are fp32 for every problem dtype.
// Expert parallelism: where the dispatch stores each pair's row instead of
// x_perm (the owner's arena, slot rank*C + position inside the owner's
// run), with its routing weight and local expert id; the empty slots of
// every owner's region, the y-offset mailbox and the rows flag as for
// moe_ep_send (ep_peer.cu builds it).
struct EpDest {
  uint8_t* const* arenas;  // device array of the G arena base addresses
  int G, rank, El;
  int64_t C;               // slots per source: T*k
  size_t x_off, w_off, id_off, yoff_off, flag_off;
  const float* rw;         // routing weights [T, k]
  uint32_t* done;          // this rank's completed-block counter
  uint64_t* epoch;         // this rank's epoch (advanced and published)
};
// Expert parallelism, the other way: where a down GEMM's weighted rows go
// instead of y_perm. Sorted row p came from slot j = scale_idx[p] = s*C + i
// of this rank's arena; its row goes to source s's arena, y region, row
// yoff[s] + i (yoff: this rank's mailbox).
struct EpRet {
  uint8_t* const* arenas;
  int64_t C;
  size_t y_off;
  const int32_t* yoff;
};
// This rank's arena regions (expert parallelism), for moe_ep_experts.
struct EpViews {
  void* x;          // received rows [G*C][H]
  float* w;         // their routing weights [G*C]
  int64_t* id;      // their local expert ids [G*C], -1 for empty slots
  int32_t* yoff;    // the sources' y offsets [G]
  size_t y_off, ret_flag_off;
  uint64_t* epoch;  // this rank's epoch
  int64_t C;
};
bool ep_views(const moe_problem& p, int G, void* own_arena, EpViews* v);
// Publish this rank's epoch (not advanced) into flag slot `rank` at byte
// offset flag_off of every arena, after a system-scope fence.
cudaError_t launch_ep_publish(uint8_t* const* arenas, int G, int rank, size_t flag_off, const uint64_t* epoch,
                              cudaStream_t s);
// moe_ep_dispatch_send's layout helper; false if the problem or G is invalid.
bool ep_dest(const moe_problem& p, int G, int rank, void* const* arenas, void* own_arena, const float* rw,
             EpDest* d);
// The dispatch (histogram, scan, ranking) with each row stored to its
// owner's arena; x_perm is not written.
cudaError_t launch_dispatch_ep(int dtype, const int64_t* selected, const void* x, int64_t T, int64_t H, int64_t E,
                               int64_t k, int32_t* local, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                               int32_t* pair_pos, int32_t* err, uint32_t* ticket, const EpDest& ep, cudaStream_t s);
cudaError_t launch_combine(int dtype, const float* y_perm, const int32_t* pair_pos, const float* shared_out,
                           void* out, int64_t T, int64_t H, int64_t k, cudaStream_t s);

// ---- grouped GEMMs ----------------------------------------------------
// A segment table is either `offsets` [E+1] on the device, or (offsets ==
// nullptr) one segment of `single_rows` rows.
struct Segments {
  const int32_t* offsets;
  int32_t E;
  int32_t single_rows;
  int64_t rows_total;  // rows of the A / out buffers (bound for TMA)
};

// SIMT fp32: h = silu(A Wg^T) * (A Wu^T) and y = scale * (h Wd^T).
cudaError_t launch_simt_gate_up(const Segments& sg, const float* A, const float* w_gate_up, float* h, int64_t I,
                                int64_t H, int32_t* err, cudaStream_t s);
cudaError_t launch_simt_down(const Segments& sg, const float* h, const float* w_down, float* y,
                             const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                             cudaStream_t s);

// tcgen05 / TMEM bf16 grouped GEMMs: h is bf16, y is fp32.
// Variant: 1 = one CTA per 128-row tile; 2 = CTA pairs (cta_group::2) per
// 256-row tile, for segments averaging at least 192 rows.
int tc_gemm_variant(const Segments& sg, bool down);
int tc_gemm_launches(const Segments& sg);
bool get_encode();
bool make_tensor_map_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box);
int num_sms();
// CTA-pair GEMMs; A is the row-major operand (x_perm or h), the tensor maps
// are built inside.
cudaError_t launch_tc2_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                               int64_t I, int64_t H, int32_t* err, int num_sms, cudaStream_t s);
cudaError_t launch_tc2_down(const Segments& sg, const void* A, const void* w_down, int64_t E_w, void* y,
                            const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                            int num_sms, cudaStream_t s);
cudaError_t launch_tc_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                              int64_t I, int64_t H, int32_t* err, cudaStream_t s);
int tc_router_splits(int64_t T, int64_t H, int64_t E);
cudaError_t launch_tc_logits(const void* x, const void* gate_w, int64_t T, int64_t H, int64_t E, float* partial,
                             int64_t ldo, int splits, int32_t* err, cudaStream_t s);
// Weight-gradient GEMM: out[e][m][n] = sum_{k in [koff[e], koff[e+1])}
// A[k][m] * B[k][n]; A [rows][lda] and B [rows][ldb] bf16 row-major (read
// MN-major; rows at or past `rows` read as zero), koff [E+1] on the device
// (non-decreasing multiples of 64, at most k_extent), out fp32 [E][M][N]; an
// expert with an empty range gets zeros.
cudaError_t launch_wgrad(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t rows, const int32_t* koff,
                         int64_t k_extent, int E, int64_t M, int64_t N, float* out, int32_t* err, cudaStream_t s);
// y[p][n] = scale(p) * sum_k A[p][k] * W[e][k][n] over the segments, with W
// stored [E_w][K][N] (N innermost, read MN-major: no transposed copy); A
// [rows][lda] bf16 (K used columns, lda a multiple of 8), y fp32 [rows][N].
// The one-CTA or pair kernel as for down.
cudaError_t launch_tc_down_kn(const Segments& sg, const void* A, int64_t lda, const void* w_kn, int64_t E_w, void* y,
                              const float* row_scale, const int32_t* scale_idx, int64_t N, int64_t K, int32_t* err,
                              cudaStream_t s);
// The down GEMM with each weighted row stored into its source's arena (EpRet)
// instead of y; every epilogue warp fences its stores at system scope last.
// The one-CTA or pair kernel as for down.
cudaError_t launch_tc_down_ep(const Segments& sg, const void* h, const void* w_down, int64_t E_w,
                              const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, const EpRet& ep,
                              int32_t* err, cudaStream_t s);
cudaError_t launch_tc2_down_ep(const Segments& sg, const void* A, const void* w_down, int64_t E_w,
                               const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I,
                               const EpRet& ep, int32_t* err, int num_sms, cudaStream_t s);
cudaError_t launch_tc2_down_kn(const Segments& sg, const void* A, int64_t lda, const void* w_kn, int64_t E_w, void* y,
                               const float* row_scale, const int32_t* scale_idx, int64_t N, int64_t K, int32_t* err,
                               int num_sms, cudaStream_t s);
cudaError_t launch_tc_down(const Segments& sg, const void* h, const void* w_down, int64_t E_w, void* y,
                           const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                           cudaStream_t s);

}  // namespace stm
