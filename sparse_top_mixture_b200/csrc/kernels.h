// Internal launch wrappers (host side). Not part of the public C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

namespace stm {

// ---- router -----------------------------------------------------------
struct RouterSplit {
  int splits;       // partial sums along H
  int k_per_split;  // H elements per partial
};
RouterSplit router_split(int64_t T, int64_t H, int64_t Ecols);

cudaError_t launch_router_logits(int dtype, const void* x, const void* gate_w, const void* extra_row,
                                 float* partial, int64_t T, int64_t H, int64_t E, int64_t Ecols,
                                 const RouterSplit& sp, cudaStream_t s);
cudaError_t launch_topk(const float* partial, int splits, int64_t T, int64_t E, int64_t Ecols, int64_t k,
                        int score, int bias_mode, int renorm, const float* bias, float* weights,
                        int64_t* selected, float* gamma, cudaStream_t s);

// ---- dispatch ---------------------------------------------------------
int64_t dispatch_tokens_per_block(int64_t k);
int64_t dispatch_num_blocks(int64_t T, int64_t k);
cudaError_t launch_dispatch(int dtype, const int64_t* selected, const void* x, int64_t T, int64_t H, int64_t E,
                            int64_t k, int32_t* local, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                            int32_t* pair_pos, void* x_perm, int32_t* err, cudaStream_t s);

// ---- combine ----------------------------------------------------------
// y_perm [T*k, H] and shared_out [T, H] are fp32 for every problem dtype.
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
cudaError_t launch_tc_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                              int64_t I, int64_t H, int32_t* err, cudaStream_t s);
cudaError_t launch_tc_down(const Segments& sg, const void* h, const void* w_down, int64_t E_w, void* y,
                           const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                           cudaStream_t s);

}  // namespace stm
