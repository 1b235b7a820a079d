// Device-side tile table of a grouped GEMM over per-expert row segments.
//
// Segment e covers rows [off[e], off[e+1]) of the permuted activations. It is
// cut into ceil(count_e / BM) row tiles; pre[e] is the exclusive prefix of
// those tile counts, so pre[E] is the number of row tiles. Experts with no
// rows own no tiles and their weights are never read (the empty-expert rule
// of "feat: Phase 43 -- Sparse/Grouped MoE Dispatch", Tests). The table is
// rebuilt by every CTA from the device offsets, so the host never needs the
// counts (no host synchronisation, as in the grouped path of "Sparse MoE FFN
// for DFlash-family drafters").
#pragma once

#include "common.cuh"

namespace stm {

// Called by one full warp. off/pre are shared-memory arrays of E+1 entries.
// A table that is not monotone or leaves [0, rows_total] gets no tiles and
// raises MOE_DEVERR_BAD_EXPERT_ID (bit 1) in `err`, so that a malformed
// caller-supplied table can never steer a load or store out of bounds.
__device__ __forceinline__ void warp_build_tile_table(const int32_t* __restrict__ offsets, int E, int single_rows,
                                                      int BM, int* off, int* pre, int64_t rows_total,
                                                      int32_t* err) {
  const int lane = threadIdx.x & 31;
  if (offsets == nullptr) {  // one segment [0, single_rows)
    if (lane == 0) {
      off[0] = 0;
      off[1] = single_rows;
      pre[0] = 0;
      pre[1] = (int)ceil_div(single_rows, BM);
    }
    return;
  }
  int c[8];
  int local = 0;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    c[i] = 0;
    if (e < E) {
      const int a = offsets[e], b = offsets[e + 1];
      bad |= a < 0 || b < a || (int64_t)b > rows_total;
      off[e] = a;
      c[i] = (b - a + BM - 1) / BM;
      if (e == E - 1) off[E] = b;
    }
    local += c[i];
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) {
      raise_error(err, 1);
      for (int e = 0; e <= E; ++e) pre[e] = 0;
    }
    return;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - local;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    if (e < E) pre[e] = run;
    run += c[i];
  }
  if (lane == 31) pre[E] = incl;
}

// Row tile mt -> expert e with pre[e] <= mt < pre[e+1].
__device__ __forceinline__ int find_segment(const int* pre, int E, int mt) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= mt) lo = mid;
    else hi = mid;
  }
  return lo;
}

}  // namespace stm
