// The counting sort's scan: per-block expert counts -> segment offsets and
// the base position of every (block, expert) run. Done by the one CTA of a
// 1024-thread grid that finishes last (the dispatch's histogram kernel, or
// the forward's top-k kernel when it also counts).
#pragma once

#include "common.cuh"

namespace stm {

// Threads per scan CTA.
constexpr int kScanThreads = 1024;

// Threads that share one expert's column in the scan: the largest power of
// two up to 32 with next_pow2(E) x tpe <= kScanThreads.
inline int scan_threads_per_expert(int64_t E) {
  int ep = 1;
  while (ep < E) ep <<= 1;
  return ep >= kScanThreads ? 1 : (kScanThreads / ep < 32 ? kScanThreads / ep : 32);
}

// Exclusive scan of the [nblk x E] per-block counts by one CTA of
// kScanThreads threads: counts, offsets, and (in place) the base position of
// every (block, expert) run. Each expert's column is split among `tpe`
// threads of one warp (tpe = 4..32), which read their ranges with independent
// loads, combine through a segmented warp scan, and write the running bases.
// The counts were written by other CTAs of the same grid: read through L2.
// A range of up to kScanRegs entries is read once, in one round of loads,
// and kept in registers for the second pass; longer ranges (more than
// kScanRegs x tpe blocks) are read twice, in rounds of kScanRegs.
constexpr int kScanRegs = 16;

static __device__ void block_scan_counts(int32_t* __restrict__ local, int nblk, int E, int tpe,
                                         int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int* tot) {
  const int tid = threadIdx.x;
  const int e = tid / tpe, part = tid % tpe;
  const bool active = e < E;
  const int chunk = (nblk + tpe - 1) / tpe;
  const int b0 = min(nblk, part * chunk), b1 = min(nblk, b0 + chunk);
  const bool in_regs = b1 - b0 <= kScanRegs;
  int v[kScanRegs];
  int sum = 0;
  if (active) {
    for (int b = b0; b < b1; b += kScanRegs) {
#pragma unroll
      for (int i = 0; i < kScanRegs; ++i) v[i] = (b + i < b1) ? __ldcg(local + (int64_t)(b + i) * E + e) : 0;
#pragma unroll
      for (int i = 0; i < kScanRegs; ++i) sum += v[i];
    }
  }
  // segmented inclusive scan over the tpe parts of one expert (same warp)
  int incl = sum;
  for (int o = 1; o < tpe; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (part >= o) incl += x;
  }
  if (active && part == tpe - 1) tot[e] = incl;
  __syncthreads();
  if (tid < 32) {  // exclusive scan of the expert totals, 8 per lane
    int c[8], loc = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = tid * 8 + i;
      c[i] = ee < E ? tot[ee] : 0;
      loc += c[i];
    }
    int inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, inc, o);
      if (tid >= o) inc += x;
    }
    int run = inc - loc;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = tid * 8 + i;
      if (ee < E) {
        counts[ee] = c[i];
        offsets[ee] = run;
        tot[ee] = run;
      }
      run += c[i];
    }
    if (tid == 31) offsets[E] = inc;
  }
  __syncthreads();
  if (!active) return;
  int run = tot[e] + incl - sum;
  for (int b = b0; b < b1; b += kScanRegs) {
    if (!in_regs) {
#pragma unroll
      for (int i = 0; i < kScanRegs; ++i) v[i] = (b + i < b1) ? __ldcg(local + (int64_t)(b + i) * E + e) : 0;
    }
#pragma unroll
    for (int i = 0; i < kScanRegs; ++i) {
      if (b + i < b1) local[(int64_t)(b + i) * E + e] = run;
      run += v[i];
    }
  }
}

}  // namespace stm
