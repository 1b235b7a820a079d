// Sorted-segment dispatch: histogram, exclusive scan, stable permutation and
// the gather of token copies into contiguous per-expert segments.
//
// Follows "Sparse MoE FFN for DFlash-family drafters" (What's here, SparseMoE:
// one argsort of the routed expert ids into contiguous per-expert segments)
// and "feat: Phase 43 -- Sparse/Grouped MoE Dispatch" (Neural Network:
// arg_sort grouping, then index_select of each expert's tokens).
//
// The argsort is done as a counting sort, which is stable by construction and
// needs no comparison passes. Two launches:
//   1. hist_scan_kernel: each 256-pair dispatch block counts the experts of
//      its own pairs (four dispatch blocks per 1024-thread CTA); the last CTA
//      to finish (an atomic ticket, no waiting on other CTAs) turns the
//      [blocks x E] counts into segment offsets and the base position of
//      every (block, expert) run, and resets the ticket;
//   2. permute_gather_kernel: each dispatch block ranks its pairs inside each
//      expert run in pair order (warp match + prefix counts across warps),
//      writes the permutation and its inverse, and copies its tokens' rows to
//      their k segment slots with 16-byte vector loads and stores. Several
//      CTAs share one dispatch block, each copying a slice of the columns (the
//      ranking, a few hundred integer operations, is repeated by each), so
//      that the copy spreads over the whole GPU even for a 16-token batch.
// Every dispatch block handles whole tokens and at most 256 pairs, so the
// ranking is a single pass. Counts are order-independent and positions are a
// pure function of the pair order: the result is deterministic.
#include "common.cuh"
#include "kernels.h"
#include "peer.cuh"

namespace stm {

namespace {

constexpr int DTHREADS = 256;     // pairs per dispatch block
constexpr int HIST_SUB = 4;       // dispatch blocks per histogram CTA
constexpr int SCAN_THREADS = DTHREADS * HIST_SUB;

// Exclusive scan of the [nblk x E] per-block counts by one CTA of
// SCAN_THREADS threads: counts, offsets, and (in place) the base position of
// every (block, expert) run. Each expert's column is split among `tpe`
// threads of one warp (tpe = 4..32), which read their ranges with independent
// loads, combine through a segmented warp scan, and write the running bases.
// The counts were written by other CTAs of the same grid: read through L2.
// A range of up to kScanRegs entries is read once, in one round of loads,
// and kept in registers for the second pass; longer ranges (more than
// kScanRegs x tpe blocks) are read twice, in rounds of kScanRegs.
constexpr int kScanRegs = 16;

__device__ void block_scan_counts(int32_t* __restrict__ local, int nblk, int E, int tpe,
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

__global__ void __launch_bounds__(SCAN_THREADS) hist_scan_kernel(const int64_t* __restrict__ sel, int64_t P, int k,
                                                                 int E, int tok_per_blk, int nblk, int tpe,
                                                                 int32_t* __restrict__ local,
                                                                 int32_t* __restrict__ counts,
                                                                 int32_t* __restrict__ offsets,
                                                                 uint32_t* __restrict__ ticket, int32_t* err) {
  __shared__ int cnt[HIST_SUB][kMaxExperts];
  __shared__ int last;
  const int sub = threadIdx.x / DTHREADS, t = threadIdx.x % DTHREADS;
  for (int e = t; e < E; e += DTHREADS) cnt[sub][e] = 0;
  __syncthreads();
  const int b = blockIdx.x * HIST_SUB + sub;
  if (b < nblk) {
    const int64_t q0 = (int64_t)b * tok_per_blk * k;
    const int64_t q1 = min(P, q0 + (int64_t)tok_per_blk * k);
    for (int64_t q = q0 + t; q < q1; q += DTHREADS) {
      const int64_t e = sel[q];
      if (e < 0 || e >= E) raise_error(err, 1);
      else atomicAdd(&cnt[sub][e], 1);
    }
  }
  __syncthreads();
  if (b < nblk)
    for (int e = t; e < E; e += DTHREADS) local[(int64_t)b * E + e] = cnt[sub][e];
  // Publish this CTA's counts, then take a ticket: the CTA that draws the
  // last one sees every other CTA's counts and does the scan.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  block_scan_counts(local, nblk, E, tpe, counts, offsets, &cnt[0][0]);
  if (threadIdx.x == 0) *ticket = 0u;  // ready for the next dispatch on this workspace
}

// Rank the block's pairs, write sorted_pairs / pair_pos (column slice 0
// only), and copy column slice blockIdx.y of each token row to the slots of
// its k pairs: x_perm[pair_pos[t*k + j]] = x[t]. With EP (expert
// parallelism), the row of sorted position p of expert e goes instead to
// owner q = e / El's arena, slot rank*C + p - offsets[q*El] (plain peer
// stores), with its routing weight and local id; every CTA then marks its
// share of the owners' empty slots, and the last one publishes the epoch.
template <typename T, bool EP>
__global__ void __launch_bounds__(DTHREADS) permute_gather_kernel(const int64_t* __restrict__ sel, int64_t P, int k,
                                                                  int E, int tok_per_blk,
                                                                  const int32_t* __restrict__ bases,
                                                                  int32_t* __restrict__ sorted_pairs,
                                                                  int32_t* __restrict__ pair_pos,
                                                                  const T* __restrict__ x, T* __restrict__ x_perm,
                                                                  int64_t Tn, int H, int vec_per_slice,
                                                                  const int32_t* __restrict__ offsets, EpDest ep) {
  // Per-warp counts of each expert (at most 32, so 16 bits) and the slot of
  // every pair: 5 KB of shared memory, small enough to sit beside a
  // persistent GEMM CTA on the same SM.
  __shared__ __align__(16) uint16_t wcnt[DTHREADS / 32][kMaxExperts];
  __shared__ int s_pos[DTHREADS];
  __shared__ int s_dst[EP ? DTHREADS : 1];  // EP: the pair's arena slot, owner in the top bits
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (DTHREADS / 32) * kMaxExperts / 2; i += DTHREADS)
    reinterpret_cast<uint32_t*>(&wcnt[0][0])[i] = 0u;
  __syncthreads();

  const int64_t q0 = (int64_t)blockIdx.x * tok_per_blk * k;
  const int64_t q1 = min(P, q0 + (int64_t)tok_per_blk * k);
  const int64_t q = q0 + tid;
  const bool active = q < q1;
  int e = -1;
  if (active) {
    const int64_t v = sel[q];
    e = (v >= 0 && v < E) ? (int)v : -1;
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && rank == 0) wcnt[warp][e] = (uint16_t)__popc(peers);
  __syncthreads();
  // slot = this block's base for the expert + pairs of earlier warps + rank
  int pos = -1;
  if (e >= 0) {
    pos = bases[(int64_t)blockIdx.x * E + e] + rank;
    for (int w = 0; w < warp; ++w) pos += wcnt[w][e];
  }
  s_pos[tid] = pos;
  if (blockIdx.y == 0) {
    if (e >= 0) sorted_pairs[pos] = (int32_t)q;
    if (active) pair_pos[q] = pos;
  }
  if constexpr (EP) {
    int owner = -1;
    int64_t slot = -1;
    if (e >= 0) {
      owner = e / ep.El;
      slot = (int64_t)ep.rank * ep.C + (pos - offsets[owner * ep.El]);
      if (blockIdx.y == 0) {
        reinterpret_cast<float*>(ep.arenas[owner] + ep.w_off)[slot] = ep.rw[q];
        reinterpret_cast<int64_t*>(ep.arenas[owner] + ep.id_off)[slot] = e - owner * ep.El;
      }
    }
    s_dst[tid] = owner;  // the slot follows from pos and the owner's offset below
  } else {
    if (x_perm == nullptr) return;
  }
  __syncthreads();
  // Copy: work items (token of the block, 16-byte vector of this slice),
  // consecutive threads on consecutive vectors of one row.
  constexpr int V = Elem<T>::kPerVec;
  const int nvec = H / V;
  const int v0 = blockIdx.y * vec_per_slice;
  const int nv = min(nvec, v0 + vec_per_slice) - v0;
  if (!EP && nv <= 0) return;  // (with EP every CTA must reach the publication below)
  const int64_t t0 = (int64_t)blockIdx.x * tok_per_blk;
  const int ntok = (int)min((int64_t)tok_per_blk, Tn - t0);
  const int items = ntok * max(nv, 0);
  for (int it = tid; it < items; it += DTHREADS) {
    const int i = it / nv, v = v0 + (it - i * nv);
    const uint4 val = reinterpret_cast<const uint4*>(x + (t0 + i) * (int64_t)H)[v];
    for (int j = 0; j < k; ++j) {
      const int p = s_pos[i * k + j];
      if (p < 0) continue;
      if constexpr (EP) {
        const int owner = s_dst[i * k + j];
        const int64_t slot = (int64_t)ep.rank * ep.C + (p - offsets[owner * ep.El]);
        reinterpret_cast<uint4*>(reinterpret_cast<T*>(ep.arenas[owner] + ep.x_off) + slot * H)[v] = val;
      } else {
        reinterpret_cast<uint4*>(x_perm + (int64_t)p * H)[v] = val;
      }
    }
  }
  if constexpr (EP) {
    // the owners' empty slots and where their rows sit in our sorted order
    const int64_t nb = (int64_t)gridDim.x * gridDim.y;
    const int64_t b = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    for (int64_t jj = b * DTHREADS + tid; jj < (int64_t)ep.G * ep.C; jj += nb * DTHREADS) {
      const int o = (int)(jj / ep.C);
      const int64_t i = jj - (int64_t)o * ep.C;
      if (i >= offsets[(o + 1) * ep.El] - offsets[o * ep.El])
        reinterpret_cast<int64_t*>(ep.arenas[o] + ep.id_off)[(int64_t)ep.rank * ep.C + i] = -1;
      if (i == 0) reinterpret_cast<int32_t*>(ep.arenas[o] + ep.yoff_off)[ep.rank] = offsets[o * ep.El];
    }
    publish_when_done(ep.done, ep.epoch, true, ep.arenas, ep.G, ep.flag_off, ep.rank);
  }
}

// out[t] = sum_j y_perm[pair_pos[t*k+j]] + shared_out[t]: fp32 rows, summed in
// slot order in fp32, rounded once to the output type. A work unit is one
// token's 4 KB column chunk (256 threads x one 16-byte vector of each of its
// k rows), so each y row is read as 4 KB contiguous runs; units are strided
// over a grid of a few CTAs per SM, so every SM gets the same share. A
// thread loads up to eight slots' pair positions and then issues those rows'
// loads together, before adding them in slot order.
constexpr int CTHREADS = 256;

template <typename T>
__global__ void __launch_bounds__(CTHREADS) combine_kernel(const float* __restrict__ y_perm,
                                                           const int32_t* __restrict__ pair_pos,
                                                           const float* __restrict__ shared_out,
                                                           T* __restrict__ out, int64_t Tn, int H, int k) {
  const int nvec = H / 4;
  const int chunks = (nvec + CTHREADS - 1) / CTHREADS;
  const int64_t units = Tn * chunks;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t t = u / chunks;
    const int v = (int)(u - t * chunks) * CTHREADS + threadIdx.x;
    if (v >= nvec) continue;
    const int32_t* pp = pair_pos + t * k;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < k; j0 += 8) {
      int p[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) p[j] = j0 + j < k ? __ldg(pp + j0 + j) : -1;
      float4 y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        y[j] = p[j] >= 0 ? __ldcs(reinterpret_cast<const float4*>(y_perm + (int64_t)p[j] * H) + v)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (p[j] < 0) continue;  // skipped pairs and slots past k add nothing
        acc.x += y[j].x;
        acc.y += y[j].y;
        acc.z += y[j].z;
        acc.w += y[j].w;
      }
    }
    if (shared_out != nullptr) {
      const float4 y = __ldcs(reinterpret_cast<const float4*>(shared_out + t * H) + v);
      acc.x += y.x;
      acc.y += y.y;
      acc.z += y.z;
      acc.w += y.w;
    }
    if constexpr (sizeof(T) == 2) {
      uint2 o;
      o.x = pack_bf16x2(acc.x, acc.y);
      o.y = pack_bf16x2(acc.z, acc.w);
      reinterpret_cast<uint2*>(out + t * H)[v] = o;
    } else {
      reinterpret_cast<float4*>(out + t * H)[v] = acc;
    }
  }
}

}  // namespace

int64_t dispatch_tokens_per_block(int64_t k) { return std::max<int64_t>(1, DTHREADS / k); }
int64_t dispatch_num_blocks(int64_t T, int64_t k) { return ceil_div(T, dispatch_tokens_per_block(k)); }

cudaError_t launch_dispatch(int dtype, const int64_t* selected, const void* x, int64_t T, int64_t H, int64_t E,
                            int64_t k, int32_t* local, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                            int32_t* pair_pos, void* x_perm, int32_t* err, uint32_t* ticket, cudaStream_t s) {
  const int tpb = (int)dispatch_tokens_per_block(k);
  const int nblk = (int)dispatch_num_blocks(T, k);
  const int64_t P = T * k;
  int ep = 1;
  while (ep < E) ep <<= 1;
  const int tpe = std::min(32, SCAN_THREADS / ep);
  hist_scan_kernel<<<(unsigned)ceil_div(nblk, HIST_SUB), SCAN_THREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, nblk,
                                                                             tpe, local, counts, offsets, ticket, err);
  // Column slices per dispatch block: enough CTAs for about eight per SM,
  // each slice at least 32 vectors (512 bytes) of a row.
  const int V = dtype == 0 ? 4 : 8;
  const int64_t nvec = H / V;
  int slices = 1;
  if (x_perm != nullptr)
    slices = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(148 * 8, nblk), nvec / 32));
  const int vps = (int)ceil_div(nvec, slices);
  slices = (int)ceil_div(nvec, vps);
  const dim3 grid((unsigned)nblk, (unsigned)slices);
  if (dtype == 0)
    permute_gather_kernel<float, false><<<grid, DTHREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, local,
                                                                  sorted_pairs, pair_pos, (const float*)x,
                                                                  (float*)x_perm, T, (int)H, vps, nullptr, EpDest{});
  else
    permute_gather_kernel<__nv_bfloat16, false><<<grid, DTHREADS, 0, s>>>(
        selected, P, (int)k, (int)E, tpb, local, sorted_pairs, pair_pos, (const __nv_bfloat16*)x,
        (__nv_bfloat16*)x_perm, T, (int)H, vps, nullptr, EpDest{});
  return cudaGetLastError();
}

cudaError_t launch_dispatch_ep(int dtype, const int64_t* selected, const void* x, int64_t T, int64_t H, int64_t E,
                               int64_t k, int32_t* local, int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
                               int32_t* pair_pos, int32_t* err, uint32_t* ticket, const EpDest& ep, cudaStream_t s) {
  const int tpb = (int)dispatch_tokens_per_block(k);
  const int nblk = (int)dispatch_num_blocks(T, k);
  const int64_t P = T * k;
  int ep2 = 1;
  while (ep2 < E) ep2 <<= 1;
  const int tpe = std::min(32, SCAN_THREADS / ep2);
  hist_scan_kernel<<<(unsigned)ceil_div(nblk, HIST_SUB), SCAN_THREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, nblk,
                                                                             tpe, local, counts, offsets, ticket, err);
  const int V = dtype == 0 ? 4 : 8;
  const int64_t nvec = H / V;
  int slices = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(148 * 8, std::max(nblk, 1)), nvec / 32));
  const int vps = (int)ceil_div(nvec, slices);
  slices = (int)ceil_div(nvec, vps);
  const dim3 grid((unsigned)std::max(nblk, 1), (unsigned)slices);
  if (dtype == 0)
    permute_gather_kernel<float, true><<<grid, DTHREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, local,
                                                                 sorted_pairs, pair_pos, (const float*)x, nullptr, T,
                                                                 (int)H, vps, offsets, ep);
  else
    permute_gather_kernel<__nv_bfloat16, true><<<grid, DTHREADS, 0, s>>>(
        selected, P, (int)k, (int)E, tpb, local, sorted_pairs, pair_pos, (const __nv_bfloat16*)x, nullptr, T, (int)H,
        vps, offsets, ep);
  return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const float* y_perm, const int32_t* pair_pos, const float* shared_out,
                           void* out, int64_t T, int64_t H, int64_t k, cudaStream_t s) {
  const int64_t units = T * ceil_div(H / 4, CTHREADS);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, 148 * 8));
  if (dtype == 0)
    combine_kernel<float><<<grid, CTHREADS, 0, s>>>(y_perm, pair_pos, shared_out, (float*)out, T, (int)H, (int)k);
  else
    combine_kernel<__nv_bfloat16><<<grid, CTHREADS, 0, s>>>(y_perm, pair_pos, shared_out, (__nv_bfloat16*)out, T,
                                                           (int)H, (int)k);
  return cudaGetLastError();
}

}  // namespace stm
