// Sorted-segment dispatch: histogram, exclusive scan, stable permutation and
// the gather of token copies into contiguous per-expert segments.
//
// Follows "Sparse MoE FFN for DFlash-family drafters" (What's here, SparseMoE:
// one argsort of the routed expert ids into contiguous per-expert segments)
// and "feat: Phase 43 -- Sparse/Grouped MoE Dispatch" (Neural Network:
// arg_sort grouping, then index_select of each expert's tokens).
//
// The argsort is done as a counting sort, which is stable by construction and
// needs no comparison passes:
//   1. each block counts the experts of its own pairs (block-local histogram);
//   2. one block turns the [blocks x E] counts into segment offsets and the
//      base position of every (block, expert) run;
//   3. each block ranks its pairs inside each expert run in pair order (warp
//      match + prefix counts across warps), writes the permutation and its
//      inverse, then copies each token row once into its k destinations with
//      16-byte vector loads and stores.
// Every block handles whole tokens and at most 256 pairs, so the ranking is a
// single pass. Counts are order-independent and positions are a pure function
// of the pair order: the result is deterministic.
#include "common.cuh"
#include "kernels.h"

namespace stm {

namespace {

constexpr int DTHREADS = 256;

__global__ void __launch_bounds__(DTHREADS) hist_kernel(const int64_t* __restrict__ sel, int64_t P, int k, int E,
                                                        int tok_per_blk, int32_t* __restrict__ local,
                                                        int32_t* err) {
  __shared__ int cnt[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += DTHREADS) cnt[e] = 0;
  __syncthreads();
  const int64_t q0 = (int64_t)blockIdx.x * tok_per_blk * k;
  const int64_t q1 = min(P, q0 + (int64_t)tok_per_blk * k);
  for (int64_t q = q0 + threadIdx.x; q < q1; q += DTHREADS) {
    const int64_t e = sel[q];
    if (e < 0 || e >= E) raise_error(err, 1);
    else atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += DTHREADS) local[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// One block: counts, offsets, and (in place) per-(block, expert) base positions.
__global__ void __launch_bounds__(DTHREADS) scan_kernel(int32_t* __restrict__ local, int nblk, int E,
                                                        int32_t* __restrict__ counts,
                                                        int32_t* __restrict__ offsets) {
  __shared__ int s[DTHREADS];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    for (int b = 0; b < nblk; ++b) {
      const int v = local[(int64_t)b * E + e];
      local[(int64_t)b * E + e] = run;
      run += v;
    }
  }
  s[e] = (e < E) ? run : 0;
  __syncthreads();
  for (int o = 1; o < DTHREADS; o <<= 1) {  // inclusive Hillis-Steele scan
    const int v = (e >= o) ? s[e - o] : 0;
    __syncthreads();
    s[e] += v;
    __syncthreads();
  }
  const int excl = s[e] - ((e < E) ? run : 0);
  if (e < E) {
    counts[e] = run;
    offsets[e] = excl;
    for (int b = 0; b < nblk; ++b) local[(int64_t)b * E + e] += excl;
  }
  if (e == DTHREADS - 1) offsets[E] = s[e];
}

template <typename T>
__global__ void __launch_bounds__(DTHREADS) permute_kernel(const int64_t* __restrict__ sel, int64_t P, int k,
                                                           int E, int tok_per_blk,
                                                           const int32_t* __restrict__ bases,
                                                           int32_t* __restrict__ sorted_pairs,
                                                           int32_t* __restrict__ pair_pos, const T* __restrict__ x,
                                                           T* __restrict__ x_perm, int H) {
  __shared__ int wcnt[DTHREADS / 32][kMaxExperts];
  __shared__ int pos_s[DTHREADS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (DTHREADS / 32) * kMaxExperts; i += DTHREADS) (&wcnt[0][0])[i] = 0;
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
  if (e >= 0 && rank == 0) wcnt[warp][e] = __popc(peers);
  __syncthreads();
  if (tid < E) {
    int run = bases[(int64_t)blockIdx.x * E + tid];
#pragma unroll
    for (int w = 0; w < DTHREADS / 32; ++w) {
      const int c = wcnt[w][tid];
      wcnt[w][tid] = run;
      run += c;
    }
  }
  __syncthreads();
  int pos = -1;
  if (e >= 0) {
    pos = wcnt[warp][e] + rank;
    sorted_pairs[pos] = (int32_t)q;
  }
  if (active) pair_pos[q] = pos;
  pos_s[tid] = pos;
  __syncthreads();

  if (x_perm == nullptr) return;
  constexpr int V = Elem<T>::kPerVec;
  const int nvec = H / V;
  const int ntok = (int)((q1 - q0) / k);
  const int64_t t0 = q0 / k;
  for (int tt = warp; tt < ntok; tt += DTHREADS / 32) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (t0 + tt) * (int64_t)H);
    for (int v = lane; v < nvec; v += 32) {
      const uint4 val = src[v];
      for (int j = 0; j < k; ++j) {
        const int p = pos_s[tt * k + j];
        if (p >= 0) reinterpret_cast<uint4*>(x_perm + (int64_t)p * H)[v] = val;
      }
    }
  }
}

// out[t] = sum_j y_perm[pair_pos[t*k+j]] + shared_out[t]: fp32 rows, summed in
// slot order in fp32, rounded once to the output type. Four columns per
// thread (16-byte fp32 loads).
template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ y_perm,
                                                      const int32_t* __restrict__ pair_pos,
                                                      const float* __restrict__ shared_out, T* __restrict__ out,
                                                      int H, int k) {
  __shared__ int pp[kMaxExperts];
  const int64_t t = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) pp[j] = pair_pos[t * k + j];
  __syncthreads();
  const int nvec = H / 4;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < nvec; v += gridDim.y * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int p = pp[j];
      if (p < 0) continue;
      const float4 y = reinterpret_cast<const float4*>(y_perm + (int64_t)p * H)[v];
      acc.x += y.x;
      acc.y += y.y;
      acc.z += y.z;
      acc.w += y.w;
    }
    if (shared_out != nullptr) {
      const float4 y = reinterpret_cast<const float4*>(shared_out + t * H)[v];
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
                            int32_t* pair_pos, void* x_perm, int32_t* err, cudaStream_t s) {
  const int tpb = (int)dispatch_tokens_per_block(k);
  const int nblk = (int)dispatch_num_blocks(T, k);
  const int64_t P = T * k;
  hist_kernel<<<nblk, DTHREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, local, err);
  scan_kernel<<<1, DTHREADS, 0, s>>>(local, nblk, (int)E, counts, offsets);
  if (dtype == 0)
    permute_kernel<float><<<nblk, DTHREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, local, sorted_pairs, pair_pos,
                                                    (const float*)x, (float*)x_perm, (int)H);
  else
    permute_kernel<__nv_bfloat16><<<nblk, DTHREADS, 0, s>>>(selected, P, (int)k, (int)E, tpb, local, sorted_pairs,
                                                            pair_pos, (const __nv_bfloat16*)x,
                                                            (__nv_bfloat16*)x_perm, (int)H);
  return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const float* y_perm, const int32_t* pair_pos, const float* shared_out,
                           void* out, int64_t T, int64_t H, int64_t k, cudaStream_t s) {
  const int64_t nvec = H / 4;
  const unsigned gy = (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(nvec, 128), T < 148 ? 16 : 1));
  dim3 grid((unsigned)T, gy);
  if (dtype == 0)
    combine_kernel<float><<<grid, 128, 0, s>>>(y_perm, pair_pos, shared_out, (float*)out, (int)H, (int)k);
  else
    combine_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(y_perm, pair_pos, shared_out, (__nv_bfloat16*)out, (int)H,
                                                       (int)k);
  return cudaGetLastError();
}

}  // namespace stm
