// Router: logits GEMM and warp-per-token score + top-k.
//
// Follows "mstar.model.components.moe" (Router contract, TopKRouter: softmax
// top-k with optional renormalisation, int64 indices) and "Sparse MoE FFN for
// DFlash-family drafters" (What's here, MoEGate: sqrtsoftplus scores and an
// fp32 aux-loss-free bias that only ranks experts). The shared-expert gate of
// SparseMoeBlockWithSharedExpert, sigmoid(shared_gate(x)), is a per-token dot
// product computed by the top-k kernel.
//
// Logits: for bf16 problems the tcgen05 GEMM (fp32 accumulate) computes x .
// gate_w^T; it reads x once, so the router costs about one pass over the
// hidden states. fp32 problems use the SIMT tile below. Both split the H
// reduction into a few partial sums when there are too few token/expert tiles
// to fill the GPU (the 16-token decode batch), and the top-k kernel adds the
// partials in a fixed order, so routing is bit-reproducible run to run.
#include "common.cuh"
#include "kernels.h"

namespace stm {

namespace {

constexpr int RBM = 64, RBN = 64, RBK = 32, RTHREADS = 256;

template <typename T>
__global__ void __launch_bounds__(RTHREADS) router_logits_kernel(const T* __restrict__ x,
                                                                 const T* __restrict__ gate_w,
                                                                 float* __restrict__ partial, int Tn, int H,
                                                                 int E, int ldo, int k_per_split) {
  __shared__ float As[RBK][RBM + 4];
  __shared__ float Bs[RBK][RBN + 4];
  constexpr int V = Elem<T>::kPerVec;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.x * RBM, n0 = blockIdx.y * RBN;
  const int kb = blockIdx.z * k_per_split;
  const int ke = min(H, kb + k_per_split);

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  constexpr int VPR = RBK / V;         // vectors per tile row
  constexpr int NV = RBM * VPR;        // vectors per tile
  static_assert(RBM == RBN && NV % RTHREADS == 0, "tile loads: whole vectors per thread");
  constexpr int PV = NV / RTHREADS;
  // The next K slice is read into registers while the current one is
  // multiplied out of shared memory (the same products in the same order).
  uint4 va[PV], vb[PV];
  auto load_slice = [&](int k0) {
#pragma unroll
    for (int u = 0; u < PV; ++u) {
      const int i = tid + u * RTHREADS;
      const int r = i / VPR, kk = k0 + (i % VPR) * V;
      const int row = m0 + r, col = n0 + r;
      va[u] = (row < Tn && kk < ke) ? *reinterpret_cast<const uint4*>(x + (int64_t)row * H + kk)
                                    : make_uint4(0u, 0u, 0u, 0u);
      vb[u] = (col < E && kk < ke) ? *reinterpret_cast<const uint4*>(gate_w + (int64_t)col * H + kk)
                                   : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto store_slice = [&]() {
#pragma unroll
    for (int u = 0; u < PV; ++u) {
      const int i = tid + u * RTHREADS;
      const int r = i / VPR, c = (i % VPR) * V;
      float f[8];
      if constexpr (V == 8) unpack16_bf16(va[u], f); else unpack16(va[u], f, nullptr);
#pragma unroll
      for (int q = 0; q < V; ++q) As[c + q][r] = f[q];
      if constexpr (V == 8) unpack16_bf16(vb[u], f); else unpack16(vb[u], f, nullptr);
#pragma unroll
      for (int q = 0; q < V; ++q) Bs[c + q][r] = f[q];
    }
  };
  if (kb < ke) load_slice(kb);
  for (int k0 = kb; k0 < ke; k0 += RBK) {
    store_slice();
    __syncthreads();
    if (k0 + RBK < ke) load_slice(k0 + RBK);
#pragma unroll 8
    for (int kk = 0; kk < RBK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* dst = partial + (int64_t)blockIdx.z * Tn * ldo;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty + 16 * i;
    if (row >= Tn) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx + 16 * j;
      if (col < E) dst[(int64_t)row * ldo + col] = acc[i][j];
    }
  }
}

// The top-k orders experts by (key descending, index ascending). A float key
// maps to an unsigned integer with the same order (sign bit flipped for
// non-negative values, all bits for negative ones; -0 joins +0 and NaN ranks
// below every number), so one warp-wide integer max finds the best key and one
// integer min over the lanes holding it finds the lowest index among equals.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int TOPK_WARPS = 8;

// One warp per token; lane l owns experts [l*NS, l*NS + NS), NS = 1, 2, 4 or
// 8 (E up to 32, 64, 128 or 256), so a lane reads its logits of one partial
// with one or two 16-byte loads when rows are 16-byte aligned.
template <typename TX, int NS>
__global__ void __launch_bounds__(TOPK_WARPS * 32) topk_kernel(const float* __restrict__ partial, int splits,
                                                                int64_t ldo, int vec4, int Tn, int E, int k,
                                                                int score, int bias_mode, int renorm,
                                                                const float* __restrict__ bias,
                                                                float* __restrict__ weights,
                                                                int64_t* __restrict__ selected,
                                                                const TX* __restrict__ x,
                                                                const TX* __restrict__ shared_gate, int H,
                                                                float* __restrict__ gamma) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * TOPK_WARPS + (threadIdx.x >> 5);
  if (t >= Tn) return;
  const int e0 = lane * NS;

  float logit[NS], sc[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) logit[i] = 0.f;
  if (NS >= 4 && vec4 && e0 + NS <= E) {
    for (int s = 0; s < splits; ++s) {
      const float4* src = reinterpret_cast<const float4*>(partial + ((int64_t)s * Tn + t) * ldo + e0);
#pragma unroll
      for (int v = 0; v < NS / 4; ++v) {
        const float4 q = src[v];
        logit[4 * v] += q.x;
        logit[4 * v + 1] += q.y;
        logit[4 * v + 2] += q.z;
        logit[4 * v + 3] += q.w;
      }
    }
  } else {
    for (int s = 0; s < splits; ++s) {
      const float* src = partial + ((int64_t)s * Tn + t) * ldo;
#pragma unroll
      for (int i = 0; i < NS; ++i)
        if (e0 + i < E) logit[i] += src[e0 + i];
    }
  }
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    if (e0 + i >= E) logit[i] = -INFINITY;
    else if (bias_mode == 1) logit[i] += bias[e0 + i];
  }
  if (score == 0) {  // softmax over all E experts
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NS; ++i) m = fmaxf(m, logit[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      sc[i] = (e0 + i < E) ? expf(logit[i] - m) : 0.f;
      z += sc[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
    for (int i = 0; i < NS; ++i) sc[i] = sc[i] / z;
  } else if (score == 1) {  // sigmoid
#pragma unroll
    for (int i = 0; i < NS; ++i) sc[i] = 1.0f / (1.0f + expf(-logit[i]));
  } else {  // sqrtsoftplus: sqrt(log(1 + e^l)), stable form
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const float l = logit[i];
      sc[i] = sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
    }
  }
  // Selection key. Without a selection bias every score function is
  // increasing in the logit, so ranking by the logit ranks by the score and
  // avoids ties introduced by rounding the scores.
  uint32_t key[NS];
  uint32_t live = 0;  // bit i: expert e0 + i exists and is not yet taken
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    const int e = e0 + i;
    key[i] = order_key((bias_mode == 2 && e < E) ? sc[i] + bias[e] : logit[i]);
    if (e < E) live |= 1u << i;
  }

  // Slot j's expert and raw weight go to shared memory, written by the lane
  // that owns the expert; the renormalising sum runs in slot order.
  __shared__ float s_w[TOPK_WARPS][kMaxExperts];
  __shared__ int s_e[TOPK_WARPS][kMaxExperts];
  const int wid = threadIdx.x >> 5;
  for (int j = 0; j < k; ++j) {
    // This lane's best live expert: largest key, then lowest index.
    uint32_t bk = 0;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if (((live >> i) & 1u) && (bi < 0 || key[i] > bk)) { bk = key[i]; bi = i; }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bi >= 0 ? bk : 0u);
    const int cand = (bi >= 0 && bk == wk) ? e0 + bi : 0x7fffffff;
    const int we = (int)__reduce_min_sync(0xffffffffu, (uint32_t)cand);
    if (we == cand) {  // the owning lane
      float w = 0.f;
#pragma unroll
      for (int i = 0; i < NS; ++i)
        if (i == bi) w = sc[i];
      live &= ~(1u << bi);
      s_w[wid][j] = w;
      s_e[wid][j] = we;
    }
  }
  __syncwarp();
  float tot = 0.f;
  if (renorm)
    for (int j = 0; j < k; ++j) tot += s_w[wid][j];
  for (int j = lane; j < k; j += 32) {
    float w = s_w[wid][j];
    if (renorm) w = tot > 0.f ? w / tot : 0.f;
    weights[(int64_t)t * k + j] = w;
    selected[(int64_t)t * k + j] = (int64_t)s_e[wid][j];
  }
  if (gamma != nullptr) {
    // gamma[t] = sigmoid(x[t] . shared_gate): fp32 dot product, lanes over
    // 16-byte vectors, butterfly sum (same result in every lane).
    constexpr int V = Elem<TX>::kPerVec;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    const uint4* gr = reinterpret_cast<const uint4*>(shared_gate);
    float acc = 0.f;
    for (int v = lane; v < H / V; v += 32) {
      float a[8], b[8];
      if constexpr (V == 8) {
        unpack16_bf16(xr[v], a);
        unpack16_bf16(gr[v], b);
      } else {
        unpack16(xr[v], a, nullptr);
        unpack16(gr[v], b, nullptr);
      }
#pragma unroll
      for (int q = 0; q < V; ++q) acc = fmaf(a[q], b[q], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) gamma[t] = 1.0f / (1.0f + expf(-acc));
  }
}

// gamma[t] = sigmoid(x[t] . g), one warp per token.
template <typename TX>
__global__ void __launch_bounds__(256) shared_gate_kernel(const TX* __restrict__ x, const TX* __restrict__ g, int Tn,
                                                          int H, float* __restrict__ gamma) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= Tn) return;
  constexpr int V = Elem<TX>::kPerVec;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
  const uint4* gr = reinterpret_cast<const uint4*>(g);
  float acc = 0.f;
  for (int v = lane; v < H / V; v += 32) {
    float a[8], b[8];
    if constexpr (V == 8) {
      unpack16_bf16(xr[v], a);
      unpack16_bf16(gr[v], b);
    } else {
      unpack16(xr[v], a, nullptr);
      unpack16(gr[v], b, nullptr);
    }
#pragma unroll
    for (int q = 0; q < V; ++q) acc = fmaf(a[q], b[q], acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) gamma[t] = 1.0f / (1.0f + expf(-acc));
}

}  // namespace

cudaError_t launch_shared_gate(int dtype, const void* x, const void* g, int64_t T, int64_t H, float* gamma,
                               cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(T, 8));
  if (dtype == 0)
    shared_gate_kernel<float><<<grid, 256, 0, s>>>((const float*)x, (const float*)g, (int)T, (int)H, gamma);
  else
    shared_gate_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)g,
                                                           (int)T, (int)H, gamma);
  return cudaGetLastError();
}

RouterPlan router_plan(int dtype, int64_t T, int64_t H, int64_t E) {
  RouterPlan r;
  T = std::max<int64_t>(T, 1);
  r.ldo = round_up(E, 4);
  if (dtype == 1) {
    r.tensor_cores = true;
    r.splits = tc_router_splits(T, H, E);
    r.k_per_split = 0;
    return r;
  }
  r.tensor_cores = false;
  const int64_t blocks_mn = ceil_div(T, RBM) * ceil_div(E, RBN);
  int64_t splits = 1;
  const int64_t target = 2 * 148;
  if (blocks_mn < target) splits = ceil_div(target, blocks_mn);
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, ceil_div(H, 256)));
  const int64_t kps = round_up(ceil_div(H, splits), RBK);
  r.splits = (int)ceil_div(H, kps);
  r.k_per_split = (int)kps;
  return r;
}

size_t router_partial_bytes(int dtype, int64_t T, int64_t H, int64_t E) {
  const RouterPlan r = router_plan(dtype, T, H, E);
  return (size_t)r.splits * (size_t)T * (size_t)r.ldo * 4;
}

namespace {

template <typename TX, int NS>
void launch_topk_ns(dim3 grid, const float* partial, int splits, int64_t ldo, int vec4, int64_t T, int64_t E,
                    int64_t k, int score, int bias_mode, int renorm, const float* bias, float* weights,
                    int64_t* selected, const void* x, const void* shared_gate, int64_t H, float* gamma,
                    cudaStream_t s) {
  topk_kernel<TX, NS><<<grid, TOPK_WARPS * 32, 0, s>>>(partial, splits, ldo, vec4, (int)T, (int)E, (int)k, score,
                                                       bias_mode, renorm, bias, weights, selected,
                                                       (const TX*)x, (const TX*)shared_gate, (int)H, gamma);
}

template <typename TX>
void launch_topk_t(dim3 grid, const float* partial, int splits, int64_t ldo, int vec4, int64_t T, int64_t E,
                   int64_t k, int score, int bias_mode, int renorm, const float* bias, float* weights,
                   int64_t* selected, const void* x, const void* shared_gate, int64_t H, float* gamma,
                   cudaStream_t s) {
  if (E <= 32)
    launch_topk_ns<TX, 1>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights,
                          selected, x, shared_gate, H, gamma, s);
  else if (E <= 64)
    launch_topk_ns<TX, 2>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights,
                          selected, x, shared_gate, H, gamma, s);
  else if (E <= 128)
    launch_topk_ns<TX, 4>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights,
                          selected, x, shared_gate, H, gamma, s);
  else
    launch_topk_ns<TX, 8>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights,
                          selected, x, shared_gate, H, gamma, s);
}

}  // namespace

cudaError_t launch_topk(const float* partial, int splits, int64_t ldo, int64_t T, int64_t E, int64_t k, int score,
                        int bias_mode, int renorm, const float* bias, float* weights, int64_t* selected,
                        const void* x, const void* shared_gate, int64_t H, int dtype, float* gamma, cudaStream_t s) {
  const dim3 grid((unsigned)ceil_div(T, TOPK_WARPS));
  const int vec4 = (ldo % 4 == 0 && (reinterpret_cast<uintptr_t>(partial) & 15u) == 0) ? 1 : 0;
  if (dtype == 0)
    launch_topk_t<float>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights, selected,
                         x, shared_gate, H, gamma, s);
  else
    launch_topk_t<__nv_bfloat16>(grid, partial, splits, ldo, vec4, T, E, k, score, bias_mode, renorm, bias, weights,
                                 selected, x, shared_gate, H, gamma, s);
  return cudaGetLastError();
}

cudaError_t launch_route(int dtype, const void* x, const void* gate_w, const void* shared_gate, const float* bias,
                         int64_t T, int64_t H, int64_t E, int64_t k, int score, int bias_mode, int renorm,
                         float* partial, float* weights, int64_t* selected, float* gamma, int32_t* err,
                         cudaStream_t s) {
  const RouterPlan plan = router_plan(dtype, T, H, E);
  cudaError_t e;
  if (plan.tensor_cores) {
    e = launch_tc_logits(x, gate_w, T, H, E, partial, plan.ldo, plan.splits, err, s);
  } else {
    dim3 grid((unsigned)ceil_div(T, RBM), (unsigned)ceil_div(E, RBN), (unsigned)plan.splits);
    router_logits_kernel<float><<<grid, RTHREADS, 0, s>>>((const float*)x, (const float*)gate_w, partial, (int)T,
                                                          (int)H, (int)E, (int)plan.ldo, plan.k_per_split);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  return launch_topk(partial, plan.splits, plan.ldo, T, E, k, score, bias_mode, renorm, bias, weights, selected, x,
                     shared_gate, H, dtype, shared_gate ? gamma : nullptr, s);
}

}  // namespace stm
