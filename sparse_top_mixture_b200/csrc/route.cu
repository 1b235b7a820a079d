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
  for (int k0 = kb; k0 < ke; k0 += RBK) {
    for (int i = tid; i < NV; i += RTHREADS) {
      const int r = i / VPR, c = (i % VPR) * V;
      const int kk = k0 + c;
      float f[8];
      // A: token rows
      {
        const int row = m0 + r;
        if (row < Tn && kk < ke) {
          const uint4 v = *reinterpret_cast<const uint4*>(x + (int64_t)row * H + kk);
          if constexpr (V == 8) unpack16_bf16(v, f); else unpack16(v, f, nullptr);
        } else {
#pragma unroll
          for (int q = 0; q < V; ++q) f[q] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < V; ++q) As[c + q][r] = f[q];
      }
      // B: expert rows
      {
        const int col = n0 + r;
        if (col < E && kk < ke) {
          const T* src = gate_w + (int64_t)col * H;
          const uint4 v = *reinterpret_cast<const uint4*>(src + kk);
          if constexpr (V == 8) unpack16_bf16(v, f); else unpack16(v, f, nullptr);
        } else {
#pragma unroll
          for (int q = 0; q < V; ++q) f[q] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < V; ++q) Bs[c + q][r] = f[q];
      }
    }
    __syncthreads();
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

// (key, index) order of the top-k: larger key first, lower index on ties.
__device__ __forceinline__ bool ranks_before(float ka, int ea, float kb, int eb) {
  return ka > kb || (ka == kb && ea < eb);
}

constexpr int TOPK_WARPS = 8;

template <typename TX>
__global__ void __launch_bounds__(TOPK_WARPS * 32) topk_kernel(const float* __restrict__ partial, int splits,
                                                                int64_t ldo, int Tn, int E, int k, int score,
                                                                int bias_mode, int renorm,
                                                                const float* __restrict__ bias,
                                                                float* __restrict__ weights,
                                                                int64_t* __restrict__ selected,
                                                                const TX* __restrict__ x,
                                                                const TX* __restrict__ shared_gate, int H,
                                                                float* __restrict__ gamma) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * TOPK_WARPS + (threadIdx.x >> 5);
  if (t >= Tn) return;

  float logit[8], sc[8], key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    float l = -INFINITY;
    if (e < E) {
      l = 0.f;
      for (int s = 0; s < splits; ++s) l += partial[((int64_t)s * Tn + t) * ldo + e];
      if (bias_mode == 1) l += bias[e];
    }
    logit[i] = l;
  }
  if (score == 0) {  // softmax over all E experts
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, logit[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sc[i] = (lane + 32 * i < E) ? expf(logit[i] - m) : 0.f;
      z += sc[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i] = sc[i] / z;
  } else if (score == 1) {  // sigmoid
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i] = 1.0f / (1.0f + expf(-logit[i]));
  } else {  // sqrtsoftplus: sqrt(log(1 + e^l)), stable form
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float l = logit[i];
      sc[i] = sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
    }
  }
  // Selection key. Without a selection bias every score function is
  // increasing in the logit, so ranking by the logit ranks by the score and
  // avoids ties introduced by rounding the scores.
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    key[i] = (bias_mode == 2 && e < E) ? sc[i] + bias[e] : logit[i];
  }

  // Slot j's expert and raw weight go to shared memory; the renormalising
  // sum runs in slot order (identical in every lane).
  __shared__ float s_w[TOPK_WARPS][kMaxExperts];
  __shared__ int s_e[TOPK_WARPS][kMaxExperts];
  const int wid = threadIdx.x >> 5;
  uint32_t taken = 0;
  float tot = 0.f;
  for (int j = 0; j < k; ++j) {
    float bk = -INFINITY, bs = 0.f;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && ranks_before(key[i], e, bk, be)) {
        bk = key[i]; be = e; bs = sc[i];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      if (ranks_before(ok, oe, bk, be)) { bk = ok; be = oe; bs = os; }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == 0) {
      s_w[wid][j] = bs;
      s_e[wid][j] = be;
    }
    tot += bs;
  }
  __syncwarp();
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

cudaError_t launch_topk(const float* partial, int splits, int64_t ldo, int64_t T, int64_t E, int64_t k, int score,
                        int bias_mode, int renorm, const float* bias, float* weights, int64_t* selected,
                        const void* x, const void* shared_gate, int64_t H, int dtype, float* gamma, cudaStream_t s) {
  dim3 grid((unsigned)ceil_div(T, TOPK_WARPS));
  if (dtype == 0)
    topk_kernel<float><<<grid, TOPK_WARPS * 32, 0, s>>>(partial, splits, ldo, (int)T, (int)E, (int)k, score,
                                                        bias_mode, renorm, bias, weights, selected, (const float*)x,
                                                        (const float*)shared_gate, (int)H, gamma);
  else
    topk_kernel<__nv_bfloat16><<<grid, TOPK_WARPS * 32, 0, s>>>(
        partial, splits, ldo, (int)T, (int)E, (int)k, score, bias_mode, renorm, bias, weights, selected,
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)shared_gate, (int)H, gamma);
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
