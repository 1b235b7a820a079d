// Backward pass of the sparse top-k MoE FFN for fp32 problems (SIMT).
//
// Gradients of sum(dout * out) for the forward of moe_forward with the expert
// choice held fixed (top-k selection is piecewise constant in its keys, so no
// gradient flows through the choice, nor through an aux-loss-free selection
// bias: "Sparse MoE FFN for DFlash-family drafters", What's here, MoEGate,
// whose bias is moved by a sign controller and never by gradients; the same
// page's tests check grouped-GEMM gradients against a per-expert loop). The
// chain rule of the forward, written out:
//   expert e on token t: g = x Wg^T, u = x Wu^T, h = silu(g) u, y = h Wd^T,
//   out_t += w y;  dy = w dout;  dWd += dy^T h;  dh = dy Wd;
//   dg = dh u silu'(g), du = dh silu(g);  dWgu += [dg du]^T x;
//   dx += dg Wg + du Wu;  dw = dout . y;
//   renormalised weights w_j = s_j / sum s: ds_i = (dw_i - sum_j dw_j w_j) / sum s;
//   scores S = f(L): softmax dL = S (dS - sum dS S), sigmoid dL = dS S (1 - S),
//   sqrtsoftplus dL = dS sig(L) / (2 S);  dgate_w = dL^T x, dx += dL gate_w,
//   a logit bias gets sum_t dL;  shared expert: out += gamma Y_s(x), with
//   gamma = sig(x . g) when gated: dz = (dout . Y_s) gamma (1 - gamma).
// Every output element is computed by one thread looping over its reduction
// in a fixed order (no atomics): the result is deterministic. This is the
// reference-grade path for fp32 problems; bf16 problems are not supported.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int BT = 256;

__device__ __forceinline__ float sig_f(float a) { return 1.0f / (1.0f + expf(-a)); }
__device__ __forceinline__ float silu_grad_f(float g) {
  const float s = sig_f(g);
  return s * (1.0f + g * (1.0f - s));
}

// Router forward for one token per block: logits, scores, and the routing
// weights of its k selected experts (slot order), as in the forward.
__global__ void __launch_bounds__(BT) bw_router_fwd(const float* __restrict__ x, const float* __restrict__ gw,
                                                   const float* __restrict__ bias, int bias_mode, int score,
                                                   int renorm, const int64_t* __restrict__ sel, int H, int E, int k,
                                                   float* __restrict__ L, float* __restrict__ S,
                                                   float* __restrict__ w) {
  __shared__ float red[BT];
  __shared__ float s_sc[kMaxExperts];
  const int t = blockIdx.x, e = threadIdx.x;
  float l = -INFINITY;
  if (e < E) {
    float acc = 0.f;
    for (int h = 0; h < H; ++h) acc = fmaf(x[(int64_t)t * H + h], gw[(int64_t)e * H + h], acc);
    if (bias_mode == MOE_BIAS_LOGIT) acc += bias[e];
    l = acc;
    L[(int64_t)t * E + e] = l;
  }
  float sc = 0.f;
  if (score == MOE_SCORE_SOFTMAX) {
    red[e] = l;
    __syncthreads();
    for (int o = BT / 2; o > 0; o >>= 1) {
      if (e < o) red[e] = fmaxf(red[e], red[e + o]);
      __syncthreads();
    }
    const float m = red[0];
    __syncthreads();
    const float z = e < E ? expf(l - m) : 0.f;
    red[e] = z;
    __syncthreads();
    for (int o = BT / 2; o > 0; o >>= 1) {
      if (e < o) red[e] += red[e + o];
      __syncthreads();
    }
    sc = z / red[0];
  } else if (score == MOE_SCORE_SIGMOID) {
    sc = sig_f(l);
  } else {
    sc = sqrtf(fmaxf(l, 0.f) + log1pf(expf(-fabsf(l))));
  }
  if (e < E) {
    S[(int64_t)t * E + e] = sc;
    s_sc[e] = sc;
  }
  __syncthreads();
  if (e == 0) {
    float tot = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      tot += (ej >= 0 && ej < E) ? s_sc[ej] : 0.f;
    }
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      float v = (ej >= 0 && ej < E) ? s_sc[ej] : 0.f;
      if (renorm) v = tot > 0.f ? v / tot : 0.f;
      w[(int64_t)t * k + j] = v;
    }
  }
}

// gu[r][j] = x[token(r)] . Wgu[e(r)][j], r over rows of a segment-sorted or
// token-ordered row set (tok/ex give each row's token and expert).
__global__ void __launch_bounds__(BT) bw_gate_up(const float* __restrict__ x, const float* __restrict__ wgu,
                                               const int32_t* __restrict__ tok, const int32_t* __restrict__ ex,
                                               int64_t R, int H, int I2, float* __restrict__ gu) {
  const int64_t n = R * I2;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t r = i / I2;
    const int j = (int)(i - r * I2);
    const int e = ex ? ex[r] : 0;
    const int t = tok ? tok[r] : (int)r;
    if (e < 0) { gu[i] = 0.f; continue; }
    const float* xr = x + (int64_t)t * H;
    const float* wr = wgu + ((int64_t)e * I2 + j) * H;
    float acc = 0.f;
    for (int h = 0; h < H; ++h) acc = fmaf(xr[h], wr[h], acc);
    gu[i] = acc;
  }
}

// y[r][n] = (silu(g) u)[r] . Wd[e(r)][n]   (unscaled expert output)
__global__ void __launch_bounds__(BT) bw_down_fwd(const float* __restrict__ gu, const float* __restrict__ wd,
                                                const int32_t* __restrict__ ex, int64_t R, int H, int I,
                                                float* __restrict__ y) {
  const int64_t n = R * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t r = i / H;
    const int c = (int)(i - r * H);
    const int e = ex ? ex[r] : 0;
    if (e < 0) { y[i] = 0.f; continue; }
    const float* g = gu + r * 2 * I;
    const float* wr = wd + ((int64_t)e * H + c) * I;
    float acc = 0.f;
    for (int m = 0; m < I; ++m) acc = fmaf(silu_f32(g[m]) * g[I + m], wr[m], acc);
    y[i] = acc;
  }
}

// dgu[r] = [dh u silu'(g) | dh silu(g)] with dh = scale(r) * (dout[token(r)] . Wd[e(r)][:, m])
__global__ void __launch_bounds__(BT) bw_dgu(const float* __restrict__ dout, const float* __restrict__ gu,
                                           const float* __restrict__ wd, const int32_t* __restrict__ tok,
                                           const int32_t* __restrict__ ex, const float* __restrict__ scale,
                                           int64_t R, int H, int I, float* __restrict__ dgu) {
  const int64_t n = R * I;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t r = i / I;
    const int m = (int)(i - r * I);
    const int e = ex ? ex[r] : 0;
    float* d = dgu + r * 2 * I;
    if (e < 0) { d[m] = 0.f; d[I + m] = 0.f; continue; }
    const int t = tok ? tok[r] : (int)r;
    const float* dr = dout + (int64_t)t * H;
    const float* wcol = wd + (int64_t)e * H * I + m;
    float acc = 0.f;
    for (int c = 0; c < H; ++c) acc = fmaf(dr[c], wcol[(int64_t)c * I], acc);
    const float dh = scale[r] * acc;
    const float g = gu[r * 2 * I + m], u = gu[r * 2 * I + I + m];
    d[m] = dh * u * silu_grad_f(g);
    d[I + m] = dh * silu_f32(g);
  }
}

// Routed dx[t][h] = sum_j dgu[row(t,j)] . Wgu[e_j][:, h]  (written, not added)
__global__ void __launch_bounds__(BT) bw_dx_routed(const float* __restrict__ dgu, const float* __restrict__ wgu,
                                                 const int64_t* __restrict__ sel, const int32_t* __restrict__ pair_pos,
                                                 int T, int H, int E, int k, int I2, float* __restrict__ dx) {
  const int64_t n = (int64_t)T * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t t = i / H;
    const int h = (int)(i - t * H);
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t e = sel[t * k + j];
      const int p = pair_pos[t * k + j];
      if (e < 0 || e >= E || p < 0) continue;
      const float* d = dgu + (int64_t)p * I2;
      const float* wc = wgu + (int64_t)e * I2 * H + h;
      for (int m = 0; m < I2; ++m) acc = fmaf(d[m], wc[(int64_t)m * H], acc);
    }
    dx[i] = acc;
  }
}

// dWd[e][n][m] = sum over e's rows r of scale(r) dout[token(r)][n] h[r][m]
__global__ void __launch_bounds__(BT) bw_dwd(const float* __restrict__ dout, const float* __restrict__ gu,
                                           const int32_t* __restrict__ tok, const float* __restrict__ scale,
                                           const int32_t* __restrict__ offsets, int nseg, int64_t rows_single,
                                           int H, int I, float* __restrict__ dwd) {
  const int64_t n = (int64_t)nseg * H * I;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t e = i / ((int64_t)H * I);
    const int64_t rem = i - e * H * I;
    const int c = (int)(rem / I), m = (int)(rem - (int64_t)c * I);
    const int64_t r0 = offsets ? offsets[e] : 0, r1 = offsets ? offsets[e + 1] : rows_single;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; ++r) {
      const int t = tok ? tok[r] : (int)r;
      const float* g = gu + r * 2 * I;
      acc = fmaf(scale[r] * dout[(int64_t)t * H + c], silu_f32(g[m]) * g[I + m], acc);
    }
    dwd[i] = acc;
  }
}

// dWgu[e][m][h] = sum over e's rows r of dgu[r][m] x[token(r)][h]
__global__ void __launch_bounds__(BT) bw_dwgu(const float* __restrict__ dgu, const float* __restrict__ x,
                                            const int32_t* __restrict__ tok, const int32_t* __restrict__ offsets,
                                            int nseg, int64_t rows_single, int H, int I2,
                                            float* __restrict__ dwgu) {
  const int64_t n = (int64_t)nseg * I2 * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t e = i / ((int64_t)I2 * H);
    const int64_t rem = i - e * I2 * H;
    const int m = (int)(rem / H), h = (int)(rem - (int64_t)m * H);
    const int64_t r0 = offsets ? offsets[e] : 0, r1 = offsets ? offsets[e + 1] : rows_single;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; ++r) {
      const int t = tok ? tok[r] : (int)r;
      acc = fmaf(dgu[r * I2 + m], x[(int64_t)t * H + h], acc);
    }
    dwgu[i] = acc;
  }
}

// Per sorted row: token, expert and routing weight of its pair.
// Rows at or past offsets[E] (pairs skipped for a bad expert id) get expert -1.
__global__ void __launch_bounds__(BT) bw_rows(const int32_t* __restrict__ sorted_pairs,
                                            const int32_t* __restrict__ offsets, const int64_t* __restrict__ sel,
                                            const float* __restrict__ w, int64_t P, int E, int k,
                                            int32_t* __restrict__ tok, int32_t* __restrict__ ex,
                                            float* __restrict__ scale) {
  const int64_t used = offsets[E];
  for (int64_t p = blockIdx.x * (int64_t)BT + threadIdx.x; p < P; p += (int64_t)gridDim.x * BT) {
    if (p >= used) {
      tok[p] = 0;
      ex[p] = -1;
      scale[p] = 0.f;
      continue;
    }
    const int q = sorted_pairs[p];
    const int64_t e = sel[q];
    tok[p] = q / k;
    ex[p] = (e >= 0 && e < E) ? (int)e : -1;
    scale[p] = w[q];
  }
}

// dw[q] = dout[token(q)] . y[pair_pos[q]]
__global__ void __launch_bounds__(BT) bw_dw(const float* __restrict__ dout, const float* __restrict__ y,
                                          const int32_t* __restrict__ pair_pos, int64_t P, int H, int k,
                                          float* __restrict__ dw) {
  for (int64_t q = blockIdx.x * (int64_t)BT + threadIdx.x; q < P; q += (int64_t)gridDim.x * BT) {
    const int p = pair_pos[q];
    float acc = 0.f;
    if (p >= 0) {
      const float* d = dout + (q / k) * H;
      const float* yr = y + (int64_t)p * H;
      for (int c = 0; c < H; ++c) acc = fmaf(d[c], yr[c], acc);
    }
    dw[q] = acc;
  }
}

// Router backward, one token per block: dS from dw (renormalisation), dL from dS.
__global__ void __launch_bounds__(BT) bw_router_bwd(const float* __restrict__ L, const float* __restrict__ S,
                                                  const float* __restrict__ w, const float* __restrict__ dw,
                                                  const int64_t* __restrict__ sel, int score, int renorm, int E,
                                                  int k, float* __restrict__ dL) {
  __shared__ float dS[kMaxExperts];
  __shared__ float red[BT];
  const int t = blockIdx.x, e = threadIdx.x;
  if (e < E) dS[e] = 0.f;
  __syncthreads();
  if (e == 0) {
    float tot = 0.f, dww = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      if (ej >= 0 && ej < E) tot += S[(int64_t)t * E + ej];
      dww += dw[(int64_t)t * k + j] * w[(int64_t)t * k + j];
    }
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      if (ej < 0 || ej >= E) continue;
      const float d = dw[(int64_t)t * k + j];
      dS[ej] += renorm ? (tot > 0.f ? (d - dww) / tot : 0.f) : d;
    }
  }
  __syncthreads();
  const float s = e < E ? S[(int64_t)t * E + e] : 0.f;
  const float ds = e < E ? dS[e] : 0.f;
  float dl;
  if (score == MOE_SCORE_SOFTMAX) {
    red[e] = ds * s;
    __syncthreads();
    for (int o = BT / 2; o > 0; o >>= 1) {
      if (e < o) red[e] += red[e + o];
      __syncthreads();
    }
    dl = s * (ds - red[0]);
  } else if (score == MOE_SCORE_SIGMOID) {
    dl = ds * s * (1.f - s);
  } else {
    dl = (e < E && s > 0.f) ? ds * sig_f(L[(int64_t)t * E + e]) / (2.f * s) : 0.f;
  }
  if (e < E) dL[(int64_t)t * E + e] = dl;
}

// dgate_w[e][h] = sum_t dL[t][e] x[t][h]; d_bias[e] = sum_t dL[t][e]
__global__ void __launch_bounds__(BT) bw_dgate(const float* __restrict__ dL, const float* __restrict__ x, int T,
                                             int H, int E, float* __restrict__ dgw, float* __restrict__ dbias) {
  const int64_t n = (int64_t)E * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t e = i / H;
    const int h = (int)(i - e * H);
    float acc = 0.f, sb = 0.f;
    for (int t = 0; t < T; ++t) {
      const float d = dL[(int64_t)t * E + e];
      acc = fmaf(d, x[(int64_t)t * H + h], acc);
      sb += d;
    }
    dgw[i] = acc;
    if (dbias && h == 0) dbias[e] = sb;
  }
}

// dx[t][h] += sum_e dL[t][e] gate_w[e][h]  (+ dz[t] g[h] for a gated shared expert)
__global__ void __launch_bounds__(BT) bw_dx_router(const float* __restrict__ dL, const float* __restrict__ gw,
                                                 const float* __restrict__ dz, const float* __restrict__ g, int T,
                                                 int H, int E, float* __restrict__ dx) {
  const int64_t n = (int64_t)T * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t t = i / H;
    const int h = (int)(i - t * H);
    float acc = 0.f;
    for (int e = 0; e < E; ++e) acc = fmaf(dL[t * E + e], gw[(int64_t)e * H + h], acc);
    if (dz) acc = fmaf(dz[t], g[h], acc);
    dx[i] += acc;
  }
}

// Shared expert gate: gamma[t] (1 plain, sig(x.g) gated) and dz[t]
// = (dout[t] . Y_s[t]) gamma (1 - gamma) (gated only).
__global__ void __launch_bounds__(BT) bw_shared_gate(const float* __restrict__ x, const float* __restrict__ g,
                                                   const float* __restrict__ dout, const float* __restrict__ ys,
                                                   int T, int H, int gated, float* __restrict__ gamma,
                                                   float* __restrict__ dz) {
  for (int t = blockIdx.x * BT + threadIdx.x; t < T; t += gridDim.x * BT) {
    float gm = 1.f, d = 0.f;
    if (gated) {
      float z = 0.f, dy = 0.f;
      for (int h = 0; h < H; ++h) {
        z = fmaf(x[(int64_t)t * H + h], g[h], z);
        dy = fmaf(dout[(int64_t)t * H + h], ys[(int64_t)t * H + h], dy);
      }
      gm = sig_f(z);
      d = dy * gm * (1.f - gm);
    }
    gamma[t] = gm;
    dz[t] = d;
  }
}

// Shared expert dx: dx[t][h] += dgu_s[t] . Wsgu[:, h]
__global__ void __launch_bounds__(BT) bw_dx_shared(const float* __restrict__ dgus, const float* __restrict__ wsgu,
                                                 int T, int H, int I2, float* __restrict__ dx) {
  const int64_t n = (int64_t)T * H;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t t = i / H;
    const int h = (int)(i - t * H);
    const float* d = dgus + t * I2;
    float acc = 0.f;
    for (int m = 0; m < I2; ++m) acc = fmaf(d[m], wsgu[(int64_t)m * H + h], acc);
    dx[i] += acc;
  }
}

// d_shared_gate[h] = sum_t dz[t] x[t][h]
__global__ void __launch_bounds__(BT) bw_dgvec(const float* __restrict__ dz, const float* __restrict__ x, int T,
                                             int H, float* __restrict__ dg) {
  for (int h = blockIdx.x * BT + threadIdx.x; h < H; h += gridDim.x * BT) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc = fmaf(dz[t], x[(int64_t)t * H + h], acc);
    dg[h] = acc;
  }
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, BT), 148 * 32)); }

struct BwLayout {
  size_t header, local, counts, offsets, sorted_pairs, pair_pos, tok, ex, scale, w, dw, L, S, dL, gu, y, dgu, gus,
      ys, dgus, gamma, dz, total;
};

size_t a256(size_t v) { return (v + 255) & ~size_t(255); }

BwLayout bw_layout(const moe_problem& p) {
  BwLayout b;
  const int64_t P = p.T * p.k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = a256(off + bytes);
    return at;
  };
  b.header = take(sizeof(WsHeader));
  b.local = take((size_t)dispatch_num_blocks(p.T, p.k) * p.E * 4);
  b.counts = take((size_t)p.E * 4);
  b.offsets = take((size_t)(p.E + 1) * 4);
  b.sorted_pairs = take((size_t)P * 4);
  b.pair_pos = take((size_t)P * 4);
  b.tok = take((size_t)P * 4);
  b.ex = take((size_t)P * 4);
  b.scale = take((size_t)P * 4);
  b.w = take((size_t)P * 4);
  b.dw = take((size_t)P * 4);
  b.L = take((size_t)p.T * p.E * 4);
  b.S = take((size_t)p.T * p.E * 4);
  b.dL = take((size_t)p.T * p.E * 4);
  b.gu = take((size_t)P * 2 * p.I * 4);
  b.y = take((size_t)P * p.H * 4);
  b.dgu = take((size_t)P * 2 * p.I * 4);
  const bool sh = p.shared != MOE_SHARED_NONE;
  b.gus = take(sh ? (size_t)p.T * 2 * p.I_shared * 4 : 0);
  b.ys = take(sh ? (size_t)p.T * p.H * 4 : 0);
  b.dgus = take(sh ? (size_t)p.T * 2 * p.I_shared * 4 : 0);
  b.gamma = take(sh ? (size_t)p.T * 4 : 0);
  b.dz = take(sh ? (size_t)p.T * 4 : 0);
  b.total = off;
  return b;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

bool ok16(const void* q) { return q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }
// NULL or 4-byte aligned
bool ok4(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 3u) == 0; }

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_backward_workspace_size(const moe_problem* p, size_t* bytes) {
  size_t fwd = 0;
  const moe_status st = moe_workspace_size(p, &fwd);  // validates the problem
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = bw_layout(*p).total;
  return MOE_OK;
}

MOE_API moe_status moe_backward(const moe_problem* p, const moe_weights* w, const void* x_, const void* dout_,
                                const int64_t* selected, moe_grads* g, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  size_t need = 0;
  const moe_status st = moe_backward_workspace_size(p, &need);
  if (st != MOE_OK) return st;
  if (p->dtype != MOE_DTYPE_F32) return MOE_ERR_UNSUPPORTED;
  if (w == nullptr || g == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  const bool sh = p->shared != MOE_SHARED_NONE, gated = p->shared == MOE_SHARED_SIGMOID_GATED;
  const bool has_tokens = p->T > 0;  // per-token arrays and the workspace may be NULL without tokens
  if ((has_tokens && (!ok16(x_) || !ok16(dout_) || !ok16(selected) || !ok16(g->dx) || !ok16(ws))) || !ok16(w->gate_w) ||
      !ok16(w->gate_up) || !ok16(w->down) || !ok16(g->d_gate_w) || !ok16(g->d_gate_up) || !ok16(g->d_down))
    return MOE_ERR_INVALID_ARGUMENT;
  if ((p->bias_mode != MOE_BIAS_NONE) != (w->bias != nullptr) || !ok4(w->bias)) return MOE_ERR_INVALID_ARGUMENT;
  if ((p->bias_mode == MOE_BIAS_LOGIT) != (g->d_bias != nullptr) || !ok4(g->d_bias))
    return MOE_ERR_INVALID_ARGUMENT;
  if (sh && (!ok16(w->shared_gate_up) || !ok16(w->shared_down) || !ok16(g->d_shared_gate_up) ||
             !ok16(g->d_shared_down)))
    return MOE_ERR_INVALID_ARGUMENT;
  if (gated != (w->shared_gate != nullptr) || gated != (g->d_shared_gate != nullptr) || !ok4(w->shared_gate) ||
      !ok4(g->d_shared_gate))
    return MOE_ERR_INVALID_ARGUMENT;
  if (has_tokens && ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->T == 0) {  // no tokens: every weight gradient is zero
    const size_t f = sizeof(float);
    cudaError_t e = cudaMemsetAsync(g->d_gate_w, 0, (size_t)(p->E * p->H) * f, s);
    if (e == cudaSuccess && g->d_bias) e = cudaMemsetAsync(g->d_bias, 0, (size_t)p->E * f, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->d_gate_up, 0, (size_t)(p->E * 2 * p->I * p->H) * f, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->d_down, 0, (size_t)(p->E * p->H * p->I) * f, s);
    if (e == cudaSuccess && sh) e = cudaMemsetAsync(g->d_shared_gate_up, 0, (size_t)(2 * p->I_shared * p->H) * f, s);
    if (e == cudaSuccess && sh) e = cudaMemsetAsync(g->d_shared_down, 0, (size_t)(p->H * p->I_shared) * f, s);
    if (e == cudaSuccess && gated) e = cudaMemsetAsync(g->d_shared_gate, 0, (size_t)p->H * f, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const BwLayout b = bw_layout(*p);
  const int T = (int)p->T, H = (int)p->H, E = (int)p->E, k = (int)p->k, I = (int)p->I, Is = (int)p->I_shared;
  const int64_t P = p->T * p->k;
  const float* x = static_cast<const float*>(x_);
  const float* dout = static_cast<const float*>(dout_);
  const float* gw = static_cast<const float*>(w->gate_w);
  const float* wgu = static_cast<const float*>(w->gate_up);
  const float* wd = static_cast<const float*>(w->down);
  int32_t* err = at<int32_t>(ws, b.header);
  int32_t* offsets = at<int32_t>(ws, b.offsets);
  int32_t* sorted_pairs = at<int32_t>(ws, b.sorted_pairs);
  int32_t* pair_pos = at<int32_t>(ws, b.pair_pos);
  int32_t* tok = at<int32_t>(ws, b.tok);
  int32_t* ex = at<int32_t>(ws, b.ex);
  float* scale = at<float>(ws, b.scale);
  float* wts = at<float>(ws, b.w);
  float* dw = at<float>(ws, b.dw);
  float* L = at<float>(ws, b.L);
  float* S = at<float>(ws, b.S);
  float* dL = at<float>(ws, b.dL);
  float* gu = at<float>(ws, b.gu);
  float* y = at<float>(ws, b.y);
  float* dgu = at<float>(ws, b.dgu);
  auto chk = [](cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; };

  // routing weights of the given choice, and its sorted segments
  bw_router_fwd<<<T, BT, 0, s>>>(x, gw, w->bias, p->bias_mode, p->score, p->renormalize ? 1 : 0, selected, H, E, k,
                                 L, S, wts);
  if (launch_dispatch(MOE_DTYPE_F32, selected, nullptr, p->T, p->H, p->E, p->k, at<int32_t>(ws, b.local),
                      at<int32_t>(ws, b.counts), offsets, sorted_pairs, pair_pos, nullptr, err, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  bw_rows<<<grid_for(P), BT, 0, s>>>(sorted_pairs, offsets, selected, wts, P, E, k, tok, ex, scale);
  // routed experts, rows in segment order
  bw_gate_up<<<grid_for(P * 2 * I), BT, 0, s>>>(x, wgu, tok, ex, P, H, 2 * I, gu);
  bw_down_fwd<<<grid_for(P * H), BT, 0, s>>>(gu, wd, ex, P, H, I, y);
  bw_dw<<<grid_for(P), BT, 0, s>>>(dout, y, pair_pos, P, H, k, dw);
  bw_dgu<<<grid_for(P * I), BT, 0, s>>>(dout, gu, wd, tok, ex, scale, P, H, I, dgu);
  bw_dx_routed<<<grid_for((int64_t)T * H), BT, 0, s>>>(dgu, wgu, selected, pair_pos, T, H, E, k, 2 * I, g->dx);
  bw_dwd<<<grid_for((int64_t)E * H * I), BT, 0, s>>>(dout, gu, tok, scale, offsets, E, 0, H, I, g->d_down);
  bw_dwgu<<<grid_for((int64_t)E * 2 * I * H), BT, 0, s>>>(dgu, x, tok, offsets, E, 0, H, 2 * I, g->d_gate_up);
  // router
  bw_router_bwd<<<T, BT, 0, s>>>(L, S, wts, dw, selected, p->score, p->renormalize ? 1 : 0, E, k, dL);
  bw_dgate<<<grid_for((int64_t)E * H), BT, 0, s>>>(dL, x, T, H, E, g->d_gate_w, g->d_bias);
  float* dz = nullptr;
  if (sh) {
    const float* wsgu = static_cast<const float*>(w->shared_gate_up);
    const float* wsd = static_cast<const float*>(w->shared_down);
    float* gus = at<float>(ws, b.gus);
    float* ys = at<float>(ws, b.ys);
    float* dgus = at<float>(ws, b.dgus);
    float* gamma = at<float>(ws, b.gamma);
    dz = at<float>(ws, b.dz);
    bw_gate_up<<<grid_for((int64_t)T * 2 * Is), BT, 0, s>>>(x, wsgu, nullptr, nullptr, T, H, 2 * Is, gus);
    bw_down_fwd<<<grid_for((int64_t)T * H), BT, 0, s>>>(gus, wsd, nullptr, T, H, Is, ys);
    bw_shared_gate<<<grid_for(T), BT, 0, s>>>(x, static_cast<const float*>(w->shared_gate), dout, ys, T, H,
                                              gated ? 1 : 0, gamma, dz);
    bw_dgu<<<grid_for((int64_t)T * Is), BT, 0, s>>>(dout, gus, wsd, nullptr, nullptr, gamma, T, H, Is, dgus);
    bw_dx_shared<<<grid_for((int64_t)T * H), BT, 0, s>>>(dgus, wsgu, T, H, 2 * Is, g->dx);
    bw_dwd<<<grid_for((int64_t)H * Is), BT, 0, s>>>(dout, gus, nullptr, gamma, nullptr, 1, T, H, Is,
                                                   g->d_shared_down);
    bw_dwgu<<<grid_for((int64_t)2 * Is * H), BT, 0, s>>>(dgus, x, nullptr, nullptr, 1, T, H, 2 * Is,
                                                        g->d_shared_gate_up);
    if (gated) bw_dgvec<<<grid_for(H), BT, 0, s>>>(dz, x, T, H, g->d_shared_gate);
  }
  bw_dx_router<<<grid_for((int64_t)T * H), BT, 0, s>>>(dL, gw, gated ? dz : nullptr,
                                                      gated ? static_cast<const float*>(w->shared_gate) : nullptr,
                                                      T, H, E, g->dx);
  return chk(cudaGetLastError());
}
