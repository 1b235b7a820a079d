// Backward pass of the sparse top-k MoE FFN for fp32 problems (SIMT tiles).
//
// Gradients of sum(dout * out) for the forward of moe_forward with the expert
// choice held fixed (top-k selection is piecewise constant in its keys, so no
// gradient flows through the choice, nor through an aux-loss-free selection
// bias: "Sparse MoE FFN for DFlash-family drafters", What's here, MoEGate,
// whose bias is moved by a sign controller and never by gradients; the same
// page's tests check grouped-GEMM gradients against a per-expert loop). The
// chain rule of the forward, written out for expert e on token t:
//   g = x Wg^T, u = x Wu^T, h = silu(g) u, y = h Wd^T, out_t += w y;
//   dhu = dout Wd (unscaled);  dh = w dhu;  dWd += (w dout)^T h;
//   dg = dh u silu'(g), du = dh silu(g);  dWgu += [dg du]^T x;
//   dx += dg Wg + du Wu;  dw = dout . y = h . dhu;
//   renormalised weights w_j = s_j / sum s: ds_i = (dw_i - sum_j dw_j w_j) / sum s;
//   scores S = f(L): softmax dL = S (dS - sum dS S), sigmoid dL = dS S (1 - S),
//   sqrtsoftplus dL = dS sig(L) / (2 S);  dgate_w = dL^T x, dx += dL gate_w,
//   a logit bias gets sum_t dL;  shared expert: out += gamma Y_s(x), with
//   gamma = sig(x . g) when gated: dz = (h_s . dhu_s) gamma (1 - gamma).
//
// Layout of the work: the routed rows are sorted into per-expert segments by
// the forward's dispatch kernels. Data gradients are grouped GEMMs over those
// rows (one 128-row tile never crosses a segment, as in the forward); weight
// gradients are per-expert GEMMs whose reduction walks the expert's segment
// rows; dx is put back in token order by the forward's combine kernel. The
// router and shared expert use the same two GEMM kernels over one all-token
// segment. Every GEMM is 128x128 output tiles, 8-deep k slices
// double-buffered in shared memory, 8x8 fp32 outputs per thread; every output
// element is one thread's fixed-order sum (dgate_w: row-chunk partials added
// in chunk order), with no atomics, so results are deterministic. bf16
// problems take the tensor-core variant at the end of this file.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "tiles.cuh"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace stm {
namespace {

constexpr int BT = 256;                    // threads of every backward kernel
constexpr int TM = 128, TN = 128, TK = 8;  // GEMM tile
constexpr int TP = TM + 4;                 // padded shared row (keeps float4 alignment)

__device__ __forceinline__ float sig_f(float a) { return 1.0f / (1.0f + expf(-a)); }
__device__ __forceinline__ float silu_grad_f(float g) {
  const float s = sig_f(g);
  return s * (1.0f + g * (1.0f - s));
}

// 8 x 8 outputs per thread from one TK-deep slice of the A [TK][TM] and
// B [TK][TN] shared tiles. Thread (tx, ty) owns rows ty*4+{0..3}, 64+ty*4+{0..3}
// and columns tx*4+{0..3}, 64+tx*4+{0..3}.
__device__ __forceinline__ void mma_slice(const float (*As)[TP], const float (*Bs)[TP], int tx, int ty,
                                          float (&acc)[8][8]) {
#pragma unroll
  for (int kk = 0; kk < TK; ++kk) {
    const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
    const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
    const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
    const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
    const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

__device__ __forceinline__ int out_idx(int t, int i) { return i < 4 ? t * 4 + i : 64 + t * 4 + (i - 4); }

// ---- grouped row GEMM ---------------------------------------------------------
// C[r, n] = sum_k A[amap(r), k] * B_e[n, k]   (B_NT: B_e is [N, K])
//        or sum_k A[amap(r), k] * B_e[k, n]   (otherwise: B_e is [K, N])
// over rows r of each segment e (or one segment of single_rows rows).
enum { EPI_STORE = 0, EPI_ADD = 1, EPI_DGU = 2 };

struct RowGemm {
  const float* A;
  const int32_t* amap;  // row r reads A row amap[r] (NULL: row r)
  int64_t lda;
  const float* B;
  int64_t b_stride;  // elements between experts' B
  int N, K;
  const int32_t* offsets;  // [E+1] segment table, or NULL for one segment
  int E, single_rows;
  int64_t rows_total;
  float* C;  // EPI_STORE / EPI_ADD: C[r * ldc + n]
  int64_t ldc;
  const float* dz;    // EPI_ADD: optional C += dz[r] * gvec[n]
  const float* gvec;
  const float* GU;     // EPI_DGU (N == I): [g | u] rows [*, 2I]
  const float* scale;  // EPI_DGU: dh = scale[r] * acc
  float* DGU;          // EPI_DGU: [dg | du] rows [*, 2I]
  float* DHU;          // EPI_DGU: acc rows [*, I]
  float* Hact;         // EPI_DGU: h = silu(g) u rows [*, I]
  int32_t* err;
};

template <bool B_NT, int EPI>
__global__ void __launch_bounds__(BT, 2) bw_row_gemm(RowGemm a) {
  __shared__ int off[kMaxExperts + 1], pre[kMaxExperts + 1];
  __shared__ __align__(16) float As[2][TK][TP];
  __shared__ __align__(16) float Bs[2][TK][TP];
  const int tid = threadIdx.x;
  if (tid < 32) warp_build_tile_table(a.offsets, a.E, a.single_rows, TM, off, pre, a.rows_total, a.err);
  __syncthreads();
  const int nseg = a.offsets ? a.E : 1;
  const int mt = blockIdx.x;
  if (mt >= pre[nseg]) return;
  const int e = find_segment(pre, nseg, mt);
  const int row0 = off[e] + (mt - pre[e]) * TM, row_end = off[e + 1];
  const int n0 = blockIdx.y * TN;
  const int N = a.N, K = a.K;
  const float* Be = a.B + (int64_t)e * a.b_stride;

  // A loads: 8 consecutive k of rows (tid >> 3) + 32p.
  const int ac = tid & 7;
  const float* arow[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int r = row0 + (tid >> 3) + 32 * p;
    arow[p] = r < row_end ? a.A + (int64_t)(a.amap ? a.amap[r] : r) * a.lda : nullptr;
  }
  float ra[4], rb[4];
  auto load = [&](int k0) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int kk = k0 + ac;
      ra[p] = (arow[p] != nullptr && kk < K) ? arow[p][kk] : 0.f;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (B_NT) {
        const int n = n0 + (tid >> 3) + 32 * p, kk = k0 + ac;
        rb[p] = (n < N && kk < K) ? Be[(int64_t)n * K + kk] : 0.f;
      } else {
        const int n = n0 + (tid & 127), kk = k0 + (tid >> 7) + 2 * p;
        rb[p] = (n < N && kk < K) ? Be[(int64_t)kk * N + n] : 0.f;
      }
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      As[buf][ac][(tid >> 3) + 32 * p] = ra[p];
      if (B_NT) Bs[buf][ac][(tid >> 3) + 32 * p] = rb[p];
      else Bs[buf][(tid >> 7) + 2 * p][tid & 127] = rb[p];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int tx = tid & 15, ty = tid >> 4;
  load(0);
  store(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < K; k0 += TK) {
    const bool more = k0 + TK < K;
    if (more) load(k0 + TK);
    mma_slice(As[buf], Bs[buf], tx, ty, acc);
    if (more) store(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = row0 + out_idx(ty, i);
    if (r >= row_end) continue;
    const float sc = EPI == EPI_DGU ? a.scale[r] : 1.f;
    const float dzr = (EPI == EPI_ADD && a.dz != nullptr) ? a.dz[r] : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + out_idx(tx, j);
      if (n >= N) continue;
      const float v = acc[i][j];
      if (EPI == EPI_STORE) {
        a.C[r * a.ldc + n] = v;
      } else if (EPI == EPI_ADD) {
        float add = v;
        if (a.dz != nullptr) add = fmaf(dzr, a.gvec[n], add);
        a.C[r * a.ldc + n] += add;
      } else {
        const float* gu = a.GU + (int64_t)r * 2 * N;
        const float g = gu[n], u = gu[N + n];
        const float dh = sc * v;
        a.DGU[(int64_t)r * 2 * N + n] = dh * u * silu_grad_f(g);
        a.DGU[(int64_t)r * 2 * N + N + n] = dh * silu_f32(g);
        a.DHU[(int64_t)r * N + n] = v;
        a.Hact[(int64_t)r * N + n] = silu_f32(g) * u;
      }
    }
  }
}

// ---- per-segment weight-gradient GEMM -------------------------------------------
// C_e[i, j] = sum over rows r of segment e of Aop(r, i) * Bop(r, j), with
//   Aop(r, i) = A[amap(r) * lda + i] * (ascale ? ascale[r] : 1)
//   Bop(r, j) = B[bmap(r) * ldb + j]
// C_e is [M, N] at C + e * M * N. Segments without rows write zeros. Without
// a segment table, segment e is rows [e * chunk, min((e + 1) * chunk,
// single_rows)): a split of one long reduction into partial sums that
// bw_sum_parts adds up in order.
struct WGemm {
  const float* A;
  const int32_t* amap;
  const float* ascale;
  int64_t lda;
  int M;
  const float* B;
  const int32_t* bmap;
  int64_t ldb;
  int N;
  const int32_t* offsets;  // [E+1], or NULL: chunks of single_rows rows
  int single_rows, chunk;
  int64_t rows_total;
  float* C;
  int32_t* err;
};

__global__ void __launch_bounds__(BT, 2) bw_wgrad_gemm(WGemm a) {
  __shared__ __align__(16) float As[2][TK][TP];
  __shared__ __align__(16) float Bs[2][TK][TP];
  const int tid = threadIdx.x;
  const int e = blockIdx.y;
  int r0 = a.offsets ? a.offsets[e] : e * a.chunk;
  int r1 = a.offsets ? a.offsets[e + 1] : min(a.single_rows, r0 + a.chunk);
  if (r0 < 0 || r1 < r0 || (int64_t)r1 > a.rows_total) {  // malformed table: no rows are read
    if (tid == 0) raise_error(a.err, MOE_DEVERR_BAD_EXPERT_ID);
    r0 = r1 = 0;
  }
  const int M = a.M, N = a.N;
  const int mtiles = (M + TM - 1) / TM;
  const int m0 = (blockIdx.x % mtiles) * TM, n0 = (blockIdx.x / mtiles) * TN;
  const int li = tid & 127, lc = tid >> 7;  // loads: column li of slice rows lc + 2p

  float ra[4], rb[4];
  auto load = [&](int k0) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int r = r0 + k0 + lc + 2 * p;
      const bool rv = r < r1;
      const int i = m0 + li, j = n0 + li;
      float av = 0.f, bv = 0.f;
      if (rv && i < M) {
        av = a.A[(int64_t)(a.amap ? a.amap[r] : r) * a.lda + i];
        if (a.ascale) av *= a.ascale[r];
      }
      if (rv && j < N) bv = a.B[(int64_t)(a.bmap ? a.bmap[r] : r) * a.ldb + j];
      ra[p] = av;
      rb[p] = bv;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      As[buf][lc + 2 * p][li] = ra[p];
      Bs[buf][lc + 2 * p][li] = rb[p];
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int tx = tid & 15, ty = tid >> 4;
  const int K = r1 - r0;
  if (K > 0) {
    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < K; k0 += TK) {
      const bool more = k0 + TK < K;
      if (more) load(k0 + TK);
      mma_slice(As[buf], Bs[buf], tx, ty, acc);
      if (more) store(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
  float* Ce = a.C + (int64_t)e * M * N;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + out_idx(ty, i);
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + out_idx(tx, j);
      if (n < N) Ce[(int64_t)m * N + n] = acc[i][j];
    }
  }
}

// ---- router and small per-row kernels ---------------------------------------------

// Warps per block and experts per lane of the per-token router kernels
// (one warp per token; lane l owns experts l, l + 32, ...).
constexpr int kTokWarps = BT / 32;
constexpr int kExpPerLane = kMaxExperts / 32;

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One token per warp: logits L (+ logit bias, in place), scores S and the
// routing weights w of its k chosen experts (slot order), as in the forward.
__global__ void __launch_bounds__(BT) bw_scores(float* __restrict__ L, const float* __restrict__ bias, int bias_mode,
                                              int score, int renorm, const int64_t* __restrict__ sel, int T, int E,
                                              int k, float* __restrict__ S, float* __restrict__ w) {
  __shared__ float s_sc[kTokWarps][kMaxExperts];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTokWarps + wid;
  if (t >= T) return;  // the whole warp; no block-wide barrier follows
  float l[kExpPerLane], sc[kExpPerLane];
#pragma unroll
  for (int i = 0; i < kExpPerLane; ++i) {
    const int e = i * 32 + lane;
    l[i] = -INFINITY;
    if (e < E) {
      float v = L[(int64_t)t * E + e];
      if (bias_mode == MOE_BIAS_LOGIT) {
        v += bias[e];
        L[(int64_t)t * E + e] = v;
      }
      l[i] = v;
    }
  }
  if (score == MOE_SCORE_SOFTMAX) {
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) m = fmaxf(m, l[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) {
      sc[i] = i * 32 + lane < E ? expf(l[i] - m) : 0.f;
      z += sc[i];
    }
    z = warp_sum_f(z);
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) sc[i] = sc[i] / z;
  } else if (score == MOE_SCORE_SIGMOID) {
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) sc[i] = sig_f(l[i]);
  } else {
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) sc[i] = sqrtf(fmaxf(l[i], 0.f) + log1pf(expf(-fabsf(l[i]))));
  }
#pragma unroll
  for (int i = 0; i < kExpPerLane; ++i) {
    const int e = i * 32 + lane;
    if (e < E) {
      S[(int64_t)t * E + e] = sc[i];
      s_sc[wid][e] = sc[i];
    }
  }
  __syncwarp();
  if (lane == 0) {
    float tot = 0.f;
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      tot += (ej >= 0 && ej < E) ? s_sc[wid][ej] : 0.f;
    }
    for (int j = 0; j < k; ++j) {
      const int64_t ej = sel[(int64_t)t * k + j];
      float v = (ej >= 0 && ej < E) ? s_sc[wid][ej] : 0.f;
      if (renorm) v = tot > 0.f ? v / tot : 0.f;
      w[(int64_t)t * k + j] = v;
    }
  }
}

// Per sorted row p < offsets[E]: its token and routing weight.
__global__ void __launch_bounds__(BT) bw_rows(const int32_t* __restrict__ sorted_pairs,
                                            const int32_t* __restrict__ offsets, const float* __restrict__ w,
                                            int E, int k, int32_t* __restrict__ tok, float* __restrict__ scale) {
  const int64_t used = offsets[E];
  for (int64_t p = blockIdx.x * (int64_t)BT + threadIdx.x; p < used; p += (int64_t)gridDim.x * BT) {
    const int q = sorted_pairs[p];
    tok[p] = q / k;
    scale[p] = w[q];
  }
}

// One warp per output q: out[q] = sum_m h dhu over row p = map(q) (0 when
// p < 0), times gamma (1 - gamma) when gamma is given.
__global__ void __launch_bounds__(BT) bw_rowdot(const float* __restrict__ Hact, const float* __restrict__ DHU, int I,
                                              const int32_t* __restrict__ map, int64_t R,
                                              const float* __restrict__ gamma, float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  for (int64_t q = (blockIdx.x * (int64_t)BT + threadIdx.x) >> 5; q < R; q += ((int64_t)gridDim.x * BT) >> 5) {
    const int64_t p = map ? map[q] : q;
    float acc = 0.f;
    if (p >= 0) {
      const float* h = Hact + p * I;
      const float* d = DHU + p * I;
      for (int m = lane; m < I; m += 32) acc = fmaf(h[m], d[m], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      if (gamma) acc *= gamma[q] * (1.f - gamma[q]);
      out[q] = acc;
    }
  }
}

// Router backward, one token per warp: dS from dw (renormalisation), dL from
// dS; also dL rounded to bf16 into dL16 (row pitch ld16) when given.
__global__ void __launch_bounds__(BT) bw_router_bwd(const float* __restrict__ L, const float* __restrict__ S,
                                                  const float* __restrict__ w, const float* __restrict__ dw,
                                                  const int64_t* __restrict__ sel, int score, int renorm, int T,
                                                  int E, int k, float* __restrict__ dL,
                                                  __nv_bfloat16* __restrict__ dL16, int ld16) {
  __shared__ float s_dS[kTokWarps][kMaxExperts];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTokWarps + wid;
  if (t >= T) return;  // the whole warp; no block-wide barrier follows
  float* dS = s_dS[wid];
  for (int e = lane; e < E; e += 32) dS[e] = 0.f;
  __syncwarp();
  if (lane == 0) {
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
  __syncwarp();
  float sv[kExpPerLane], ds[kExpPerLane];
#pragma unroll
  for (int i = 0; i < kExpPerLane; ++i) {
    const int e = i * 32 + lane;
    sv[i] = e < E ? S[(int64_t)t * E + e] : 0.f;
    ds[i] = e < E ? dS[e] : 0.f;
  }
  float red = 0.f;
  if (score == MOE_SCORE_SOFTMAX) {
#pragma unroll
    for (int i = 0; i < kExpPerLane; ++i) red += ds[i] * sv[i];
    red = warp_sum_f(red);
  }
#pragma unroll
  for (int i = 0; i < kExpPerLane; ++i) {
    const int e = i * 32 + lane;
    if (e >= E) continue;
    float dl;
    if (score == MOE_SCORE_SOFTMAX) dl = sv[i] * (ds[i] - red);
    else if (score == MOE_SCORE_SIGMOID) dl = ds[i] * sv[i] * (1.f - sv[i]);
    else dl = sv[i] > 0.f ? ds[i] * sig_f(L[(int64_t)t * E + e]) / (2.f * sv[i]) : 0.f;
    dL[(int64_t)t * E + e] = dl;
    if (dL16) dL16[(int64_t)t * ld16 + e] = __float2bfloat16_rn(dl);
  }
}

// out[i] = sum_{s < S} part[s * n + i], in order of s
__global__ void __launch_bounds__(BT) bw_sum_parts(const float* __restrict__ part, int S, int64_t n,
                                                 float* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    float acc = 0.f;
#pragma unroll 4
    for (int q = 0; q < S; ++q) acc += part[q * n + i];  // in part order; unrolled so loads overlap
    out[i] = acc;
  }
}

// out[c] = sum_t v[t * ldv + c] for c < C (fixed order over t)
__global__ void __launch_bounds__(BT) bw_colsum(const float* __restrict__ v, int64_t ldv, int T, int C,
                                              float* __restrict__ out) {
  for (int c = blockIdx.x * BT + threadIdx.x; c < C; c += gridDim.x * BT) {
    float acc = 0.f;
    for (int t = 0; t < T; ++t) acc += v[(int64_t)t * ldv + c];
    out[c] = acc;
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

// gamma[t] = sig(x[t] . g) when g is given, else 1. One warp per token.
__global__ void __launch_bounds__(BT) bw_gamma(const float* __restrict__ x, const float* __restrict__ g, int T, int H,
                                             float* __restrict__ gamma) {
  const int lane = threadIdx.x & 31;
  for (int64_t t = (blockIdx.x * (int64_t)BT + threadIdx.x) >> 5; t < T; t += ((int64_t)gridDim.x * BT) >> 5) {
    if (g == nullptr) {
      if (lane == 0) gamma[t] = 1.f;
      continue;
    }
    float acc = 0.f;
    for (int h = lane; h < H; h += 32) acc = fmaf(x[t * H + h], g[h], acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) gamma[t] = sig_f(acc);
  }
}

unsigned grid_for(int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, BT), 148 * 32)); }

template <bool B_NT, int EPI>
cudaError_t run_rows(const RowGemm& a, cudaStream_t s) {
  const int64_t nseg = a.offsets ? a.E : 1;
  const dim3 grid((unsigned)(a.rows_total / TM + nseg), (unsigned)ceil_div(a.N, TN));
  bw_row_gemm<B_NT, EPI><<<grid, BT, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t run_wgrad(const WGemm& a, int nseg, cudaStream_t s) {
  const dim3 grid((unsigned)(ceil_div(a.M, TM) * ceil_div(a.N, TN)), (unsigned)nseg);
  bw_wgrad_gemm<<<grid, BT, 0, s>>>(a);
  return cudaGetLastError();
}

// Row chunks of the router's dgate_w = dL^T x: its [E, H] output has few
// tiles, so its T-long reduction is split until about two blocks per SM are
// busy (at least 64 rows a chunk, at most 32 chunks).
int router_chunks(const moe_problem& p) {
  const int64_t tiles = ceil_div(p.E, TM) * ceil_div(p.H, TN);
  int64_t S = std::min<int64_t>({ceil_div(2 * 148, tiles), ceil_div(p.T, 64), 32});
  S = std::max<int64_t>(S, 1);
  const int64_t chunk = ceil_div(p.T, S);
  return (int)ceil_div(p.T, std::max<int64_t>(chunk, 1));
}

struct BwLayout {
  size_t header, local, counts, offsets, sorted_pairs, pair_pos, tok, scale, w, dw, L, S, dL, parts, gu, dgu, dhu,
      hact, dxr, extra, gus, dgus, dhus, hacts, gamma, dz, total;
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
  b.scale = take((size_t)P * 4);
  b.w = take((size_t)P * 4);
  b.dw = take((size_t)P * 4);
  b.L = take((size_t)p.T * p.E * 4);
  b.S = take((size_t)p.T * p.E * 4);
  b.dL = take((size_t)p.T * p.E * 4);
  const int S = router_chunks(p);
  b.parts = take(S > 1 ? (size_t)S * p.E * p.H * 4 : 0);
  b.gu = take((size_t)P * 2 * p.I * 4);
  b.dgu = take((size_t)P * 2 * p.I * 4);
  b.dhu = take((size_t)P * p.I * 4);
  b.hact = take((size_t)P * p.I * 4);
  b.dxr = take((size_t)P * p.H * 4);
  b.extra = take((size_t)p.T * p.H * 4);
  const bool sh = p.shared != MOE_SHARED_NONE;
  const size_t Is = sh ? (size_t)p.I_shared : 0;
  b.gus = take((size_t)p.T * 2 * Is * 4);
  b.dgus = take((size_t)p.T * 2 * Is * 4);
  b.dhus = take((size_t)p.T * Is * 4);
  b.hacts = take((size_t)p.T * Is * 4);
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

RowGemm row_gemm(const float* A, const int32_t* amap, int64_t lda, const float* B, int64_t b_stride, int N, int K,
                 const int32_t* offsets, int E, int single_rows, int64_t rows_total, int32_t* err) {
  RowGemm a{};
  a.A = A;
  a.amap = amap;
  a.lda = lda;
  a.B = B;
  a.b_stride = b_stride;
  a.N = N;
  a.K = K;
  a.offsets = offsets;
  a.E = E;
  a.single_rows = single_rows;
  a.rows_total = rows_total;
  a.err = err;
  return a;
}

WGemm wgrad(const float* A, const int32_t* amap, const float* ascale, int64_t lda, int M, const float* B,
            const int32_t* bmap, int64_t ldb, int N, const int32_t* offsets, int single_rows, int64_t rows_total,
            float* C, int32_t* err, int chunk = 0) {
  WGemm a{};
  a.A = A;
  a.amap = amap;
  a.ascale = ascale;
  a.lda = lda;
  a.M = M;
  a.B = B;
  a.bmap = bmap;
  a.ldb = ldb;
  a.N = N;
  a.offsets = offsets;
  a.single_rows = single_rows;
  a.chunk = chunk > 0 ? chunk : single_rows;
  a.rows_total = rows_total;
  a.C = C;
  a.err = err;
  return a;
}


// ---- bf16 problems: tensor-core backward ------------------------------------------
// The same chain rule on the 5th-generation tensor cores. bf16 inputs (x,
// dout, weights) stay bf16 as GEMM operands, products accumulate in fp32:
//   [g | u] = x_perm Wgu^T and dhu = dout_perm Wd (fp32), then per row h =
//   silu(g) u and dw = h . dhu (fp32) and [dg | du] rounded to bf16 (the next
//   GEMM's operand), dx rows = [dg du] Wgu (fp32) -- on the forward's grouped
//   kernels over the dispatch's segments, with Wd [E][H][I] and Wgu
//   [E][2I][H] read as stored (MN-major B operands: no transposed copies);
//   weight gradients on the weight-gradient mode of the one-CTA kernel, whose
//   K loop walks an expert's rows and reads both operands MN-major from row
//   buffers: dWd = (w dout)^T h and dWgu = [dg du]^T x, from copies in which
//   every expert's rows start at a multiple of 64 and are zero-padded up to
//   the next (w dout and h rounded to bf16 there), and dgate_w = dlogits^T x
//   over one segment of all tokens (dlogits rounded to bf16, x as given). The
//   router's scores and dx and the gate vector keep the fp32 SIMT code above,
//   on fp32 copies of x and gate_w. Gradients are fp32. Still no atomics:
//   results are deterministic.

// out[i] = float(in[i])
__global__ void __launch_bounds__(BT) bw16_to_f32(const __nv_bfloat16* __restrict__ in, int64_t n,
                                                float* __restrict__ out) {
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT)
    out[i] = __bfloat162float(in[i]);
}

// L[t][e] = sum over splits s (in order) of part[s][t][e], row pitch ldo.
__global__ void __launch_bounds__(BT) bw16_sum_logits(const float* __restrict__ part, int splits, int64_t ldo,
                                                    int T, int E, float* __restrict__ L) {
  const int64_t n = (int64_t)T * E;
  for (int64_t i = blockIdx.x * (int64_t)BT + threadIdx.x; i < n; i += (int64_t)gridDim.x * BT) {
    const int64_t t = i / E;
    const int e = (int)(i - t * E);
    float acc = 0.f;
#pragma unroll 4
    for (int sp = 0; sp < splits; ++sp) acc += part[((int64_t)sp * T + t) * ldo + e];  // in split order
    L[i] = acc;
  }
}

// Padded row offsets of the weight-gradient GEMMs: koff[e] = sum over e' < e
// of round_up(count[e'], 64); also the one-segment range of all tokens,
// ranges = {0, T, 0, round_up(T, 64)}, and its split into `splits` row
// chunks of `chunk` rows (a multiple of 64) for the router's weight gradient:
// rsplit[i] = min(i * chunk, round_up(T, 64)), i = 0..splits.
// One warp: lane l scans experts [l*per, l*per + per), per = ceil(E / 32),
// then the lanes' totals are scanned with shuffles.
__global__ void bw16_koff(const int32_t* __restrict__ offsets, int E, int T, int32_t* __restrict__ koff,
                          int32_t* __restrict__ ranges, int splits, int chunk, int32_t* __restrict__ rsplit) {
  const int lane = threadIdx.x;
  if (lane >= 32 || blockIdx.x != 0) return;
  constexpr int kPer = kMaxExperts / 32;
  const int per = (E + 31) / 32;
  int padded[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane * per + i;
    padded[i] = (i < per && e < E) ? (offsets[e + 1] - offsets[e] + 63) / 64 * 64 : 0;
    sum += padded[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane * per + i;
    if (i < per && e < E) koff[e] = run;
    run += padded[i];
  }
  if (lane == 31) koff[E] = incl;
  if (lane == 0) {
    const int Tpad = (T + 63) / 64 * 64;
    ranges[0] = 0;
    ranges[1] = T;
    ranges[2] = 0;
    ranges[3] = Tpad;
    for (int i = 0; i <= splits; ++i) rsplit[i] = min(i * chunk, Tpad);
  }
}

// Padded row buffers, one block per 64-row group (an expert's run starts at a
// multiple of 64, so a group lies in one expert e). Row q = koff[e] + j holds,
// for j < count_e and r = off[e] + j: x_pad[q] = x[tok[r]] and dy_pad[q] =
// bf16(scale[r] * dout[tok[r]]); also dout_perm[r] = dout[tok[r]] (the sorted
// rows of dout, dense). Rows with j >= count_e are zero in x_pad, dy_pad,
// h_pad [*, I] and dgdu_pad [*, 2I] (the SwiGLU backward writes the others).
// 16-byte vectors (H and I are multiples of 8).
constexpr int kPadBatch = 4;

__global__ void __launch_bounds__(BT) bw16_pad_rows(const __nv_bfloat16* __restrict__ x,
                                                  const __nv_bfloat16* __restrict__ dout,
                                                  const int32_t* __restrict__ tok, const float* __restrict__ scale,
                                                  const int32_t* __restrict__ off, const int32_t* __restrict__ koff,
                                                  int E, int H, int I, __nv_bfloat16* __restrict__ dout_perm,
                                                  __nv_bfloat16* __restrict__ x_pad,
                                                  __nv_bfloat16* __restrict__ dy_pad,
                                                  __nv_bfloat16* __restrict__ h_pad,
                                                  __nv_bfloat16* __restrict__ dgdu_pad) {
  __shared__ int s_src[64];
  __shared__ float s_sc[64];
  __shared__ int s_e;
  const int q0 = blockIdx.x * 64;
  if (q0 >= koff[E]) return;  // past the last expert's run (the same for the whole block)
  if (threadIdx.x == 0) {
    int lo = 0, hi = E;  // koff[lo] <= q0 < koff[lo + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (koff[mid] <= q0) lo = mid;
      else hi = mid;
    }
    s_e = lo;
  }
  __syncthreads();
  const int e = s_e;
  const int j0 = q0 - koff[e];
  const int cnt = off[e + 1] - off[e];
  if (threadIdx.x < 64) {
    const int j = j0 + (int)threadIdx.x;
    int src = -1;
    float sc = 0.f;
    if (j < cnt) {
      const int r = off[e] + j;
      src = tok[r];
      sc = scale[r];
    }
    s_src[threadIdx.x] = src;
    s_sc[threadIdx.x] = sc;
  }
  __syncthreads();
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  const int hv = H / 8;
  const int total = 64 * hv;
  // kPadBatch vectors a thread at a time: their loads are all issued before
  // the first store, so each thread keeps several rows' loads in flight.
  for (int base = threadIdx.x; base < total; base += BT * kPadBatch) {
    uint4 xv[kPadBatch], dv[kPadBatch];
#pragma unroll
    for (int u = 0; u < kPadBatch; ++u) {
      const int idx = base + u * BT;
      xv[u] = zero;
      dv[u] = zero;
      if (idx < total) {
        const int i = idx / hv, v = idx - i * hv;
        const int src = s_src[i];
        if (src >= 0) {
          xv[u] = reinterpret_cast<const uint4*>(x + (int64_t)src * H)[v];
          dv[u] = reinterpret_cast<const uint4*>(dout + (int64_t)src * H)[v];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPadBatch; ++u) {
      const int idx = base + u * BT;
      if (idx >= total) break;
      const int i = idx / hv, v = idx - i * hv;
      const int64_t q = q0 + i;
      uint4 yo = zero;
      if (s_src[i] >= 0) {
        reinterpret_cast<uint4*>(dout_perm + (int64_t)(off[e] + j0 + i) * H)[v] = dv[u];
        float f[8];
        unpack16_bf16(dv[u], f);
        const float sc = s_sc[i];
        yo = make_uint4(pack_bf16x2(sc * f[0], sc * f[1]), pack_bf16x2(sc * f[2], sc * f[3]),
                        pack_bf16x2(sc * f[4], sc * f[5]), pack_bf16x2(sc * f[6], sc * f[7]));
      }
      reinterpret_cast<uint4*>(x_pad + q * H)[v] = xv[u];
      reinterpret_cast<uint4*>(dy_pad + q * H)[v] = yo;
    }
  }
  const int nvalid = max(0, min(64, cnt - j0));
  const int iv = I / 8, rv = 3 * iv;  // one row: I/8 vectors of h, 2I/8 of [dg | du]
  for (int idx = threadIdx.x; idx < (64 - nvalid) * rv; idx += BT) {
    const int i = nvalid + idx / rv, v = idx % rv;
    const int64_t q = q0 + i;
    if (v < iv) reinterpret_cast<uint4*>(h_pad + q * I)[v] = zero;
    else reinterpret_cast<uint4*>(dgdu_pad + q * 2 * I)[v - iv] = zero;
  }
}

// SwiGLU backward, one warp per row p < R (R = *nrows when given, else rows),
// with g, u from gu [*, 2I], dhu [*, I] and the row's weight scale[p]: h =
// silu(g) u and dh = scale dhu in fp32; [dg | du] = [dh u silu'(g) | dh silu(g)]
// rounded to bf16 into dgdu [*, 2I]; h rounded to bf16 into h_rows [*, I] and
// [dg | du] into dgdu_rows (when given) at row q = koff[e] + p - off[e] of p's
// segment e (q = p without off); dot = sum_i h dhu (fp32, h unrounded) into
// dot_out[dot_idx[p]] (or [p]; nothing without dot_out), times gamma (1 -
// gamma) with dot_gamma = gamma. Lanes take 4 columns at a time (I is a
// multiple of 8): 16-byte loads, 8-byte stores.
__global__ void __launch_bounds__(BT) bw16_swiglu_rows(const float* __restrict__ gu, const float* __restrict__ dhu,
                                                     const float* __restrict__ scale, const int32_t* __restrict__ nrows,
                                                     int64_t rows, int I, const int32_t* __restrict__ off,
                                                     const int32_t* __restrict__ koff, int E,
                                                     const int32_t* __restrict__ dot_idx,
                                                     const float* __restrict__ dot_gamma, float* __restrict__ dot_out,
                                                     __nv_bfloat16* __restrict__ dgdu,
                                                     __nv_bfloat16* __restrict__ h_rows,
                                                     __nv_bfloat16* __restrict__ dgdu_rows) {
  __shared__ int s_off[kMaxExperts + 1], s_koff[kMaxExperts + 1];
  if (off) {
    for (int e = threadIdx.x; e <= E; e += BT) {
      s_off[e] = off[e];
      s_koff[e] = koff[e];
    }
  }
  __syncthreads();
  const int64_t R = nrows ? (int64_t)*nrows : rows;
  const int lane = threadIdx.x & 31;
  for (int64_t p = (blockIdx.x * (int64_t)BT + threadIdx.x) >> 5; p < R; p += ((int64_t)gridDim.x * BT) >> 5) {
    int64_t q = p;
    if (off) {
      int lo = 0, hi = E;  // s_off[lo] <= p < s_off[lo + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= p) lo = mid;
        else hi = mid;
      }
      q = s_koff[lo] + (p - s_off[lo]);
    }
    const float sc = scale[p];
    const float* grow = gu + p * 2 * I;
    const float* drow = dhu + p * I;
    float dot = 0.f;
    for (int i = lane * 4; i < I; i += 128) {
      const float4 g4 = *reinterpret_cast<const float4*>(grow + i);
      const float4 u4 = *reinterpret_cast<const float4*>(grow + I + i);
      const float4 d4 = *reinterpret_cast<const float4*>(drow + i);
      const float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w}, d[4] = {d4.x, d4.y, d4.z, d4.w};
      float h[4], dg[4], du[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float sg = silu_f32(g[c]);
        const float dh = sc * d[c];
        h[c] = sg * u[c];
        dg[c] = dh * u[c] * silu_grad_f(g[c]);
        du[c] = dh * sg;
        dot = fmaf(h[c], d[c], dot);
      }
      const uint2 dg2 = make_uint2(pack_bf16x2(dg[0], dg[1]), pack_bf16x2(dg[2], dg[3]));
      const uint2 du2 = make_uint2(pack_bf16x2(du[0], du[1]), pack_bf16x2(du[2], du[3]));
      *reinterpret_cast<uint2*>(dgdu + p * 2 * I + i) = dg2;
      *reinterpret_cast<uint2*>(dgdu + p * 2 * I + I + i) = du2;
      *reinterpret_cast<uint2*>(h_rows + q * I + i) = make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
      if (dgdu_rows) {
        *reinterpret_cast<uint2*>(dgdu_rows + q * 2 * I + i) = dg2;
        *reinterpret_cast<uint2*>(dgdu_rows + q * 2 * I + I + i) = du2;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0 && dot_out) {
      if (dot_gamma) dot *= dot_gamma[p] * (1.f - dot_gamma[p]);
      dot_out[dot_idx ? dot_idx[p] : p] = dot;
    }
  }
}

// out[t][h] += add[t][h] (+ dz[t] * g[h] when dz is given), fp32.
__global__ void __launch_bounds__(BT) bw16_add_rows(float* __restrict__ out, const float* __restrict__ add,
                                                  const float* __restrict__ dz, const float* __restrict__ g, int T,
                                                  int H) {
  const int hv = H / 4;
  const int64_t n = (int64_t)T * hv;
  for (int64_t idx = blockIdx.x * (int64_t)BT + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * BT) {
    const int64_t t = idx / hv;
    const int h = (int)(idx - t * hv) * 4;
    float4 o = reinterpret_cast<float4*>(out)[idx];
    const float4 a = reinterpret_cast<const float4*>(add)[idx];
    o.x += a.x;
    o.y += a.y;
    o.z += a.z;
    o.w += a.w;
    if (dz) {
      const float z = dz[t];
      o.x = fmaf(z, g[h], o.x);
      o.y = fmaf(z, g[h + 1], o.y);
      o.z = fmaf(z, g[h + 2], o.z);
      o.w = fmaf(z, g[h + 3], o.w);
    }
    reinterpret_cast<float4*>(out)[idx] = o;
  }
}

// out[t][h] = bf16(gamma[t] * in[t][h]), eight columns per thread (H a multiple of 8).
__global__ void __launch_bounds__(BT) bw16_scale_rows(const __nv_bfloat16* __restrict__ in,
                                                    const float* __restrict__ gamma, int T, int H,
                                                    __nv_bfloat16* __restrict__ out) {
  const int hv = H / 8;
  const int64_t n = (int64_t)T * hv;
  for (int64_t idx = blockIdx.x * (int64_t)BT + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * BT) {
    const int64_t t = idx / hv;
    float f[8];
    unpack16_bf16(reinterpret_cast<const uint4*>(in)[idx], f);
    const float sc = gamma[t];
    reinterpret_cast<uint4*>(out)[idx] =
        make_uint4(pack_bf16x2(sc * f[0], sc * f[1]), pack_bf16x2(sc * f[2], sc * f[3]),
                   pack_bf16x2(sc * f[4], sc * f[5]), pack_bf16x2(sc * f[6], sc * f[7]));
  }
}

// Row chunks of the bf16 router weight gradient dgate_w = dL^T x: its [E, H]
// output has few tiles and a T-long reduction, so the reduction is split
// into at most 16 chunks of whole 64-row steps until about one tile per SM
// is busy; the partial sums are added in chunk order.
struct RouterSplit16 {
  int splits, chunk;
};
RouterSplit16 router_split16(const moe_problem& p) {
  const int64_t tiles = ceil_div(p.E, 128) * ceil_div(p.H, 256);
  const int64_t steps = ceil_div(p.T, 64);
  const int64_t want = std::max<int64_t>(1, std::min<int64_t>({ceil_div(148, tiles), steps, 16}));
  const int64_t chunk = ceil_div(steps, want) * 64;
  return {(int)ceil_div(round_up(p.T, 64), chunk), (int)chunk};
}

struct BwLayout16 {
  size_t header, local, counts, offsets, sorted_pairs, pair_pos, tok, scale, w, dw, L, S, dL, dL16, lpart, x32, g32,
      koff, ranges, rsplit, parts, xperm, doutperm, gu, dhu, dgdu, dxr, extra, xpad, dypad, hpad, dgdupad, gus, dhus, hs, dgdus, dys,
      rdx, gamma, dz, total;
  int64_t Ppad, Tpad, Epad;
};

BwLayout16 bw_layout16(const moe_problem& p) {
  BwLayout16 b;
  const int64_t P = p.T * p.k;
  b.Ppad = round_up(P + 63 * p.E, 64);
  b.Tpad = round_up(p.T, 64);
  b.Epad = round_up(p.E, 8);  // 16-byte rows of the bf16 dlogits
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = a256(off + bytes);
    return at;
  };
  const size_t f = 4, h2 = 2;
  b.header = take(sizeof(WsHeader));
  b.local = take((size_t)dispatch_num_blocks(p.T, p.k) * p.E * 4);
  b.counts = take((size_t)p.E * 4);
  b.offsets = take((size_t)(p.E + 1) * 4);
  b.sorted_pairs = take((size_t)P * 4);
  b.pair_pos = take((size_t)P * 4);
  b.tok = take((size_t)P * 4);
  b.scale = take((size_t)P * f);
  b.w = take((size_t)P * f);
  b.dw = take((size_t)P * f);
  b.L = take((size_t)p.T * p.E * f);
  b.S = take((size_t)p.T * p.E * f);
  b.dL = take((size_t)p.T * p.E * f);
  b.dL16 = take((size_t)p.T * b.Epad * h2);
  b.lpart = take(router_partial_bytes(MOE_DTYPE_BF16, p.T, p.H, p.E));
  const bool sh = p.shared != MOE_SHARED_NONE, gated = p.shared == MOE_SHARED_SIGMOID_GATED;
  b.x32 = take(gated ? (size_t)p.T * p.H * f : 0);  // fp32 x for the shared gate's SIMT kernels
  b.g32 = take(gated ? (size_t)p.H * f : 0);
  b.koff = take((size_t)(p.E + 1) * 4);
  b.ranges = take(4 * 4);
  const RouterSplit16 rs = router_split16(p);
  b.rsplit = take((size_t)(rs.splits + 1) * 4);
  b.parts = take(rs.splits > 1 ? (size_t)rs.splits * p.E * p.H * f : 0);
  b.xperm = take((size_t)P * p.H * h2);
  b.doutperm = take((size_t)P * p.H * h2);
  b.gu = take((size_t)P * 2 * p.I * f);
  b.dhu = take((size_t)P * p.I * f);
  b.dgdu = take((size_t)P * 2 * p.I * h2);
  b.dxr = take((size_t)P * p.H * f);
  b.extra = take((size_t)p.T * p.H * f);
  b.xpad = take((size_t)b.Ppad * p.H * h2);
  b.dypad = take((size_t)b.Ppad * p.H * h2);
  b.hpad = take((size_t)b.Ppad * p.I * h2);
  b.dgdupad = take((size_t)b.Ppad * 2 * p.I * h2);
  const size_t Is = sh ? (size_t)p.I_shared : 0;
  b.gus = take((size_t)p.T * 2 * Is * f);
  b.dhus = take((size_t)p.T * Is * f);
  b.hs = take((size_t)p.T * Is * h2);
  b.dgdus = take((size_t)p.T * 2 * Is * h2);
  b.dys = take(gated ? (size_t)p.T * p.H * h2 : 0);
  b.rdx = take(sh ? (size_t)p.T * p.H * f : 0);  // the router's dx beside the shared expert's
  b.gamma = take(sh ? (size_t)p.T * f : 0);
  b.dz = take(sh ? (size_t)p.T * f : 0);
  b.total = off;
  return b;
}

#define BW16_CUDA(...)                                     \
  do {                                                     \
    if ((__VA_ARGS__) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

moe_status backward_bf16(const moe_problem* p, const moe_weights* w, const void* x_, const void* dout_,
                         const int64_t* selected, moe_grads* g, void* ws, cudaStream_t s) {
  const BwLayout16 b = bw_layout16(*p);
  const bool sh = p->shared != MOE_SHARED_NONE, gated = p->shared == MOE_SHARED_SIGMOID_GATED;
  const int T = (int)p->T, H = (int)p->H, E = (int)p->E, k = (int)p->k, I = (int)p->I, Is = (int)p->I_shared;
  const int64_t P = p->T * p->k;
  using bf = __nv_bfloat16;
  const bf* x = static_cast<const bf*>(x_);
  const bf* dout = static_cast<const bf*>(dout_);
  WsHeader* hdr = at<WsHeader>(ws, b.header);
  int32_t* err = &hdr->error_bits;
  int32_t* offsets = at<int32_t>(ws, b.offsets);
  int32_t* sorted_pairs = at<int32_t>(ws, b.sorted_pairs);
  int32_t* pair_pos = at<int32_t>(ws, b.pair_pos);
  int32_t* tok = at<int32_t>(ws, b.tok);
  float* scale = at<float>(ws, b.scale);
  float* wts = at<float>(ws, b.w);
  float* dw = at<float>(ws, b.dw);
  float* L = at<float>(ws, b.L);
  float* S = at<float>(ws, b.S);
  float* dL = at<float>(ws, b.dL);
  bf* dL16 = at<bf>(ws, b.dL16);
  float* x32 = gated ? at<float>(ws, b.x32) : nullptr;
  float* g32 = gated ? at<float>(ws, b.g32) : nullptr;
  int32_t* koff = at<int32_t>(ws, b.koff);
  int32_t* ranges = at<int32_t>(ws, b.ranges);
  bf* xperm = at<bf>(ws, b.xperm);
  bf* doutperm = at<bf>(ws, b.doutperm);
  float* gu = at<float>(ws, b.gu);
  float* dhu = at<float>(ws, b.dhu);
  bf* dgdu = at<bf>(ws, b.dgdu);
  float* dxr = at<float>(ws, b.dxr);
  float* extra = at<float>(ws, b.extra);
  bf* xpad = at<bf>(ws, b.xpad);
  bf* dypad = at<bf>(ws, b.dypad);
  bf* hpad = at<bf>(ws, b.hpad);
  bf* dgdupad = at<bf>(ws, b.dgdupad);

  // fp32 copies of x and the gate vector for the shared gate's SIMT kernels
  if (gated) {
    bw16_to_f32<<<grid_for((int64_t)T * H), BT, 0, s>>>(x, (int64_t)T * H, x32);
    bw16_to_f32<<<grid_for(H), BT, 0, s>>>(static_cast<const bf*>(w->shared_gate), H, g32);
  }
  // Router: logits on the tensor cores (the forward's split-K GEMM, its
  // partials summed in split order), then scores and the routing weights of
  // the given choice.
  {
    const RouterPlan rp = router_plan(MOE_DTYPE_BF16, T, H, E);
    float* lpart = at<float>(ws, b.lpart);
    BW16_CUDA(launch_tc_logits(x, w->gate_w, T, H, E, lpart, rp.ldo, rp.splits, err, s));
    bw16_sum_logits<<<grid_for((int64_t)T * E), BT, 0, s>>>(lpart, rp.splits, rp.ldo, T, E, L);
  }
  bw_scores<<<(unsigned)ceil_div(T, kTokWarps), BT, 0, s>>>(L, w->bias, p->bias_mode, p->score,
                                                              p->renormalize ? 1 : 0, selected, (int)T, E, k, S, wts);
  // Sorted segments of the choice with x_perm.
  BW16_CUDA(launch_dispatch(MOE_DTYPE_BF16, selected, x, p->T, p->H, p->E, p->k, at<int32_t>(ws, b.local),
                            at<int32_t>(ws, b.counts), offsets, sorted_pairs, pair_pos, xperm, err,
                            &hdr->dispatch_ticket, s));
  bw_rows<<<grid_for(P), BT, 0, s>>>(sorted_pairs, offsets, wts, E, k, tok, scale);
  const RouterSplit16 rs = router_split16(*p);
  int32_t* rsplit = at<int32_t>(ws, b.rsplit);
  bw16_koff<<<1, 32, 0, s>>>(offsets, E, T, koff, ranges, rs.splits, rs.chunk, rsplit);
  // The sorted rows of dout; the padded rows of x and w dout for the weight gradients.
  bw16_pad_rows<<<(unsigned)(b.Ppad / 64), BT, 0, s>>>(x, dout, tok, scale, offsets, koff, E, H, I, doutperm, xpad,
                                                       dypad, hpad, dgdupad);
  // Routed experts on the tensor cores; the weights are read as stored.
  const Segments sg{offsets, (int32_t)E, 0, P};
  BW16_CUDA(launch_tc_down(sg, xperm, w->gate_up, E, gu, nullptr, nullptr, 2 * I, H, err, s));  // [g | u]
  BW16_CUDA(launch_tc_down_kn(sg, doutperm, H, w->down, E, dhu, nullptr, nullptr, I, H, err, s));  // dhu
  // dw of pairs the dispatch dropped (bad expert ids) stays 0
  BW16_CUDA(cudaMemsetAsync(dw, 0, (size_t)P * sizeof(float), s));
  bw16_swiglu_rows<<<grid_for(P * 32), BT, 0, s>>>(gu, dhu, scale, offsets + E, P, I, offsets, koff, E, sorted_pairs,
                                                    nullptr, dw, dgdu, hpad, dgdupad);
  BW16_CUDA(launch_tc_down_kn(sg, dgdu, 2 * I, w->gate_up, E, dxr, nullptr, nullptr, H, 2 * I, err, s));  // dx rows
  // Routed weight gradients: dWd = (w dout)^T h, dWgu = [dg du]^T x.
  BW16_CUDA(launch_wgrad(dypad, H, hpad, I, b.Ppad, koff, b.Ppad, E, H, I, g->d_down, err, s));
  BW16_CUDA(launch_wgrad(dgdupad, 2 * I, xpad, H, b.Ppad, koff, b.Ppad, E, 2 * I, H, g->d_gate_up, err, s));
  // Router backward: dL (fp32, and rounded to bf16 for the tensor cores:
  // dgate_w = dL^T x over all tokens, the router's dx = dL gate_w with gate_w
  // [E][H] read as stored); d_bias = sum_t dL in fp32. The router's dx goes
  // to `extra`, or beside the shared expert's when there is one.
  bw_router_bwd<<<(unsigned)ceil_div(T, kTokWarps), BT, 0, s>>>(L, S, wts, dw, selected, p->score,
                                                                  p->renormalize ? 1 : 0, (int)T, E, k, dL, dL16,
                                                                  (int)b.Epad);
  if (rs.splits > 1) {
    float* parts = at<float>(ws, b.parts);
    BW16_CUDA(launch_wgrad(dL16, b.Epad, x, H, T, rsplit, b.Tpad, rs.splits, E, H, parts, err, s));
    bw_sum_parts<<<grid_for((int64_t)E * H), BT, 0, s>>>(parts, rs.splits, (int64_t)E * H, g->d_gate_w);
  } else {
    BW16_CUDA(launch_wgrad(dL16, b.Epad, x, H, T, ranges + 2, b.Tpad, 1, E, H, g->d_gate_w, err, s));
  }
  if (g->d_bias) bw_colsum<<<grid_for(E), BT, 0, s>>>(dL, E, T, E, g->d_bias);
  const Segments one{nullptr, 1, (int32_t)T, p->T};
  float* rdx = sh ? at<float>(ws, b.rdx) : extra;
  BW16_CUDA(launch_tc_down_kn(one, dL16, b.Epad, w->gate_w, 1, rdx, nullptr, nullptr, H, E, err, s));
  // Shared expert over all tokens (one segment), scaled by gamma; its dx goes to `extra`.
  float* dz = nullptr;
  if (sh) {
    float* gus = at<float>(ws, b.gus);
    float* dhus = at<float>(ws, b.dhus);
    bf* hs = at<bf>(ws, b.hs);
    bf* dgdus = at<bf>(ws, b.dgdus);
    float* gamma = at<float>(ws, b.gamma);
    dz = at<float>(ws, b.dz);
    bw_gamma<<<grid_for((int64_t)T * 32), BT, 0, s>>>(x32, g32, T, H, gamma);
    BW16_CUDA(launch_tc_down(one, x, w->shared_gate_up, 1, gus, nullptr, nullptr, 2 * Is, H, err, s));
    BW16_CUDA(launch_tc_down_kn(one, dout, H, w->shared_down, 1, dhus, nullptr, nullptr, Is, H, err, s));
    bw16_swiglu_rows<<<grid_for((int64_t)T * 32), BT, 0, s>>>(gus, dhus, gamma, nullptr, T, Is, nullptr, nullptr, 0,
                                                               nullptr, gamma, gated ? dz : nullptr, dgdus, hs,
                                                               nullptr);
    BW16_CUDA(launch_tc_down_kn(one, dgdus, 2 * Is, w->shared_gate_up, 1, extra, nullptr, nullptr, H, 2 * Is, err, s));
    // w dout for the shared expert is gamma dout (dout itself when ungated)
    const bf* dys = dout;
    if (gated) {
      bf* dyg = at<bf>(ws, b.dys);
      bw16_scale_rows<<<grid_for((int64_t)T * H / 8), BT, 0, s>>>(dout, gamma, T, H, dyg);
      dys = dyg;
    }
    BW16_CUDA(launch_wgrad(dys, H, hs, Is, T, ranges + 2, b.Tpad, 1, H, Is, g->d_shared_down, err, s));
    BW16_CUDA(launch_wgrad(dgdus, 2 * Is, x, H, T, ranges + 2, b.Tpad, 1, 2 * Is, H, g->d_shared_gate_up, err, s));
    if (gated) bw_dgvec<<<grid_for(H), BT, 0, s>>>(dz, x32, T, H, g->d_shared_gate);
    // extra = the shared expert's dx + the router's (+ the shared gate's dz g)
    bw16_add_rows<<<grid_for((int64_t)T * H / 4), BT, 0, s>>>(extra, rdx, gated ? dz : nullptr, g32, T, H);
  }
  // dx = sum of each token's rows + extra.
  BW16_CUDA(launch_combine(MOE_DTYPE_F32, dxr, pair_pos, extra, g->dx, p->T, p->H, p->k, s));
  return MOE_OK;
}

}  // namespace
}  // namespace stm

using namespace stm;

MOE_API moe_status moe_backward_workspace_size(const moe_problem* p, size_t* bytes) {
  size_t fwd = 0;
  const moe_status st = moe_workspace_size(p, &fwd);  // validates the problem
  if (st != MOE_OK) return st;
  if (bytes == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = p->dtype == MOE_DTYPE_BF16 ? bw_layout16(*p).total : bw_layout(*p).total;
  return MOE_OK;
}

#define BW_CUDA(...)                                       \
  do {                                                     \
    if ((__VA_ARGS__) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

MOE_API moe_status moe_backward(const moe_problem* p, const moe_weights* w, const void* x_, const void* dout_,
                                const int64_t* selected, moe_grads* g, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  size_t need = 0;
  const moe_status st = moe_backward_workspace_size(p, &need);
  if (st != MOE_OK) return st;
  if (w == nullptr || g == nullptr) return MOE_ERR_INVALID_ARGUMENT;
  const bool sh = p->shared != MOE_SHARED_NONE, gated = p->shared == MOE_SHARED_SIGMOID_GATED;
  const bool has_tokens = p->T > 0;  // per-token arrays and the workspace may be NULL without tokens
  if ((has_tokens && (!ok16(x_) || !ok16(dout_) || !ok16(selected) || !ok16(g->dx) || !ok16(ws))) ||
      !ok16(w->gate_w) || !ok16(w->gate_up) || !ok16(w->down) || !ok16(g->d_gate_w) || !ok16(g->d_gate_up) ||
      !ok16(g->d_down))
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
  if (!has_tokens) {  // no tokens: every weight gradient is zero
    const size_t f = sizeof(float);
    BW_CUDA(cudaMemsetAsync(g->d_gate_w, 0, (size_t)(p->E * p->H) * f, s));
    if (g->d_bias) BW_CUDA(cudaMemsetAsync(g->d_bias, 0, (size_t)p->E * f, s));
    BW_CUDA(cudaMemsetAsync(g->d_gate_up, 0, (size_t)(p->E * 2 * p->I * p->H) * f, s));
    BW_CUDA(cudaMemsetAsync(g->d_down, 0, (size_t)(p->E * p->H * p->I) * f, s));
    if (sh) BW_CUDA(cudaMemsetAsync(g->d_shared_gate_up, 0, (size_t)(2 * p->I_shared * p->H) * f, s));
    if (sh) BW_CUDA(cudaMemsetAsync(g->d_shared_down, 0, (size_t)(p->H * p->I_shared) * f, s));
    if (gated) BW_CUDA(cudaMemsetAsync(g->d_shared_gate, 0, (size_t)p->H * f, s));
    return MOE_OK;
  }
  NvtxRange range("moe_backward");
  if (p->dtype == MOE_DTYPE_BF16) return backward_bf16(p, w, x_, dout_, selected, g, ws, s);
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
  float* scale = at<float>(ws, b.scale);
  float* wts = at<float>(ws, b.w);
  float* dw = at<float>(ws, b.dw);
  float* L = at<float>(ws, b.L);
  float* S = at<float>(ws, b.S);
  float* dL = at<float>(ws, b.dL);
  float* gu = at<float>(ws, b.gu);
  float* dgu = at<float>(ws, b.dgu);
  float* dhu = at<float>(ws, b.dhu);
  float* hact = at<float>(ws, b.hact);
  float* dxr = at<float>(ws, b.dxr);
  float* extra = at<float>(ws, b.extra);

  // Router: logits, scores and the routing weights of the given choice.
  BW_CUDA(run_rows<true, EPI_STORE>(
      [&] {
        RowGemm a = row_gemm(x, nullptr, H, gw, 0, E, H, nullptr, 1, T, T, err);
        a.C = L;
        a.ldc = E;
        return a;
      }(),
      s));
  bw_scores<<<(unsigned)ceil_div(T, kTokWarps), BT, 0, s>>>(L, w->bias, p->bias_mode, p->score,
                                                              p->renormalize ? 1 : 0, selected, (int)T, E, k, S, wts);
  // Sorted segments of the choice, each row's token and weight.
  BW_CUDA(launch_dispatch(MOE_DTYPE_F32, selected, nullptr, p->T, p->H, p->E, p->k, at<int32_t>(ws, b.local),
                          at<int32_t>(ws, b.counts), offsets, sorted_pairs, pair_pos, nullptr, err,
                          &at<WsHeader>(ws, b.header)->dispatch_ticket, s));
  bw_rows<<<grid_for(P), BT, 0, s>>>(sorted_pairs, offsets, wts, E, k, tok, scale);
  // Routed experts: recompute [g | u]; dhu and [dg | du]; dx rows; dw.
  BW_CUDA(run_rows<true, EPI_STORE>(
      [&] {
        RowGemm a = row_gemm(x, tok, H, wgu, (int64_t)2 * I * H, 2 * I, H, offsets, E, 0, P, err);
        a.C = gu;
        a.ldc = 2 * I;
        return a;
      }(),
      s));
  BW_CUDA(run_rows<false, EPI_DGU>(
      [&] {
        RowGemm a = row_gemm(dout, tok, H, wd, (int64_t)H * I, I, H, offsets, E, 0, P, err);
        a.GU = gu;
        a.scale = scale;
        a.DGU = dgu;
        a.DHU = dhu;
        a.Hact = hact;
        return a;
      }(),
      s));
  BW_CUDA(run_rows<false, EPI_STORE>(
      [&] {
        RowGemm a = row_gemm(dgu, nullptr, 2 * I, wgu, (int64_t)2 * I * H, H, 2 * I, offsets, E, 0, P, err);
        a.C = dxr;
        a.ldc = H;
        return a;
      }(),
      s));
  bw_rowdot<<<grid_for(P * 32), BT, 0, s>>>(hact, dhu, I, pair_pos, P, nullptr, dw);
  // Routed weight gradients: dWd_e = (w dout)^T h, dWgu_e = [dg du]^T x.
  BW_CUDA(run_wgrad(wgrad(dout, tok, scale, H, H, hact, nullptr, I, I, offsets, 0, P, g->d_down, err), E, s));
  BW_CUDA(run_wgrad(wgrad(dgu, nullptr, nullptr, 2 * I, 2 * I, x, tok, H, H, offsets, 0, P, g->d_gate_up, err), E,
                    s));
  // Router backward: dL, dgate_w = dL^T x (in row chunks summed in order), d_bias = sum_t dL.
  bw_router_bwd<<<(unsigned)ceil_div(T, kTokWarps), BT, 0, s>>>(L, S, wts, dw, selected, p->score,
                                                                  p->renormalize ? 1 : 0, (int)T, E, k, dL, nullptr, 0);
  const int nchunk = router_chunks(*p);
  if (nchunk == 1) {
    BW_CUDA(run_wgrad(wgrad(dL, nullptr, nullptr, E, E, x, nullptr, H, H, nullptr, T, T, g->d_gate_w, err), 1, s));
  } else {
    float* parts = at<float>(ws, b.parts);
    const int chunk = (int)ceil_div(T, nchunk);
    BW_CUDA(run_wgrad(wgrad(dL, nullptr, nullptr, E, E, x, nullptr, H, H, nullptr, T, T, parts, err, chunk), nchunk,
                      s));
    bw_sum_parts<<<grid_for((int64_t)E * H), BT, 0, s>>>(parts, nchunk, (int64_t)E * H, g->d_gate_w);
  }
  if (g->d_bias) bw_colsum<<<grid_for(E), BT, 0, s>>>(dL, E, T, E, g->d_bias);
  // Shared expert over all tokens, scaled by gamma; its dx goes to `extra`.
  float* dz = nullptr;
  const float* gvec = static_cast<const float*>(w->shared_gate);
  if (sh) {
    const float* wsgu = static_cast<const float*>(w->shared_gate_up);
    const float* wsd = static_cast<const float*>(w->shared_down);
    float* gus = at<float>(ws, b.gus);
    float* dgus = at<float>(ws, b.dgus);
    float* dhus = at<float>(ws, b.dhus);
    float* hacts = at<float>(ws, b.hacts);
    float* gamma = at<float>(ws, b.gamma);
    dz = at<float>(ws, b.dz);
    bw_gamma<<<grid_for((int64_t)T * 32), BT, 0, s>>>(x, gated ? gvec : nullptr, T, H, gamma);
    BW_CUDA(run_rows<true, EPI_STORE>(
        [&] {
          RowGemm a = row_gemm(x, nullptr, H, wsgu, 0, 2 * Is, H, nullptr, 1, T, T, err);
          a.C = gus;
          a.ldc = 2 * Is;
          return a;
        }(),
        s));
    BW_CUDA(run_rows<false, EPI_DGU>(
        [&] {
          RowGemm a = row_gemm(dout, nullptr, H, wsd, 0, Is, H, nullptr, 1, T, T, err);
          a.GU = gus;
          a.scale = gamma;
          a.DGU = dgus;
          a.DHU = dhus;
          a.Hact = hacts;
          return a;
        }(),
        s));
    BW_CUDA(run_rows<false, EPI_STORE>(
        [&] {
          RowGemm a = row_gemm(dgus, nullptr, 2 * Is, wsgu, 0, H, 2 * Is, nullptr, 1, T, T, err);
          a.C = extra;
          a.ldc = H;
          return a;
        }(),
        s));
    if (gated) bw_rowdot<<<grid_for((int64_t)T * 32), BT, 0, s>>>(hacts, dhus, Is, nullptr, T, gamma, dz);
    BW_CUDA(run_wgrad(wgrad(dout, nullptr, gamma, H, H, hacts, nullptr, Is, Is, nullptr, T, T, g->d_shared_down,
                            err),
                      1, s));
    BW_CUDA(run_wgrad(wgrad(dgus, nullptr, nullptr, 2 * Is, 2 * Is, x, nullptr, H, H, nullptr, T, T,
                            g->d_shared_gate_up, err),
                      1, s));
    if (gated) bw_dgvec<<<grid_for(H), BT, 0, s>>>(dz, x, T, H, g->d_shared_gate);
  }
  // Router (and shared gate) dx into `extra`, then dx = sum of each token's rows + extra.
  RowGemm rd = row_gemm(dL, nullptr, E, gw, 0, H, E, nullptr, 1, T, T, err);
  rd.C = extra;
  rd.ldc = H;
  rd.dz = gated ? dz : nullptr;
  rd.gvec = gated ? gvec : nullptr;
  if (sh) BW_CUDA(run_rows<false, EPI_ADD>(rd, s));
  else BW_CUDA(run_rows<false, EPI_STORE>(rd, s));
  BW_CUDA(launch_combine(MOE_DTYPE_F32, dxr, pair_pos, extra, g->dx, p->T, p->H, p->k, s));
  return MOE_OK;
}
