// fp32 grouped SwiGLU on the SIMT pipes, for fp32 problems.
//
// The tensor cores have no fp32-in, fp32-accurate mode that meets an fp32
// problem's 1e-5 relative bar, so fp32 problems use plain FFMA tiles: 64 rows
// x 64 columns per block, 16-deep k slices in shared memory, 4x4 outputs per
// thread. Same segment table as the tensor-core path.
//   gate_up: h[p, n] = silu(sum_h A[p,h] Wg[e,n,h]) * sum_h A[p,h] Wu[e,n,h]
//   down:    y[p, n] = scale(p) * sum_i h[p,i] Wd[e,n,i]
// ("mstar.model.components.moe", SparseMoeBlock fused gate_up/down layout and
// dispatch_experts_fused's per-expert SwiGLU.)
#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace stm {

namespace {

constexpr int SBM = 64, SBN = 64, SBK = 16, STHREADS = 256;
static_assert(SBM == SBN && SBM * SBK % STHREADS == 0, "tile loads: whole elements per thread");

template <bool GATE_UP>
__global__ void __launch_bounds__(STHREADS) simt_grouped_kernel(const float* __restrict__ A,
                                                                const int32_t* __restrict__ offsets, int E,
                                                                int single_rows, const float* __restrict__ W,
                                                                float* __restrict__ out, int N, int K,
                                                                const float* __restrict__ row_scale,
                                                                const int32_t* __restrict__ scale_idx,
                                                                int64_t rows_total, int32_t* err) {
  __shared__ int off[kMaxExperts + 1], pre[kMaxExperts + 1];
  __shared__ float As[SBK][SBM + 4];
  __shared__ float Bs[GATE_UP ? 2 : 1][SBK][SBN + 4];
  const int tid = threadIdx.x;
  if (tid < 32) warp_build_tile_table(offsets, E, single_rows, SBM, off, pre, rows_total, err);
  __syncthreads();
  const int Eseg = offsets ? E : 1;
  const int mt = blockIdx.x;
  if (mt >= pre[Eseg]) return;
  const int e = find_segment(pre, Eseg, mt);
  const int row0 = off[e] + (mt - pre[e]) * SBM;
  const int row_end = off[e + 1];
  const int n0 = blockIdx.y * SBN;
  const int tx = tid & 15, ty = tid >> 4;
  // Weights of expert e: gate_up [2N, K] (gate rows then up rows) or down [N, K].
  const float* We = W + (int64_t)e * (GATE_UP ? 2 : 1) * N * K;

  float acc[GATE_UP ? 2 : 1][4][4];
#pragma unroll
  for (int g = 0; g < (GATE_UP ? 2 : 1); ++g)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[g][i][j] = 0.f;

  // The next K slice is read into registers while the current one is
  // multiplied out of shared memory (the same products in the same order).
  constexpr int G = GATE_UP ? 2 : 1;
  constexpr int PER = SBM * SBK / STHREADS;  // elements of a tile per thread (SBN == SBM)
  float ra[PER], rb[G][PER];
  auto load_slice = [&](int k0) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int i = tid + u * STHREADS;
      const int r = i / SBK, c = i % SBK;
      const int row = row0 + r, kk = k0 + c;
      ra[u] = (row < row_end && kk < K) ? A[(int64_t)row * K + kk] : 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int n = n0 + r;
        rb[g][u] = (n < N && kk < K) ? We[((int64_t)g * N + n) * K + kk] : 0.f;
      }
    }
  };
  auto store_slice = [&]() {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int i = tid + u * STHREADS;
      const int r = i / SBK, c = i % SBK;
      As[c][r] = ra[u];
#pragma unroll
      for (int g = 0; g < G; ++g) Bs[g][c][r] = rb[g][u];
    }
  };
  load_slice(0);
  store_slice();
  __syncthreads();
  for (int k0 = 0; k0 < K; k0 += SBK) {
    const bool more = k0 + SBK < K;
    if (more) load_slice(k0 + SBK);
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int g = 0; g < (GATE_UP ? 2 : 1); ++g) {
        float b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[g][kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[g][i][j] = fmaf(a[i], b[j], acc[g][i][j]);
      }
    }
    __syncthreads();
    if (more) {
      store_slice();
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = row0 + ty + 16 * i;
    if (row >= row_end) continue;
    float sc = 1.f;
    if (!GATE_UP && row_scale != nullptr) sc = row_scale[scale_idx ? scale_idx[row] : row];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      float v;
      if (GATE_UP) v = silu_f32(acc[0][i][j]) * acc[GATE_UP ? 1 : 0][i][j];
      else v = sc * acc[0][i][j];
      out[(int64_t)row * N + n] = v;
    }
  }
}

dim3 simt_grid(const Segments& sg, int64_t N) {
  // Row tiles are bounded by rows/BM + (number of segments).
  const int64_t nseg = sg.offsets ? sg.E : 1;
  const int64_t mt = sg.rows_total / SBM + nseg;
  return dim3((unsigned)mt, (unsigned)ceil_div(N, SBN));
}

}  // namespace

cudaError_t launch_simt_gate_up(const Segments& sg, const float* A, const float* w_gate_up, float* h, int64_t I,
                                int64_t H, int32_t* err, cudaStream_t s) {
  simt_grouped_kernel<true><<<simt_grid(sg, I), STHREADS, 0, s>>>(A, sg.offsets, sg.E, sg.single_rows, w_gate_up,
                                                                   h, (int)I, (int)H, nullptr, nullptr,
                                                                   sg.rows_total, err);
  return cudaGetLastError();
}

cudaError_t launch_simt_down(const Segments& sg, const float* h, const float* w_down, float* y,
                             const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                             cudaStream_t s) {
  simt_grouped_kernel<false><<<simt_grid(sg, H), STHREADS, 0, s>>>(h, sg.offsets, sg.E, sg.single_rows, w_down, y,
                                                                    (int)H, (int)I, row_scale, scale_idx,
                                                                    sg.rows_total, err);
  return cudaGetLastError();
}

}  // namespace stm
