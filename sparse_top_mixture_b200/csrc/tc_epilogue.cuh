// Epilogues of the tensor-core grouped GEMMs: one thread owns one accumulator
// row (one TMEM lane) and walks its 256 fp32 columns 32 at a time.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace stm {
namespace tc {

// Each epilogue warp owns 32 consecutive output rows (one per lane, i.e. per
// TMEM lane) and walks the accumulator 32 columns at a time. The fp32 down
// output goes through a per-warp staging block in shared memory, so that a
// warp store instruction writes whole 128-byte row segments instead of one
// 16-byte piece of 32 different rows (half-filled 32-byte sectors doubled
// the L2 write traffic of that GEMM).
constexpr int kStageStride = 36;                        // floats per staged row (144 B, keeps 16-byte alignment)
constexpr int kStageFloatsPerWarp = 32 * kStageStride;  // 4608 B per epilogue warp

// Write this lane's 32 fp32 values (row `lane` of the warp block) to
// out_row0[r * ldo + j] for rows r < nrows and columns j < ncols (ncols a
// multiple of 4).
__device__ __forceinline__ void store_block_f32(const float (&v)[32], float* stage, float* out_row0, int64_t ldo,
                                                int nrows, int ncols, int lane) {
  float4* srow = reinterpret_cast<float4*>(stage + lane * kStageStride);
#pragma unroll
  for (int q = 0; q < 8; ++q) srow[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int c4 = lane & 7;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = it * 4 + (lane >> 3);
    if (r < nrows && c4 * 4 < ncols)
      *reinterpret_cast<float4*>(out_row0 + (int64_t)r * ldo + c4 * 4) =
          reinterpret_cast<const float4*>(stage + r * kStageStride)[c4];
  }
  __syncwarp();
}

// gate_up: TMEM columns gcol + j (gate) and ucol + j (up) hold output column
// col0 + j; h = silu(gate) * up rounded to bf16. `nchunks` chunks of 32.
// Each lane stores its own row directly (the bf16 output is small; staging
// it through shared memory was measured slower than the write traffic it
// saves). out_row0: output row of lane 0; nrows: valid rows of the warp.
__device__ __forceinline__ void epilogue_swiglu(uint32_t tbase, int gcol, int ucol, int nchunks,
                                                __nv_bfloat16* out_row0, int64_t ldo, int nrows, int col0, int N,
                                                int lane) {
  __nv_bfloat16* orow = out_row0 + (int64_t)lane * ldo;
  const bool valid = lane < nrows;
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    uint32_t g[32], u[32];
    tmem_ld32(tbase + gcol + c * 32, g);
    tmem_ld32(tbase + ucol + c * 32, u);
    tmem_ld_wait();
    const int cb = col0 + c * 32;
    if (!valid) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      if (cb + v * 8 < N) {
        float hv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          hv[q] = silu_f32(__uint_as_float(g[v * 8 + q])) * __uint_as_float(u[v * 8 + q]);
        uint4 o;
        o.x = pack_bf16x2(hv[0], hv[1]);
        o.y = pack_bf16x2(hv[2], hv[3]);
        o.z = pack_bf16x2(hv[4], hv[5]);
        o.w = pack_bf16x2(hv[6], hv[7]);
        *reinterpret_cast<uint4*>(orow + cb + v * 8) = o;
      }
    }
  }
}

// down: y = sc * accumulator in fp32 for `nchunks` chunks of 32 columns
// starting at TMEM column 0 and output column col0. sc is this lane's row
// scale. Two register buffers: the next chunk's TMEM load is in flight while
// this one is staged and stored (the loads' latency, not the stores, bounded
// the epilogue when the K loop is short).
__device__ __forceinline__ void epilogue_scale_f32(uint32_t tbase, int nchunks, float sc, float* stage,
                                                   float* out_row0, int64_t ldo, int nrows, int col0, int N,
                                                   int lane) {
  auto store = [&](const uint32_t(&d)[32], int c) {
    const int cb = col0 + c * 32;
    if (cb >= N || nrows <= 0) return;  // warp-uniform
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = sc * __uint_as_float(d[q]);
    store_block_f32(v, stage, out_row0 + cb, ldo, nrows, N - cb, lane);
  };
  uint32_t a[32], b[32];
  tmem_ld32(tbase, a);
  tmem_ld_wait_regs(a);
#pragma unroll 1
  for (int c = 0; c < nchunks; c += 2) {  // a holds chunk c
    const bool two = c + 1 < nchunks;
    if (two) tmem_ld32(tbase + (c + 1) * 32, b);
    store(a, c);
    if (!two) break;
    tmem_ld_wait_regs(b);
    const bool more = c + 2 < nchunks;
    if (more) tmem_ld32(tbase + (c + 2) * 32, a);
    store(b, c + 1);
    if (more) tmem_ld_wait_regs(a);
  }
}

// store_block_f32 with a destination per row: row r of the warp block goes
// to row_ptr of lane r (NULL: not stored) + column offset cb (ncols of the
// 32 columns, a multiple of 4). The row pointers are exchanged by shuffles.
__device__ __forceinline__ void store_block_f32_rows(const float (&v)[32], float* stage, float* row_ptr, int cb,
                                                     int nrows, int ncols, int lane) {
  float4* srow = reinterpret_cast<float4*>(stage + lane * kStageStride);
#pragma unroll
  for (int q = 0; q < 8; ++q) srow[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  __syncwarp();
  const int c4 = lane & 7;
  const unsigned long long mine = reinterpret_cast<unsigned long long>(row_ptr);
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int r = it * 4 + (lane >> 3);
    float* dst = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, mine, r));
    if (r < nrows && dst != nullptr && c4 * 4 < ncols)
      *reinterpret_cast<float4*>(dst + cb + c4 * 4) = reinterpret_cast<const float4*>(stage + r * kStageStride)[c4];
  }
  __syncwarp();
}

// epilogue_scale_f32 into per-row destinations (this lane's row at row_ptr,
// NULL for none), the same pipelined TMEM loads.
__device__ __forceinline__ void epilogue_scale_f32_rows(uint32_t tbase, int nchunks, float sc, float* stage,
                                                        float* row_ptr, int nrows, int col0, int N, int lane) {
  auto store = [&](const uint32_t(&d)[32], int c) {
    const int cb = col0 + c * 32;
    if (cb >= N || nrows <= 0) return;  // warp-uniform
    float v[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = sc * __uint_as_float(d[q]);
    store_block_f32_rows(v, stage, row_ptr, cb, nrows, N - cb, lane);
  };
  uint32_t a[32], b[32];
  tmem_ld32(tbase, a);
  tmem_ld_wait_regs(a);
#pragma unroll 1
  for (int c = 0; c < nchunks; c += 2) {  // a holds chunk c
    const bool two = c + 1 < nchunks;
    if (two) tmem_ld32(tbase + (c + 1) * 32, b);
    store(a, c);
    if (!two) break;
    tmem_ld_wait_regs(b);
    const bool more = c + 2 < nchunks;
    if (more) tmem_ld32(tbase + (c + 2) * 32, a);
    store(b, c + 1);
    if (more) tmem_ld_wait_regs(a);
  }
}

// Epilogues of swapped tiles (the weights as the MMA's M operand, a segment
// tail's tokens as its N columns): TMEM lane = output feature, column = row
// of the tile. `ncols` accumulator columns are read 32 at a time (columns
// past the tile's rows are read and dropped); `nrows` rows are stored.

// gate_up: lanes 0-15 of this warp hold the gate pre-activations of features
// f0 .. f0+15 and lanes 16-31 the up pre-activations of the same features.
// A lane swaps its values with lane ^ 16, so lane L < 16 finishes rows j and
// lane L + 16 rows j + 16 of feature f0 + L; h = silu(gate) * up rounded to
// bf16, as in epilogue_swiglu. out_row0: output row of column 0.
__device__ __forceinline__ void epilogue_swiglu_swapped(uint32_t tbase, int ncols, __nv_bfloat16* out_row0,
                                                        int64_t ldo, int nrows, int f0, int N, int lane) {
  const bool lo = lane < 16;
  const int f = f0 + (lane & 15);
  __nv_bfloat16* ocol = out_row0 + f;
#pragma unroll 1
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tbase + c0, v);
    tmem_ld_wait_regs(v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float a = __uint_as_float(v[j]), b = __uint_as_float(v[j + 16]);
      const float ao = __shfl_xor_sync(0xffffffffu, a, 16);
      const float bo = __shfl_xor_sync(0xffffffffu, b, 16);
      const float g = lo ? a : bo, u = lo ? ao : b;
      const int r = c0 + j + (lo ? 0 : 16);
      if (r < nrows && f < N) ocol[(int64_t)r * ldo] = __float2bfloat16_rn(silu_f32(g) * u);
    }
  }
}

// down: y = sc * accumulator for feature f0 + lane of rows 0 .. nrows-1,
// each row's scale read by the lane of the same index and passed round by
// shuffles. Row r goes to row_ptr(r) + f0 + lane, where row_ptr gives the
// row's base pointer (NULL: not stored); a warp store writes 128 contiguous
// bytes of one row.
template <typename RowScale, typename RowPtr>
__device__ __forceinline__ void epilogue_scale_f32_swapped(uint32_t tbase, int ncols, int nrows, int f0, int N,
                                                           int lane, RowScale row_scale, RowPtr row_ptr) {
  const int f = f0 + lane;
#pragma unroll 1
  for (int c0 = 0; c0 < ncols; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tbase + c0, v);
    const int mine = c0 + lane;
    float sc = 1.f;
    float* dst = nullptr;
    if (mine < nrows) {
      sc = row_scale(mine);
      dst = row_ptr(mine);
    }
    const unsigned long long dbits = reinterpret_cast<unsigned long long>(dst);
    tmem_ld_wait_regs(v);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float s = __shfl_sync(0xffffffffu, sc, j);
      float* d = reinterpret_cast<float*>(__shfl_sync(0xffffffffu, dbits, j));
      if (c0 + j < nrows && d != nullptr && f < N) d[f] = s * __uint_as_float(v[j]);
    }
  }
}

}  // namespace tc
}  // namespace stm
