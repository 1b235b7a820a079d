// Epilogues of the tensor-core grouped GEMMs: one thread owns one accumulator
// row (one TMEM lane) and walks its 256 fp32 columns 32 at a time.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace stm {
namespace tc {

// gate_up: accumulator columns j (gate) and 128 + j (up) of output column
// col0 + j; h = silu(gate) * up rounded to bf16, 16-byte stores, columns
// past N skipped (N is a multiple of 8).
__device__ __forceinline__ void epilogue_swiglu(uint32_t tbase, bool valid, __nv_bfloat16* orow, int col0, int N) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t g[32], u[32];
    tmem_ld32(tbase + c * 32, g);
    tmem_ld32(tbase + 128 + c * 32, u);
    tmem_ld_wait();
    const int cb = col0 + c * 32;
    if (valid) {
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
}

// down: y = sc * accumulator in fp32, 16-byte stores, columns past N skipped
// (N is a multiple of 8).
__device__ __forceinline__ void epilogue_scale_f32(uint32_t tbase, bool valid, float sc, float* orow, int col0,
                                                   int N) {
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    uint32_t d[32];
    tmem_ld32(tbase + c * 32, d);
    tmem_ld_wait();
    const int cb = col0 + c * 32;
    if (valid) {
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        if (cb + v * 4 < N) {
          float4 o;
          o.x = sc * __uint_as_float(d[v * 4 + 0]);
          o.y = sc * __uint_as_float(d[v * 4 + 1]);
          o.z = sc * __uint_as_float(d[v * 4 + 2]);
          o.w = sc * __uint_as_float(d[v * 4 + 3]);
          *reinterpret_cast<float4*>(orow + cb + v * 4) = o;
        }
      }
    }
  }
}

}  // namespace tc
}  // namespace stm
