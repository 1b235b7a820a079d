// Device helpers shared by the MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace stm {

constexpr int kMaxExperts = 256;  // warp top-k keeps E/32 <= 8 keys per lane

// Workspace header: the first 256 bytes of every workspace.
struct WsHeader {
  int32_t error_bits;
  int32_t wait_site;         // which pipeline wait gave up, when one did
  uint32_t dispatch_ticket;  // CTAs of the running dispatch histogram that are done (0 between calls)
  int32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "the workspace header is 256 bytes");

__host__ __device__ constexpr inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

__device__ __forceinline__ void raise_error(int32_t* flag, int32_t bits) {
  if (flag) atomicOr(flag, bits);
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float v) { return v; }
  static __device__ __forceinline__ float from_f32(float v) { return v; }
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
};
template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
  static constexpr int kPerVec = 8;
};

// 16-byte vector <-> 4 or 8 floats.
__device__ __forceinline__ void unpack16(const uint4& v, float* f, float*) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ void unpack16_bf16(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

}  // namespace stm
