// bf16 grouped SwiGLU GEMMs on the 5th-generation tensor cores (sm_100a).
//
// What is computed ("mstar.model.components.moe", SparseMoeBlock fused layout
// gate_up_proj [E,2I,H] and down_proj [E,H,I]; "Sparse MoE FFN for
// DFlash-family drafters", GroupedExperts / SparseMoE grouped GEMM with no host
// syncs; "feat: Phase 43", only routed segments are computed):
//   gate_up: h[p, n] = bf16( silu(A[p] . Wg[e,n]) * (A[p] . Wu[e,n]) )
//   down:    y[p, n] = scale(p) * (h[p] . Wd[e,n])          (kept in fp32)
// for every row p of every non-empty segment e of the device segment table.
//
// Design (one CTA per SM, persistent, warp-specialised, 192 threads):
//   warp 0      TMA producer: A tile [128 x 64] and B tile [256 x 64] bf16 per
//               k-step into a 4-stage ring of 128-byte-swizzled smem buffers.
//               For gate_up the B tile is the gate rows n0..n0+127 followed by
//               the up rows n0..n0+127 of expert e (two boxes of a 4-D tensor
//               map [E][2][I][H]), so accumulator columns j and 128+j pair up.
//   warp 1      TMEM allocator and MMA issuer: one thread issues
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16, fp32
//               accumulate) and commits each smem stage back to the producer.
//               Two TMEM accumulators (2 x 256 columns) let the epilogue of
//               one tile overlap the main loop of the next.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time, SwiGLU or
//               the routing-weight scale in fp32; h is packed to bf16 (it is
//               the next GEMM's operand), y stays fp32; 16-byte stores;
//               rows past the segment end belong to the next expert and are
//               dropped.
// Row tiles straddle nothing: each tile starts inside one segment; the TMA
// box may read rows of the next segment (or zero fill past the buffer) and
// the epilogue masks them.
//
// Every wait on an mbarrier is bounded (about a second of SM clocks). On a
// timeout the kernel raises MOE_DEVERR_WAIT_TIMEOUT in the workspace header,
// the other roles stop at their next wait, in-flight TMA copies and MMAs are
// drained with bounded waits, and TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace stm {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;          // 64 bf16 = 128 bytes = one swizzle row
constexpr int UMMA_N = 256;
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = UMMA_N * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * UMMA_N;
constexpr int NTHREADS = 192;
constexpr long long kWaitLimitCycles = 2000000000LL;

enum { MODE_GATE_UP = 0, MODE_DOWN = 1 };

struct Args {
  const int32_t* offsets;
  int32_t E;
  int32_t single_rows;
  int32_t N;        // output columns
  int32_t n_tiles;  // column tiles per row tile
  int32_t k_tiles;
  void* out;  // gate_up: bf16 h; down: fp32 y
  const float* row_scale;
  const int32_t* scale_idx;
  int32_t* err;
  int64_t rows_total;
};

struct __align__(8) Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int off[kMaxExperts + 1];
  int pre[kMaxExperts + 1];
};

constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Ctl);

// ---- PTX wrappers --------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete.
// Gives up when another role has aborted (unless draining) or after about a
// second of SM clocks, in which case it records the error and aborts.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, Ctl* ctl, int32_t* err, int site,
                                            bool draining) {
  const long long start = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (!draining && *reinterpret_cast<volatile int*>(&ctl->abort)) return false;
      if (clock64() - start > kWaitLimitCycles) {
        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
        if (err) {
          atomicOr(err, 2);
          atomicExch(err + 1, site);
        }
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Ctl* ctl, int32_t* err, int site,
                                          bool draining = false) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ctl, err, site, draining);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
      "%6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every previously issued tcgen05.mma of this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart (tcgen05 descriptor format:
// start>>4 in bits 0-13, LBO>>4 in 16-29, SBO>>4 in 32-45, version 1 in
// 46-47, layout type 2 = SWIZZLE_128B in 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B bf16
// (bits 7-9 and 10-12 = 1), both K-major, N>>3 in bits 17-22, M>>4 in 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(UMMA_N >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

struct TileCoord {
  int e, row0, row_end, n_idx;
};

__device__ __forceinline__ TileCoord decode_tile(const Ctl* ctl, int Eseg, int n_tiles, int tile) {
  TileCoord c;
  const int mt = tile / n_tiles;
  c.n_idx = tile - mt * n_tiles;
  c.e = find_segment(ctl->pre, Eseg, mt);
  c.row0 = ctl->off[c.e] + (mt - ctl->pre[c.e]) * BM;
  c.row_end = ctl->off[c.e + 1];
  return c;
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Eseg = args.offsets ? args.E : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], 128);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) warp_build_tile_table(args.offsets, args.E, args.single_rows, BM, ctl->off, ctl->pre, args.rows_total,
                                        args.err);
  if (warp == 1) tmem_alloc(&ctl->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total_tiles = ctl->pre[Eseg] * args.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;  // per stage: ever issued, parity of the last issue
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileCoord tc = decode_tile(ctl, Eseg, args.n_tiles, tile);
        for (int kt = 0; kt < args.k_tiles; ++kt) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, ctl, args.err, 1)) { ok = false; break; }
          uint8_t* sa = base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&ctl->full[stage], STAGE_BYTES);
          const int k0 = kt * BK;
          tma_load_2d(sa, &tmA, &ctl->full[stage], k0, tc.row0);
          if (MODE == MODE_GATE_UP) {
            const int n0 = tc.n_idx * 128;
            tma_load_4d(sb, &tmB, &ctl->full[stage], k0, n0, 0, tc.e);
            tma_load_4d(sb + B_BYTES / 2, &tmB, &ctl->full[stage], k0, n0, 1, tc.e);
          } else {
            tma_load_3d(sb, &tmB, &ctl->full[stage], k0, tc.n_idx * UMMA_N, tc.e);
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Drain: every copy this thread issued has landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (last_parity >> s) & 1u, ctl, args.err, 6, true);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, ctl, args.err, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * UMMA_N);
        for (int kt = 0; kt < args.k_tiles; ++kt) {
          if (!mbar_wait(&ctl->full[stage], phase, ctl, args.err, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + stage * STAGE_BYTES);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // advance K by 16 bf16 = 32 bytes inside the swizzled 128-byte row
            umma_bf16(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(kk * 2), kIdesc,
                      (kt > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Drain: all MMAs issued here are complete before TMEM is freed.
      umma_commit(&ctl->drain);
      mbar_wait(&ctl->drain, 0, ctl, args.err, 7, true);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord tc = decode_tile(ctl, Eseg, args.n_tiles, tile);
      if (!mbar_wait(&ctl->tfull[acc], acc_phase, ctl, args.err, 4)) break;
      tc_fence_after();
      const int row = tc.row0 + r;
      const bool valid = row < tc.row_end;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * UMMA_N);
      if (MODE == MODE_GATE_UP) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c * 32, g);
          tmem_ld32(tbase + 128 + c * 32, u);
          tmem_ld_wait();
          const int col0 = tc.n_idx * 128 + c * 32;
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.out) + (int64_t)row * args.N;
          if (valid) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              if (col0 + v * 8 < args.N) {
                float hv[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  hv[q] = silu_f32(__uint_as_float(g[v * 8 + q])) * __uint_as_float(u[v * 8 + q]);
                uint4 o;
                o.x = pack_bf16x2(hv[0], hv[1]);
                o.y = pack_bf16x2(hv[2], hv[3]);
                o.z = pack_bf16x2(hv[4], hv[5]);
                o.w = pack_bf16x2(hv[6], hv[7]);
                *reinterpret_cast<uint4*>(orow + col0 + v * 8) = o;
              }
            }
          }
        }
      } else {
        float sc = 1.f;
        if (valid && args.row_scale != nullptr) sc = args.row_scale[args.scale_idx ? args.scale_idx[row] : row];
#pragma unroll 1
        for (int c = 0; c < UMMA_N / 32; ++c) {
          uint32_t d[32];
          tmem_ld32(tbase + c * 32, d);
          tmem_ld_wait();
          const int col0 = tc.n_idx * UMMA_N + c * 32;
          float* orow = reinterpret_cast<float*>(args.out) + (int64_t)row * args.N;
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              if (col0 + v * 4 < args.N) {
                float4 o;
                o.x = sc * __uint_as_float(d[v * 4 + 0]);
                o.y = sc * __uint_as_float(d[v * 4 + 1]);
                o.z = sc * __uint_as_float(d[v * 4 + 2]);
                o.w = sc * __uint_as_float(d[v * 4 + 3]);
                *reinterpret_cast<float4*>(orow + col0 + v * 4) = o;
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---- host side -----------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  const uint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r =
      g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr), dims, strides_bytes,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

template <int MODE>
cudaError_t launch_tc(const Segments& sg, const CUtensorMap& tmA, const CUtensorMap& tmB, int64_t N, int64_t K,
                      void* out, const float* row_scale, const int32_t* scale_idx, int32_t* err, cudaStream_t s) {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(tc_grouped_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  Args a;
  a.offsets = sg.offsets;
  a.E = sg.E;
  a.single_rows = sg.single_rows;
  a.N = (int32_t)N;
  a.n_tiles = (int32_t)ceil_div(N, MODE == MODE_GATE_UP ? 128 : UMMA_N);
  a.k_tiles = (int32_t)ceil_div(K, BK);
  a.out = out;
  a.row_scale = row_scale;
  a.scale_idx = scale_idx;
  a.err = err;
  a.rows_total = sg.rows_total;
  const int64_t nseg = sg.offsets ? sg.E : 1;
  const int64_t max_tiles = (sg.rows_total / BM + nseg) * a.n_tiles;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_tiles));
  tc_grouped_gemm_kernel<MODE><<<grid, NTHREADS, kSmemBytes, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                              int64_t I, int64_t H, int32_t* err, cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)H, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)H * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_map(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // gate_up [E][2][I][H]: dim0 = H, dim1 = I (row within a half), dim2 = half, dim3 = expert
    const uint64_t dims[4] = {(uint64_t)H, (uint64_t)I, 2, (uint64_t)E_w};
    const uint64_t strides[3] = {(uint64_t)H * 2, (uint64_t)I * H * 2, (uint64_t)2 * I * H * 2};
    const uint32_t box[4] = {BK, 128, 1, 1};
    if (!make_map(&tmB, w_gate_up, 4, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_GATE_UP>(sg, tmA, tmB, I, H, h, nullptr, nullptr, err, s);
}

cudaError_t launch_tc_down(const Segments& sg, const void* h, const void* w_down, int64_t E_w, void* y,
                           const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                           cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)I, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)I * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_map(&tmA, h, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // down [E][H][I]: dim0 = I, dim1 = H, dim2 = expert
    const uint64_t dims[3] = {(uint64_t)I, (uint64_t)H, (uint64_t)E_w};
    const uint64_t strides[2] = {(uint64_t)I * 2, (uint64_t)H * I * 2};
    const uint32_t box[3] = {BK, UMMA_N, 1};
    if (!make_map(&tmB, w_down, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_DOWN>(sg, tmA, tmB, H, I, y, row_scale, scale_idx, err, s);
}

}  // namespace stm
