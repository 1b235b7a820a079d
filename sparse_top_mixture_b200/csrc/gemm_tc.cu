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
#include "tc_ptx.cuh"
#include "tc_epilogue.cuh"

namespace stm {

namespace {

using namespace tc;

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

// MODE_DOWN_KN: the down epilogue over B stored [E][K][N] (N innermost, read
// MN-major). MODE_WGRAD: both operands stored [K rows][M] and [K rows][N]
// (read MN-major), K running over each expert's row range.
// MODE_DOWN_EP: the down GEMM with each weighted row stored into its
// source's arena (expert parallelism; EpRet) instead of y.
enum { MODE_GATE_UP = 0, MODE_DOWN = 1, MODE_LOGITS = 2, MODE_WGRAD = 3, MODE_DOWN_KN = 4, MODE_DOWN_EP = 5 };
constexpr int MN_CHUNK_BYTES = BK * 64 * 2;  // 64 MN elements x 64 K rows of an MN-major operand

struct Args {
  const int32_t* offsets;
  int32_t E;
  int32_t single_rows;
  int32_t N;        // output columns
  int32_t n_tiles;  // column tiles per row tile
  int32_t k_tiles;  // BK-deep k-steps over the whole K
  int32_t k_splits; // independent partial sums along K (LOGITS only; else 1)
  int32_t kps;      // k-steps per split
  int64_t ldo;      // output row pitch in elements
  void* out;  // gate_up: bf16 h; down: fp32 y
  const float* row_scale;
  const int32_t* scale_idx;
  int32_t* err;
  int64_t rows_total;
  int32_t M;        // WGRAD: output rows per expert
  int32_t m_tiles;  // WGRAD: 128-row tiles of M
  int32_t n_mma;    // LOGITS: MMA N (the expert count rounded up to 16); else UMMA_N
  EpRet ep;         // DOWN_EP only
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

constexpr int EPI_BYTES = 4 * kStageFloatsPerWarp * 4;  // epilogue staging, one block per warp
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + sizeof(Ctl);

// Tiles of M=128, or M=64 for a segment's last 64 rows or fewer: the
// accumulator then occupies TMEM lanes 0-15 of each 32-lane sub-partition
// (tile row r -> lane (r % 16) + 32 * (r / 16)).

struct TileCoord {
  int e, row0, row_end, n_idx, kt0, kt1, split;
  bool m64;  // at most 64 rows of the segment left: M=64 MMA
};

// Tile index -> (row tile, column tile, k split); the split varies fastest.
// WGRAD: tile index -> (expert, row tile of M, column tile of N); the K range
// is the expert's padded segment [off[e], off[e+1]) (multiples of BK).
template <int MODE>
__device__ __forceinline__ TileCoord decode_tile(const Ctl* ctl, int Eseg, const Args& a, int tile) {
  TileCoord c;
  if constexpr (MODE == MODE_WGRAD) {
    const int per_e = a.m_tiles * a.n_tiles;
    c.e = tile / per_e;
    const int rest = tile - c.e * per_e;
    const int mt = rest / a.n_tiles;
    c.n_idx = rest - mt * a.n_tiles;
    c.split = 0;
    c.kt0 = ctl->off[c.e] / BK;
    c.kt1 = ctl->off[c.e + 1] / BK;
    c.row0 = mt * BM;
    c.row_end = a.M;
    c.m64 = c.row_end - c.row0 <= 64;
    return c;
  }
  c.split = tile % a.k_splits;
  const int rest = tile / a.k_splits;
  const int mt = rest / a.n_tiles;
  c.n_idx = rest - mt * a.n_tiles;
  c.kt0 = c.split * a.kps;
  c.kt1 = min(a.k_tiles, c.kt0 + a.kps);
  c.e = find_segment(ctl->pre, Eseg, mt);
  c.row0 = ctl->off[c.e] + (mt - ctl->pre[c.e]) * BM;
  c.row_end = ctl->off[c.e + 1];
  c.m64 = c.row_end - c.row0 <= 64;
  return c;
}

// WGRAD: the padded K offsets [E+1] into shared memory (one warp). They must
// be non-decreasing multiples of BK inside [0, rows_total] (the operands' K
// extent); otherwise every expert gets an empty range and MOE_DEVERR_BAD_EXPERT_ID
// is raised.
__device__ __forceinline__ void warp_load_k_ranges(const int32_t* __restrict__ offsets, int E, int64_t k_extent,
                                                   int* off, int32_t* err) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  for (int e = lane; e <= E; e += 32) {
    const int v = offsets[e];
    off[e] = v;
    bad |= v < 0 || (v % BK) != 0 || (int64_t)v > k_extent || (e > 0 && offsets[e - 1] > v);
  }
  if (__any_sync(0xffffffffu, bad)) {
    __syncwarp();
    if (lane == 0) raise_error(err, 1);
    for (int e = lane; e <= E; e += 32) off[e] = 0;
  }
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi_stage = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES);
  Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * STAGE_BYTES + EPI_BYTES);
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
  if (warp == 2) {
    if constexpr (MODE == MODE_WGRAD)
      warp_load_k_ranges(args.offsets, args.E, args.rows_total, ctl->off, args.err);
    else
      warp_build_tile_table(args.offsets, args.E, args.single_rows, BM, ctl->off, ctl->pre, args.rows_total,
                            args.err);
  }
  if (warp == 1) tmem_alloc(&ctl->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total_tiles = MODE == MODE_WGRAD ? args.E * args.m_tiles * args.n_tiles
                                             : ctl->pre[Eseg] * args.n_tiles * args.k_splits;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;  // per stage: ever issued, parity of the last issue
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        const TileCoord tc = decode_tile<MODE>(ctl, Eseg, args, tile);
        for (int kt = tc.kt0; kt < tc.kt1; ++kt) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, args.err, 1)) { ok = false; break; }
          uint8_t* sa = base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          // the router's B box has only n_mma rows (its N is the expert count)
          mbar_arrive_expect_tx(&ctl->full[stage],
                                MODE == MODE_LOGITS ? (uint32_t)(A_BYTES + args.n_mma * BK * 2) : STAGE_BYTES);
          const int k0 = kt * BK;
          if (MODE == MODE_WGRAD) {
            // 64-column chunks of the [K rows][M] and [K rows][N] operands
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)
              tma_load_2d(sa + j * MN_CHUNK_BYTES, &tmA, &ctl->full[stage], tc.row0 + 64 * j, k0);
#pragma unroll
            for (int j = 0; j < UMMA_N / 64; ++j)
              tma_load_2d(sb + j * MN_CHUNK_BYTES, &tmB, &ctl->full[stage], tc.n_idx * UMMA_N + 64 * j, k0);
          } else {
            tma_load_2d(sa, &tmA, &ctl->full[stage], k0, tc.row0);
            if (MODE == MODE_GATE_UP) {
              const int n0 = tc.n_idx * 128;  // gate rows, then the matching up rows
              tma_load_4d(sb, &tmB, &ctl->full[stage], k0, n0, 0, tc.e);
              tma_load_4d(sb + B_BYTES / 2, &tmB, &ctl->full[stage], k0, n0, 1, tc.e);
            } else if (MODE == MODE_DOWN_KN) {
#pragma unroll
              for (int j = 0; j < UMMA_N / 64; ++j)
                tma_load_3d(sb + j * MN_CHUNK_BYTES, &tmB, &ctl->full[stage], tc.n_idx * UMMA_N + 64 * j, k0, tc.e);
            } else {
              tma_load_3d(sb, &tmB, &ctl->full[stage], k0, tc.n_idx * UMMA_N, MODE == MODE_LOGITS ? 0 : tc.e);
            }
          }
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Drain: every copy this thread issued has landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (last_parity >> s) & 1u, &ctl->abort, args.err, 6, true);
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
        const TileCoord tc = decode_tile<MODE>(ctl, Eseg, args, tile);
        if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, args.err, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * UMMA_N);
        constexpr bool a_mn = MODE == MODE_WGRAD;
        constexpr bool b_mn = MODE == MODE_WGRAD || MODE == MODE_DOWN_KN;
        const uint32_t idesc = MODE == MODE_LOGITS ? make_idesc(tc.m64 ? 64 : 128, args.n_mma)
                                                   : make_idesc_mn(tc.m64 ? 64 : 128, UMMA_N, a_mn, b_mn);
        for (int kt = tc.kt0; kt < tc.kt1; ++kt) {
          if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, args.err, 3)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + stage * STAGE_BYTES);
          const uint64_t adesc = a_mn ? sw128_mn_desc(sa, MN_CHUNK_BYTES) : sw128_desc(sa);
          const uint64_t bdesc = b_mn ? sw128_mn_desc(sa + A_BYTES, MN_CHUNK_BYTES) : sw128_desc(sa + A_BYTES);
          // K by 16: 32 bytes along a K-major 128-byte row, or 16 rows (2048
          // bytes) of an MN-major chunk (descriptor units of 16 bytes)
          constexpr uint64_t a_step = a_mn ? 128 : 2;
          constexpr uint64_t b_step = b_mn ? 128 : 2;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            umma_bf16(d_tmem, adesc + a_step * kk, bdesc + b_step * kk, idesc, (kt > tc.kt0 || kk > 0) ? 1u : 0u);
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
      mbar_wait(&ctl->drain, 0, &ctl->abort, args.err, 7, true);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord tc = decode_tile<MODE>(ctl, Eseg, args, tile);
      if (!mbar_wait(&ctl->tfull[acc], acc_phase, &ctl->abort, args.err, 4)) break;
      tc_fence_after();
      // this warp's rows: 32 consecutive (16 for an M=64 tile), lane = row
      const int rows_w = tc.m64 ? 16 : 32;
      const int row_w0 = tc.row0 + quarter * rows_w;
      const int nrows = max(0, min(rows_w, tc.row_end - row_w0));
      const int row = row_w0 + lane;
      const bool valid = lane < nrows;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * UMMA_N);
      float* stage = epi_stage + (warp - 2) * kStageFloatsPerWarp;
      if (MODE == MODE_GATE_UP) {
        epilogue_swiglu(tbase, 0, 128, 4, reinterpret_cast<__nv_bfloat16*>(args.out) + (int64_t)row_w0 * args.ldo,
                        args.ldo, nrows, tc.n_idx * 128, args.N, lane);
      } else if (MODE == MODE_WGRAD) {
        // dW[e] rows row_w0.. of M, fp32, row pitch N; an expert without rows
        // (empty K range, no MMA issued) gets zeros, not the stale accumulator
        float* orow0 = reinterpret_cast<float*>(args.out) + (int64_t)tc.e * args.M * args.ldo +
                       (int64_t)row_w0 * args.ldo;
        if (tc.kt1 > tc.kt0) {
          epilogue_scale_f32(tbase, UMMA_N / 32, 1.f, stage, orow0, args.ldo, nrows, tc.n_idx * UMMA_N, args.N,
                             lane);
        } else {
          float z[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) z[q] = 0.f;
#pragma unroll 1
          for (int c = 0; c < UMMA_N / 32; ++c) {
            const int cb = tc.n_idx * UMMA_N + c * 32;
            if (cb >= args.N || nrows <= 0) break;  // warp-uniform
            store_block_f32(z, stage, orow0 + cb, args.ldo, nrows, args.N - cb, lane);
          }
        }
      } else if (MODE == MODE_DOWN || MODE == MODE_DOWN_KN) {
        float sc = 1.f;
        if (valid && args.row_scale != nullptr) sc = args.row_scale[args.scale_idx ? args.scale_idx[row] : row];
        epilogue_scale_f32(tbase, UMMA_N / 32, sc, stage,
                           reinterpret_cast<float*>(args.out) + (int64_t)row_w0 * args.ldo, args.ldo, nrows,
                           tc.n_idx * UMMA_N, args.N, lane);
      } else if (MODE == MODE_DOWN_EP) {
        // this lane's row came from slot j = s*C + i: to source s's y, row yoff[s] + i
        float sc = 1.f;
        float* rp = nullptr;
        if (valid) {
          const int64_t j = args.scale_idx[row];
          sc = args.row_scale[j];
          const int64_t src = j / args.ep.C;
          rp = reinterpret_cast<float*>(args.ep.arenas[src] + args.ep.y_off) +
               (args.ep.yoff[src] + (j - src * args.ep.C)) * args.N;
        }
        epilogue_scale_f32_rows(tbase, UMMA_N / 32, sc, stage, rp, nrows, tc.n_idx * UMMA_N, args.N, lane);
      } else {
        // router logits: fp32 partial sum of this k split; the row pitch is a
        // multiple of 4 floats, columns past N are not written.
        float* orow = reinterpret_cast<float*>(args.out) + (int64_t)tc.split * args.rows_total * args.ldo +
                      (int64_t)row * args.ldo;
#pragma unroll 1
        for (int c = 0; c < UMMA_N / 32; ++c) {
          const int col0 = tc.n_idx * UMMA_N + c * 32;
          if (col0 >= args.N) break;  // warp-uniform
          uint32_t d[32];
          tmem_ld32(tbase + c * 32, d);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const int cv = col0 + v * 4;
              if (cv + 3 < args.N) {
                *reinterpret_cast<float4*>(orow + cv) =
                    make_float4(__uint_as_float(d[v * 4 + 0]), __uint_as_float(d[v * 4 + 1]),
                                __uint_as_float(d[v * 4 + 2]), __uint_as_float(d[v * 4 + 3]));
              } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  if (cv + q < args.N) orow[cv + q] = __uint_as_float(d[v * 4 + q]);
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
    if (MODE == MODE_DOWN_EP) __threadfence_system();  // the rows stored to peers, before any flag
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int MODE>
cudaError_t launch_tc(const Segments& sg, const CUtensorMap& tmA, const CUtensorMap& tmB, int64_t N, int64_t K,
                      void* out, int64_t ldo, const float* row_scale, const int32_t* scale_idx, int32_t* err,
                      cudaStream_t s, int k_splits = 1, const EpRet* ep = nullptr) {
  static std::once_flag attr_once[kSmemAttrDevices];  // one set per kernel instance (MODE)
  static cudaError_t attr_status[kSmemAttrDevices];
  const void* kernel = reinterpret_cast<const void*>(tc_grouped_gemm_kernel<MODE>);
  const cudaError_t attr_err = set_max_dynamic_smem_once(kernel, (int)kSmemBytes, attr_once, attr_status);
  if (attr_err != cudaSuccess) return attr_err;
  Args a{};
  a.offsets = sg.offsets;
  a.E = sg.E;
  a.single_rows = sg.single_rows;
  a.N = (int32_t)N;
  a.n_tiles = (int32_t)ceil_div(N, MODE == MODE_GATE_UP ? 128 : UMMA_N);
  a.k_tiles = (int32_t)ceil_div(K, BK);
  a.k_splits = std::max(1, k_splits);
  a.kps = (int32_t)ceil_div(a.k_tiles, a.k_splits);
  a.ldo = ldo;
  a.out = out;
  a.row_scale = row_scale;
  a.scale_idx = scale_idx;
  a.err = err;
  a.rows_total = sg.rows_total;
  a.M = 0;
  a.m_tiles = 0;
  a.n_mma = MODE == MODE_LOGITS ? (int32_t)std::min<int64_t>(UMMA_N, round_up(N, 16)) : UMMA_N;
  if (ep != nullptr) a.ep = *ep;
  const int64_t nseg = sg.offsets ? sg.E : 1;
  const int64_t max_tiles = (sg.rows_total / BM + nseg) * a.n_tiles * a.k_splits;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), max_tiles));
  tc_grouped_gemm_kernel<MODE><<<grid, NTHREADS, kSmemBytes, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

}  // namespace

// Weight gradients: out[e][m][n] = sum over rows k in [koff[e], koff[e+1])
// of A[k][m] * B[k][n]. A [rows][lda] and B [rows][ldb] are bf16 row-major
// (M and N used columns, read MN-major); rows at or past `rows` read as zero,
// so a K range may run past the last row. koff: E+1 non-decreasing multiples
// of 64 within [0, k_extent]. out fp32 [E][M][N]; an expert with an empty
// range gets zeros.
cudaError_t launch_wgrad(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t rows, const int32_t* koff,
                         int64_t k_extent, int E, int64_t M, int64_t N, float* out, int32_t* err, cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  static std::once_flag attr_once[kSmemAttrDevices];
  static cudaError_t attr_status[kSmemAttrDevices];
  const void* kernel = reinterpret_cast<const void*>(tc_grouped_gemm_kernel<MODE_WGRAD>);
  const cudaError_t attr_err = set_max_dynamic_smem_once(kernel, (int)kSmemBytes, attr_once, attr_status);
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)M, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)lda * 2};
    const uint32_t box[2] = {64, BK};
    if (!make_tensor_map_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)ldb * 2};
    const uint32_t box[2] = {64, BK};
    if (!make_tensor_map_bf16(&tmB, B, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  Args a{};
  a.offsets = koff;
  a.E = E;
  a.N = (int32_t)N;
  a.n_tiles = (int32_t)ceil_div(N, UMMA_N);
  a.k_splits = 1;
  a.ldo = N;
  a.out = out;
  a.err = err;
  a.rows_total = k_extent;  // bound of the K ranges
  a.M = (int32_t)M;
  a.m_tiles = (int32_t)ceil_div(M, BM);
  a.n_mma = UMMA_N;
  const int64_t tiles = (int64_t)E * a.m_tiles * a.n_tiles;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms(), tiles));
  tc_grouped_gemm_kernel<MODE_WGRAD><<<grid, NTHREADS, kSmemBytes, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}


// ---- host side -----------------------------------------------------------

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

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

bool make_tensor_map_bf16(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box) {
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

// Launches one grouped GEMM takes.
int tc_gemm_launches(const Segments&) { return 1; }

int tc_gemm_variant(const Segments& sg, bool) {
  // CTA pairs halve the operand bytes per SM (and the TMA loads in flight
  // per unit of MMA work) but work on 256-row tiles: both GEMMs gain from
  // segments of about 192 rows on.
  const int64_t nseg = sg.offsets ? sg.E : 1;
  return sg.rows_total >= 192 * nseg ? 2 : 1;
}

cudaError_t launch_tc_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                              int64_t I, int64_t H, int32_t* err, cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  if (tc_gemm_variant(sg, false) == 2) return launch_tc2_gate_up(sg, A, w_gate_up, E_w, h, I, H, err, num_sms(), s);
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)H, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)H * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // gate_up [E][2][I][H]: dim0 = H, dim1 = I (row within a half), dim2 = half, dim3 = expert
    const uint64_t dims[4] = {(uint64_t)H, (uint64_t)I, 2, (uint64_t)E_w};
    const uint64_t strides[3] = {(uint64_t)H * 2, (uint64_t)I * H * 2, (uint64_t)2 * I * H * 2};
    const uint32_t box[4] = {BK, 128, 1, 1};
    if (!make_tensor_map_bf16(&tmB, w_gate_up, 4, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_GATE_UP>(sg, tmA, tmB, I, H, h, I, nullptr, nullptr, err, s);
}

cudaError_t launch_tc_down(const Segments& sg, const void* h, const void* w_down, int64_t E_w, void* y,
                           const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                           cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  if (tc_gemm_variant(sg, true) == 2)
    return launch_tc2_down(sg, h, w_down, E_w, y, row_scale, scale_idx, H, I, err, num_sms(), s);
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)I, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)I * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&tmA, h, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // down [E][H][I]: dim0 = I, dim1 = H, dim2 = expert
    const uint64_t dims[3] = {(uint64_t)I, (uint64_t)H, (uint64_t)E_w};
    const uint64_t strides[2] = {(uint64_t)I * 2, (uint64_t)H * I * 2};
    const uint32_t box[3] = {BK, UMMA_N, 1};
    if (!make_tensor_map_bf16(&tmB, w_down, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_DOWN>(sg, tmA, tmB, H, I, y, H, row_scale, scale_idx, err, s);
}

cudaError_t launch_tc_down_kn(const Segments& sg, const void* A, int64_t lda, const void* w_kn, int64_t E_w, void* y,
                              const float* row_scale, const int32_t* scale_idx, int64_t N, int64_t K, int32_t* err,
                              cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  if (tc_gemm_variant(sg, true) == 2)
    return launch_tc2_down_kn(sg, A, lda, w_kn, E_w, y, row_scale, scale_idx, N, K, err, num_sms(), s);
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)lda * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&tmA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // B [E][K][N]: dim0 = N, dim1 = K, dim2 = expert; 64-column chunks of BK rows
    const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E_w};
    const uint64_t strides[2] = {(uint64_t)N * 2, (uint64_t)K * N * 2};
    const uint32_t box[3] = {64, BK, 1};
    if (!make_tensor_map_bf16(&tmB, w_kn, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_DOWN_KN>(sg, tmA, tmB, N, K, y, N, row_scale, scale_idx, err, s);
}

cudaError_t launch_tc_down_ep(const Segments& sg, const void* h, const void* w_down, int64_t E_w,
                              const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, const EpRet& ep,
                              int32_t* err, cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  if (row_scale == nullptr || scale_idx == nullptr) return cudaErrorInvalidValue;
  if (tc_gemm_variant(sg, true) == 2)
    return launch_tc2_down_ep(sg, h, w_down, E_w, row_scale, scale_idx, H, I, ep, err, num_sms(), s);
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)I, (uint64_t)sg.rows_total};
    const uint64_t strides[1] = {(uint64_t)I * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&tmA, h, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)I, (uint64_t)H, (uint64_t)E_w};
    const uint64_t strides[2] = {(uint64_t)I * 2, (uint64_t)H * I * 2};
    const uint32_t box[3] = {BK, UMMA_N, 1};
    if (!make_tensor_map_bf16(&tmB, w_down, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  return launch_tc<MODE_DOWN_EP>(sg, tmA, tmB, H, I, nullptr, H, row_scale, scale_idx, err, s, 1, &ep);
}

int tc_router_splits(int64_t T, int64_t H, int64_t E) {
  const int64_t k_tiles = ceil_div(H, BK);
  const int64_t tiles_mn = ceil_div(T, BM) * ceil_div(E, UMMA_N);
  // At most 16 partials: the top-k kernel adds them serially per logit.
  int64_t splits = std::max<int64_t>(1, std::min<int64_t>({k_tiles, (int64_t)16, 148 / std::max<int64_t>(1, tiles_mn)}));
  const int64_t kps = ceil_div(k_tiles, splits);
  return (int)ceil_div(k_tiles, kps);  // every split gets at least one k-step
}

cudaError_t launch_tc_logits(const void* x, const void* gate_w, int64_t T, int64_t H, int64_t E, float* partial,
                             int64_t ldo, int splits, int32_t* err, cudaStream_t s) {
  if (!get_encode()) return cudaErrorNotSupported;
  CUtensorMap tmA, tmB;
  {
    const uint64_t dims[2] = {(uint64_t)H, (uint64_t)T};
    const uint64_t strides[1] = {(uint64_t)H * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_tensor_map_bf16(&tmA, x, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    // N of the router's MMA: the expert count rounded up to 16 (at most 256);
    // the B box has that many rows (zero fill past E)
    const uint64_t dims[3] = {(uint64_t)H, (uint64_t)E, 1};
    const uint64_t strides[2] = {(uint64_t)H * 2, (uint64_t)E * H * 2};
    const uint32_t box[3] = {BK, (uint32_t)std::min<int64_t>(UMMA_N, round_up(E, 16)), 1};
    if (!make_tensor_map_bf16(&tmB, gate_w, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  Segments sg{nullptr, 1, (int32_t)T, T};
  return launch_tc<MODE_LOGITS>(sg, tmA, tmB, E, H, partial, ldo, nullptr, nullptr, err, s, splits);
}

}  // namespace stm
