// bf16 grouped SwiGLU GEMMs on CTA pairs (tcgen05.mma.cta_group::2).
//
// Same computation as the one-CTA kernel in gemm_tc.cu (gate_up with the
// SwiGLU epilogue, down with the routing-weight epilogue, over the device
// segment table; "mstar.model.components.moe", SparseMoeBlock fused layout;
// "Sparse MoE FFN for DFlash-family drafters", grouped GEMM with no host
// syncs), but each tile is 256 rows x 256 accumulator columns computed by two
// CTAs on two SMs of a cluster:
//   - each CTA loads its own 128 rows of A and its own half of B (128 of the
//     256 B rows: for gate_up the leader loads the gate rows n0..n0+127 and
//     the peer the matching up rows), so a k-step moves 32 KB per CTA instead
//     of 48 KB for the same MMA work per SM and the stage ring is 6 deep;
//   - both CTAs' TMA loads complete on the leader's full barrier; the leader
//     posts the pair's transaction bytes and issues the M=256 MMA, whose
//     commits arrive on the empty / accumulator barriers of both CTAs;
//   - each CTA's epilogue drains its own TMEM rows and arrives on the
//     leader's accumulator-empty barrier.
// No TMA multicast is used: every CTA fetches its own tiles.
// The kernel takes the number of 64-element K atoms per stage as a template
// parameter (two atoms: a 3-D tensor-map view [K/64][rows][64] whose box
// spans both); it is launched with one (see kAtomsPerStage).
//
// Used when segments average at least 192 rows. A row tile is 256 rows of one
// segment. A tile with at most 128 rows left (a segment's tail) runs with the
// operands swapped: the tile's weight rows are the M=256 operand (128 per
// CTA, loaded as for a full tile) and its r rows the N operand, N = r rounded
// up to 16 (each CTA supplies N/2 of them from a 64-row load), so the MMA
// costs N/256 of a full tile's instead of the whole of it. TMEM lane is then
// the output feature and column the row. For gate_up each CTA's 128 weight
// rows are 4 groups of [16 gate rows | the matching 16 up rows] (one 5-D
// load), so that every epilogue warp holds a gate value and its up value in
// lanes L and L + 16 and combines them with one shuffle. Modes that read B
// MN-major keep the unswapped tail: an M=128 pair MMA, 64 rows per CTA, whose
// accumulator holds output columns 0..127 in TMEM lanes 0-63 and 128..255 in
// lanes 64-127. Handing tails to a separate launch was measured slower: the
// tail experts' weights had left L2 by then.
// All waits are bounded as in the one-CTA kernel; a cluster barrier before
// TMEM is freed guarantees no remote arrive or MMA still targets a CTA that
// is about to exit.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "tc_epilogue.cuh"
#include "tc_ptx.cuh"
#include "tiles.cuh"

namespace stm {

namespace {

using namespace tc;

constexpr int BM2 = 256;         // rows per pair tile
constexpr int HALF = 128;        // rows of A (and of B) per CTA
constexpr int BK = 64;           // K elements per atom (128 bytes: one swizzle row)
constexpr int ATOM_BYTES = HALF * BK * 2;  // one 128-row x 64-element K atom
constexpr int UMMA_N = 256;
constexpr int UMMA_K = 16;
constexpr int RING_BYTES = 6 * 2 * ATOM_BYTES;  // 192 KB of stages per CTA
constexpr int MAX_STAGES = 6;
constexpr int TMEM_COLS = 2 * UMMA_N;
constexpr int NTHREADS = 192;
constexpr uint32_t kIdesc256 = make_idesc(256, UMMA_N);
constexpr uint32_t kIdesc128 = make_idesc(128, UMMA_N);  // unswapped tails: 64 rows per CTA
constexpr int SWAP_ROWS = HALF / 2;                     // tail rows loaded per CTA (a swapped tile's N <= 128)
constexpr int SWAP_ROW_BYTES = SWAP_ROWS * BK * 2;       // 8 KB per K atom

// KA K atoms per stage: stage = KA atoms of A then KA atoms of B.
template <int KA>
struct Ring {
  static constexpr int A_BYTES = KA * ATOM_BYTES;
  static constexpr int B_BYTES = KA * ATOM_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = RING_BYTES / STAGE_BYTES;
  static_assert(STAGES >= 2 && STAGES <= MAX_STAGES, "ring depth");
};

// MODE_DOWN_KN: the down epilogue over B stored [E][K][N] (N innermost),
// read MN-major: each CTA's 128 B columns are two 64-column chunks of 64 K
// rows (one K atom per stage only).
// MODE_DOWN_EP: the down GEMM with each weighted row stored into its
// source's arena (expert parallelism; EpRet) instead of y.
enum { MODE_GATE_UP = 0, MODE_DOWN = 1, MODE_DOWN_KN = 2, MODE_DOWN_EP = 3 };
constexpr int MN_CHUNK_BYTES = 64 * BK * 2;

struct Args2 {
  const int32_t* offsets;
  int32_t E;
  int32_t single_rows;
  int32_t N;
  int32_t n_tiles;
  int32_t k_tiles;  // stages (KA atoms each) over the whole K
  int64_t ldo;
  void* out;
  const float* row_scale;
  const int32_t* scale_idx;
  int32_t* err;
  int64_t rows_total;
  int32_t swap_tails;  // tails run swapped (K-major B only, one K atom per stage)
  EpRet ep;            // MODE_DOWN_EP only
};

struct __align__(8) Ctl2 {
  uint64_t full[MAX_STAGES];   // leader only: both CTAs' bytes of a stage landed
  uint64_t empty[MAX_STAGES];  // both: the pair MMA finished reading a stage
  uint64_t tfull[2];           // both: accumulator ready
  uint64_t tempty[2];          // leader only: both CTAs' epilogues drained it
  uint64_t drain;              // both: every pair MMA complete
  uint32_t tmem_base;
  int abort;
  int off[kMaxExperts + 1];
  int pre[kMaxExperts + 1];
};

// Shared memory: the stage ring (its base 1024-byte aligned: the 128-byte
// swizzle repeats every 1024 bytes), the epilogue staging blocks (one per
// epilogue warp; down only: gate_up stores its bf16 rows directly), then
// Ctl2. down declares the dynamic shared memory 1024-byte aligned and checks
// it (doing nothing if it is not); gate_up requests 1 KB more and rounds its
// base up. Each variant measured 3-9% faster for its GEMM than the other
// layout (the same code otherwise). gate_up's ~200 KB leave room on the SM
// for the dispatch kernels that run beside a shared expert's GEMM.
template <int MODE>
constexpr int epi_bytes2() {
  return MODE != MODE_GATE_UP ? 4 * kStageFloatsPerWarp * 4 : 0;
}
template <int MODE>
constexpr size_t smem_bytes2() {
  return (MODE == MODE_GATE_UP ? 1024 : 0) + (size_t)RING_BYTES + epi_bytes2<MODE>() + sizeof(Ctl2);
}
static_assert(smem_bytes2<MODE_GATE_UP>() <= 232448, "dynamic shared memory above the 227 KB per-block limit");
static_assert(smem_bytes2<MODE_DOWN>() <= 232448, "dynamic shared memory above the 227 KB per-block limit");
static_assert(smem_bytes2<MODE_DOWN_KN>() <= 232448, "dynamic shared memory above the 227 KB per-block limit");
static_assert(smem_bytes2<MODE_DOWN_EP>() <= 232448, "dynamic shared memory above the 227 KB per-block limit");

struct Tile2 {
  int e, row0, row_end, n_idx;
  bool tail;       // at most 128 rows left
  bool swap;       // a tail run swapped: ncols = its rows rounded up to 16
  int ncols;
  int rows_cta;    // unswapped: rows per CTA, 128, or 64 for a tail
  bool peer_rows;  // unswapped: the peer's rows hold any row of the segment
};

__device__ __forceinline__ Tile2 decode_tile2(const Ctl2* ctl, int Eseg, int n_tiles, int tile, bool swap_tails) {
  Tile2 t;
  const int mt = tile / n_tiles;
  t.n_idx = tile - mt * n_tiles;
  t.e = find_segment(ctl->pre, Eseg, mt);
  t.row0 = ctl->off[t.e] + (mt - ctl->pre[t.e]) * BM2;
  t.row_end = ctl->off[t.e + 1];
  t.tail = t.row_end - t.row0 <= HALF;
  t.swap = swap_tails && t.tail;
  t.ncols = (t.row_end - t.row0 + 15) & ~15;
  t.rows_cta = t.tail ? HALF / 2 : HALF;
  t.peer_rows = t.row0 + t.rows_cta < t.row_end;
  return t;
}

template <int MODE, int KA>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    tc2_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA64,
                            const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB64,
                            const Args2 args) {
  constexpr int STAGES = Ring<KA>::STAGES;
  constexpr int A_BYTES = Ring<KA>::A_BYTES;
  constexpr int B_BYTES = Ring<KA>::B_BYTES;
  constexpr int STAGE_BYTES = Ring<KA>::STAGE_BYTES;
  static_assert(MODE != MODE_DOWN_KN || KA == 1, "MN-major B takes one K atom per stage");
  const bool swap_tails = KA == 1 && MODE != MODE_DOWN_KN && args.swap_tails != 0;
  uint8_t* base;
  if constexpr (MODE == MODE_GATE_UP) {
    extern __shared__ uint8_t smem_gu[];
    base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_gu) + 1023) & ~uintptr_t(1023));
  } else {
    extern __shared__ __align__(1024) uint8_t smem_dn[];
    // The same shared-window offset in every CTA of the grid: all of them
    // return here, or none.
    if ((smem_u32(smem_dn) & 1023u) != 0) {
      if (threadIdx.x == 0) raise_error(args.err, MOE_DEVERR_SMEM_LAYOUT);
      return;
    }
    base = smem_dn;
  }
  float* epi_stage = reinterpret_cast<float*>(base + RING_BYTES);
  Ctl2* ctl = reinterpret_cast<Ctl2*>(base + RING_BYTES + epi_bytes2<MODE>());
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int Eseg = args.offsets ? args.E : 1;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl->tfull[a], 1);
      mbar_init(&ctl->tempty[a], 8);  // one arrive per epilogue warp, 4 warps x 2 CTAs
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 2)
    warp_build_tile_table(args.offsets, args.E, args.single_rows, BM2, ctl->off, ctl->pre, args.rows_total,
                          args.err);
  if (warp == 1) tmem_alloc2(&ctl->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int total_tiles = ctl->pre[Eseg] * args.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_parity = 0;
      for (int tile = pair; tile < total_tiles; tile += npairs) {
        const Tile2 tc = decode_tile2(ctl, Eseg, args.n_tiles, tile, swap_tails);
        bool ok = true;
        for (int kt = 0; kt < args.k_tiles; ++kt) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, args.err, 11)) { ok = false; break; }
          uint8_t* sa = base + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          const uint32_t full_leader = mapa_shared(smem_u32(&ctl->full[stage]), 0);
          if (leader)
            mbar_arrive_expect_tx(&ctl->full[stage],
                                  tc.swap ? (uint32_t)(2 * B_BYTES + 2 * SWAP_ROW_BYTES)
                                          : (uint32_t)(2 * B_BYTES + A_BYTES + (tc.peer_rows ? A_BYTES : 0)));
          // K coordinates: with two atoms per stage the views are [atoms][rows][64]
          // and the stage starts at atom kt*2; with one, K is the innermost
          // dimension and the stage starts at element kt*64.
          const int ka = kt * KA;
          const int cx = KA == 2 ? 0 : ka * BK;
          const int cz = KA == 2 ? ka : 0;
          if (tc.swap) {
            // this CTA's half of the N columns: rows row0 + rank*ncols/2 on
            // (64 loaded, the first ncols/2 read by the MMA)
            tma2_load_3d(sa, &tmA64, full_leader, cx, tc.row0 + (int)rank * (tc.ncols / 2), cz);
          } else if (leader || tc.peer_rows) {
            tma2_load_3d(sa, &tmA, full_leader, cx, tc.row0 + (int)rank * tc.rows_cta, cz);
          }
          if (MODE == MODE_GATE_UP) {
            if (tc.swap) {
              // features n_idx*128 + rank*64 .. +63 as 4 x [16 gate rows | 16 up rows]
              tma2_load_5d(sb, &tmB64, full_leader, cx, 0, 0, (tc.n_idx * 128 + (int)rank * 64) / 16, tc.e);
            } else if (!tc.tail) {
              // leader: gate rows n0..n0+127; peer: the matching up rows
              tma2_load_5d(sb, &tmB, full_leader, cx, tc.n_idx * 128, cz, (int)rank, tc.e);
            } else {
              // each CTA, per atom: 64 gate rows then the matching 64 up rows
              const int n0 = tc.n_idx * 128 + (int)rank * 64;
#pragma unroll
              for (int a = 0; a < KA; ++a) {
                tma2_load_5d(sb + a * ATOM_BYTES, &tmB64, full_leader, cx, n0, cz + a, 0, tc.e);
                tma2_load_5d(sb + a * ATOM_BYTES + ATOM_BYTES / 2, &tmB64, full_leader, cx, n0, cz + a, 1, tc.e);
              }
            }
          } else if (MODE == MODE_DOWN_KN) {
            const int n0 = tc.n_idx * UMMA_N + (int)rank * HALF;
            tma2_load_3d(sb, &tmB, full_leader, n0, ka * BK, tc.e);
            tma2_load_3d(sb + MN_CHUNK_BYTES, &tmB, full_leader, n0 + 64, ka * BK, tc.e);
          } else {
            tma2_load_4d(sb, &tmB, full_leader, cx, tc.n_idx * UMMA_N + (int)rank * HALF, cz, tc.e);
          }
          if (leader) {
            issued |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // Drain (leader): the full barriers count both CTAs' bytes, so every
      // copy of the pair has landed once they complete.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (last_parity >> s) & 1u, &ctl->abort, args.err, 16, true);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (leader) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += npairs) {
        const Tile2 tc = decode_tile2(ctl, Eseg, args.n_tiles, tile, swap_tails);
        constexpr uint32_t b_mn = MODE == MODE_DOWN_KN ? 1u << 16 : 0u;  // B MN-major
        const uint32_t idesc = tc.swap ? make_idesc(256, tc.ncols) : (tc.tail ? kIdesc128 : kIdesc256) | b_mn;
        if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, args.err, 12)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * UMMA_N);
        for (int kt = 0; kt < args.k_tiles; ++kt) {
          if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, args.err, 13)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + stage * STAGE_BYTES);
#pragma unroll
          for (int a = 0; a < KA; ++a) {
            const uint64_t adesc = sw128_desc(sa + a * ATOM_BYTES);
            const uint64_t bdesc = MODE == MODE_DOWN_KN ? sw128_mn_desc(sa + A_BYTES, MN_CHUNK_BYTES)
                                                        : sw128_desc(sa + A_BYTES + a * ATOM_BYTES);
            // K by 16: 32 bytes along a K-major row; 16 rows (2048 bytes) of an
            // MN-major chunk (descriptor units of 16 bytes)
            constexpr uint64_t b_step = MODE == MODE_DOWN_KN ? 128 : 2;
            if (tc.swap) {
              // the stage's weight rows (K-major) as the M operand, its rows of A as the N operand
#pragma unroll
              for (int kk = 0; kk < BK / UMMA_K; ++kk)
                umma2_bf16(d_tmem, bdesc + (uint64_t)(kk * 2), adesc + (uint64_t)(kk * 2), idesc,
                           (kt > 0 || a > 0 || kk > 0) ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < BK / UMMA_K; ++kk)
                umma2_bf16(d_tmem, adesc + (uint64_t)(kk * 2), bdesc + b_step * kk, idesc,
                           (kt > 0 || a > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma2_commit_mc(&ctl->empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_mc(&ctl->tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma2_commit_mc(&ctl->drain, 0x3);
      mbar_wait(&ctl->drain, 0, &ctl->abort, args.err, 17, true);
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    const int quarter = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&ctl->tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&ctl->tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs) {
      const Tile2 tc = decode_tile2(ctl, Eseg, args.n_tiles, tile, swap_tails);
      if (!mbar_wait(&ctl->tfull[acc], acc_phase, &ctl->abort, args.err, 14)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * UMMA_N);
      if (tc.swap) {
        // lane = this CTA's weight row 32*quarter + lane, column = row of the tile
        const int nrows = tc.row_end - tc.row0;
        if constexpr (MODE == MODE_GATE_UP) {
          __nv_bfloat16* orow0 = reinterpret_cast<__nv_bfloat16*>(args.out) + (int64_t)tc.row0 * args.ldo;
          epilogue_swiglu_swapped(tbase, tc.ncols, orow0, args.ldo, nrows,
                                  tc.n_idx * 128 + (int)rank * 64 + 16 * quarter, args.N, lane);
        } else {
          const int f0 = tc.n_idx * UMMA_N + (int)rank * HALF + 32 * quarter;
          const int row0 = tc.row0;
          auto scale = [&](int r) -> float {
            if (args.row_scale == nullptr) return 1.f;
            return args.row_scale[args.scale_idx ? args.scale_idx[row0 + r] : row0 + r];
          };
          if constexpr (MODE == MODE_DOWN_EP) {
            auto dest = [&](int r) -> float* {
              const int64_t j = args.scale_idx[row0 + r];
              const int64_t src = j / args.ep.C;
              return reinterpret_cast<float*>(args.ep.arenas[src] + args.ep.y_off) +
                     (args.ep.yoff[src] + (j - src * args.ep.C)) * args.N;
            };
            epilogue_scale_f32_swapped(tbase, tc.ncols, nrows, f0, args.N, lane, scale, dest);
          } else {
            auto dest = [&](int r) -> float* {
              return reinterpret_cast<float*>(args.out) + (int64_t)(row0 + r) * args.ldo;
            };
            epilogue_scale_f32_swapped(tbase, tc.ncols, nrows, f0, args.N, lane, scale, dest);
          }
        }
      } else {
        // This warp's 32 consecutive rows (lane = row). Full tile: rows
        // rank*128 + quarter*32 of the 256. Tail (M=128 pair): TMEM lane L holds
        // row L % 64 of this CTA's 64 and column half L / 64.
        const int half = tc.tail ? (quarter >> 1) : 0;
        const int row_w0 = tc.tail ? tc.row0 + (int)rank * (HALF / 2) + 32 * (quarter & 1)
                                   : tc.row0 + (int)rank * HALF + quarter * 32;
        const int nrows = max(0, min(32, tc.row_end - row_w0));
        const int row = row_w0 + lane;
        float* stage = epi_stage + (warp - 2) * kStageFloatsPerWarp;
        if (MODE == MODE_GATE_UP) {
          __nv_bfloat16* orow0 = reinterpret_cast<__nv_bfloat16*>(args.out) + (int64_t)row_w0 * args.ldo;
          if (!tc.tail)
            epilogue_swiglu(tbase, 0, 128, 4, orow0, args.ldo, nrows, tc.n_idx * 128, args.N, lane);
          else
            epilogue_swiglu(tbase, 0, 64, 2, orow0, args.ldo, nrows, tc.n_idx * 128 + half * 64, args.N, lane);
        } else {
          float sc = 1.f;
          if (lane < nrows && args.row_scale != nullptr)
            sc = args.row_scale[args.scale_idx ? args.scale_idx[row] : row];
          if constexpr (MODE == MODE_DOWN_EP) {
            // this lane's row came from slot j = s*C + i: to source s's y, row yoff[s] + i
            float* rp = nullptr;
            if (lane < nrows) {
              const int64_t j = args.scale_idx[row];
              const int64_t src = j / args.ep.C;
              rp = reinterpret_cast<float*>(args.ep.arenas[src] + args.ep.y_off) +
                   (args.ep.yoff[src] + (j - src * args.ep.C)) * args.N;
            }
            if (!tc.tail)
              epilogue_scale_f32_rows(tbase, 8, sc, stage, rp, nrows, tc.n_idx * UMMA_N, args.N, lane);
            else
              epilogue_scale_f32_rows(tbase, 4, sc, stage, rp, nrows, tc.n_idx * UMMA_N + half * 128, args.N, lane);
          } else {
            float* orow0 = reinterpret_cast<float*>(args.out) + (int64_t)row_w0 * args.ldo;
            if (!tc.tail)
              epilogue_scale_f32(tbase, 8, sc, stage, orow0, args.ldo, nrows, tc.n_idx * UMMA_N, args.N, lane);
            else
              epilogue_scale_f32(tbase, 4, sc, stage, orow0, args.ldo, nrows, tc.n_idx * UMMA_N + half * 128, args.N,
                                 lane);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      // down releases at CTA scope (its staged fp32 stores need not be
      // visible to the leader first); gate_up measured faster with a
      // cluster-scope release after its direct bf16 stores.
      if (lane == 0) {
        if (MODE != MODE_GATE_UP) mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
        else mbar_arrive_remote_release(acc ? tempty_leader1 : tempty_leader0);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (MODE == MODE_DOWN_EP) __threadfence_system();  // the rows stored to peers, before any flag
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote arrive or pair MMA still targets either CTA
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc2(tmem_base, TMEM_COLS);
  }
}

// tmA64: the A operand with a 64-row box (swapped tails); swap_tails: run
// tails swapped (then tmB64 is the gate_up map of 16-row gate/up groups).
template <int MODE, int KA>
cudaError_t launch_tc2(const Segments& sg, const CUtensorMap& tmA, const CUtensorMap& tmA64, const CUtensorMap& tmB,
                       const CUtensorMap& tmB64, bool swap_tails, int64_t N, int64_t K, void* out, int64_t ldo,
                       const float* row_scale, const int32_t* scale_idx, int32_t* err, int num_sms, cudaStream_t s,
                       const EpRet* ep = nullptr) {
  static std::once_flag attr_once[kSmemAttrDevices];  // one set per kernel instance
  static cudaError_t attr_status[kSmemAttrDevices];
  const void* kernel = reinterpret_cast<const void*>(tc2_grouped_gemm_kernel<MODE, KA>);
  const cudaError_t attr_err = set_max_dynamic_smem_once(kernel, (int)smem_bytes2<MODE>(), attr_once, attr_status);
  if (attr_err != cudaSuccess) return attr_err;
  Args2 a{};
  if (ep != nullptr) a.ep = *ep;
  a.offsets = sg.offsets;
  a.E = sg.E;
  a.single_rows = sg.single_rows;
  a.N = (int32_t)N;
  a.n_tiles = (int32_t)ceil_div(N, MODE == MODE_GATE_UP ? 128 : UMMA_N);
  a.k_tiles = (int32_t)ceil_div(K, BK * KA);
  a.ldo = ldo;
  a.out = out;
  a.row_scale = row_scale;
  a.scale_idx = scale_idx;
  a.err = err;
  a.rows_total = sg.rows_total;
  a.swap_tails = swap_tails && KA == 1 && MODE != MODE_DOWN_KN ? 1 : 0;
  const int64_t nseg = sg.offsets ? sg.E : 1;
  const int64_t max_tiles = (sg.rows_total / BM2 + nseg) * a.n_tiles;
  const int pairs = (int)std::max<int64_t>(1, std::min<int64_t>(num_sms / 2, max_tiles));
  tc2_grouped_gemm_kernel<MODE, KA><<<2 * pairs, NTHREADS, smem_bytes2<MODE>(), s>>>(tmA, tmA64, tmB, tmB64, a);
  return cudaGetLastError();
}

// K atoms per stage. Two atoms per stage (3 stages of 64 KB: half the TMA
// operations and barrier round trips for the same bytes in flight; the view
// [K/64][rows][64], for K a multiple of 64) were measured against one atom
// per stage (6 stages of 32 KB): no gain on the DSV4- and Zipf-shaped
// problems and 3-5% slower on the Qwen3-shaped one (its 12-32-step K loops),
// so the kernels are launched with one atom per stage; the kernel and the map
// builder keep the atom count as a parameter.
constexpr int kAtomsPerStage = 1;

// Tensor maps over a K-major operand of `rows` rows (row pitch K elements),
// with the gate_up halves as a further dimension when `halves` is 2 and
// `nslab` consecutive operand slabs `slab_bytes` apart as the last one when
// nslab > 0 (none for the activations). Two atoms per stage: dims {64, rows,
// K/64, (halves,) (slabs)}, the atom dimension 128 bytes apart, box {64,
// box_rows, 2 or 1, 1, 1}. One atom: dims {K, rows, 1, ...}, box {64,
// box_rows, 1, ...}, reading zeros past K. The map's rank must equal the
// rank of the TMA instruction the kernel issues on it (3 for the
// activations, 5 for gate_up, 4 for down): a mismatch is rejected here, on
// the host, before any launch.
bool map_kmajor(CUtensorMap* m, const void* ptr, int KA, int64_t K, int64_t rows, int64_t row_pitch_bytes,
                int halves, int64_t half_bytes, int64_t nslab, int64_t slab_bytes, uint32_t box_rows,
                int expect_rank) {
  uint64_t dims[5], strides[4];
  uint32_t box[5];
  dims[0] = KA == 2 ? (uint64_t)BK : (uint64_t)K;
  box[0] = BK;
  dims[1] = (uint64_t)rows;
  strides[0] = (uint64_t)row_pitch_bytes;
  box[1] = box_rows;
  dims[2] = KA == 2 ? (uint64_t)(K / BK) : 1;
  strides[1] = KA == 2 ? (uint64_t)BK * 2 : (uint64_t)row_pitch_bytes * rows;
  box[2] = (uint32_t)(KA == 2 && box_rows == HALF ? 2 : 1);
  int r = 3;
  if (halves == 2) {
    dims[r] = 2;
    strides[r - 1] = (uint64_t)half_bytes;
    box[r] = 1;
    ++r;
  }
  if (nslab > 0) {
    dims[r] = (uint64_t)nslab;
    strides[r - 1] = (uint64_t)slab_bytes;
    box[r] = 1;
    ++r;
  }
  if (r != expect_rank) return false;
  return make_tensor_map_bf16(m, ptr, r, dims, strides, box);
}

// gate_up [E][2][I][H] seen as {H, 16 rows, 2 halves, I/16 groups, E} with
// box {64, 16, 2, 4, 1}: one load brings 64 features as 4 x [16 gate rows |
// the matching 16 up rows], 128 rows of 128 bytes in the swizzled layout.
// Needs I % 16 == 0 (every group inside its half); groups past I/16 read
// zeros.
bool map_gate_up_groups(CUtensorMap* m, const void* w_gate_up, int64_t H, int64_t I, int64_t E_w) {
  if (I % 16 != 0) return false;
  const uint64_t dims[5] = {(uint64_t)H, 16, 2, (uint64_t)(I / 16), (uint64_t)E_w};
  const uint64_t strides[4] = {(uint64_t)H * 2, (uint64_t)I * H * 2, (uint64_t)16 * H * 2, (uint64_t)2 * I * H * 2};
  const uint32_t box[5] = {BK, 16, 2, 4, 1};
  return make_tensor_map_bf16(m, w_gate_up, 5, dims, strides, box);
}

}  // namespace


cudaError_t launch_tc2_gate_up(const Segments& sg, const void* A, const void* w_gate_up, int64_t E_w, void* h,
                               int64_t I, int64_t H, int32_t* err, int num_sms, cudaStream_t s) {
  constexpr int KA = kAtomsPerStage;
  CUtensorMap tmA, tmA64, tmB, tmB64;
  // A: x_perm [rows, H] (3-D loads, 128 or 64 rows); gate_up [E][2][I][H]
  // (5-D loads): 128 rows of gate or of up per CTA (full tiles); for tails,
  // 4 x [16 gate | 16 up] rows per CTA (swapped, I % 16 == 0), else 64 gate +
  // 64 up rows per CTA and atom
  const bool swap = KA == 1 && I % 16 == 0;
  if (!map_kmajor(&tmA, A, KA, H, sg.rows_total, H * 2, 1, 0, 0, 0, HALF, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmA64, A, KA, H, sg.rows_total, H * 2, 1, 0, 0, 0, SWAP_ROWS, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmB, w_gate_up, KA, H, I, H * 2, 2, I * H * 2, E_w, 2 * I * H * 2, HALF, 5))
    return cudaErrorInvalidValue;
  if (swap ? !map_gate_up_groups(&tmB64, w_gate_up, H, I, E_w)
           : !map_kmajor(&tmB64, w_gate_up, KA, H, I, H * 2, 2, I * H * 2, E_w, 2 * I * H * 2, HALF / 2, 5))
    return cudaErrorInvalidValue;
  return launch_tc2<MODE_GATE_UP, KA>(sg, tmA, tmA64, tmB, tmB64, swap, I, H, h, I, nullptr, nullptr, err, num_sms,
                                      s);
}

cudaError_t launch_tc2_down(const Segments& sg, const void* A, const void* w_down, int64_t E_w, void* y,
                            const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I, int32_t* err,
                            int num_sms, cudaStream_t s) {
  constexpr int KA = kAtomsPerStage;
  CUtensorMap tmA, tmA64, tmB;
  // A: h [rows, I] (3-D loads, 128 or 64 rows); down [E][H][I] (4-D loads),
  // 128 of the tile's 256 output rows per CTA
  if (!map_kmajor(&tmA, A, KA, I, sg.rows_total, I * 2, 1, 0, 0, 0, HALF, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmA64, A, KA, I, sg.rows_total, I * 2, 1, 0, 0, 0, SWAP_ROWS, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmB, w_down, KA, I, H, I * 2, 1, 0, E_w, H * I * 2, HALF, 4)) return cudaErrorInvalidValue;
  return launch_tc2<MODE_DOWN, KA>(sg, tmA, tmA64, tmB, tmB, true, H, I, y, H, row_scale, scale_idx, err, num_sms,
                                   s);
}

cudaError_t launch_tc2_down_ep(const Segments& sg, const void* A, const void* w_down, int64_t E_w,
                               const float* row_scale, const int32_t* scale_idx, int64_t H, int64_t I,
                               const EpRet& ep, int32_t* err, int num_sms, cudaStream_t s) {
  constexpr int KA = kAtomsPerStage;
  CUtensorMap tmA, tmA64, tmB;
  // as launch_tc2_down: h [rows, I] (3-D loads), down [E][H][I] (4-D loads)
  if (!map_kmajor(&tmA, A, KA, I, sg.rows_total, I * 2, 1, 0, 0, 0, HALF, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmA64, A, KA, I, sg.rows_total, I * 2, 1, 0, 0, 0, SWAP_ROWS, 3)) return cudaErrorInvalidValue;
  if (!map_kmajor(&tmB, w_down, KA, I, H, I * 2, 1, 0, E_w, H * I * 2, HALF, 4)) return cudaErrorInvalidValue;
  return launch_tc2<MODE_DOWN_EP, KA>(sg, tmA, tmA64, tmB, tmB, true, H, I, nullptr, H, row_scale, scale_idx, err,
                                      num_sms, s, &ep);
}

cudaError_t launch_tc2_down_kn(const Segments& sg, const void* A, int64_t lda, const void* w_kn, int64_t E_w, void* y,
                               const float* row_scale, const int32_t* scale_idx, int64_t N, int64_t K, int32_t* err,
                               int num_sms, cudaStream_t s) {
  CUtensorMap tmA, tmB;
  // A: [rows, K] of pitch lda (3-D loads); B [E][K][N] (3-D loads of 64 columns x 64 K rows)
  if (!map_kmajor(&tmA, A, 1, K, sg.rows_total, lda * 2, 1, 0, 0, 0, HALF, 3)) return cudaErrorInvalidValue;
  const uint64_t dims[3] = {(uint64_t)N, (uint64_t)K, (uint64_t)E_w};
  const uint64_t strides[2] = {(uint64_t)N * 2, (uint64_t)K * N * 2};
  const uint32_t box[3] = {64, BK, 1};
  if (!make_tensor_map_bf16(&tmB, w_kn, 3, dims, strides, box)) return cudaErrorInvalidValue;
  return launch_tc2<MODE_DOWN_KN, 1>(sg, tmA, tmA, tmB, tmB, false, N, K, y, N, row_scale, scale_idx, err, num_sms,
                                     s);
}

}  // namespace stm
