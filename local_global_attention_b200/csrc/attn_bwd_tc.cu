// PACK3D backward on the Blackwell tensor cores (bf16 in, fp32 accumulate).
//
// "Geometry Matters in Packed 3D Attention" (abstract) calls the operator
// trainable at scale; its gradients, with P the softmax weights over a query's
// window keys and unmasked block summaries, delta_i = sum_c dO_ic O_ic and
// tau the softmax scale:
//   dS = P (dO V^T - delta)                    (keys and summaries alike)
//   dq~_i = tau sum_j dS_ij k~_j + tau sum_B dT_iB kbar_B
//   dk~_j = tau sum_i dS_ij q~_i + dkbar_B(j) / |B(j)|,  dkbar_B = tau sum_i dT_iB q~_i
//   dv_j  = sum_i P_ij dO_i + dvbar_B(j) / |B(j)|,       dvbar_B = sum_i P_iB dO_i
//   dq = R(c)^T dq~, dk = R(c)^T dk~ (the rotation is orthogonal).
//
// Kernels of one call:
//   staging: the rotated keys and the values in grid order with the block
//     summaries (the forward's staging kernel), and k_bwd_stage_q: the rotated
//     queries and dO in grid order, and per voxel (lse log2 e, delta) in fp32
//     and as statistic channels (below).
//   k_bwd_tc<DSUM>: rows = 128 block summaries, columns = every query of the
//     volume in chunks, split over CTAs; partial dkbar, dvbar per split, added
//     in split order by k_bwd_sum_reduce (deterministic).
//   k_bwd_tc<DQ>: rows = the 128 queries of a 4 x 4 x 8 tile, columns = the
//     keys of its halo, then the summaries; dq.
//   k_bwd_tc<DKDV>: rows = the 128 keys of a tile, columns = the queries of
//     its halo (the window is symmetric); dk, dv plus the summary gradients
//     spread over each block.
//
// One kernel template serves the three roles.  Per column chunk of 64:
//   S = A1 C1^T and dP = A2 C2^T (tcgen05, fp32 in tensor memory; A1 in tensor
//   memory with the window's penalty channels, A2 in shared memory); the
//   elementwise warps form P = 2^(S tau log2 e - L) and dS = P (dP - delta) and
//   write both as bf16 over S and dP; then acc1 += dS C1 and (dk/dv and the
//   summary role) acc2 += P C2, with C1, C2 the chunk's rows read as
//   channel-contiguous B operands.  S and dP are double-buffered, so the next
//   chunk's products run while the elementwise warps work on this one.
//
//   Where L and delta belong to the columns (dk/dv and the summary role) they
//   ride in the products: 16 more contraction channels hold, per column,
//   -L / (tau log2 e) and -delta, each split into three bf16 parts (their sum is
//   the fp32 value), against ones in the rows' channels (A1's in tensor memory,
//   A2's in shared memory).  S and dP then arrive as S - L / (tau log2 e) and
//   dP - delta, so the elementwise warps read no per-column statistics.
//
//   role  A1 (TMEM)   A2 (smem)  C1         C2      L, delta    acc1     acc2
//   DQ    q~ tile     dO tile    k~ / kbar  v / vbar per row    dq~      -
//   DKDV  k~ tile     v tile     q~ chunk   dO      per column  dk~      dv
//   DSUM  kbar rows   vbar rows  q~ chunk   dO      per column  dkbar    dvbar
//
// Tensor memory (512 columns, one CTA per SM): acc1 [0, 96), acc2 [96, 192),
// buffers b = 0, 1 at 192 + 128 b (S: 64 columns, dP: 64 columns), A1 [448, 512)
// (96 channels, 16 penalty channels, 16 statistic channels).
// Warps 0-7 elementwise (warp w: TMEM lanes 32 (w % 4) .., columns of half
// w / 4 of the chunk), warp 8 MMA issue, warp 9 TMA producer.  Every wait is
// bounded; a CTA that gives up sets the timeout bit of the index error word.
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "pack3d_internal.cuh"
#include "tc_attn_common.cuh"
#include "tc_primitives.cuh"

namespace p3d {

namespace {

using namespace tc;
using namespace tca;

constexpr int D = 96;
constexpr int NSTAGE = 6;
constexpr int SEGC = KCH * 64;    // one 32-channel segment of a 64-row chunk (4 KB)
constexpr int SEGR = 128 * 64;    // one 32-channel segment of the 128-row tile (8 KB)
constexpr uint32_t CHUNK_BYTES = 6 * SEGC;
constexpr uint32_t STAT_BYTES = KCH * 32;  // 16 bf16 statistic channels per column
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_ACC1 = 0, COL_ACC2 = 96, COL_BUF = 192, BUF_COLS = 128, COL_A1 = 448;
constexpr int NSOFT_WARPS = 8, MMA_WARP = 8, TMA_WARP = 9, NTHREADS = 320;
constexpr uint32_t WAIT_LIMIT = 1u << 20;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int ERR_TIMEOUT_BIT = 4;

enum Role { ROLE_DQ = 0, ROLE_DKDV = 1, ROLE_DSUM = 2 };

struct Smem {
  uint8_t a2[3 * SEGR];          // row operand 2 (K-major, 64-byte swizzle)
  uint8_t c1[NSTAGE][3 * SEGC];  // column operand 1 of each stage
  uint8_t c2[NSTAGE][3 * SEGC];  // column operand 2
  uint8_t cp[NSTAGE][KCH * 32];  // penalty channels of the column rows (32-byte swizzle)
  uint8_t cs[NSTAGE][KCH * 32];  // statistic channels of the column rows (32-byte swizzle)
  uint8_t a2x[128 * 32];         // the rows' statistic channels of the dP product
  PenaltyTable pt;               // the tile's penalty channels per axis (dense volumes)
  uint64_t a_full;               // A1 in tensor memory and A2 loaded
  uint64_t kv_full[NSTAGE], kv_empty[NSTAGE];
  uint64_t s_full[2];    // S and dP of the buffer's chunk computed
  uint64_t p_full[2];    // P and dS of the buffer's chunk written
  uint64_t acc_done[2];  // the accumulations reading the buffer are done
  uint64_t acc_final;    // every accumulation of the CTA is done
  uint64_t drain;         // a CTA that gave up: its issued MMAs are done
  uint32_t tmem_base;
  int32_t abort;
};
constexpr size_t SMEM_REQUEST = sizeof(Smem) + 1024;
static_assert(SMEM_REQUEST <= 232448, "shared memory of one CTA");
static_assert(offsetof(Smem, cs) % 1024 == 0 && offsetof(Smem, a2x) % 256 == 0 &&
                  offsetof(Smem, cp) % 1024 == 0,
              "32-byte-swizzled operands start on their pattern's boundary");

// Pointers of one backward kernel launch (which ones a role reads is in the
// role table above).
struct BwdArgs {
  const __nv_bfloat16* a1;  // row operand 1: DQ q~, DKDV k~ (grid order), DSUM kbar (bf16)
  const float4* stat;       // per voxel (lse log2 e, delta, 0, 0), grid order
  __nv_bfloat16* out1;      // DQ dq, DKDV dk (packed order)
  __nv_bfloat16* out2;      // DKDV dv
  const float* dks;         // DKDV: dkbar (tau included), fp32 [B][H][nb][96]
  const float* dvs;         // DKDV: dvbar
  float* part;              // DSUM: partial sums [split][B][H][nb][2][96]
  int nsplit;               // DSUM: splits of the volume's chunks
};

struct BwdMaps {
  CUtensorMap c1, c2;    // column chunks: grid-order volumes, box {32, 16, 2, 2, 1}
  CUtensorMap c1s, c2s;  // DQ summary columns: bf16 summaries, box {32, 64, 1}
  CUtensorMap st;        // per-column statistic channels: [B*H][Z][Y][X][16] bf16, box {16, 16, 2, 2, 1}
  CUtensorMap a2;        // row operand 2: box {32, 8, 2, 2, 1} (tile) or {32, 128, 1} (summaries)
};

__device__ __forceinline__ int dist_to_range(int v, int lo, int hi) {
  return v < lo ? lo - v : (v > hi ? v - hi : 0);
}

// Rows of a tile-role warp (2 x 2 x 8 box of the tile, clipped): extent of its
// active rows, for skipping chunk halves no row of the warp reaches.
struct WarpExtent {
  int zlo, zhi, ylo, yhi, xlo, xhi;
  bool any;
};

__device__ __forceinline__ WarpExtent warp_extent(bool active, int z, int y, int x) {
  constexpr int BIG = 1 << 29;
  WarpExtent e;
  e.zlo = __reduce_min_sync(0xffffffffu, active ? z : BIG);
  e.zhi = __reduce_max_sync(0xffffffffu, active ? z : -BIG);
  e.ylo = __reduce_min_sync(0xffffffffu, active ? y : BIG);
  e.yhi = __reduce_max_sync(0xffffffffu, active ? y : -BIG);
  e.xlo = __reduce_min_sync(0xffffffffu, active ? x : BIG);
  e.xhi = __reduce_max_sync(0xffffffffu, active ? x : -BIG);
  e.any = __any_sync(0xffffffffu, active);
  return e;
}

// Rotate a whole row back (R^T) in place: axial mode, segment a pairs
// (j, j + 16) turned by the table row of coordinate c_a; packed mode, pairs
// (j, j + 48) by the row of the packed position.
__device__ __forceinline__ void rotate_back(float (&v)[96], const float* rope, const Geo& g,
                                            int cz, int cy, int cx, int pos) {
  if (g.rope_mode == PACK3D_ROPE_PACKED) {
    const float2* t = rope_row96(rope, g, 0, 0, pos);
#pragma unroll
    for (int j = 0; j < 48; ++j) {
      const float2 cs = t[j];
      const float y1 = v[j], y2 = v[j + 48];
      v[j] = y1 * cs.x + y2 * cs.y;
      v[j + 48] = y2 * cs.x - y1 * cs.y;
    }
  } else {
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      const float2* t = rope_row96(rope, g, a, a == 0 ? cz : (a == 1 ? cy : cx), pos);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 cs = t[j];
        const float y1 = v[32 * a + j], y2 = v[32 * a + j + 16];
        v[32 * a + j] = y1 * cs.x + y2 * cs.y;
        v[32 * a + j + 16] = y2 * cs.x - y1 * cs.y;
      }
    }
  }
}

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float (&v)[96]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 12; ++i)
    d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                      pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

// Row of an accumulator (96 fp32 columns) of this thread's TMEM lane.
__device__ __forceinline__ void load_acc_row(uint32_t taddr, float (&v)[96]) {
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    uint32_t r[32];
    tmem_ld32(taddr + 32 * part, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[32 * part + i] = __uint_as_float(r[i]);
  }
}

// PARTIAL: a partly occupied volume (empty voxels and blocks masked; compiled
// out of the dense kernels).
template <int ROLE, bool PARTIAL>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_bwd_tc(Geo g, pack3d_index ix, const __grid_constant__ BwdMaps maps, BwdArgs args) {
  if (ix.err[0]) return;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~(uintptr_t)1023);
  volatile int32_t* abort_flag = &sm.abort;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int h = blockIdx.y, b = blockIdx.z, bh = b * g.H + h;
  constexpr bool TILE_ROWS = ROLE != ROLE_DSUM;   // rows are a 4 x 4 x 8 tile
  constexpr bool PENALTY = ROLE != ROLE_DSUM;     // local chunks masked by penalty channels
  constexpr bool COL_STATS = ROLE != ROLE_DQ;     // L, delta per column
  constexpr bool TWO_ACC = ROLE != ROLE_DQ;

  // ---- row tile and column chunks ----
  TileBox tb{};
  int B0 = 0, split = 0;
  int cz0, cy0, cx0, nyc, nxc, j_begin, n_local;
  if (TILE_ROWS) {
    tb = tile_box(g, blockIdx.x);
    cz0 = tb.hz0;
    cy0 = tb.hy0;
    cx0 = tb.hx0;
    const int nzc = (tb.hz + BZK - 1) / BZK;
    nyc = (tb.hy + BYK - 1) / BYK;
    nxc = (tb.hx + BXK - 1) / BXK;
    j_begin = 0;
    n_local = nzc * nyc * nxc;
  } else {
    const int nrt = (g.nb + 127) / 128;
    const int rt = blockIdx.x % nrt;
    split = blockIdx.x / nrt;
    B0 = rt * 128;
    // the queries of the owned planes (all planes unless the call is a z-slab)
    cz0 = g.own_lo;
    cy0 = cx0 = 0;
    const int nzc = (g.own_hi - g.own_lo + BZK - 1) / BZK;
    nyc = (g.Y + BYK - 1) / BYK;
    nxc = (g.X + BXK - 1) / BXK;
    const int total = nzc * nyc * nxc;
    j_begin = (int)((int64_t)split * total / args.nsplit);
    n_local = (int)((int64_t)(split + 1) * total / args.nsplit) - j_begin;
  }
  const int n_sum = ROLE == ROLE_DQ ? (g.nb + KCH - 1) / KCH : 0;
  const int nch = n_local + n_sum;
  // origin of local chunk j of the column box
  auto chunk_origin = [&](int j, int& z, int& y, int& x) {
    const int jj = j_begin + j;
    const int xc = jj % nxc, rest = jj / nxc;
    x = cx0 + BXK * xc;
    y = cy0 + BYK * (rest % nyc);
    z = cz0 + BZK * (rest / nyc);
  };

  if (tid == 0) {
    mbar_init(&sm.a_full, NSOFT_WARPS + 1);  // elementwise warps (A1) + the A2 copies
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&sm.kv_full[s], 2);  // TMA bytes + the penalty rows
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], NSOFT_WARPS);
      mbar_init(&sm.acc_done[i], 1);
    }
    mbar_init(&sm.acc_final, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  if (warp == TMA_WARP) {
    // ================= TMA producer (lane 0) and penalty rows (all lanes) =================
    if (lane == 0) {
      tma_prefetch_map(&maps.c1);
      tma_prefetch_map(&maps.c2);
      // row operand 2: four 2 x 2 x 8 boxes per segment in TMEM-lane order, or
      // 128 summary rows
      mbar_arrive_expect_tx(&sm.a_full, 3 * SEGR);
#pragma unroll
      for (int seg = 0; seg < 3; ++seg) {
        if (TILE_ROWS) {
#pragma unroll
          for (int w = 0; w < 4; ++w)
            tma_load_5d(sm.a2 + seg * SEGR + w * 2048, &maps.a2, seg * 32, tb.x0,
                        tb.y0 + 2 * (w & 1), tb.z0 + 2 * (w >> 1), bh, &sm.a_full);
        } else {
          tma_load_3d(sm.a2 + seg * SEGR, &maps.a2, seg * 32, B0, bh, &sm.a_full);
        }
      }
    }
    // dense volumes whose halo box fits the per-axis tables: penalty rows by
    // table lookups
    const bool table = PENALTY && !PARTIAL && tb.hz <= PEN_TAB && tb.hy <= PEN_TAB &&
                       tb.hx <= PEN_TAB;
    if (table) {
      penalty_table(sm.pt, g, tb, lane);
      __syncwarp();
    }
    int issued = 0;
    for (int j = 0; j < nch; ++j) {
      const int s = j % NSTAGE, round = j / NSTAGE;
      bool ok = true;
      if (lane == 0 && round > 0)
        ok = mbar_wait_or_abort(&sm.kv_empty[s], (round - 1) & 1, WAIT_LIMIT, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      int z = 0, y = 0, x = 0;
      if (j < n_local) chunk_origin(j, z, y, x);
      if (lane == 0) {
        if (j < n_local) {
          mbar_arrive_expect_tx(&sm.kv_full[s], CHUNK_BYTES + (COL_STATS ? STAT_BYTES : 0));
#pragma unroll
          for (int seg = 0; seg < 3; ++seg) {
            tma_load_5d(sm.c1[s] + seg * SEGC, &maps.c1, seg * 32, x, y, z, bh, &sm.kv_full[s]);
            tma_load_5d(sm.c2[s] + seg * SEGC, &maps.c2, seg * 32, x, y, z, bh, &sm.kv_full[s]);
          }
          if (COL_STATS) tma_load_5d(sm.cs[s], &maps.st, 0, x, y, z, bh, &sm.kv_full[s]);
        } else {
          mbar_arrive_expect_tx(&sm.kv_full[s], CHUNK_BYTES);
          const int Bs = (j - n_local) * KCH;
#pragma unroll
          for (int seg = 0; seg < 3; ++seg) {
            tma_load_3d(sm.c1[s] + seg * SEGC, &maps.c1s, seg * 32, Bs, bh, &sm.kv_full[s]);
            tma_load_3d(sm.c2[s] + seg * SEGC, &maps.c2s, seg * 32, Bs, bh, &sm.kv_full[s]);
          }
        }
      }
      if (PENALTY && j < n_local) {
        if (table)
          penalty_rows_table(sm.cp[s], sm.pt, tb, z, y, x, lane);
        else
          penalty_rows<PARTIAL>(sm.cp[s], g, tb, z, y, x, lane, ix.vol + (int64_t)b * g.V);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.kv_full[s]);
      issued = j + 1;
    }
    // Copies still in flight must land before the CTA ends (bounded: they
    // complete unless the memory system has failed).
    if (lane == 0) {
      mbar_wait(&sm.a_full, 0, WAIT_LIMIT);
      for (int j = max(0, issued - NSTAGE); j < issued; ++j)
        mbar_wait(&sm.kv_full[j % NSTAGE], (j / NSTAGE) & 1, WAIT_LIMIT);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ================= MMA issue (the whole warp, converged; one lane issues) =================
    constexpr uint32_t idesc_s = idesc_bf16(128, KCH, false);
    constexpr uint32_t idesc_o = idesc_bf16(128, D, true);
    // a descriptor's low field is the address in 16-byte units: an operand at a
    // byte offset is the base descriptor plus offset / 16
    const uint64_t c1k = sdesc_sw64(smem_u32(sm.c1[0]), 16, 512);
    const uint64_t c2k = sdesc_sw64(smem_u32(sm.c2[0]), 16, 512);
    const uint64_t c1m = sdesc_sw64(smem_u32(sm.c1[0]), SEGC, 512);
    const uint64_t c2m = sdesc_sw64(smem_u32(sm.c2[0]), SEGC, 512);
    const uint64_t a2d = sdesc_sw64(smem_u32(sm.a2), 16, 512);
    const uint64_t cpd = sdesc_sw32(smem_u32(sm.cp[0]), 16, 256);
    const uint64_t csd = sdesc_sw32(smem_u32(sm.cs[0]), 16, 256);
    const uint64_t a2xd = sdesc_sw32(smem_u32(sm.a2x), 16, 256);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, parity, WAIT_LIMIT, abort_flag));
    };
    bool ok = wait_all(&sm.a_full, 0);
    for (int j = 0; j <= nch && ok; ++j) {
      if (j < nch) {
        // S_j and dP_j into buffer j % 2 once the accumulations of chunk j - 2
        // have read it
        const int s = j % NSTAGE, bf = j & 1;
        if (!(ok = wait_all(&sm.kv_full[s], (j / NSTAGE) & 1))) break;
        if (j >= 2 && !(ok = wait_all(&sm.acc_done[bf], ((j - 2) >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t tS = tbase + COL_BUF + BUF_COLS * bf, tdP = tS + 64;
        const uint32_t so = (uint32_t)(s * 3 * SEGC);
#pragma unroll
        for (int st = 0; st < D / 16; ++st) {
          const uint32_t ko = so + (st >> 1) * SEGC + (st & 1) * 32;
          mma_ts_warp(tS, tbase + COL_A1 + 8 * st, c1k + (ko >> 4), idesc_s, st > 0);
        }
        if (PENALTY && j < n_local)
          mma_ts_warp(tS, tbase + COL_A1 + 48, cpd + ((uint32_t)(s * KCH * 32) >> 4), idesc_s, 1u);
        // S - L / (tau log2 e) and dP - delta: the column statistics ride in
        // 16 more contraction channels (ones in the rows' channels)
        if (COL_STATS)
          mma_ts_warp(tS, tbase + COL_A1 + 56, csd + ((uint32_t)(s * KCH * 32) >> 4), idesc_s, 1u);
#pragma unroll
        for (int st = 0; st < D / 16; ++st) {
          const uint32_t ao = (st >> 1) * SEGR + (st & 1) * 32;
          const uint32_t ko = so + (st >> 1) * SEGC + (st & 1) * 32;
          mma_ss_warp(tdP, a2d + (ao >> 4), c2k + (ko >> 4), idesc_s, st > 0);
        }
        if (COL_STATS)
          mma_ss_warp(tdP, a2xd, csd + ((uint32_t)(s * KCH * 32) >> 4), idesc_s, 1u);
        mma_commit_warp(&sm.s_full[bf]);
      }
      if (j >= 1) {
        // accumulations of chunk j - 1 once its P and dS are written
        const int jp = j - 1, sp = jp % NSTAGE, bp = jp & 1;
        if (!(ok = wait_all(&sm.p_full[bp], (jp >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t tS = tbase + COL_BUF + BUF_COLS * bp, tdP = tS + 64;
        const uint32_t so = (uint32_t)(sp * 3 * SEGC);
#pragma unroll
        for (int st = 0; st < KCH / 16; ++st) {
          // keys (columns) 16 st .. 16 st + 15: bf16 pairs written by half st / 2
          const uint32_t col = 32 * (st >> 1) + 8 * (st & 1);
          const uint32_t bo = so + st * 16 * 64;
          const uint32_t acc = (jp > 0 || st > 0) ? 1u : 0u;
          mma_ts_warp(tbase + COL_ACC1, tdP + col, c1m + (bo >> 4), idesc_o, acc);
          if (TWO_ACC) mma_ts_warp(tbase + COL_ACC2, tS + col, c2m + (bo >> 4), idesc_o, acc);
        }
        mma_commit_warp(&sm.acc_done[bp]);
        mma_commit_warp(&sm.kv_empty[sp]);
        if (jp == nch - 1) mma_commit_warp(&sm.acc_final);
      }
    }
    __syncwarp();
  } else {
    // ================= elementwise warps =================
    const int q4 = warp & 3, hf = warp >> 2;
    const int r = q4 * 32 + lane;  // TMEM lane = row of the tile
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    int rz = 0, ry = 0, rx = 0, lzi = 0, lyi = 0, lxi = 0;
    bool active;
    int64_t vox = 0;  // grid index of the row (tile roles)
    if (TILE_ROWS) {
      lane_pos(r, lzi, lyi, lxi);
      active = lzi < tb.lz && lyi < tb.ly && lxi < tb.lx && tb.z0 + lzi >= g.own_lo &&
               tb.z0 + lzi < g.own_hi;  // (a z-slab gives its owned planes only)
      rz = tb.z0 + lzi;
      ry = tb.y0 + lyi;
      rx = tb.x0 + lxi;
      vox = (((int64_t)bh * g.Z + rz) * g.Y + ry) * g.X + rx;
      // an empty voxel of a partly occupied volume is no row
      if (PARTIAL && active && !occupied(g, ix.vol, b, rz, ry, rx)) active = false;
    } else {
      // an empty block has no summary
      active = B0 + r < g.nb && (!PARTIAL || ix.bcount[(int64_t)b * g.nb + B0 + r] > 0);
    }
    {
      // A1 row into this lane: channels 0-63 from half 0, 64-95 and the
      // one-hot penalty channels from half 1
      const uint4* src = nullptr;
      if (active)
        src = reinterpret_cast<const uint4*>(args.a1 + (TILE_ROWS ? vox : (int64_t)bh * g.nb + B0 + r) * D);
      const uint32_t tq = tbase + lane_base + COL_A1;
      if (hf == 0) {
        uint32_t w32[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = active ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
          w32[4 * i] = v.x;
          w32[4 * i + 1] = v.y;
          w32[4 * i + 2] = v.z;
          w32[4 * i + 3] = v.w;
        }
        tmem_st32(tq, w32);
      } else {
        uint32_t w16[16], w8[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = active ? __ldg(src + 8 + i) : make_uint4(0, 0, 0, 0);
          w16[4 * i] = v.x;
          w16[4 * i + 1] = v.y;
          w16[4 * i + 2] = v.z;
          w16[4 * i + 3] = v.w;
        }
        if (PENALTY && active) {
          onehot_words(lzi, lyi, lxi, w8);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) w8[i] = 0u;
        }
        tmem_st16(tq + 32, w16);
        tmem_st8(tq + 48, w8);
        if (COL_STATS) {
          // statistic channels: ones at 0-2 (the S product's -L / (tau log2 e)
          // parts), and in shared memory ones at 3-5 for the dP product (-delta)
          uint32_t ws[8] = {0x3f803f80u, 0x00003f80u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st8(tq + 56, ws);
          const uint32_t rr = (uint32_t)r;
          *reinterpret_cast<uint4*>(sm.a2x + sw32_off(rr, 0)) =
              make_uint4(0u, 0x3f800000u, 0x3f803f80u, 0u);
          *reinterpret_cast<uint4*>(sm.a2x + sw32_off(rr, 1)) = make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.a_full);
    }
    const float c2 = g.tau * LOG2E;  // logits -> log2 units
    float Lrow = 0.f, Drow = 0.f;   // DQ: this query's lse log2 e and delta
    if (ROLE == ROLE_DQ && active) {
      const float4 sv = args.stat[vox];
      Lrow = sv.x;
      Drow = sv.y;
    }
    WarpExtent we{};
    if (TILE_ROWS) we = warp_extent(active, rz, ry, rx);
    // DQ summary chunks: the box of blocks this query's window touches
    // (global planes: the block grid of a z-slab is the whole volume's)
    const int bzlo = max(rz + g.zo - g.rz, 0) / g.bz, bzhi = min(rz + g.zo + g.rz, g.Zt - 1) / g.bz;
    const int bylo = max(ry - g.ry, 0) / g.by, byhi = min(ry + g.ry, g.Y - 1) / g.by;
    const int bxlo = max(rx - g.rx, 0) / g.bx, bxhi = min(rx + g.rx, g.X - 1) / g.bx;
    // DSUM: the range of query coordinates whose window meets this row's block
    int mzlo = 0, mzhi = -1, mylo = 0, myhi = -1, mxlo = 0, mxhi = -1;
    if (ROLE == ROLE_DSUM) {
      const int Br = B0 + r;
      const int bz = Br / (g.nby * g.nbx), by = (Br / g.nbx) % g.nby, bx = Br % g.nbx;
      mzlo = bz * g.bz - g.zo - g.rz;  // local planes of a z-slab
      mzhi = bz * g.bz - g.zo + g.bz - 1 + g.rz;
      mylo = by * g.by - g.ry;
      myhi = by * g.by + g.by - 1 + g.ry;
      mxlo = bx * g.bx - g.rx;
      mxhi = bx * g.bx + g.bx - 1 + g.rx;
    }

    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int bf = j & 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(&sm.s_full[bf], (j >> 1) & 1, WAIT_LIMIT, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // which of this half's 32 columns count: all (the penalty channels mask
      // the window), or the bits of the summary masks
      bool use_bits = false, skip = false;
      uint32_t bits = 0xffffffffu;
      if (j < n_local) {
        int z, y, x;
        chunk_origin(j, z, y, x);
        const int qz = z + hf;  // this half's plane of the chunk box
        if (TILE_ROWS) {
          skip = !we.any || qz >= g.Z || dist_to_range(qz, we.zlo, we.zhi) > g.rz ||
                 (dist_to_range(y, we.ylo, we.yhi) > g.ry &&
                  dist_to_range(y + 1, we.ylo, we.yhi) > g.ry) ||
                 x > we.xhi + g.rx || x + BXK - 1 < we.xlo - g.rx;
        } else {
          use_bits = true;
          bits = 0u;
          // partly occupied volume: the half's 32 query voxels that hold a token
          // (lane n looks up column n)
          uint32_t occ = 0xffffffffu;
          if (PARTIAL) {
            const int oz = qz, oy = y + (lane >> 4), ox = x + (lane & 15);
            const bool in = oz < g.Z && oy < g.Y && ox < g.X && occupied(g, ix.vol, b, oz, oy, ox);
            occ = __ballot_sync(0xffffffffu, in);
          }
          if (active && qz < g.own_hi) {
            const bool zin = qz >= mzlo && qz <= mzhi;
            const uint32_t xs = bit_range(0, min(BXK, g.X - x) - 1);  // in the volume
            const int elo = max(mxlo - x, 0), ehi = min(mxhi - x, BXK - 1);
            const uint32_t xm = elo <= ehi ? bit_range(elo, ehi) : 0u;  // x meets the block
#pragma unroll
            for (int dy = 0; dy < 2; ++dy) {
              const int qy = y + dy;
              if (qy >= g.Y) continue;
              const bool meets_zy = zin && qy >= mylo && qy <= myhi;
              bits |= (xs & (meets_zy ? ~xm : 0xffffu)) << (16 * dy);
            }
            bits &= occ;
          }
          skip = __ballot_sync(0xffffffffu, bits != 0u) == 0u;
          // (most chunks mask nothing for any row of the warp)
          use_bits = __any_sync(0xffffffffu, bits != 0xffffffffu);
        }
      } else {
        // DQ: summaries B .. B + 31 of this half
        const int Bs = (j - n_local) * KCH + 32 * hf;
        bits = active ? (uint32_t)(summary_mask64(g, (j - n_local) * KCH, bzlo, bzhi, bylo, byhi,
                                                  bxlo, bxhi) >>
                                   (32 * hf))
                      : 0u;
        // empty blocks have no summary (Bs is a multiple of 32)
        if (PARTIAL && Bs < g.nb) bits &= ix.bocc[(int64_t)b * ((g.nb + 31) / 32) + Bs / 32];
        use_bits = __any_sync(0xffffffffu, bits != 0xffffffffu);
        skip = __ballot_sync(0xffffffffu, bits != 0u) == 0u;
      }
      const uint32_t tS = tbase + lane_base + COL_BUF + BUF_COLS * bf + 32 * hf;
      const uint32_t tdP = tS + 64;
      uint32_t pw[16], dw[16];
      if (skip) {
#pragma unroll
        for (int i = 0; i < 16; ++i) pw[i] = dw[i] = 0u;
      } else {
        uint32_t sv[32], dv[32];
        tmem_ld32(tS, sv);
        tmem_ld32(tdP, dv);
        tmem_wait_ld();
        const float2 c2p = make_float2(c2, c2);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 sp = make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
          const float2 dpp = make_float2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1]));
          // column roles: the products already hold S - L / (tau log2 e) and dP - delta
          float2 a = COL_STATS ? f2_mul(sp, c2p) : f2_fma(sp, c2p, make_float2(-Lrow, -Lrow));
          if (use_bits) {
            if (!((bits >> (2 * i)) & 1u)) a.x = -INFINITY;
            if (!((bits >> (2 * i + 1)) & 1u)) a.y = -INFINITY;
          }
          const float2 p = make_float2(ex2(a.x), ex2(a.y));
          const float2 ds = f2_mul(p, COL_STATS ? dpp : f2_add(dpp, make_float2(-Drow, -Drow)));
          if (TWO_ACC) pw[i] = pack_bf16x2(p.x, p.y);
          dw[i] = pack_bf16x2(ds.x, ds.y);
        }
      }
      // P over this half's S columns (only the roles whose second product reads
      // it), dS over its dP columns (each half writes only columns it has read)
      if (TWO_ACC) tmem_st16(tS, pw);
      tmem_st16(tdP, dw);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[bf]);
    }

    // ---- epilogue ----
    if (ok && nch > 0)
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(&sm.acc_final, 0, WAIT_LIMIT, abort_flag));
    if (ok) {
      tc_fence_after();
      if (ROLE == ROLE_DSUM) {
        // partial sums of this split: acc1 (dkbar / tau) from half 0, acc2 from half 1
        float v[96];
        if (nch > 0) {
          load_acc_row(tbase + lane_base + (hf == 0 ? COL_ACC1 : COL_ACC2), v);
        } else {
#pragma unroll
          for (int i = 0; i < 96; ++i) v[i] = 0.f;
        }
        if (active) {
          float* dst = args.part + ((((int64_t)split * g.B + b) * g.H + h) * g.nb + B0 + r) * 2 * D +
                       hf * D;
#pragma unroll
          for (int i = 0; i < 24; ++i)
            reinterpret_cast<float4*>(dst)[i] =
                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      } else if (ROLE == ROLE_DQ) {
        if (hf == 0) {
          float v[96];
          load_acc_row(tbase + lane_base + COL_ACC1, v);
          if (active) {
            const int qi = ix.vol[((int64_t)b * g.Z + rz) * g.Y * g.X + (int64_t)ry * g.X + rx];
#pragma unroll
            for (int i = 0; i < 96; ++i) v[i] *= g.tau;
            rotate_back(v, ix.rope, g, rz, ry, rx, qi);
            store_row_bf16(args.out1 + (((int64_t)b * g.N + qi) * g.H + h) * D, v);
          }
        }
      } else {
        // dk (half 0): tau acc1 + dkbar / |B|, rotated back; dv (half 1): acc2 + dvbar / |B|
        float v[96];
        load_acc_row(tbase + lane_base + (hf == 0 ? COL_ACC1 : COL_ACC2), v);
        if (active) {
          const int kj = ix.vol[((int64_t)b * g.Z + rz) * g.Y * g.X + (int64_t)ry * g.X + rx];
          const int Bk = (((rz + g.zo) / g.bz) * g.nby + ry / g.by) * g.nbx + rx / g.bx;
          // the tokens the key's block holds (cut at the volume's edge; in a
          // partly occupied volume, the tokens present)
          const BlockExt be = block_ext(g, (rz + g.zo) / g.bz, ry / g.by, rx / g.bx);
          const int held = PARTIAL ? ix.bcount[(int64_t)b * g.nb + Bk] : be.ez * be.ey * be.ex;
          const float inv = 1.f / (float)held;
          const float4* srow = reinterpret_cast<const float4*>(
              (hf == 0 ? args.dks : args.dvs) + (((int64_t)b * g.H + h) * g.nb + Bk) * D);
          const float sc = hf == 0 ? g.tau : 1.f;
#pragma unroll
          for (int i = 0; i < 24; ++i) {
            const float4 a = srow[i];
            v[4 * i] = v[4 * i] * sc + a.x * inv;
            v[4 * i + 1] = v[4 * i + 1] * sc + a.y * inv;
            v[4 * i + 2] = v[4 * i + 2] * sc + a.z * inv;
            v[4 * i + 3] = v[4 * i + 3] * sc + a.w * inv;
          }
          if (hf == 0) rotate_back(v, ix.rope, g, rz, ry, rx, kj);
          store_row_bf16((hf == 0 ? args.out1 : args.out2) + (((int64_t)b * g.N + kj) * g.H + h) * D,
                         v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (sm.abort && tid == 0) atomicOr(&ix.err[0], ERR_TIMEOUT_BIT);
  if (warp == MMA_WARP) {
    // A CTA that gave up may still have products in flight (no role waited
    // for the last one): they land before the columns are freed (bounded).
    if (sm.abort) {
      mma_commit_warp(&sm.drain);
      if (lane == 0) mbar_wait(&sm.drain, 0, WAIT_LIMIT);
      __syncwarp();
    }
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

// dkbar = tau * sum over splits of the partials, dvbar = the same without tau
// (splits added in order, so the result does not depend on scheduling).
__global__ void k_bwd_sum_reduce(Geo g, const int32_t* __restrict__ err, int nsplit,
                                 const float* __restrict__ part, float* __restrict__ dks,
                                 float* __restrict__ dvs) {
  if (err[0]) return;
  const int64_t rows = (int64_t)g.B * g.H * g.nb;
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= rows * D) return;
  const int64_t row = e / D;
  const int c = (int)(e % D);
  float sk = 0.f, sv = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* src = part + ((int64_t)s * rows + row) * 2 * D;
    sk += src[c];
    sv += src[D + c];
  }
  dks[e] = g.tau * sk;
  dvs[e] = sv;
}

// Rotated queries and dO in grid order ([B][H][Z][Y][X][96] bf16) and per voxel
// (lse log2 e, delta = sum_c dO_c out_c, 0, 0), read once through the
// coordinate volume.  One CTA per (64-voxel piece of an x row and group of up
// to 8 heads, row z * Y + y, batch item), as the forward's staging of keys and
// values.  delta is summed per 16-channel item of a row as its dO and out
// pieces arrive, then over the six items in item order.
constexpr int STAGE_XS = 64, STAGE_HG = 8;

// x as hi + mid + lo, each the bf16 rounding of what is left (bit patterns).
__device__ __forceinline__ void split3_bf16(float x, uint32_t (&w)[3]) {
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    w[i] = (uint32_t)__bfloat16_as_ushort(h);
    x -= __bfloat162float(h);
  }
}

template <typename TO>
__global__ void __launch_bounds__(256)
    k_bwd_stage_q(Geo g, pack3d_index ix, const __nv_bfloat16* __restrict__ q,
                  const __nv_bfloat16* __restrict__ dout, const TO* __restrict__ out,
                  const float* __restrict__ lse, __nv_bfloat16* __restrict__ qg,
                  __nv_bfloat16* __restrict__ dog, float4* __restrict__ stat,
                  uint4* __restrict__ schan) {
  if (ix.err[0]) return;
  __shared__ int32_t tok[STAGE_XS];
  // delta partials: per (voxel, head of the group) the dot products of the six items
  __shared__ float part[STAGE_XS][STAGE_HG][6];
  const int nxb = (g.X + STAGE_XS - 1) / STAGE_XS;
  const int xb = (blockIdx.x % nxb) * STAGE_XS, h0 = (blockIdx.x / nxb) * STAGE_HG;
  const int zy = blockIdx.y, b = blockIdx.z;
  const int nh = min(STAGE_HG, g.H - h0);  // this CTA's heads h0 ..
  const int z = zy / g.Y, y = zy % g.Y;
  const int nx = min(STAGE_XS, g.X - xb);
  const int64_t vox0 = ((int64_t)b * g.Z * g.Y + zy) * g.X + xb;
  for (int i = threadIdx.x; i < nx; i += blockDim.x) tok[i] = ix.vol[vox0 + i];
  __syncthreads();
  const int H = g.H;
  // (hh: a head of the group)
  auto grid_row = [&](int hh) {
    return ((((int64_t)b * H + h0 + hh) * g.Z + z) * g.Y + y) * g.X + xb;
  };
  // an empty voxel (token -1, partly occupied volumes) gets zero rows and
  // statistics (0, 0)
  for (int it = threadIdx.x; it < nh * nx * 6; it += blockDim.x) {
    const int w = it % 6, rem = it / 6;
    const int x = rem % nx, hh = rem / nx;
    const Item96 item = item96(g, w);
    const int tk = tok[x];
    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo, dlo = lo, dhi = lo;
    float dot = 0.f;
    if (tk >= 0) {
      const int64_t row = (((int64_t)b * g.N + tk) * H + h0 + hh) * D;
      const uint4* src = reinterpret_cast<const uint4*>(q + row);
      const uint4* dsrc = reinterpret_cast<const uint4*>(dout + row);
      lo = __ldg(src + item.c1);
      hi = __ldg(src + item.c2);
      dlo = __ldg(dsrc + item.c1);
      dhi = __ldg(dsrc + item.c2);
      // dO . O over this item's 16 channels
      float o[16];
      if constexpr (sizeof(TO) == 4) {
        const float4* os = reinterpret_cast<const float4*>(out + row);
        const float4 a0 = __ldg(os + 2 * item.c1), a1 = __ldg(os + 2 * item.c1 + 1);
        const float4 b0 = __ldg(os + 2 * item.c2), b1 = __ldg(os + 2 * item.c2 + 1);
        o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
        o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
        o[8] = b0.x; o[9] = b0.y; o[10] = b0.z; o[11] = b0.w;
        o[12] = b1.x; o[13] = b1.y; o[14] = b1.z; o[15] = b1.w;
      } else {
        const uint4* os = reinterpret_cast<const uint4*>(out + row);
        const uint4 oa = __ldg(os + item.c1), ob = __ldg(os + item.c2);
        const uint32_t* pa = reinterpret_cast<const uint32_t*>(&oa);
        const uint32_t* pb = reinterpret_cast<const uint32_t*>(&ob);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 fa = unpack_bf16x2(pa[u]), fb = unpack_bf16x2(pb[u]);
          o[2 * u] = fa.x;
          o[2 * u + 1] = fa.y;
          o[8 + 2 * u] = fb.x;
          o[8 + 2 * u + 1] = fb.y;
        }
      }
      const uint32_t* dl = reinterpret_cast<const uint32_t*>(&dlo);
      const uint32_t* dh = reinterpret_cast<const uint32_t*>(&dhi);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 fa = unpack_bf16x2(dl[u]), fb = unpack_bf16x2(dh[u]);
        dot += fa.x * o[2 * u];
        dot += fa.y * o[2 * u + 1];
        dot += fb.x * o[8 + 2 * u];
        dot += fb.y * o[8 + 2 * u + 1];
      }
      const int c = item.a == 0 ? z : (item.a == 1 ? y : xb + x);
      rot_chunk(lo, hi, rope_row96(ix.rope, g, item.a, c, tk), item.j0);
    }
    part[x][hh][w] = dot;
    uint4* qd = reinterpret_cast<uint4*>(qg + (grid_row(hh) + x) * D);
    uint4* dd = reinterpret_cast<uint4*>(dog + (grid_row(hh) + x) * D);
    qd[item.c1] = lo;
    qd[item.c2] = hi;
    dd[item.c1] = dlo;
    dd[item.c2] = dhi;
  }
  __syncthreads();
  for (int it = threadIdx.x; it < nh * nx; it += blockDim.x) {
    const int x = it % nx, hh = it / nx;
    if (tok[x] < 0) {
      stat[grid_row(hh) + x] = make_float4(0.f, 0.f, 0.f, 0.f);
      schan[2 * (grid_row(hh) + x)] = make_uint4(0u, 0u, 0u, 0u);
      schan[2 * (grid_row(hh) + x) + 1] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    // the items' partial dot products added in item order
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 6; ++w) acc += part[x][hh][w];
    const float L = lse[((int64_t)b * H + h0 + hh) * g.N + tok[x]] * LOG2E;
    stat[grid_row(hh) + x] = make_float4(L, acc, 0.f, 0.f);
    // the column roles' statistic channels: -L / (tau log2 e) and -delta, each
    // as three bf16 parts whose sum is the fp32 value (to fp32 precision)
    uint32_t wl[3], wd[3];
    split3_bf16(-L / (g.tau * LOG2E), wl);
    split3_bf16(-acc, wd);
    schan[2 * (grid_row(hh) + x)] =
        make_uint4(wl[0] | (wl[1] << 16), wl[2] | (wd[0] << 16), wd[1] | (wd[2] << 16), 0u);
    schan[2 * (grid_row(hh) + x) + 1] = make_uint4(0u, 0u, 0u, 0u);
  }
}

struct BwdWs {
  size_t kg, vg, qg, dog, stat, schan, ksum, vsum, ksb, vsb, dks, dvs, part, total;
};

// Splits of the summary role: as many CTAs as fill one wave (one per SM), at
// most one chunk each, at most 64.
int dsum_splits(const Geo& g) {
  const int nrt = (g.nb + 127) / 128;
  const int64_t chunks =
      (int64_t)((g.own_hi - g.own_lo + 1) / 2) * ((g.Y + 1) / 2) * ((g.X + 15) / 16);
  const int64_t groups = (int64_t)g.B * g.H * nrt;
  int64_t s = (148 + groups - 1) / groups;
  s = std::min<int64_t>(s, std::min<int64_t>(chunks, 64));
  return (int)std::max<int64_t>(s, 1);
}

BwdWs bwd_layout(const Geo& g) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t vox = (size_t)g.B * g.H * g.V;  // grid order: one row per voxel
  const size_t vol = vox * D * 2;
  const size_t sum32 = (size_t)g.B * g.H * g.nb * D * 4;
  const size_t sum16 = sum32 / 2;
  BwdWs w;
  size_t o = 0;
  w.kg = o;   o += al(vol);
  w.vg = o;   o += al(vol);
  w.qg = o;   o += al(vol);
  w.dog = o;  o += al(vol);
  w.stat = o; o += al(vox * 16);
  w.schan = o; o += al(vox * 32);
  w.ksum = o; o += al(sum32);
  w.vsum = o; o += al(sum32);
  w.ksb = o;  o += al(sum16);
  w.vsb = o;  o += al(sum16);
  w.dks = o;  o += al(sum32);
  w.dvs = o;  o += al(sum32);
  w.part = o; o += al((size_t)dsum_splits(g) * 2 * sum32);
  w.total = o;
  return w;
}

template <int ROLE>
int launch_role(const Geo& g, const pack3d_index* idx, const BwdMaps& maps, const BwdArgs& args,
                dim3 grid, cudaStream_t s) {
  auto kern = g.partial ? k_bwd_tc<ROLE, true> : k_bwd_tc<ROLE, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_REQUEST) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  kern<<<grid, NTHREADS, SMEM_REQUEST, s>>>(g, *idx, maps, args);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

}  // namespace

bool backward_tc_supported(const Geo& g) { return g.d == D && g.dtype == PACK3D_BF16; }

size_t backward_tc_workspace_bytes(const Geo& g) {
  return backward_tc_supported(g) ? bwd_layout(g).total : 0;
}

namespace {

// The three roles' tensor maps over a staged workspace.
struct RoleMaps {
  BwdMaps q, k, s;  // dq, dk/dv, summary gradients
};

bool encode_role_maps(const Geo& g, uint8_t* base, const BwdWs& w, RoleMaps& m) {
  const uint64_t BH = (uint64_t)g.B * g.H;
  const uint64_t vdims[5] = {(uint64_t)D, (uint64_t)g.X, (uint64_t)g.Y, (uint64_t)g.Z, BH};
  const uint32_t cbox[5] = {32, BXK, BYK, BZK, 1};
  const uint32_t rbox[5] = {32, TX, 2, 2, 1};
  const uint64_t sdims[3] = {(uint64_t)D, (uint64_t)g.nb, BH};
  const uint32_t scbox[3] = {32, KCH, 1};
  const uint32_t srbox[3] = {32, 128, 1};
  const uint64_t tdims[5] = {16, (uint64_t)g.X, (uint64_t)g.Y, (uint64_t)g.Z, BH};
  const uint32_t tbox[5] = {16, BXK, BYK, BZK, 1};
  m = RoleMaps{};
  bool ok = true;
  // summary role: columns q~ / dO, stats; rows kbar (a1), vbar (A2)
  ok &= encode_bf16(&m.s.c1, base + w.qg, 5, vdims, cbox);
  ok &= encode_bf16(&m.s.c2, base + w.dog, 5, vdims, cbox);
  ok &= encode_map(&m.s.st, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base + w.schan, 5, tdims, tbox,
                   CU_TENSOR_MAP_SWIZZLE_32B);
  ok &= encode_bf16(&m.s.a2, base + w.vsb, 3, sdims, srbox);
  m.s.c1s = m.s.c1;
  m.s.c2s = m.s.c2;
  // dk / dv role: columns q~ / dO, stats; rows k~ (a1), v (A2)
  m.k = m.s;
  ok &= encode_bf16(&m.k.a2, base + w.vg, 5, vdims, rbox);
  // dq role: columns k~ / v then kbar / vbar; rows q~ (a1), dO (A2)
  ok &= encode_bf16(&m.q.c1, base + w.kg, 5, vdims, cbox);
  ok &= encode_bf16(&m.q.c2, base + w.vg, 5, vdims, cbox);
  ok &= encode_bf16(&m.q.c1s, base + w.ksb, 3, sdims, scbox);
  ok &= encode_bf16(&m.q.c2s, base + w.vsb, 3, sdims, scbox);
  ok &= encode_bf16(&m.q.a2, base + w.dog, 5, vdims, rbox);
  m.q.st = m.s.st;
  return ok;
}

// fp32 summaries -> the bf16 copies the MMAs read.
__global__ void k_bwd_summary_copies(const float* __restrict__ ks, const float* __restrict__ vs,
                                     __nv_bfloat16* __restrict__ kb, __nv_bfloat16* __restrict__ vb,
                                     int64_t n, const int32_t* __restrict__ err) {
  if (err[0]) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    kb[i] = __float2bfloat16_rn(ks[i]);
    vb[i] = __float2bfloat16_rn(vs[i]);
  }
}

}  // namespace

int backward_tc_summary_grads(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                              const void* v, const void* out, const float* lse, const void* dout,
                              const float* ksum, const float* vsum, float* dks, float* dvs,
                              void* workspace, cudaStream_t s) {
  const BwdWs w = bwd_layout(g);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(base + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(base + off); };
  // rotated keys and values in grid order, with the block summaries (fp32 and bf16)
  int rc = launch_block_summaries_staged(g, idx, k, v, f32(w.ksum), f32(w.vsum), base + w.kg,
                                         base + w.vg, base + w.ksb, base + w.vsb, s);
  if (rc) return rc;
  if (ksum) {
    // given summaries (the whole volume's, e.g. summed over z-slabs) replace
    // the ones computed from this call's tokens
    const int64_t n = (int64_t)g.B * g.H * g.nb * D;
    k_bwd_summary_copies<<<(unsigned)std::min<int64_t>((n + 255) / 256, 148 * 8), 256, 0, s>>>(
        ksum, vsum, bf(w.ksb), bf(w.vsb), n, idx->err);
    count_launches(1);
    if ((rc = cuda_status(cudaGetLastError()))) return rc;
  }
  {
    dim3 grid(((g.X + STAGE_XS - 1) / STAGE_XS) * ((g.H + STAGE_HG - 1) / STAGE_HG), g.Z * g.Y,
              g.B);
    if (g.out_fp32)
      k_bwd_stage_q<float><<<grid, 256, 0, s>>>(
          g, *idx, (const __nv_bfloat16*)q, (const __nv_bfloat16*)dout, (const float*)out, lse,
          bf(w.qg), bf(w.dog), reinterpret_cast<float4*>(base + w.stat),
          reinterpret_cast<uint4*>(base + w.schan));
    else
      k_bwd_stage_q<__nv_bfloat16><<<grid, 256, 0, s>>>(
          g, *idx, (const __nv_bfloat16*)q, (const __nv_bfloat16*)dout,
          (const __nv_bfloat16*)out, lse, bf(w.qg), bf(w.dog),
          reinterpret_cast<float4*>(base + w.stat), reinterpret_cast<uint4*>(base + w.schan));
    count_launches(1);
    if ((rc = cuda_status(cudaGetLastError()))) return rc;
  }
  RoleMaps m;
  if (!encode_role_maps(g, base, w, m)) return PACK3D_ERR_CUDA;
  // summary gradients, then their reduction in split order
  const int nsplit = dsum_splits(g);
  BwdArgs a{};
  a.a1 = bf(w.ksb);
  a.stat = reinterpret_cast<const float4*>(base + w.stat);
  a.part = f32(w.part);
  a.nsplit = nsplit;
  const int nrt = (g.nb + 127) / 128;
  if ((rc = launch_role<ROLE_DSUM>(g, idx, m.s, a, dim3(nrt * nsplit, g.H, g.B), s))) return rc;
  const int64_t n = (int64_t)g.B * g.H * g.nb * D;
  k_bwd_sum_reduce<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(g, idx->err, nsplit, f32(w.part),
                                                                dks, dvs);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

int backward_tc_from_summary_grads(const Geo& g, const pack3d_index* idx, const float* dks,
                                   const float* dvs, void* dq, void* dk, void* dv,
                                   void* workspace, cudaStream_t s) {
  const BwdWs w = bwd_layout(g);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(base + off); };
  RoleMaps m;
  if (!encode_role_maps(g, base, w, m)) return PACK3D_ERR_CUDA;
  const float4* stat = reinterpret_cast<const float4*>(base + w.stat);
  int rc;
  {
    BwdArgs a{};
    a.a1 = bf(w.qg);
    a.stat = stat;
    a.out1 = (__nv_bfloat16*)dq;
    if ((rc = launch_role<ROLE_DQ>(g, idx, m.q, a, dim3(g.nT, g.H, g.B), s))) return rc;
  }
  BwdArgs a{};
  a.a1 = bf(w.kg);
  a.stat = stat;
  a.out1 = (__nv_bfloat16*)dk;
  a.out2 = (__nv_bfloat16*)dv;
  a.dks = dks;
  a.dvs = dvs;
  return launch_role<ROLE_DKDV>(g, idx, m.k, a, dim3(g.nT, g.H, g.B), s);
}

int launch_backward_tc(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                       const void* v, const void* out, const float* lse, const void* dout,
                       void* dq, void* dk, void* dv, void* workspace, cudaStream_t s) {
  const BwdWs w = bwd_layout(g);
  float* dks = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.dks);
  float* dvs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.dvs);
  int rc = backward_tc_summary_grads(g, idx, q, k, v, out, lse, dout, nullptr, nullptr, dks, dvs,
                                     workspace, s);
  if (rc) return rc;
  return backward_tc_from_summary_grads(g, idx, dks, dvs, dq, dk, dv, workspace, s);
}

}  // namespace p3d
