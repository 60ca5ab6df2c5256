// PACK3D forward on the Blackwell tensor cores (bf16 in, fp32 accumulate).
//
// "Geometry Matters in Packed 3D Attention" (abstract): each query attends
// exactly to its clipped 3D window and to the summaries of the blocks its
// window misses, in one softmax, with axial RoPE on grid coordinates.
//
// Two kernels per call:
//
//   k_grid_kv: reads every key and value row once through the coordinate
//     volume, applies the axial rotation to the key (fp32 arithmetic, the
//     table built in fp64 by the index build) and writes both in grid order,
//     one [Z][Y][X][96] bf16 volume per (batch item, head).  With the packing
//     undone here, the halo of a query tile is a 3-D box of the grid, which the
//     tensor-memory accelerator (TMA) copies as tiled loads; no key is gathered
//     or rotated twice.
//
//   k_forward_tc: one CTA per 4 x 4 x 8 query tile (M = 128 rows) of one
//     (batch item, head).  The tile's clipped halo box is covered by chunks of
//     16 (x) x 2 (y) x 2 (z) = 64 keys, then the block summaries (bf16 copies,
//     64 per chunk), all streamed through one online softmax.  Roles:
//
//     * TMA (warp 5): per chunk six box loads by one thread (three 32-channel
//       segments of K and of V, 64-byte swizzle: exactly the K-major operand
//       layout of the MMAs) into a 3-stage shared-memory ring; positions
//       outside the volume are filled with zeros by the copy and masked.  The
//       warp also writes the chunk's penalty rows (below), assembled from
//       per-axis tables built once per tile;
//     * MMA (warp 4, one thread): S_j = Q K_j^T (six tcgen05.mma, K = 16, plus
//       one for the window penalty) into one of two TMEM S buffers, with both
//       Q and K read from shared memory, and O += P_j V_j (four tcgen05.mma,
//       A = P from TMEM, B = V MN-major in shared memory).  S_{j+2} is issued
//       as soon as PV_j is done, so two S products run ahead of the softmax;
//     * softmax (warps 0-3, one query row per thread, warp w = a 2 x 2 x 8 box):
//       gather and rotate the query rows once into the shared-memory Q tile;
//       per chunk form the window mask from three per-query bit sets over the
//       halo (z planes, y rows, x columns), read the chunk's 64 S values in one
//       go, keep the online max and sum, write P (bf16) over the first half of
//       the S buffer it read.  A warp whose 32 queries see none of a chunk's
//       keys (its plane or row pair outside their windows) only writes zeros.
//       Summary chunks use the mask "block box does not meet the window box";
//       there is no count bias.  The running max moves only when a row's
//       maximum grows by more than 8 (log2 units), so O is rescaled in TMEM
//       rarely; the result is the same softmax.
//
// The window mask rides in the S product: 16 extra contraction channels hold
// the query's one-hot tile position and the key's -2^14 penalties.
//
// The epilogue divides by the row sum and writes out (packed order) and the
// natural-log LSE.  Two CTAs share an SM (256 TMEM columns and ~110 KB of
// shared memory each).  Every wait
// is bounded; a CTA that gives up sets the timeout bit of the index error word.
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

constexpr int D = 96;                      // head dim handled by this path
constexpr int NSTAGE = 3;                  // K/V shared-memory ring depth
constexpr int KSEG = KCH * 64;             // one 32-channel segment of a chunk
constexpr uint32_t CHUNK_BYTES = 6 * KSEG; // K and V of one chunk
constexpr uint32_t TMEM_COLS = 256;
// Tensor memory (128 lanes = query rows, 256 columns of 32 bits): the O
// accumulator (fp32, columns [0, 96)) and two S buffers (fp32, [96, 160) and
// [160, 224)); P (bf16 pairs) is written over the first 32 columns of its S.
constexpr uint32_t COL_O = 0;
constexpr uint32_t COL_S = 96;
constexpr int QSEG = 128 * 64;             // one 32-channel segment of the Q tile
constexpr int MMA_WARP = 4;
constexpr int TMA_WARP = 5;
constexpr int NTHREADS = 192;
constexpr uint32_t WAIT_LIMIT = 1u << 20;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int ERR_TIMEOUT_BIT = 4;
constexpr int MAX_HALO = 64;               // halo extent per axis the 64-bit masks cover
// Floor of the running max (log2 units): a chunk whose keys are all masked
// never raises it, so their exponentials stay 0.  Logits below this floor
// (-693 in natural units) are outside the supported range.
constexpr float M_FLOOR = -1000.0f;

struct Smem {
  uint8_t q[3 * QSEG];           // rotated Q rows (K-major, 64-byte swizzle), row = TMEM lane
  uint8_t qp[128 * 32];          // the rows' penalty one-hot (32-byte swizzle)
  uint8_t k[NSTAGE][3 * KSEG];
  uint8_t v[NSTAGE][3 * KSEG];
  uint8_t kp[NSTAGE][KCH * 32];  // penalty channels of each stage's key rows (32-byte swizzle)
  PenaltyTable pt;               // the tile's penalty channels per axis (dense volumes)
  uint64_t q_full;               // Q is in shared memory
  uint64_t kv_full[NSTAGE];
  uint64_t kv_empty[NSTAGE];
  uint64_t s_full[2];    // S of the buffer's chunk computed
  uint64_t p_full[2];    // P of the buffer's chunk written
  uint64_t buf_free[2];  // the PV product reading the buffer's P is done
  uint64_t o_final;      // one phase: every PV product of the tile is done
  uint64_t drain;         // a CTA that gave up: its issued MMAs are done
  uint32_t tmem_base;
  int32_t abort;
};
constexpr size_t SMEM_REQUEST = sizeof(Smem) + 1024;  // + alignment slack

// ---- grid-order rotated keys and values ------------------------------------------

// One CTA per (64-voxel piece of an x row, row z * Y + y, batch item).  Key
// items are (head, voxel, item w of item96): 8 channels and their 8 rotation
// partners, rotated; value items (head, voxel, 16-byte chunk) are copied.  Consecutive
// threads cover one 192-byte row, so reads (through the volume) and writes
// (grid order) are whole rows.
constexpr int GRID_XS = 64;

__global__ void __launch_bounds__(256)
    k_grid_kv(Geo g, pack3d_index ix, const __nv_bfloat16* __restrict__ k,
              const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ kg,
              __nv_bfloat16* __restrict__ vg) {
  if (ix.err[0]) return;
  __shared__ int32_t tok[GRID_XS];
  const int xb = blockIdx.x * GRID_XS, zy = blockIdx.y, b = blockIdx.z;
  const int z = zy / g.Y, y = zy % g.Y;
  const int nx = min(GRID_XS, g.X - xb);
  const int64_t vox0 = ((int64_t)b * g.Z * g.Y + zy) * g.X + xb;
  // an empty voxel (token -1, partly occupied volumes) gets zero rows
  for (int i = threadIdx.x; i < nx; i += blockDim.x) tok[i] = ix.vol[vox0 + i];
  __syncthreads();
  const int H = g.H;
  // first element of (b, h, z, y, x = xb) in the grid-order volumes
  auto grid_row = [&](int h) {
    return ((((int64_t)b * H + h) * g.Z + z) * g.Y + y) * g.X + xb;
  };
  for (int it = threadIdx.x; it < H * nx * 6; it += blockDim.x) {
    const int w = it % 6, rem = it / 6;
    const int x = rem % nx, h = rem / nx;
    const Item96 item = item96(g, w);
    const int tk = tok[x];
    uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
    if (tk >= 0) {
      const uint4* src = reinterpret_cast<const uint4*>(k + (((int64_t)b * g.N + tk) * H + h) * D);
      lo = __ldg(src + item.c1);
      hi = __ldg(src + item.c2);
      const int c = item.a == 0 ? z : (item.a == 1 ? y : xb + x);
      rot_chunk(lo, hi, rope_row96(ix.rope, g, item.a, c, tk), item.j0);
    }
    uint4* dst = reinterpret_cast<uint4*>(kg + (grid_row(h) + x) * D);
    dst[item.c1] = lo;
    dst[item.c2] = hi;
  }
  for (int it = threadIdx.x; it < H * nx * 12; it += blockDim.x) {
    const int c = it % 12, rem = it / 12;
    const int x = rem % nx, h = rem / nx;
    uint4* dst = reinterpret_cast<uint4*>(vg + (grid_row(h) + x) * D) + c;
    *dst = tok[x] >= 0 ? __ldg(reinterpret_cast<const uint4*>(
                             v + (((int64_t)b * g.N + tok[x]) * H + h) * D) + c)
                       : make_uint4(0, 0, 0, 0);
  }
}

// fp32 summaries -> bf16 copies (the tensor-core operand type), same layout.
__global__ void k_summaries_bf16(const float4* __restrict__ ks, const float4* __restrict__ vs,
                                 uint2* __restrict__ kb, uint2* __restrict__ vb, int64_t n4,
                                 const int32_t* __restrict__ err) {
  if (err[0]) return;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = ks[i], c = vs[i];
    kb[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    vb[i] = make_uint2(pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
  }
}

// ---- softmax arithmetic ---------------------------------------------------------

// P = 2^(S c2 + mneg) for all 32 keys (masked ones carry the penalty), packed
// in pairs into p[0..15]; returns the sum.
// The scaling and the running sums use the paired fp32 arithmetic (two values
// per instruction).
__device__ __forceinline__ float exp_pack_all(const uint32_t (&sv)[32], float c2, float mneg,
                                              uint32_t* p) {
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  const float2 cc = make_float2(c2, c2), mm = make_float2(mneg, mneg);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 a = f2_fma(make_float2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])),
                            cc, mm);
    const float2 e = make_float2(ex2(a.x), ex2(a.y));
    acc[i & 1] = f2_add(acc[i & 1], e);
    p[i] = pack_bf16x2(e.x, e.y);
  }
  const float2 t = f2_add(acc[0], acc[1]);
  return t.x + t.y;
}

__device__ __forceinline__ float plain_max(const uint32_t (&sv)[32]) {
  float m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = __uint_as_float(sv[i]);
#pragma unroll
  for (int i = 4; i < 32; ++i) m[i & 3] = fmaxf(m[i & 3], __uint_as_float(sv[i]));
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

// Keys outside `bits` get S = -inf, so the unmasked max and exponentials give
// them no weight.
__device__ __forceinline__ void apply_mask(uint32_t (&sv)[32], uint32_t bits) {
#pragma unroll
  for (int i = 0; i < 32; ++i) sv[i] = ((bits >> i) & 1u) ? sv[i] : 0xff800000u;
}

struct Maps {
  CUtensorMap kg, vg;  // [B*H][Z][Y][X][96] bf16, box {32, 16, 2, 2, 1}
  CUtensorMap ks, vs;  // [B*H][nb][96] bf16, box {32, 64, 1}
};

// PARTIAL: a partly occupied volume (empty voxels masked; compiled out of the
// dense kernel).
template <bool SUMMARY, bool PARTIAL>
__global__ void __launch_bounds__(NTHREADS, 2)
    k_forward_tc(Geo g, pack3d_index ix, const __nv_bfloat16* __restrict__ q,
                 const __grid_constant__ Maps maps, void* __restrict__ out_raw,
                 float* __restrict__ lse) {
  if (ix.err[0]) return;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~(uintptr_t)1023);
  volatile int32_t* abort_flag = &sm.abort;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const TileBox tb = tile_box(g, t);
  const int nzc = (tb.hz + BZK - 1) / BZK, nyc = (tb.hy + BYK - 1) / BYK,
            nxc = (tb.hx + BXK - 1) / BXK;
  const int n_local = nzc * nyc * nxc;
  const int n_sum = SUMMARY ? (g.nb + KCH - 1) / KCH : 0;
  const int nch = n_local + n_sum;

  if (tid == 0) {
    mbar_init(&sm.q_full, 4);  // softmax barriers: one arrival per softmax warp
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&sm.kv_full[s], 2);  // TMA bytes + the penalty rows
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 4);
      mbar_init(&sm.buf_free[i], 1);
    }
    mbar_init(&sm.o_final, 1);
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
      tma_prefetch_map(&maps.kg);
      tma_prefetch_map(&maps.vg);
    }
    const int bh = b * g.H + h;
    if (!PARTIAL) {
      penalty_table(sm.pt, g, tb, lane);
      __syncwarp();
    }
    int xc = 0, yc = 0, zc = 0;
    int issued = 0;
    for (int j = 0; j < nch; ++j) {
      const int s = j % NSTAGE, round = j / NSTAGE;
      bool ok = true;
      if (lane == 0 && round > 0)
        ok = mbar_wait_or_abort(&sm.kv_empty[s], (round - 1) & 1, WAIT_LIMIT, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.kv_full[s], CHUNK_BYTES);
        if (j < n_local) {
          const int x = tb.hx0 + BXK * xc, y = tb.hy0 + BYK * yc, z = tb.hz0 + BZK * zc;
#pragma unroll
          for (int seg = 0; seg < 3; ++seg) {
            tma_load_5d(sm.k[s] + seg * KSEG, &maps.kg, seg * 32, x, y, z, bh, &sm.kv_full[s]);
            tma_load_5d(sm.v[s] + seg * KSEG, &maps.vg, seg * 32, x, y, z, bh, &sm.kv_full[s]);
          }
        } else {
          const int B0 = (j - n_local) * KCH;
#pragma unroll
          for (int seg = 0; seg < 3; ++seg) {
            tma_load_3d(sm.k[s] + seg * KSEG, &maps.ks, seg * 32, B0, bh, &sm.kv_full[s]);
            tma_load_3d(sm.v[s] + seg * KSEG, &maps.vs, seg * 32, B0, bh, &sm.kv_full[s]);
          }
        }
      }
      if (j < n_local) {
        // penalty rows of the chunk's keys (dz, dy, dx): key r = (dz * 2 + dy) * 16 + dx
        const int cz0 = tb.hz0 + BZK * zc, cy0 = tb.hy0 + BYK * yc, cx0 = tb.hx0 + BXK * xc;
        if (PARTIAL)
          penalty_rows<true>(sm.kp[s], g, tb, cz0, cy0, cx0, lane, ix.vol + (int64_t)b * g.V);
        else
          penalty_rows_table(sm.kp[s], sm.pt, tb, cz0, cy0, cx0, lane);
        fence_proxy_async_smem();
        if (++xc == nxc) {
          xc = 0;
          if (++yc == nyc) {
            yc = 0;
            ++zc;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.kv_full[s]);
      issued = j + 1;
    }
    // Copies still in flight must land before the CTA ends (bounded: they
    // complete unless the memory system has failed).
    if (lane == 0)
      for (int j = max(0, issued - NSTAGE); j < issued; ++j)
        mbar_wait(&sm.kv_full[j % NSTAGE], (j / NSTAGE) & 1, WAIT_LIMIT);
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ================= MMA issue (the whole warp, converged; one lane issues) =================
    {
      constexpr uint32_t idesc_s = idesc_bf16(128, KCH, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, D, true);
      // Descriptors are formed once: a descriptor's low field is the address
      // in 16-byte units, so an operand at a byte offset is the base
      // descriptor plus offset / 16 (all shared-memory addresses < 256 KB).
      const uint64_t kd0 = sdesc_sw64(smem_u32(sm.k[0]), 16, 512);
      const uint64_t vd0 = sdesc_sw64(smem_u32(sm.v[0]), KSEG, 512);
      const uint64_t kpd0 = sdesc_sw32(smem_u32(sm.kp[0]), 16, 256);
      const uint64_t qd0 = sdesc_sw64(smem_u32(sm.q), 16, 512);
      const uint64_t qpd = sdesc_sw32(smem_u32(sm.qp), 16, 256);
      auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, parity, WAIT_LIMIT, abort_flag));
      };
      bool ok = wait_all(&sm.q_full, 0);
      // S_j = Q K_j^T into buffer j % 2: A = the Q tile, B = the chunk's key
      // rows (both K-major, 64-byte swizzle, 16-channel steps)
      auto issue_s = [&](int j) -> bool {
        const int s = j % NSTAGE;
        if (!wait_all(&sm.kv_full[s], (j / NSTAGE) & 1)) return false;
        tc_fence_after();
        const uint32_t dS = tbase + COL_S + 64 * (j & 1);
        const uint64_t kd = kd0 + (uint64_t)((s * 3 * KSEG) >> 4);
#pragma unroll
        for (int st = 0; st < D / 16; ++st)
          mma_ss_warp(dS, qd0 + (uint64_t)(((st >> 1) * QSEG + (st & 1) * 32) >> 4),
                      kd + (uint64_t)(((st >> 1) * KSEG + (st & 1) * 32) >> 4), idesc_s, st > 0);
        if (j < n_local)  // + the window penalty (summary chunks are masked by the softmax)
          mma_ss_warp(dS, qpd, kpd0 + (uint64_t)((s * KCH * 32) >> 4), idesc_s, 1u);
        mma_commit_warp(&sm.s_full[j & 1]);
        return true;
      };
      if (ok) tc_fence_after();
      for (int j = 0; j < min(2, nch) && ok; ++j) ok = issue_s(j);
      for (int j = 0; j < nch && ok; ++j) {
        const int bi = j & 1;
        if (!(ok = wait_all(&sm.p_full[bi], (j >> 1) & 1))) break;
        tc_fence_after();
        // O += P_j V_j: A = P over the buffer's first 32 columns, B = V
        // MN-major (key rows 16 u .. 16 u + 15 at byte offset 1024 u)
        const uint64_t vd = vd0 + (uint64_t)(((j % NSTAGE) * 3 * KSEG) >> 4);
        const uint32_t pS = tbase + COL_S + 64 * bi;
#pragma unroll
        for (int st = 0; st < KCH / 16; ++st)
          mma_ts_warp(tbase + COL_O, pS + 8 * st, vd + (uint64_t)((st * 16 * 64) >> 4), idesc_o,
                      (j > 0 || st > 0) ? 1u : 0u);
        mma_commit_warp(&sm.buf_free[bi]);
        mma_commit_warp(&sm.kv_empty[j % NSTAGE]);
        if (j == nch - 1) mma_commit_warp(&sm.o_final);
        // S_{j+2} overwrites P_j: after PV_j is done
        if (j + 2 < nch) {
          if (!(ok = wait_all(&sm.buf_free[bi], (j >> 1) & 1))) break;
          tc_fence_after();
          if (!(ok = issue_s(j + 2))) break;
        }
      }
    }
    __syncwarp();
  } else {
    // ================= softmax warps (one query row per thread) =================
    // Row tid of the tile: warp w holds planes 2 (w / 2) + {0, 1}, rows
    // 2 (w % 2) + {0, 1}, all 8 columns - a 2 x 2 x 8 box, whose windows meet
    // only 4 of the 5 plane pairs and 4 of the 5 row pairs of an interior halo,
    // so the warp skips about a third of the chunks.
    const int lzi = (warp >> 1) * 2 + (lane >> 4), lyi = (warp & 1) * 2 + ((lane >> 3) & 1),
              lxi = lane & 7;
    // (a z-slab writes its owned planes only)
    bool active = lzi < tb.lz && lyi < tb.ly && lxi < tb.lx && tb.z0 + lzi >= g.own_lo &&
                  tb.z0 + lzi < g.own_hi;
    const int cz = tb.z0 + lzi, cy = tb.y0 + lyi, cx = tb.x0 + lxi;
    int qi = 0;
    if (active) qi = ix.vol[(((int64_t)b * g.Z + cz) * g.Y + cy) * g.X + cx];
    if (PARTIAL && qi < 0) {  // an empty voxel of a partly occupied volume: no query
      active = false;
      qi = 0;
    }
    {
      // this thread's query row: gathered, rotated, stored once
      uint4 r[12];
      if (active) {
        const uint4* src =
            reinterpret_cast<const uint4*>(q + (((int64_t)b * g.N + qi) * g.H + h) * D);
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = __ldg(src + i);
        if (g.rope_mode == PACK3D_ROPE_PACKED) {
          // one-dimensional rotation by the packed index: chunk w pairs with w + 6
          const float2* tp = rope_row96(ix.rope, g, 0, 0, qi);
#pragma unroll
          for (int w = 0; w < 6; ++w) rot_chunk(r[w], r[w + 6], tp, 8 * w);
        } else {
          const float2* tz = rope_row96(ix.rope, g, 0, cz, qi);
          const float2* ty = rope_row96(ix.rope, g, 1, cy, qi);
          const float2* tx = rope_row96(ix.rope, g, 2, cx, qi);
          rot_chunk(r[0], r[2], tz, 0);
          rot_chunk(r[1], r[3], tz, 8);
          rot_chunk(r[4], r[6], ty, 0);
          rot_chunk(r[5], r[7], ty, 8);
          rot_chunk(r[8], r[10], tx, 0);
          rot_chunk(r[9], r[11], tx, 8);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = make_uint4(0, 0, 0, 0);
      }
      // into the Q tile, row tid (this thread's TMEM lane): 16-byte chunk i
      // of the row is chunk i % 4 of segment i / 4; then the penalty one-hot
      const uint32_t rr = (uint32_t)tid;
#pragma unroll
      for (int i = 0; i < 12; ++i)
        *reinterpret_cast<uint4*>(sm.q + (i >> 2) * QSEG + sw64_off(rr, i & 3)) = r[i];
      uint32_t w[8];
      onehot_words(lzi, lyi, lxi, w);
      *reinterpret_cast<uint4*>(sm.qp + sw32_off(rr, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(sm.qp + sw32_off(rr, 1)) = make_uint4(w[4], w[5], w[6], w[7]);
      // visible to the tensor core (async proxy) before the arrival
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
    }
    // The window as bit sets over halo-local positions (in-volume positions
    // only, so zero-filled keys outside the volume are never selected).
    uint64_t zwin = 0, ywin = 0, xwin = 0;
    if (active) {
      zwin = bit_range64(max(cz - g.rz, 0) - tb.hz0, min(cz + g.rz, g.Z - 1) - tb.hz0);
      ywin = bit_range64(max(cy - g.ry, 0) - tb.hy0, min(cy + g.ry, g.Y - 1) - tb.hy0);
      xwin = bit_range64(max(cx - g.rx, 0) - tb.hx0, min(cx + g.rx, g.X - 1) - tb.hx0);
    }
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tbase + lane_base + COL_O;
    const float c2 = g.tau * LOG2E;  // logits -> log2 units
    float m_run = M_FLOOR, l_run = 0.f;
    // the box of blocks this query's window touches (global planes: the
    // block grid of a z-slab is the whole volume's)
    const int bzlo = max(cz + g.zo - g.rz, 0) / g.bz, bzhi = min(cz + g.zo + g.rz, g.Zt - 1) / g.bz;
    const int bylo = max(cy - g.ry, 0) / g.by, byhi = min(cy + g.ry, g.Y - 1) / g.by;
    const int bxlo = max(cx - g.rx, 0) / g.bx, bxhi = min(cx + g.rx, g.X - 1) / g.bx;
    int xc = 0, yc = 0, zc = 0;
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int bi = j & 1;
      const uint32_t tS = tbase + lane_base + COL_S + 64 * bi;
      // a warp leaves together: the TMEM accesses below are warp-collective
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(&sm.s_full[bi], (j >> 1) & 1, WAIT_LIMIT, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t bits0, bits1;
      if (!SUMMARY || j < n_local) {
        // key (dz, dy, dx) of the chunk box is bit (dz * 2 + dy) * 16 + dx
        const uint32_t xp = (uint32_t)(xwin >> (BXK * xc)) & 0xffffu;
        const uint32_t yb = (uint32_t)(ywin >> (BYK * yc)) & 3u;
        const uint32_t zb = (uint32_t)(zwin >> (BZK * zc)) & 3u;
        const uint32_t row16 = ((yb & 1u) ? xp : 0u) | ((yb & 2u) ? (xp << 16) : 0u);
        bits0 = (zb & 1u) ? row16 : 0u;
        bits1 = (zb & 2u) ? row16 : 0u;
        if (++xc == nxc) {
          xc = 0;
          if (++yc == nyc) {
            yc = 0;
            ++zc;
          }
        }
      } else {
        const int B0 = (j - n_local) * KCH;
        const uint64_t m64 = summary_mask64(g, B0, bzlo, bzhi, bylo, byhi, bxlo, bxhi);
        bits0 = (uint32_t)m64;
        bits1 = (uint32_t)(m64 >> 32);
        if (PARTIAL) {
          // empty blocks have no summary (B0 is a multiple of 64)
          const uint32_t* occ = ix.bocc + (int64_t)b * ((g.nb + 31) / 32) + B0 / 32;
          bits0 &= occ[0];
          if (B0 + 32 < g.nb) bits1 &= occ[1];
        }
        if (!active) bits0 = bits1 = 0u;
      }
      const bool skip = __ballot_sync(0xffffffffu, (bits0 | bits1) != 0u) == 0u;
      uint32_t sa[32], sb[32];
      if (!skip) {
        tmem_ld32(tS, sa);
        tmem_ld32(tS + 32, sb);
        tmem_wait_ld();
      }
      uint32_t p[32];
      float corr = 1.f;
      bool rescale_o = false;
      if (skip) {
#pragma unroll
        for (int i = 0; i < 32; ++i) p[i] = 0u;
      } else {
        const bool local = !SUMMARY || j < n_local;  // masked by the penalty channels
        // (most summary chunks mask nothing for any row of the warp)
        if (!local && __any_sync(0xffffffffu, (bits0 & bits1) != 0xffffffffu)) {
          apply_mask(sa, bits0);
          apply_mask(sb, bits1);
        }
        const float cmax = fmaxf(plain_max(sa), plain_max(sb));
        const float cmax2 = cmax * c2;
        if (cmax2 > m_run + RESCALE_THRESHOLD) {
          corr = ex2(m_run - cmax2);
          // O is exactly zero while l is (every P so far was 0)
          rescale_o = l_run != 0.f;
          l_run *= corr;
          m_run = cmax2;
        }
        const float mneg = -m_run;
        // keys 0-63 -> P columns 0-31
        l_run += exp_pack_all(sa, c2, mneg, p);
        l_run += exp_pack_all(sb, c2, mneg, p + 16);
      }
      // P over the first 32 columns of S_j (read above)
      tmem_st32(tS, p);
      if (__any_sync(0xffffffffu, rescale_o)) {
        // O may be rescaled once PV_{j-1} is done (the next product on that
        // barrier, PV_{j+1}, needs this warp's later arrivals)
        if (j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait_or_abort(&sm.buf_free[(j - 1) & 1],
                                                          ((j - 1) >> 1) & 1, WAIT_LIMIT,
                                                          abort_flag));
          if (!ok) break;
          tc_fence_after();
        }
        const float co = rescale_o ? corr : 1.f;
#pragma unroll 1
        for (int part = 0; part < 6; ++part) {
          uint32_t o[16];
          tmem_ld16(tO + part * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * co);
          tmem_st16(tO + part * 16, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[bi]);
    }
    // ---- epilogue ----
    // o_final completes once, after the last PV product.  (Waiting on a
    // buffer's buf_free here could name a phase by a parity the barrier has
    // already passed twice: a wait must never trail the barrier by two phases.)
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_or_abort(&sm.o_final, 0, WAIT_LIMIT, abort_flag));
    if (ok) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const int64_t orow = (((int64_t)b * g.N + qi) * g.H + h) * D;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        uint32_t o[32];
        tmem_ld32(tO + part * 32, o);
        tmem_wait_ld();
        if (active) {
          if (g.out_fp32) {
            float4* dst =
                reinterpret_cast<float4*>(reinterpret_cast<float*>(out_raw) + orow + part * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(
                  __uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                  __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out_raw) +
                                                  orow + part * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(
                  pack_bf16x2(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv,
                              __uint_as_float(o[8 * i + 3]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv,
                              __uint_as_float(o[8 * i + 5]) * inv),
                  pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv,
                              __uint_as_float(o[8 * i + 7]) * inv));
          }
        }
      }
      if (active) lse[((int64_t)b * g.H + h) * g.N + qi] = (m_run + log2f(l_run)) * LN2;
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

// ---- host side --------------------------------------------------------------------

struct WsLayout {
  size_t kg, vg, ks, vs, total;
};

WsLayout ws_layout(const Geo& g) {
  auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t vol = (size_t)g.B * g.H * g.Z * g.Y * g.X * D * 2;
  const size_t sum = (size_t)g.B * g.H * g.nb * D * 2;
  WsLayout w;
  w.kg = 0;
  w.vg = al(vol);
  w.ks = w.vg + al(vol);
  w.vs = w.ks + al(sum);
  w.total = w.vs + al(sum);
  return w;
}

}  // namespace

bool forward_tc_supported(const Geo& g) {
  return g.d == D && g.dtype == PACK3D_BF16 && TZ + 2 * g.rz <= MAX_HALO &&
         TY + 2 * g.ry <= MAX_HALO && TX + 2 * g.rx <= MAX_HALO;
}

size_t forward_tc_workspace_bytes(const Geo& g) {
  return forward_tc_supported(g) ? ws_layout(g).total : 0;
}

int launch_stage_kv(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                    const float* ksum, const float* vsum, void* ws, StageMode mode,
                    cudaStream_t s) {
  const WsLayout w = ws_layout(g);
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (mode == STAGE_COMPUTE)
    return launch_block_summaries_staged(g, idx, k, v, const_cast<float*>(ksum),
                                         const_cast<float*>(vsum), base + w.kg, base + w.vg,
                                         base + w.ks, base + w.vs, s);
  // staging alone: the summary kernel's bulk gather where it applies
  int rc = launch_stage_bulk(g, idx, k, v, base + w.kg, base + w.vg, s);
  if (rc == PACK3D_ERR_UNSUPPORTED) {
    dim3 ggrid((g.X + GRID_XS - 1) / GRID_XS, g.Z * g.Y, g.B);
    k_grid_kv<<<ggrid, 256, 0, s>>>(g, *idx, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                    reinterpret_cast<__nv_bfloat16*>(base + w.kg),
                                    reinterpret_cast<__nv_bfloat16*>(base + w.vg));
    count_launches(1);
  } else if (rc) {
    return rc;
  }
  if (mode == STAGE_CONVERT) {
    const int64_t n4 = (int64_t)g.B * g.H * g.nb * D / 4;
    const int blocks = (int)std::min<int64_t>((n4 + 255) / 256, 148 * 8);
    k_summaries_bf16<<<blocks, 256, 0, s>>>((const float4*)ksum, (const float4*)vsum,
                                            reinterpret_cast<uint2*>(base + w.ks),
                                            reinterpret_cast<uint2*>(base + w.vs), n4, idx->err);
    count_launches(1);
  }
  return cuda_status(cudaGetLastError());
}

int launch_attention_tc(const Geo& g, const pack3d_index* idx, const void* q, void* ws,
                        void* out, float* lse, bool summaries, cudaStream_t s) {
  const WsLayout w = ws_layout(g);
  uint8_t* base = static_cast<uint8_t*>(ws);
  Maps maps;
  const uint64_t vdims[5] = {(uint64_t)D, (uint64_t)g.X, (uint64_t)g.Y, (uint64_t)g.Z,
                             (uint64_t)g.B * g.H};
  const uint32_t vbox[5] = {32, BXK, BYK, BZK, 1};
  const uint64_t sdims[3] = {(uint64_t)D, (uint64_t)g.nb, (uint64_t)g.B * g.H};
  const uint32_t sbox[3] = {32, KCH, 1};
  if (!encode_bf16(&maps.kg, base + w.kg, 5, vdims, vbox) ||
      !encode_bf16(&maps.vg, base + w.vg, 5, vdims, vbox) ||
      !encode_bf16(&maps.ks, base + w.ks, 3, sdims, sbox) ||
      !encode_bf16(&maps.vs, base + w.vs, 3, sdims, sbox))
    return PACK3D_ERR_CUDA;
  dim3 grid(g.nT, g.H, g.B);
  auto kern = summaries ? (g.partial ? k_forward_tc<true, true> : k_forward_tc<true, false>)
                        : (g.partial ? k_forward_tc<false, true> : k_forward_tc<false, false>);
  // Two CTAs per SM: enough shared memory for both, and the largest carveout.
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_REQUEST) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  kern<<<grid, NTHREADS, SMEM_REQUEST, s>>>(g, *idx, (const __nv_bfloat16*)q, maps, out, lse);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
