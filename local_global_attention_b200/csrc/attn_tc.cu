// PACK3D forward on the Blackwell tensor cores (bf16 in, fp32 accumulate).
//
// "Geometry Matters in Packed 3D Attention" (abstract): each query attends
// exactly to its clipped 3D window and to the summaries of the blocks its
// window misses, in one softmax, with axial RoPE on grid coordinates.
//
// One CTA computes one 4 x 4 x 8 query tile (M = 128 rows) of one
// (batch item, head).  The tile's halo (the union of its windows, raster order)
// and then the block summaries are streamed in chunks of 64 keys.  Roles:
//
//   * producers (warps 5-6, one key per thread): gather the query rows once
//     (rotated in registers) and each chunk's key and value rows through the
//     index with cp.async, one chunk ahead, into the 64-byte-swizzled operand
//     layout of a 3-stage shared-memory ring; once a chunk has landed its key
//     rows are rotated in place (axial RoPE, fp32 arithmetic).  head_dim 96 is
//     three 32-channel segments, one per axis, so a rotation segment is exactly
//     one swizzle-atom column.  Summary chunks are converted from fp32 instead;
//   * MMA (warp 4, one thread): S_j = Q K_j^T (six tcgen05.mma, K = 16) into
//     one of two TMEM S buffers, and O += P_j V_j (four tcgen05.mma, A = P from
//     TMEM, B = V MN-major in shared memory), so S_{j+1} is computed while the
//     softmax works on S_j;
//   * softmax (warps 0-3, one query row per thread): builds the chunk's window
//     mask as a bit set from the halo geometry (a few operations per x-row of
//     the halo, not per key), reads S, keeps the online max and sum, writes P
//     (bf16) over S in TMEM.  A warp whose 32 rows have no key in a chunk only
//     writes zeros.  For summary chunks the mask is "block box does not meet
//     the window box"; there is no count bias.  The running max moves only when
//     a row's maximum grows by more than 8 (log2 units), so O is rescaled in
//     TMEM rarely; the result is the same softmax.
//
// The epilogue divides by the row sum and writes out (packed order) and the
// natural-log LSE.  Two CTAs share an SM (256 TMEM columns each).  Every wait
// is bounded; a CTA that gives up sets the timeout bit of the index error word.
#include <math.h>

#include "pack3d_internal.cuh"
#include "tc_primitives.cuh"

namespace p3d {

namespace {

using namespace tc;

constexpr int D = 96;                  // head dim handled by this kernel
constexpr int KCH = 64;                // keys per chunk (N of the S MMA)
constexpr int NSTAGE = 3;              // K/V shared-memory ring depth
constexpr int QSEG = 128 * 64;         // one 32-channel segment of the 128 query rows
constexpr int KSEG = KCH * 64;         // one 32-channel segment of a chunk
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_O = 0;          // O accumulator: columns [0, 96)
constexpr uint32_t COL_S = 128;        // S/P buffer b: columns [128 + 64 b, 192 + 64 b)
constexpr int MMA_WARP = 4;
constexpr int PROD0 = 160;             // first producer thread
constexpr int NPROD = KCH;             // one producer thread per key of a chunk
constexpr int NTHREADS = PROD0 + NPROD;
constexpr uint32_t WAIT_LIMIT = 1u << 20;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int ERR_TIMEOUT_BIT = 4;

struct Smem {
  uint8_t q[3 * QSEG];
  uint8_t k[NSTAGE][3 * KSEG];
  uint8_t v[NSTAGE][3 * KSEG];
  uint64_t q_full;
  uint64_t kv_full[NSTAGE];
  uint64_t kv_empty[NSTAGE];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;   // one phase per PV product
  uint64_t o_final;  // one phase: every PV product of the tile is done
  uint32_t tmem_base;
  int32_t abort;
};
constexpr size_t SMEM_REQUEST = sizeof(Smem) + 1024;  // + alignment slack

struct TileBox {
  int z0, y0, x0, lz, ly, lx;
  int hz0, hy0, hx0, hz, hy, hx;
};

__device__ __forceinline__ TileBox tile_box(const Geo& g, int t) {
  TileBox tb;
  int Tx = t % g.nTx, Ty = (t / g.nTx) % g.nTy, Tz = t / (g.nTx * g.nTy);
  tb.z0 = Tz * TZ;
  tb.y0 = Ty * TY;
  tb.x0 = Tx * TX;
  tb.lz = min(TZ, g.Z - tb.z0);
  tb.ly = min(TY, g.Y - tb.y0);
  tb.lx = min(TX, g.X - tb.x0);
  tb.hz0 = max(0, tb.z0 - g.rz);
  tb.hy0 = max(0, tb.y0 - g.ry);
  tb.hx0 = max(0, tb.x0 - g.rx);
  tb.hz = min(g.Z, tb.z0 + tb.lz + g.rz) - tb.hz0;
  tb.hy = min(g.Y, tb.y0 + tb.ly + g.ry) - tb.hy0;
  tb.hx = min(g.X, tb.x0 + tb.lx + g.rx) - tb.hx0;
  return tb;
}

// ---- producer helpers --------------------------------------------------------

// Rotate four words of pair members (lo) against their partners (hi): word u of
// lo holds channels j0 + 2u, j0 + 2u + 1 of a segment, word u of hi the same
// pairs' second members.  t = rotation table row of the segment's axis.
__device__ __forceinline__ void rot_chunk(uint4& lo, uint4& hi, const float2* __restrict__ t,
                                          int j0) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float2 x1 = unpack_bf16x2(a[u]), x2 = unpack_bf16x2(b[u]);
    float2 c0 = __ldg(t + j0 + 2 * u), c1 = __ldg(t + j0 + 2 * u + 1);
    a[u] = pack_bf16x2(x1.x * c0.x - x2.x * c0.y, x1.y * c1.x - x2.y * c1.y);
    b[u] = pack_bf16x2(x1.x * c0.y + x2.x * c0.x, x1.y * c1.y + x2.y * c1.x);
  }
}

__device__ __forceinline__ const float2* rope_row(const float2* tab, const Geo& g, int axis,
                                                  int c) {
  int off = axis == 0 ? 0 : (axis == 1 ? g.Z : g.Z + g.Y);
  return tab + (off + c) * 16;
}

// Axial rotation of a whole 96-channel row held as 12 chunks: segment a is
// chunks 4a..4a+3, and word w of a segment pairs with word w + 8.
__device__ __forceinline__ void rotate_row(uint4 (&r)[12], const float2* __restrict__ tab,
                                           const Geo& g, int cz, int cy, int cx) {
  const float2* tz = rope_row(tab, g, 0, cz);
  const float2* ty = rope_row(tab, g, 1, cy);
  const float2* tx = rope_row(tab, g, 2, cx);
  rot_chunk(r[0], r[2], tz, 0);
  rot_chunk(r[1], r[3], tz, 8);
  rot_chunk(r[4], r[6], ty, 0);
  rot_chunk(r[5], r[7], ty, 8);
  rot_chunk(r[8], r[10], tx, 0);
  rot_chunk(r[9], r[11], tx, 8);
}

// 16-byte chunk c (0..11) of a 96-channel row <-> its place in an operand
// region (three 32-channel segments of seg_bytes each, 64-byte swizzle).
__device__ __forceinline__ void store_chunk(uint8_t* region, int seg_bytes, int row, int c,
                                            const uint4& v) {
  *reinterpret_cast<uint4*>(region + (c >> 2) * seg_bytes + sw64_off(row, c & 3)) = v;
}
__device__ __forceinline__ uint4 load_chunk(const uint8_t* region, int seg_bytes, int row, int c) {
  return *reinterpret_cast<const uint4*>(region + (c >> 2) * seg_bytes + sw64_off(row, c & 3));
}

// ---- softmax helpers -------------------------------------------------------------

// Window mask of 32 consecutive halo keys [e0, e0 + 32) for one query.  The
// halo is an hz x hy x hx box in raster order; the query's window is
// |z - qz| <= rz, |y - qy| <= ry, x in [xlo, xhi] (halo-local coordinates).
// The loop walks the halo x-rows the 32 keys touch (same trip count for every
// thread); keys at or beyond nh are masked off.
__device__ __forceinline__ uint32_t local_bits(int e0, int nh, int hx, int hy, int qz, int qy,
                                               int rz, int ry, int xlo, int xhi) {
  uint32_t bits = 0;
  int r = e0 / hx;
  int z = r / hy, y = r - z * hy;
  int pos = r * hx - e0;  // bit position of x = 0 of row r (<= 0)
  while (pos < 32) {
    if (abs(z - qz) <= rz && abs(y - qy) <= ry) {
      int lo = max(pos + xlo, 0), hi = min(pos + xhi, 31);
      if (lo <= hi) bits |= bit_range(lo, hi);
    }
    pos += hx;
    if (++y == hy) {
      y = 0;
      ++z;
    }
  }
  int valid = nh - e0;
  if (valid < 32) bits &= valid <= 0 ? 0u : (0xffffffffu >> (32 - valid));
  return bits;
}

// Summary mask of 32 consecutive blocks [B0, B0 + 32) (raster order over an
// nbz x nby x nbx grid): set for blocks that do not meet the query's window,
// i.e. outside the box [blo, bhi] of blocks the window touches.
__device__ __forceinline__ uint32_t summary_bits(int B0, int nb, int nbx, int nby, int bzlo,
                                                 int bzhi, int bylo, int byhi, int bxlo,
                                                 int bxhi) {
  uint32_t bits = 0;
  int r = B0 / nbx;
  int z = r / nby, y = r - z * nby;
  int pos = r * nbx - B0;
  while (pos < 32) {
    int lo = max(pos, 0), hi = min(pos + nbx - 1, 31);
    if (lo <= hi) {
      uint32_t row = bit_range(lo, hi);
      if (z >= bzlo && z <= bzhi && y >= bylo && y <= byhi) {
        int elo = max(pos + bxlo, 0), ehi = min(pos + bxhi, 31);
        if (elo <= ehi) row &= ~bit_range(elo, ehi);
      }
      bits |= row;
    }
    pos += nbx;
    if (++y == nby) {
      y = 0;
      ++z;
    }
  }
  int valid = nb - B0;
  if (valid < 32) bits &= valid <= 0 ? 0u : (0xffffffffu >> (32 - valid));
  return bits;
}

template <bool SUMMARY>
__global__ void __launch_bounds__(NTHREADS, 2)
    k_forward_tc(Geo g, pack3d_index ix, const __nv_bfloat16* __restrict__ q,
                 const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                 const float* __restrict__ ksum, const float* __restrict__ vsum,
                 void* __restrict__ out_raw, float* __restrict__ lse) {
  if (ix.err[0]) return;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~(uintptr_t)1023);
  volatile int32_t* abort_flag = &sm.abort;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const TileBox tb = tile_box(g, t);
  const int count = tb.lz * tb.ly * tb.lx;
  const int nh = tb.hz * tb.hy * tb.hx;
  const int n_local = (nh + KCH - 1) / KCH;
  const int n_sum = SUMMARY ? (g.nb + KCH - 1) / KCH : 0;
  const int nch = n_local + n_sum;
  const int toff = ix.tile_off[(int64_t)b * (g.nT + 1) + t];

  if (tid == 0) {
    mbar_init(&sm.q_full, NPROD);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&sm.kv_full[s], NPROD);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.o_final, 1);
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

  if (tid >= PROD0) {
    // ================= producers (one key row of each chunk per thread) =================
    const int pt = tid - PROD0;
    const float2* __restrict__ tab = reinterpret_cast<const float2*>(ix.rope);
    // queries: rows pt and pt + 64, gathered, rotated, stored once
    for (int qr = pt; qr < 128; qr += NPROD) {
      uint4 r[12];
      if (qr < count) {
        const int cx = tb.x0 + qr % tb.lx, cy = tb.y0 + (qr / tb.lx) % tb.ly,
                  cz = tb.z0 + qr / (tb.lx * tb.ly);
        const int qi = ix.perm[(int64_t)b * g.N + toff + qr];
        const uint4* src =
            reinterpret_cast<const uint4*>(q + (((int64_t)b * g.N + qi) * g.H + h) * D);
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = __ldg(src + i);
        rotate_row(r, tab, g, cz, cy, cx);
      } else {
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 12; ++i) store_chunk(sm.q, QSEG, qr, i, r[i]);
    }
    fence_proxy_async_smem();
    mbar_arrive(&sm.q_full);

    const int key = pt;
    const int32_t* __restrict__ hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
    const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
    // Local chunks: the raw key and value rows are copied asynchronously into
    // the chunk's stage one chunk ahead; once they have landed the key row is
    // rotated in place.  Returns false if a wait gave up.
    auto issue = [&](int j) -> bool {
      const int s = j % NSTAGE, round = j / NSTAGE;
      if (round > 0 &&
          !mbar_wait_or_abort(&sm.kv_empty[s], (round - 1) & 1, WAIT_LIMIT, abort_flag))
        return false;
      if (j < n_local) {
        const int e = j * KCH + key;
        if (e < nh) {
          const int64_t row = (((int64_t)b * g.N + hl[e]) * g.H + h) * D;
          const uint4* ks = reinterpret_cast<const uint4*>(k + row);
          const uint4* vs = reinterpret_cast<const uint4*>(v + row);
#pragma unroll
          for (int c = 0; c < 12; ++c) {
            cp_async16(sm.k[s] + (c >> 2) * KSEG + sw64_off(key, c & 3), ks + c);
            cp_async16(sm.v[s] + (c >> 2) * KSEG + sw64_off(key, c & 3), vs + c);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 12; ++c) {
            store_chunk(sm.k[s], KSEG, key, c, make_uint4(0, 0, 0, 0));
            store_chunk(sm.v[s], KSEG, key, c, make_uint4(0, 0, 0, 0));
          }
        }
      }
      cp_async_commit();
      return true;
    };
    bool ok = issue(0);
    for (int j = 0; j < nch && ok; ++j) {
      const int s = j % NSTAGE;
      if (j + 1 < nch) {
        ok = issue(j + 1);
        if (!ok) break;
        cp_async_wait_group<1>();
      } else {
        cp_async_wait_group<0>();
      }
      if (j < n_local) {
        const int e = j * KCH + key;
        if (e < nh) {
          const int x = tb.hx0 + e % tb.hx, y = tb.hy0 + (e / tb.hx) % tb.hy,
                    z = tb.hz0 + e / (tb.hx * tb.hy);
          uint4 r[12];
#pragma unroll
          for (int c = 0; c < 12; ++c) r[c] = load_chunk(sm.k[s], KSEG, key, c);
          rotate_row(r, tab, g, z, y, x);
#pragma unroll
          for (int c = 0; c < 12; ++c) store_chunk(sm.k[s], KSEG, key, c, r[c]);
        }
      } else {
        // summaries: fp32 rows converted to bf16 (keys already rotated)
        const int B = (j - n_local) * KCH + key;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const float* src = which ? vsum : ksum;
          uint8_t* dst = which ? sm.v[s] : sm.k[s];
#pragma unroll 4
          for (int c = 0; c < 12; ++c) {
            uint4 w = make_uint4(0, 0, 0, 0);
            if (B < g.nb) {
              const float4* f = reinterpret_cast<const float4*>(src + (sbase + B) * D);
              float4 a0 = __ldg(f + 2 * c), a1 = __ldg(f + 2 * c + 1);
              w = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                             pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
            }
            store_chunk(dst, KSEG, key, c, w);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.kv_full[s]);
    }
    cp_async_wait_group<0>();
  } else if (warp == MMA_WARP) {
    // ================= MMA issue =================
    if (lane == 0) {
      const uint32_t qa = smem_u32(sm.q);
      constexpr uint32_t idesc_s = idesc_bf16(128, KCH, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, D, true);
      bool ok = mbar_wait_or_abort(&sm.q_full, 0, WAIT_LIMIT, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j % NSTAGE;
        if (!mbar_wait_or_abort(&sm.kv_full[s], (j / NSTAGE) & 1, WAIT_LIMIT, abort_flag))
          return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sm.k[s]);
        const uint32_t dst = tbase + COL_S + 64 * (j & 1);
#pragma unroll
        for (int st = 0; st < D / 16; ++st) {
          const uint32_t sub = (st & 1) * 32;
          mma_ss(dst, sdesc_sw64(qa + (st >> 1) * QSEG + sub, 16, 512),
                 sdesc_sw64(ka + (st >> 1) * KSEG + sub, 16, 512), idesc_s, st > 0);
        }
        mma_commit(&sm.s_full[j & 1]);
        return true;
      };
      if (ok) {
        tc_fence_after();
        for (int j = 0; j < nch && j < 2 && ok; ++j) ok = issue_s(j);
      }
      for (int j = 0; j < nch && ok; ++j) {
        if (!mbar_wait_or_abort(&sm.p_full[j & 1], (j >> 1) & 1, WAIT_LIMIT, abort_flag)) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sm.v[j % NSTAGE]);
        const uint32_t pa = tbase + COL_S + 64 * (j & 1);
#pragma unroll
        for (int st = 0; st < KCH / 16; ++st)
          mma_ts(tbase + COL_O, pa + 8 * st, sdesc_sw64(va + st * 16 * 64, KSEG, 512), idesc_o,
                 (j > 0 || st > 0) ? 1u : 0u);
        mma_commit(&sm.o_done);
        mma_commit(&sm.kv_empty[j % NSTAGE]);
        if (j == nch - 1) mma_commit(&sm.o_final);
        if (j + 2 < nch) {
          // S buffer j & 1 holds P_j until this PV has read it
          if (!mbar_wait_or_abort(&sm.o_done, j & 1, WAIT_LIMIT, abort_flag)) break;
          ok = issue_s(j + 2);
        }
      }
    }
    __syncwarp();
  } else {
    // ================= softmax (one query row per thread) =================
    const bool active = tid < count;
    int cz = 0, cy = 0, cx = 0, qi = 0;
    if (active) {
      cx = tb.x0 + tid % tb.lx;
      cy = tb.y0 + (tid / tb.lx) % tb.ly;
      cz = tb.z0 + tid / (tb.lx * tb.ly);
      qi = ix.perm[(int64_t)b * g.N + toff + tid];
    }
    const int qz = cz - tb.hz0, qy = cy - tb.hy0, qx = cx - tb.hx0;
    const int xlo = max(qx - g.rx, 0), xhi = min(qx + g.rx, tb.hx - 1);
    const int bzlo = max(cz - g.rz, 0) / g.bz, bzhi = min(cz + g.rz, g.Z - 1) / g.bz;
    const int bylo = max(cy - g.ry, 0) / g.by, byhi = min(cy + g.ry, g.Y - 1) / g.by;
    const int bxlo = max(cx - g.rx, 0) / g.bx, bxhi = min(cx + g.rx, g.X - 1) / g.bx;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tbase + lane_base + COL_O;
    const float c2 = g.tau * LOG2E;  // logits -> log2 units
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int buf = j & 1;
      // a warp leaves together: the TMEM accesses below are warp-collective
      ok = __all_sync(0xffffffffu,
                      mbar_wait_or_abort(&sm.s_full[buf], (j >> 1) & 1, WAIT_LIMIT, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tbase + lane_base + COL_S + 64 * buf;
      uint32_t bits0, bits1;
      if (j < n_local) {
        bits0 = local_bits(j * KCH, nh, tb.hx, tb.hy, qz, qy, g.rz, g.ry, xlo, xhi);
        bits1 = local_bits(j * KCH + 32, nh, tb.hx, tb.hy, qz, qy, g.rz, g.ry, xlo, xhi);
      } else {
        const int B0 = (j - n_local) * KCH;
        bits0 = summary_bits(B0, g.nb, g.nbx, g.nby, bzlo, bzhi, bylo, byhi, bxlo, bxhi);
        bits1 = summary_bits(B0 + 32, g.nb, g.nbx, g.nby, bzlo, bzhi, bylo, byhi, bxlo, bxhi);
      }
      if (!active) bits0 = bits1 = 0u;
      if (__ballot_sync(0xffffffffu, (bits0 | bits1) != 0u) == 0u) {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tmem_st16(tS, z);
        tmem_st16(tS + 16, z);
      } else {
        // pass 1: masked row maximum over the 64 keys
        float cmax = -INFINITY;
        {
          uint32_t sv[32];
          tmem_ld32(tS, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if ((bits0 >> i) & 1u) cmax = fmaxf(cmax, __uint_as_float(sv[i]));
          tmem_ld32(tS + 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if ((bits1 >> i) & 1u) cmax = fmaxf(cmax, __uint_as_float(sv[i]));
        }
        const float cmax2 = cmax * c2;
        float corr = 1.f;
        if (cmax2 > m_run + RESCALE_THRESHOLD) {
          if (m_run != -INFINITY) corr = ex2(m_run - cmax2);
          l_run *= corr;
          m_run = cmax2;
        }
        if (__any_sync(0xffffffffu, corr != 1.f)) {
          // O must hold every earlier PV product before it is rescaled
          ok = __all_sync(0xffffffffu,
                          mbar_wait_or_abort(&sm.o_done, (j - 1) & 1, WAIT_LIMIT, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int part = 0; part < 3; ++part) {
            uint32_t o[32];
            tmem_ld32(tO + part * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
            tmem_st32(tO + part * 32, o);
          }
        }
        const float mneg = m_run == -INFINITY ? 0.f : -m_run;
        // pass 2: P over S; keys 0-31 -> columns 0-15, keys 32-63 -> columns
        // 16-31 (columns whose S values have been read by then)
#pragma unroll 1
        for (int seg = 0; seg < 2; ++seg) {
          const uint32_t bits = seg ? bits1 : bits0;
          uint32_t sv[32], p[16];
          tmem_ld32(tS + 32 * seg, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a0 = ((bits >> (2 * i)) & 1u) ? fmaf(__uint_as_float(sv[2 * i]), c2, mneg) : -INFINITY;
            float a1 = ((bits >> (2 * i + 1)) & 1u) ? fmaf(__uint_as_float(sv[2 * i + 1]), c2, mneg) : -INFINITY;
            float e0 = ex2(a0), e1 = ex2(a1);
            l_run += e0 + e1;
            p[i] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tS + 16 * seg, p);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[buf]);
    }
    // ---- epilogue ----
    // o_final completes once, after the last PV product.  (Waiting on o_done
    // here could name a phase by a parity the barrier has already passed twice:
    // a wait must never trail the barrier by two phases.)
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
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

}  // namespace

bool forward_tc_supported(const Geo& g) { return g.d == D && g.dtype == PACK3D_BF16; }

int launch_forward_tc(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                      const void* v, const float* ksum, const float* vsum, void* out, float* lse,
                      bool summaries, cudaStream_t s) {
  dim3 grid(g.nT, g.H, g.B);
  auto kern = summaries ? k_forward_tc<true> : k_forward_tc<false>;
  // Two CTAs per SM: enough shared memory for both, and the largest carveout.
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)SMEM_REQUEST) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  kern<<<grid, NTHREADS, SMEM_REQUEST, s>>>(g, *idx, (const __nv_bfloat16*)q,
                                             (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                             ksum, vsum, out, lse);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
