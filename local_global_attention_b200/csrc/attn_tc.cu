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
//   * producers (warps 5-6, one key per thread): copy each chunk's key and
//     value rows through the index with cp.async, two chunks ahead, into the
//     64-byte-swizzled operand layout of a 3-stage shared-memory ring, and
//     rotate a chunk's key rows in place once they have landed (axial RoPE, fp32 arithmetic, the
//     rotation-table rows of the tile's halo staged in shared memory), or
//     convert summary rows from fp32.  head_dim 96 is three 32-channel
//     segments, one per axis, so a rotation segment is exactly one swizzle-atom
//     column;
//   * MMA (warp 4, one thread): S_j = Q K_j^T (six tcgen05.mma, K = 16) into
//     one of two TMEM S buffers, and O += P_j V_j (four tcgen05.mma, A = P from
//     TMEM, B = V MN-major in shared memory), so S_{j+1} is computed while the
//     softmax works on S_j;
//   * softmax warps (0-3, one query row per thread): gather and rotate the
//     query rows once; per chunk build the window mask as a bit set from the
//     halo geometry (a few operations per halo x-row, walked with a cursor, not
//     per key), read S, keep the online max and sum, write P (bf16) over S in
//     TMEM.  A warp whose 32 rows have no key in a chunk only writes zeros.
//     For summary chunks the mask is "block box does not meet the window box";
//     there is no count bias.  The running max moves only when a row's maximum
//     grows by more than 8 (log2 units), so O is rescaled in TMEM rarely; the
//     result is the same softmax.
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
constexpr int TAB_ROWS = 64;           // rotation-table rows staged in shared memory
constexpr int TAB_STRIDE = 18;         // float2 per staged row: 16 + 2 of padding, so rows
                                       // of consecutive coordinates start on different banks

struct Smem {
  uint8_t q[3 * QSEG];
  uint8_t k[NSTAGE][3 * KSEG];
  uint8_t v[NSTAGE][3 * KSEG];
  float2 tab[TAB_ROWS * TAB_STRIDE];  // rotation-table rows of the halo box
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

// ---- rotation ------------------------------------------------------------------

// Rotate four words of pair members (lo) against their partners (hi): word u of
// lo holds channels j0 + 2u, j0 + 2u + 1 of a segment, word u of hi the same
// pairs' second members.  t = rotation-table row of the segment's axis.
__device__ __forceinline__ void rot_chunk(uint4& lo, uint4& hi, const float2* t, int j0) {
  uint32_t* a = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* b = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float2 x1 = unpack_bf16x2(a[u]), x2 = unpack_bf16x2(b[u]);
    const float4 cs = *reinterpret_cast<const float4*>(t + j0 + 2 * u);  // pairs j, j + 1
    a[u] = pack_bf16x2(x1.x * cs.x - x2.x * cs.y, x1.y * cs.z - x2.y * cs.w);
    b[u] = pack_bf16x2(x1.x * cs.y + x2.x * cs.x, x1.y * cs.w + x2.y * cs.z);
  }
}

// Rows of the rotation table (16 (cos, sin) pairs per coordinate value) for the
// coordinates a tile can touch: its halo box, staged in shared memory when they
// fit (z rows, then y rows, then x rows), else read from the global table.
struct RopeRows {
  const float2* z;  // row of coordinate c is z + (c - bz) * stride
  const float2* y;
  const float2* x;
  int bz, by, bx, stride;
  __device__ __forceinline__ const float2* row(int axis, int c) const {
    return axis == 0 ? z + (c - bz) * stride
                     : (axis == 1 ? y + (c - by) * stride : x + (c - bx) * stride);
  }
};

// Axial rotation of a whole 96-channel row held as 12 chunks: segment a is
// chunks 4a..4a+3, and word w of a segment pairs with word w + 8.
__device__ __forceinline__ void rotate_row(uint4 (&r)[12], const RopeRows& rr, int cz, int cy,
                                           int cx) {
  const float2* tz = rr.row(0, cz);
  const float2* ty = rr.row(1, cy);
  const float2* tx = rr.row(2, cx);
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

// ---- masks ---------------------------------------------------------------------

// Walks the rows of a raster-ordered box (rows of `len` items, `ny` rows per
// plane) in step with 32-item segments, so no division is needed per segment.
struct RowCursor {
  int start;  // index of the first item of the current row
  int z, y;   // the current row's plane and row within the plane
  int row;    // the current row's raster index (z * ny + y)
  __device__ __forceinline__ void advance_to(int e, int len, int ny) {
    while (start + len <= e) {
      start += len;
      ++row;
      if (++y == ny) {
        y = 0;
        ++z;
      }
    }
  }
};

// Window mask of the 32 halo keys [e0, e0 + 32) for one query: the halo is an
// hz x hy x hx box in raster order and the window is |z - qz| <= rz,
// |y - qy| <= ry, x in [xlo, xhi] (halo-local).  `c` is at the row holding e0.
__device__ __forceinline__ uint32_t local_bits(RowCursor c, int e0, int nh, int hx, int hy, int qz,
                                               int qy, int rz, int ry, int xlo, int xhi) {
  uint32_t bits = 0;
  int pos = c.start - e0;  // bit of x = 0 of the current row (<= 0)
  int z = c.z, y = c.y;
  while (pos < 32) {
    if (abs(z - qz) <= rz && abs(y - qy) <= ry) {
      const int lo = max(pos + xlo, 0), hi = min(pos + xhi, 31);
      if (lo <= hi) bits |= bit_range(lo, hi);
    }
    pos += hx;
    if (++y == hy) {
      y = 0;
      ++z;
    }
  }
  const int valid = nh - e0;
  if (valid < 32) bits &= valid <= 0 ? 0u : (0xffffffffu >> (32 - valid));
  return bits;
}

// Summary mask of the 32 blocks [B0, B0 + 32) (raster order over an
// nbz x nby x nbx grid): set for blocks outside the box [blo, bhi] of blocks
// the query's window touches.  `c` is at the block row holding B0.
__device__ __forceinline__ uint32_t summary_bits(RowCursor c, int B0, int nb, int nbx, int nby,
                                                 int bzlo, int bzhi, int bylo, int byhi, int bxlo,
                                                 int bxhi) {
  uint32_t bits = 0;
  int pos = c.start - B0;
  int z = c.z, y = c.y;
  while (pos < 32) {
    const int lo = max(pos, 0), hi = min(pos + nbx - 1, 31);
    if (lo <= hi) {
      uint32_t row = bit_range(lo, hi);
      if (z >= bzlo && z <= bzhi && y >= bylo && y <= byhi) {
        const int elo = max(pos + bxlo, 0), ehi = min(pos + bxhi, 31);
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
  const int valid = nb - B0;
  if (valid < 32) bits &= valid <= 0 ? 0u : (0xffffffffu >> (32 - valid));
  return bits;
}

// Precomputed form of the masks above for boxes whose rows fit 128 bits and
// whose rows are at most 32 items long: `rows` has bit r set for the rows r
// (raster over z, y) the mask keeps or drops as a whole, and `pattern` is the
// per-row item mask repeated with period `len` over 64 bits.  For the 32 items
// [e0, e0 + 32), with the cursor at the row holding e0, the result is
// (row bit AND pattern bit) per item - a handful of bit operations, no
// data-dependent branches.
struct RowMask {
  uint32_t rows[4];
  uint64_t pattern;
  __device__ __forceinline__ uint32_t row_bit(int r) const {
    const int w = r >> 5;
    const uint32_t word = w == 0 ? rows[0] : (w == 1 ? rows[1] : (w == 2 ? rows[2] : rows[3]));
    return (word >> (r & 31)) & 1u;
  }
  // items of [e0, e0 + 32) whose row bit and pattern bit are both set
  __device__ __forceinline__ uint32_t segment(const RowCursor& c, int e0, int len) const {
    const int off = e0 - c.start;          // position of e0 inside its row
    const int r0 = c.row;                  // index of the row holding e0
    const uint32_t xb = (uint32_t)(pattern >> off);
    uint32_t rb = 0;
    for (int k = 0, lo = -off; lo < 32; ++k, lo += len) {
      const uint32_t m = bit_range(max(lo, 0), min(lo + len - 1, 31));
      rb |= row_bit(r0 + k) ? m : 0u;
    }
    return rb & xb;
  }
};

__device__ __forceinline__ uint64_t periodic(uint32_t m, int len) {
  uint64_t p = m;
  for (int s = len; s < 64; s += len) p |= (uint64_t)m << s;
  return p;
}

// P = 2^(S c2 + mneg) for the keys in `bits`, 0 elsewhere; returns the sum.
__device__ __forceinline__ float exp_pack(const uint32_t (&sv)[32], uint32_t bits, float c2,
                                          float mneg, uint32_t (&p)[16]) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float a0 = ((bits >> (2 * i)) & 1u) ? fmaf(__uint_as_float(sv[2 * i]), c2, mneg)
                                              : -INFINITY;
    const float a1 = ((bits >> (2 * i + 1)) & 1u) ? fmaf(__uint_as_float(sv[2 * i + 1]), c2, mneg)
                                                  : -INFINITY;
    const float e0 = ex2(a0), e1 = ex2(a1);
    acc[i & 3] += e0 + e1;
    p[i] = pack_bf16x2(e0, e1);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Maximum of S over the keys in `bits` (-inf if none), with independent chains.
__device__ __forceinline__ float masked_max(const uint32_t (&sv)[32], uint32_t bits) {
  float m[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if ((bits >> i) & 1u) m[i & 3] = fmaxf(m[i & 3], __uint_as_float(sv[i]));
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
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
    mbar_init(&sm.q_full, 128);
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
  // rotation-table rows of the halo box (all threads stage; producers and
  // softmax warps read)
  RopeRows rr;
  {
    const float2* gt = reinterpret_cast<const float2*>(ix.rope);
    const int rows = tb.hz + tb.hy + tb.hx;
    if (rows <= TAB_ROWS) {
      for (int e = tid; e < rows * 16; e += NTHREADS) {
        const int r = e / 16, jj = e % 16;
        const int grow = r < tb.hz ? tb.hz0 + r
                                   : (r < tb.hz + tb.hy ? g.Z + tb.hy0 + r - tb.hz
                                                        : g.Z + g.Y + tb.hx0 + r - tb.hz - tb.hy);
        sm.tab[r * TAB_STRIDE + jj] = gt[grow * 16 + jj];
      }
      rr.z = sm.tab;
      rr.y = sm.tab + tb.hz * TAB_STRIDE;
      rr.x = sm.tab + (tb.hz + tb.hy) * TAB_STRIDE;
      rr.bz = tb.hz0;
      rr.by = tb.hy0;
      rr.bx = tb.hx0;
      rr.stride = TAB_STRIDE;
    } else {
      rr.z = gt;
      rr.y = gt + g.Z * 16;
      rr.x = gt + (g.Z + g.Y) * 16;
      rr.bz = rr.by = rr.bx = 0;
      rr.stride = 16;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  if (tid >= PROD0) {
    // ================= producers (one key row of each chunk per thread) =================
    const int key = tid - PROD0;
    const int32_t* __restrict__ hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
    const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
    int next_row = (key < nh) ? hl[key] : 0;  // neighbour index of the next chunk to issue
    // Copy chunk j's raw key and value rows into its stage (zero rows past the
    // halo); one cp.async group per chunk.  False if a wait gave up.
    auto issue = [&](int j) -> bool {
      const int s = j % NSTAGE, round = j / NSTAGE;
      const int row_idx = next_row;
      if (j + 1 < n_local) {
        const int en = (j + 1) * KCH + key;
        next_row = en < nh ? hl[en] : 0;
      }
      if (round > 0 &&
          !mbar_wait_or_abort(&sm.kv_empty[s], (round - 1) & 1, WAIT_LIMIT, abort_flag))
        return false;
      if (j < n_local) {
        const int e = j * KCH + key;
        if (e < nh) {
          const int64_t row = (((int64_t)b * g.N + row_idx) * g.H + h) * D;
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
            cp_async16_zero(sm.k[s] + (c >> 2) * KSEG + sw64_off(key, c & 3), k);
            cp_async16_zero(sm.v[s] + (c >> 2) * KSEG + sw64_off(key, c & 3), v);
          }
        }
      }
      cp_async_commit();
      return true;
    };
    // Two chunks in flight: chunk j + 2 is issued after chunk j has been
    // rotated (issuing it first would wait on chunk j - 1's PV product, which
    // the MMA thread issues only after S_j, i.e. after this rotation).
    bool ok = issue(0);
    if (ok && nch > 1) ok = issue(1);
    // the halo-local coordinate of this thread's key in chunk j, advanced
    // without division
    int kx = key % tb.hx, ky = (key / tb.hx) % tb.hy, kz = key / (tb.hx * tb.hy);
    for (int j = 0; j < nch && ok; ++j) {
      const int s = j % NSTAGE;
      if (j + 1 < nch)
        cp_async_wait_group<1>();  // chunk j + 1 may still be in flight
      else
        cp_async_wait_group<0>();
      if (j < n_local) {
        if (j * KCH + key < nh) {
          uint4 r[12];
#pragma unroll
          for (int c = 0; c < 12; ++c) r[c] = load_chunk(sm.k[s], KSEG, key, c);
          rotate_row(r, rr, tb.hz0 + kz, tb.hy0 + ky, tb.hx0 + kx);
#pragma unroll
          for (int c = 0; c < 12; ++c) store_chunk(sm.k[s], KSEG, key, c, r[c]);
        }
        kx += KCH;
        while (kx >= tb.hx) {
          kx -= tb.hx;
          if (++ky == tb.hy) {
            ky = 0;
            ++kz;
          }
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
              const float4 a0 = __ldg(f + 2 * c), a1 = __ldg(f + 2 * c + 1);
              w = make_uint4(pack_bf16x2(a0.x, a0.y), pack_bf16x2(a0.z, a0.w),
                             pack_bf16x2(a1.x, a1.y), pack_bf16x2(a1.z, a1.w));
            }
            store_chunk(dst, KSEG, key, c, w);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.kv_full[s]);
      if (j + 2 < nch) ok = issue(j + 2);
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
    // ================= softmax warps (one query row per thread) =================
    const bool active = tid < count;
    int cz = 0, cy = 0, cx = 0, qi = 0;
    if (active) {
      cx = tb.x0 + tid % tb.lx;
      cy = tb.y0 + (tid / tb.lx) % tb.ly;
      cz = tb.z0 + tid / (tb.lx * tb.ly);
      qi = ix.perm[(int64_t)b * g.N + toff + tid];
    }
    {
      // this thread's query row: gathered, rotated, stored once
      uint4 r[12];
      if (active) {
        const uint4* src =
            reinterpret_cast<const uint4*>(q + (((int64_t)b * g.N + qi) * g.H + h) * D);
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = __ldg(src + i);
        rotate_row(r, rr, cz, cy, cx);
      } else {
#pragma unroll
        for (int i = 0; i < 12; ++i) r[i] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < 12; ++i) store_chunk(sm.q, QSEG, tid, i, r[i]);
      fence_proxy_async_smem();
      mbar_arrive(&sm.q_full);
    }
    const int qz = cz - tb.hz0, qy = cy - tb.hy0, qx = cx - tb.hx0;
    const int xlo = max(qx - g.rx, 0), xhi = min(qx + g.rx, tb.hx - 1);
    // Precomputed window mask (halo rows in the window; x range as a periodic
    // pattern) when the halo's rows fit, else the per-row walk.
    const bool fast_local = tb.hz * tb.hy <= 128 && tb.hx <= 32;
    RowMask lm;
    if (fast_local) {
      lm.rows[0] = lm.rows[1] = lm.rows[2] = lm.rows[3] = 0u;
      const int ylo = max(qy - g.ry, 0), yhi = min(qy + g.ry, tb.hy - 1);
      for (int z = max(qz - g.rz, 0); z <= min(qz + g.rz, tb.hz - 1); ++z) {
        // rows z * hy + [ylo, yhi] of plane z, spread over the four words
        const int a = z * tb.hy + ylo, e = z * tb.hy + yhi;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int lo = max(a - 32 * w, 0), hi = min(e - 32 * w, 31);
          if (lo <= hi) lm.rows[w] |= bit_range(lo, hi);
        }
      }
      lm.pattern = periodic(bit_range(xlo, xhi), tb.hx);
    }
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tbase + lane_base + COL_O;
    const float c2 = g.tau * LOG2E;  // logits -> log2 units
    float m_run = -INFINITY, l_run = 0.f;
    RowCursor hc = {0, 0, 0, 0};  // halo rows (hx keys each, hy rows per plane)
    RowCursor bc = {0, 0, 0, 0};  // block rows (nbx blocks each, nby rows per plane)
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
        const int e0 = j * KCH;
        hc.advance_to(e0, tb.hx, tb.hy);
        if (fast_local) {
          bits0 = lm.segment(hc, e0, tb.hx);
          hc.advance_to(e0 + 32, tb.hx, tb.hy);
          bits1 = lm.segment(hc, e0 + 32, tb.hx);
          const int valid = nh - e0;  // keys past the halo
          if (valid < 64) {
            bits0 &= valid <= 0 ? 0u : (valid >= 32 ? 0xffffffffu : (0xffffffffu >> (32 - valid)));
            bits1 &= valid <= 32 ? 0u : (0xffffffffu >> (64 - valid));
          }
        } else {
          bits0 = local_bits(hc, e0, nh, tb.hx, tb.hy, qz, qy, g.rz, g.ry, xlo, xhi);
          hc.advance_to(e0 + 32, tb.hx, tb.hy);
          bits1 = local_bits(hc, e0 + 32, nh, tb.hx, tb.hy, qz, qy, g.rz, g.ry, xlo, xhi);
        }
      } else {
        const int B0 = (j - n_local) * KCH;
        // the box of blocks this query's window touches
        const int bzlo = max(cz - g.rz, 0) / g.bz, bzhi = min(cz + g.rz, g.Z - 1) / g.bz;
        const int bylo = max(cy - g.ry, 0) / g.by, byhi = min(cy + g.ry, g.Y - 1) / g.by;
        const int bxlo = max(cx - g.rx, 0) / g.bx, bxhi = min(cx + g.rx, g.X - 1) / g.bx;
        bc.advance_to(B0, g.nbx, g.nby);
        bits0 = summary_bits(bc, B0, g.nb, g.nbx, g.nby, bzlo, bzhi, bylo, byhi, bxlo, bxhi);
        bc.advance_to(B0 + 32, g.nbx, g.nby);
        bits1 = summary_bits(bc, B0 + 32, g.nb, g.nbx, g.nby, bzlo, bzhi, bylo, byhi, bxlo, bxhi);
      }
      if (!active) bits0 = bits1 = 0u;
      if (__ballot_sync(0xffffffffu, (bits0 | bits1) != 0u) == 0u) {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tmem_st16(tS, z);
        tmem_st16(tS + 16, z);
      } else {
        // pass 1: masked row maximum (one 32-column segment in registers at a time)
        float cmax;
        {
          uint32_t sv[32];
          tmem_ld32(tS, sv);
          tmem_wait_ld();
          cmax = masked_max(sv, bits0);
          tmem_ld32(tS + 32, sv);
          tmem_wait_ld();
          cmax = fmaxf(cmax, masked_max(sv, bits1));
        }
        const float cmax2 = cmax * c2;
        float corr = 1.f;
        if (cmax2 > m_run + RESCALE_THRESHOLD) {
          if (m_run != -INFINITY) corr = ex2(m_run - cmax2);
          l_run *= corr;
          m_run = cmax2;
        }
        const float mneg = m_run == -INFINITY ? 0.f : -m_run;
        // pass 2: P over S; keys 0-31 -> columns 0-15, keys 32-63 -> columns
        // 16-31 (columns whose S values have been read by then)
        {
          uint32_t sv[32], p[16];
          tmem_ld32(tS, sv);
          tmem_wait_ld();
          l_run += exp_pack(sv, bits0, c2, mneg, p);
          tmem_st16(tS, p);
          tmem_ld32(tS + 32, sv);
          tmem_wait_ld();
          l_run += exp_pack(sv, bits1, c2, mneg, p);
          tmem_st16(tS + 16, p);
        }
        // rescale O after P and before this chunk's PV product, which is issued
        // only after p_full below
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
