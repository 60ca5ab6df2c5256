// Pieces shared by the tensor-core attention kernels (forward and backward):
// query-tile geometry, the window mask carried as extra contraction channels,
// the block-summary mask, the bf16 rotation of 16-byte chunks, and the
// tensor-map encoder for TMA box loads.
#pragma once

#include <cuda.h>

#include "pack3d_internal.cuh"
#include "tc_primitives.cuh"

namespace p3d {
namespace tca {

using namespace tc;

// Keys (or queries) per streamed chunk and the box of the grid they cover
// (x, y, z): column n of a chunk is ((dz * 2 + dy) * 16 + dx).
constexpr int KCH = 64;
constexpr int BXK = 16, BYK = 2, BZK = 2;

// Window mask as 16 extra contraction channels of a logit product S = A C^T
// ("penalty" channels): a row of A carries a one-hot of its tile-local z (4),
// y (4) and x (8) position, a row of C -2^14 in every channel whose tile
// position's window misses it (all of them outside the volume), so a masked
// logit is at most -2^14 (below -2400 in log2 units at tau = 96^-1/2) and its
// exponential is 0.  The window is symmetric, so the same channels mask
// queries against key rows and keys against query rows.
constexpr uint16_t BF16_ONE = 0x3F80, BF16_PEN = 0xC680;  // 1.0, -16384.0

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

// Tile-local position of TMEM lane (row) r: warp w = r / 32 holds the
// 2 x 2 x 8 box at planes 2 (w / 2) + {0, 1}, rows 2 (w % 2) + {0, 1}.
__device__ __forceinline__ void lane_pos(int r, int& lz, int& ly, int& lx) {
  const int w = r >> 5, l = r & 31;
  lz = (w >> 1) * 2 + (l >> 4);
  ly = (w & 1) * 2 + ((l >> 3) & 1);
  lx = l & 7;
}

// The 8 words (16 bf16 channels) of a row's one-hot tile position.
__device__ __forceinline__ void onehot_words(int lz, int ly, int lx, uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    auto hot = [&](int c) -> uint32_t {
      return (c < 4 ? c == lz : (c < 8 ? c - 4 == ly : c - 8 == lx)) ? BF16_ONE : 0u;
    };
    w[i] = hot(2 * i) | (hot(2 * i + 1) << 16);
  }
}

// Penalty rows of one chunk (64 rows of 32 bytes, 32-byte swizzle) against the
// tile `tb`: the chunk's box starts at (cz0, cy0, cx0); every lane of the warp
// writes two rows.  Rows outside the volume, and (partly occupied volumes,
// volb = the batch item's coordinate volume) rows at empty voxels, are masked
// in every channel.  PARTIAL: the volume may be partly occupied (compiled out
// of the dense kernels).
template <bool PARTIAL>
__device__ __forceinline__ void penalty_rows(uint8_t* dst, const Geo& g, const TileBox& tb,
                                             int cz0, int cy0, int cx0, int lane,
                                             const int32_t* volb) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = lane + 32 * half;
    const int kz = cz0 + (r >> 5), ky = cy0 + ((r >> 4) & 1), kx = cx0 + (r & 15);
    bool inside = kz < g.Z && ky < g.Y && kx < g.X;
    if (PARTIAL && inside) inside = volb[((int64_t)kz * g.Y + ky) * g.X + kx] >= 0;
    uint32_t w[8];
#pragma unroll
    for (int a = 0; a < 4; a += 2) {
      const uint32_t p0 = (!inside || abs(kz - (tb.z0 + a)) > g.rz) ? BF16_PEN : 0u;
      const uint32_t p1 = (!inside || abs(kz - (tb.z0 + a + 1)) > g.rz) ? BF16_PEN : 0u;
      w[a / 2] = p0 | (p1 << 16);
      const uint32_t q0 = (!inside || abs(ky - (tb.y0 + a)) > g.ry) ? BF16_PEN : 0u;
      const uint32_t q1 = (!inside || abs(ky - (tb.y0 + a + 1)) > g.ry) ? BF16_PEN : 0u;
      w[2 + a / 2] = q0 | (q1 << 16);
    }
#pragma unroll
    for (int a = 0; a < 8; a += 2) {
      const uint32_t p0 = (!inside || abs(kx - (tb.x0 + a)) > g.rx) ? BF16_PEN : 0u;
      const uint32_t p1 = (!inside || abs(kx - (tb.x0 + a + 1)) > g.rx) ? BF16_PEN : 0u;
      w[4 + a / 2] = p0 | (p1 << 16);
    }
    *reinterpret_cast<uint4*>(dst + sw32_off(r, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(dst + sw32_off(r, 1)) = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// The penalty channels of one axis depend only on the key's coordinate on
// that axis, so a tile's penalty rows are a product of three small tables over
// its halo box: entry o describes key coordinate (halo origin + o) on that axis
// - channels 0-3 (z: the tile's query planes), 4-7 (y), 8-15 (x).  A key
// outside the volume on an axis has every channel of that axis set, which masks
// it for every query.  Dense volumes only (an empty voxel does not factorise);
// halo boxes up to PEN_TAB per axis.
constexpr int PEN_TAB = 64;
struct PenaltyTable {
  uint2 z[PEN_TAB];
  uint2 y[PEN_TAB];
  uint4 x[PEN_TAB];
};

__device__ __forceinline__ uint32_t pen_pair(bool lo, bool hi) {
  return (lo ? (uint32_t)BF16_PEN : 0u) | ((hi ? (uint32_t)BF16_PEN : 0u) << 16);
}

// Fill the table of tile `tb` (the 32 lanes of one warp).
__device__ __forceinline__ void penalty_table(PenaltyTable& t, const Geo& g, const TileBox& tb,
                                              int lane) {
  for (int o = lane; o < PEN_TAB; o += 32) {
    const int kz = tb.hz0 + o, ky = tb.hy0 + o, kx = tb.hx0 + o;
    const bool zo = kz >= g.Z, yo = ky >= g.Y, xo = kx >= g.X;
    auto zm = [&](int a) { return zo || abs(kz - (tb.z0 + a)) > g.rz; };
    auto ym = [&](int a) { return yo || abs(ky - (tb.y0 + a)) > g.ry; };
    auto xm = [&](int a) { return xo || abs(kx - (tb.x0 + a)) > g.rx; };
    t.z[o] = make_uint2(pen_pair(zm(0), zm(1)), pen_pair(zm(2), zm(3)));
    t.y[o] = make_uint2(pen_pair(ym(0), ym(1)), pen_pair(ym(2), ym(3)));
    t.x[o] = make_uint4(pen_pair(xm(0), xm(1)), pen_pair(xm(2), xm(3)), pen_pair(xm(4), xm(5)),
                        pen_pair(xm(6), xm(7)));
  }
}

// penalty_rows of a dense volume from the tile's table: the same 64 rows.
__device__ __forceinline__ void penalty_rows_table(uint8_t* dst, const PenaltyTable& t,
                                                   const TileBox& tb, int cz0, int cy0, int cx0,
                                                   int lane) {
  const uint2 yw = t.y[cy0 - tb.hy0 + ((lane >> 4) & 1)];
  const uint4 xw = t.x[cx0 - tb.hx0 + (lane & 15)];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = lane + 32 * half;
    const uint2 zw = t.z[cz0 - tb.hz0 + half];
    *reinterpret_cast<uint4*>(dst + sw32_off(r, 0)) = make_uint4(zw.x, zw.y, yw.x, yw.y);
    *reinterpret_cast<uint4*>(dst + sw32_off(r, 1)) = xw;
  }
}

// Rotate four words of pair members (lo) against their partners (hi): word u of
// lo holds channels j0 + 2u, j0 + 2u + 1 of a segment, word u of hi the same
// pairs' second members.  t = rotation-table row (16 (cos, sin) pairs) of the
// segment's axis at the row's coordinate.
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

// Summary mask of the 64 blocks [B0, B0 + 64) for one query: every valid block
// except those whose box meets the query's window, i.e. the blocks
// (bz, by, bx) with bz in [bzlo, bzhi], by in [bylo, byhi], bx in [bxlo, bxhi]
// - one raster run of blocks per (bz, by).
__device__ __forceinline__ uint64_t summary_mask64(const Geo& g, int B0, int bzlo, int bzhi,
                                                   int bylo, int byhi, int bxlo, int bxhi) {
  uint64_t m = bit_range64(0, min(64, g.nb - B0) - 1);
  for (int bz = bzlo; bz <= bzhi; ++bz)
    for (int by = bylo; by <= byhi; ++by) {
      const int row = (bz * g.nby + by) * g.nbx - B0;
      const int lo = max(row + bxlo, 0), hi = min(row + bxhi, 63);
      m &= ~bit_range64(lo, hi);
    }
  return m;
}

// ---- host: tensor maps ------------------------------------------------------------

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on the driver library).
inline EncodeTiled encode_fn() {
  static EncodeTiled fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      return (EncodeTiled) nullptr;
    return reinterpret_cast<EncodeTiled>(p);
  }();
  return fn;
}

// Dense tensor of `rank` dims (innermost first), elements of `esize` bytes;
// box `box`; zero fill outside the tensor.
inline bool encode_map(CUtensorMap* m, CUtensorMapDataType type, int esize, void* base, int rank,
                       const uint64_t* dims, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[5], gstride[4];
  cuuint32_t bdim[5], estride[5];
  uint64_t stride = (uint64_t)esize;
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
    stride *= dims[i];
    if (i + 1 < rank) gstride[i] = stride;
  }
  return fn(m, type, rank, base, gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 tensor with dims[0] = 96 channels; box {32, box[1..]}, 64-byte swizzle
// (the K-major operand layout of the MMAs).
inline bool encode_bf16(CUtensorMap* m, void* base, int rank, const uint64_t* dims,
                        const uint32_t* box) {
  return encode_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rank, dims, box,
                    CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace tca
}  // namespace p3d
