// PACK3D attention on the CUDA cores in fp32: the forward used for the fp32
// mode (and for head dims the tensor-core kernel is not built for), and the
// full backward.
//
// Operator ("Geometry Matters in Packed 3D Attention", abstract): exact
// attention over each query's clipped 3D window plus the summaries of the
// blocks that do not meet the window, one softmax, axial RoPE on grid
// coordinates.  One CTA serves one 4 x 4 x 8 tile of one (batch item, head).
// G = d / 24 threads (at least 1) share a token, each owning CPT = d / G
// channels, and dot products are finished with warp shuffles inside the
// group.  The forward stages keys per chunk of KC tokens in shared memory,
// already rotated, as fp32.  The backward's dq and dk/dv kernels give each
// warp a 2 x 2 x 2 box of the tile.  They stage the halo one z-plane at a time
// and let each warp walk only the halo rows its box's windows reach.  The
// summary gradients at d = 96 have their own register-tiled kernel.  Every
// reduction runs in a fixed order.  Key coordinates come from the halo box
// and query coordinates from the tile box, so no coordinate array is read.
#include <math.h>

#include <algorithm>

#include "pack3d_internal.cuh"

namespace p3d {

namespace {

constexpr int KC = 32;            // keys (or summaries) per staged chunk
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

template <int D>
struct Split {
  static constexpr int G = D >= 48 ? D / 24 : 1;  // threads per query
  static constexpr int CPT = D / G;               // channels per thread
};

struct TileGeo {
  int z0, y0, x0, lz, ly, lx;    // tile box (clipped)
  int hz0, hy0, hx0, hz, hy, hx; // halo box (clipped)
};

__device__ __forceinline__ TileGeo tile_geo(const Geo& g, int t) {
  TileGeo tg;
  int Tx = t % g.nTx, Ty = (t / g.nTx) % g.nTy, Tz = t / (g.nTx * g.nTy);
  tg.z0 = Tz * TZ;
  tg.y0 = Ty * TY;
  tg.x0 = Tx * TX;
  tg.lz = min(TZ, g.Z - tg.z0);
  tg.ly = min(TY, g.Y - tg.y0);
  tg.lx = min(TX, g.X - tg.x0);
  tg.hz0 = max(0, tg.z0 - g.rz);
  tg.hy0 = max(0, tg.y0 - g.ry);
  tg.hx0 = max(0, tg.x0 - g.rx);
  tg.hz = min(g.Z, tg.z0 + tg.lz + g.rz) - tg.hz0;
  tg.hy = min(g.Y, tg.y0 + tg.ly + g.ry) - tg.hy0;
  tg.hx = min(g.X, tg.x0 + tg.lx + g.rx) - tg.hx0;
  return tg;
}

// Coordinate of the e-th token of the tile (raster order inside the tile).
__device__ __forceinline__ void tile_coord(const TileGeo& tg, int e, int& z, int& y, int& x) {
  x = tg.x0 + e % tg.lx;
  y = tg.y0 + (e / tg.lx) % tg.ly;
  z = tg.z0 + e / (tg.lx * tg.ly);
}

__device__ __forceinline__ void halo_coord(const TileGeo& tg, int e, int& z, int& y, int& x) {
  x = tg.hx0 + e % tg.hx;
  y = tg.hy0 + (e / tg.hx) % tg.hy;
  z = tg.hz0 + e / (tg.hx * tg.hy);
}

template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o >= 1; o /= 2) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Rotated channel c of a row, for the token with coordinate (z, y, x) and
// packed index pos - transpose = true applies R^T.  Axial mode: segment
// a = c / da, pair (j, j + da/2) of it; packed mode: pair (j, j + d/2).
template <typename T>
__device__ __forceinline__ float rot_row_channel(const T* row, const float* rope, const Geo& g,
                                                 int c, int cz, int cy, int cx, int pos,
                                                 bool transpose) {
  int base, len, p, a = 0, ca = 0;
  if (g.rope_mode == PACK3D_ROPE_PACKED) {
    base = 0;
    len = g.d / 2;
    p = c;
  } else {
    a = c / g.da;
    base = a * g.da;
    len = g.half;
    p = c % g.da;
    ca = a == 0 ? cz : (a == 1 ? cy : cx);
  }
  int j = p < len ? p : p - len;
  float2 cs = rope_cs(rope, g, a, ca, pos, j);
  float sn = transpose ? -cs.y : cs.y;
  float x1 = to_f32(row[base + j]), x2 = to_f32(row[base + j + len]);
  return p < len ? x1 * cs.x - x2 * sn : x1 * sn + x2 * cs.x;
}

template <typename T>
__device__ __forceinline__ float rot_channel(const T* row, const float* rope, const Geo& g, int c,
                                             int cz, int cy, int cx, int pos, bool transpose) {
  return rot_row_channel(row, rope, g, c, cz, cy, cx, pos, transpose);
}

__device__ __forceinline__ float rot_channel_smem(const float* row, const float* rope, const Geo& g,
                                                  int c, int cz, int cy, int cx, int pos,
                                                  bool transpose) {
  return rot_row_channel(row, rope, g, c, cz, cy, cx, pos, transpose);
}

struct ChunkCoords {
  int z[KC], y[KC], x[KC], tok[KC];
};

// The backward's local loops stage the halo box plane by plane: a whole
// z-plane of it per chunk, or as many of the plane's rows as fit in CAPK
// tokens.  Inside a chunk every warp visits only the rows its tokens' windows
// reach, so warps do not wait on rows that only other warps need.
constexpr int CAPK = 160;
struct PlaneMeta {
  int z[CAPK], y[CAPK], x[CAPK], tok[CAPK];
};

// z and y extent of a warp's active tokens (a ragged tile's warp may span rows).
struct WarpBox {
  int zlo, zhi, ylo, yhi;
};

// Token slot s (0 .. TILE-1) of a tile for the backward's token-major
// kernels: each group of 8 slots (one warp at head_dim 96) takes a 2x2x2 box
// of the 4x4x8 tile, so the union of its windows is 8 wide along every axis
// (a row of 8 along x would need 7 x 7 x 14).  Returns whether the box cell
// lies inside the clipped tile; e is its raster index there.
__device__ __forceinline__ bool box_slot(const TileGeo& tg, int s, int& z, int& y, int& x,
                                         int& e) {
  static_assert(TZ == 4 && TY == 4 && TX == 8, "slot boxes assume a 4x4x8 tile");
  const int w = s >> 3, l = s & 7;
  z = tg.z0 + 2 * (w >> 3) + ((l >> 2) & 1);
  y = tg.y0 + 2 * ((w >> 2) & 1) + ((l >> 1) & 1);
  x = tg.x0 + 2 * (w & 3) + (l & 1);
  e = ((z - tg.z0) * tg.ly + (y - tg.y0)) * tg.lx + (x - tg.x0);
  return z < tg.z0 + tg.lz && y < tg.y0 + tg.ly && x < tg.x0 + tg.lx;
}

__device__ __forceinline__ WarpBox warp_box(bool active, int cz, int cy) {
  constexpr int BIG = 1 << 29;
  WarpBox w;
  w.zlo = __reduce_min_sync(0xffffffffu, active ? cz : BIG);
  w.zhi = __reduce_max_sync(0xffffffffu, active ? cz : -BIG);
  w.ylo = __reduce_min_sync(0xffffffffu, active ? cy : BIG);
  w.yhi = __reduce_max_sync(0xffffffffu, active ? cy : -BIG);
  return w;
}

// Dot product of a thread's CPT channels with a staged fp32 row (16-byte
// aligned), summed in channel order, read 16 bytes at a time.
template <int CPT>
__device__ __forceinline__ float dot_row(const float (&r)[CPT], const float* row) {
  static_assert(CPT % 4 == 0, "channels per thread must be a multiple of 4");
  const float4* p = reinterpret_cast<const float4*>(row);
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < CPT / 4; ++v) {
    const float4 x = p[v];
    acc += r[4 * v] * x.x;
    acc += r[4 * v + 1] * x.y;
    acc += r[4 * v + 2] * x.z;
    acc += r[4 * v + 3] * x.w;
  }
  return acc;
}

// One staged token row as fp32: xr = R(c) x (the rotated row) and yr = y
// (plain), for the token with packed index i and coordinate (cz, cy, cx).
// TPR threads share the row (sub = 0 .. TPR-1), each rotation pair (both
// channels of it) read once; a thread's loads are independent of each other,
// so their latencies overlap.
template <typename T, int D, int TPR>
__device__ __forceinline__ void stage_one_row(const Geo& g, const float* __restrict__ rope,
                                              const T* __restrict__ x, const T* __restrict__ y,
                                              int b, int h, int i, int cz, int cy, int cx, int sub,
                                              float* xr, float* yr) {
  constexpr int PAIRS = D / 2, HALF = D / 6, DA = D / 3;
  const int64_t row = (((int64_t)b * g.N + i) * g.H + h) * D;
  const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
#pragma unroll
  for (int m = 0; m < (PAIRS + TPR - 1) / TPR; ++m) {
    const int pr = sub + m * TPR;
    if (pr < PAIRS) {
      int a = 0, ca = 0, j = pr, c1 = pr, c2 = pr + PAIRS;
      if (!packed) {
        a = pr / HALF;
        j = pr - a * HALF;
        c1 = a * DA + j;
        c2 = c1 + HALF;
        ca = a == 0 ? cz : (a == 1 ? cy : cx);
      }
      const float2 cs = rope_cs(rope, g, a, ca, i, j);
      const float x1 = to_f32(x[row + c1]), x2 = to_f32(x[row + c2]);
      xr[c1] = x1 * cs.x - x2 * cs.y;
      xr[c2] = x1 * cs.y + x2 * cs.x;
      yr[c1] = to_f32(y[row + c1]);
      yr[c2] = to_f32(y[row + c2]);
    }
  }
}

// Stage ROWS token rows (row stride ld floats) with NT threads, NT / ROWS per
// row; rows nrows .. ROWS-1 are zero-filled.
template <typename T, int D, int ROWS, int NT>
__device__ __forceinline__ void stage_rows(const Geo& g, const float* __restrict__ rope,
                                           const T* __restrict__ x, const T* __restrict__ y,
                                           int b, int h, const int* tok, const int* cz,
                                           const int* cy, const int* cx, int nrows, float* xo,
                                           float* yo, int ld) {
  static_assert(NT % ROWS == 0, "threads must divide evenly over the rows");
  constexpr int TPR = NT / ROWS;
  const int r = threadIdx.x / TPR, sub = threadIdx.x % TPR;
  float* xr = xo + r * ld;
  float* yr = yo + r * ld;
  if (r >= nrows) {
    for (int c = sub; c < D; c += TPR) xr[c] = yr[c] = 0.f;
    return;
  }
  stage_one_row<T, D, TPR>(g, rope, x, y, b, h, tok[r], cz[r], cy[r], cx[r], sub, xr, yr);
}

// Stage nrows token rows (row stride D) with NT threads, 16 per row, as many
// passes as needed; nothing beyond nrows is written.
template <typename T, int D, int NT>
__device__ __forceinline__ void stage_rows_n(const Geo& g, const float* __restrict__ rope,
                                             const T* __restrict__ x, const T* __restrict__ y,
                                             int b, int h, const int* tok, const int* cz,
                                             const int* cy, const int* cx, int nrows, float* xo,
                                             float* yo) {
  constexpr int TPR = 16;
  static_assert(NT % TPR == 0, "threads must divide evenly over the rows");
  const int sub = threadIdx.x % TPR;
  for (int r = threadIdx.x / TPR; r < nrows; r += NT / TPR)
    stage_one_row<T, D, TPR>(g, rope, x, y, b, h, tok[r], cz[r], cy[r], cx[r], sub, xo + r * D,
                             yo + r * D);
}

// acc[u] += a * row[u] over a thread's CPT channels of a staged fp32 row.
template <int CPT>
__device__ __forceinline__ void axpy_row(float (&acc)[CPT], float a, const float* row) {
  const float4* p = reinterpret_cast<const float4*>(row);
#pragma unroll
  for (int v = 0; v < CPT / 4; ++v) {
    const float4 x = p[v];
    acc[4 * v] += a * x.x;
    acc[4 * v + 1] += a * x.y;
    acc[4 * v + 2] += a * x.z;
    acc[4 * v + 3] += a * x.w;
  }
}

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------

template <typename T, typename TO, int D, bool SUMMARY>
__global__ void __launch_bounds__(TILE * Split<D>::G) k_forward_simt(
    Geo g, pack3d_index ix, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const float* __restrict__ ksum, const float* __restrict__ vsum,
    TO* __restrict__ out, float* __restrict__ lse) {
  constexpr int G = Split<D>::G, CPT = Split<D>::CPT;
  if (ix.err[0]) return;
  __shared__ float sk[KC][D];
  __shared__ float sv[KC][D];
  __shared__ ChunkCoords cc;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int qs = threadIdx.x / G, lane = threadIdx.x % G;
  const TileGeo tg = tile_geo(g, t);
  const int count = tg.lz * tg.ly * tg.lx;
  const bool active = qs < count;
  int cz = 0, cy = 0, cx = 0, qi = 0;
  if (active) {
    tile_coord(tg, qs, cz, cy, cx);
    qi = ix.perm[(int64_t)b * g.N + ix.tile_off[(int64_t)b * (g.nT + 1) + t] + qs];
  }
  const float qscale = g.tau * LOG2E;  // logits in log2 units
  float qr[CPT], o[CPT];
  {
    const T* qrow = q + (((int64_t)b * g.N + qi) * g.H + h) * D;
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
      int c = lane * CPT + u;
      qr[u] = active ? qscale * rot_channel(qrow, ix.rope, g, c, cz, cy, cx, qi, false) : 0.f;
      o[u] = 0.f;
    }
  }
  float m = -INFINITY, l = 0.f;

  // ---- local window keys ----
  const int nh = tg.hz * tg.hy * tg.hx;
  const int32_t* hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
  for (int base = 0; base < nh; base += KC) {
    const int nk = min(KC, nh - base);
    __syncthreads();
    for (int e = threadIdx.x; e < KC * D; e += blockDim.x) {
      int kk = e / D, c = e % D;
      float kv = 0.f, vv = 0.f;
      if (kk < nk) {
        int z, y, x;
        halo_coord(tg, base + kk, z, y, x);
        int j = hl[base + kk];
        int64_t row = (((int64_t)b * g.N + j) * g.H + h) * D;
        kv = rot_channel(k + row, ix.rope, g, c, z, y, x, j, false);
        vv = to_f32(v[row + c]);
        if (c == 0) {
          cc.z[kk] = z;
          cc.y[kk] = y;
          cc.x[kk] = x;
        }
      }
      sk[kk][c] = kv;
      sv[kk][c] = vv;
    }
    __syncthreads();
    float s[KC];
    float cmax = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < KC; ++kk) {
      float part = 0.f;
#pragma unroll
      for (int u = 0; u < CPT; ++u) part += qr[u] * sk[kk][lane * CPT + u];
      float dot = group_sum<G>(part);
      bool in = active && kk < nk && abs(cc.z[kk] - cz) <= g.rz && abs(cc.y[kk] - cy) <= g.ry &&
                abs(cc.x[kk] - cx) <= g.rx;
      s[kk] = in ? dot : -INFINITY;
      cmax = fmaxf(cmax, s[kk]);
    }
    if (cmax > m) {
      float corr = exp2f(m - cmax);  // 0 when m = -inf
      l *= corr;
#pragma unroll
      for (int u = 0; u < CPT; ++u) o[u] *= corr;
      m = cmax;
    }
    if (m > -INFINITY) {
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        float p = exp2f(s[kk] - m);
        l += p;
#pragma unroll
        for (int u = 0; u < CPT; ++u) o[u] += p * sv[kk][lane * CPT + u];
      }
    }
  }

  // ---- block summaries of blocks that miss the window ----
  if (SUMMARY) {
    const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
    for (int base = 0; base < g.nb; base += KC) {
      const int nk = min(KC, g.nb - base);
      __syncthreads();
      for (int e = threadIdx.x; e < KC * D; e += blockDim.x) {
        int kk = e / D, c = e % D;
        float kv = 0.f, vv = 0.f;
        if (kk < nk) {
          kv = ksum[(sbase + base + kk) * D + c];
          vv = vsum[(sbase + base + kk) * D + c];
          if (c == 0) {
            int B = base + kk;
            cc.z[kk] = B / (g.nby * g.nbx);
            cc.y[kk] = (B / g.nbx) % g.nby;
            cc.x[kk] = B % g.nbx;
          }
        }
        sk[kk][c] = kv;
        sv[kk][c] = vv;
      }
      __syncthreads();
      float s[KC];
      float cmax = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        float part = 0.f;
#pragma unroll
        for (int u = 0; u < CPT; ++u) part += qr[u] * sk[kk][lane * CPT + u];
        float dot = group_sum<G>(part);
        // block box meets the window box iff the intervals overlap on every axis
        int bz0 = cc.z[kk] * g.bz, by0 = cc.y[kk] * g.by, bx0 = cc.x[kk] * g.bx;
        bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                     by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                     bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
        bool in = active && kk < nk && !meets;
        s[kk] = in ? dot : -INFINITY;
        cmax = fmaxf(cmax, s[kk]);
      }
      if (cmax > m) {
        float corr = exp2f(m - cmax);
        l *= corr;
#pragma unroll
        for (int u = 0; u < CPT; ++u) o[u] *= corr;
        m = cmax;
      }
      if (m > -INFINITY) {
#pragma unroll
        for (int kk = 0; kk < KC; ++kk) {
          float p = exp2f(s[kk] - m);
          l += p;
#pragma unroll
          for (int u = 0; u < CPT; ++u) o[u] += p * sv[kk][lane * CPT + u];
        }
      }
    }
  }

  if (active) {
    float inv = 1.f / l;
    TO* orow = out + (((int64_t)b * g.N + qi) * g.H + h) * D;
#pragma unroll
    for (int u = 0; u < CPT; ++u) orow[lane * CPT + u] = from_f32<TO>(o[u] * inv);
    if (lane == 0) lse[((int64_t)b * g.H + h) * g.N + qi] = (m + log2f(l)) * LN2;
  }
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------

// delta_i = sum_c dout_ic * out_ic, fp32, [B][H][N].
template <typename T, typename TO>
__global__ void k_bwd_delta(Geo g, const int32_t* __restrict__ err, const TO* __restrict__ out,
                            const T* __restrict__ dout, float* delta) {
  if (err[0]) return;
  int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // (b, i, h) row
  if (r >= (int64_t)g.B * g.N * g.H) return;
  int h = (int)(r % g.H);
  int64_t bi = r / g.H;
  int i = (int)(bi % g.N), b = (int)(bi / g.N);
  const TO* o = out + r * g.d;
  const T* d = dout + r * g.d;
  float s = 0.f;
  for (int c = 0; c < g.d; ++c) s += to_f32(o[c]) * to_f32(d[c]);
  delta[((int64_t)b * g.H + h) * g.N + i] = s;
}

// Summary gradients dkbar_B = tau sum_i dS_iB q~_i and dvbar_B = sum_i P_iB dO_i
// over the queries i that see block B.  One CTA per (chunk of BC blocks,
// batch item, head) walks all queries tile by tile (fixed order).
constexpr int BC = 8, QC = 32;

template <typename T, int D>
__global__ void __launch_bounds__(256) k_bwd_summary(Geo g, pack3d_index ix,
                                                    const T* __restrict__ q,
                                                    const T* __restrict__ dout,
                                                    const float* __restrict__ lse,
                                                    const float* __restrict__ delta,
                                                    const float* __restrict__ ksum,
                                                    const float* __restrict__ vsum, float* dks,
                                                    float* dvs) {
  if (ix.err[0]) return;
  // rows padded to D + 1 floats: the dot products read rows kk of skb / svb at
  // the same channel from 8 threads, which would otherwise share a bank
  __shared__ float sq[QC][D + 1];
  __shared__ float sdo[QC][D + 1];
  __shared__ float skb[BC][D + 1];
  __shared__ float svb[BC][D + 1];
  __shared__ float sP[QC][BC];
  __shared__ float sdS[QC][BC];
  __shared__ int sqc[QC][3];
  __shared__ float slse[QC], sdel[QC];
  const int b = blockIdx.y, h = blockIdx.z, B0 = blockIdx.x * BC;
  const int nbc = min(BC, g.nb - B0);
  const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
  for (int e = threadIdx.x; e < BC * D; e += blockDim.x) {
    int kk = e / D, c = e % D;
    skb[kk][c] = kk < nbc ? ksum[(sbase + B0 + kk) * D + c] : 0.f;
    svb[kk][c] = kk < nbc ? vsum[(sbase + B0 + kk) * D + c] : 0.f;
  }
  // accumulators: thread owns outputs e = threadIdx.x + r * 256 of [2][BC][D]
  constexpr int NOUT = 2 * BC * D;
  constexpr int PER = (NOUT + 255) / 256;
  float acc[PER];
#pragma unroll
  for (int r = 0; r < PER; ++r) acc[r] = 0.f;
  const int64_t lbase = ((int64_t)b * g.H + h) * g.N;
  for (int t = 0; t < g.nT; ++t) {
    const TileGeo tg = tile_geo(g, t);
    const int count = tg.lz * tg.ly * tg.lx;
    const int toff = ix.tile_off[(int64_t)b * (g.nT + 1) + t];
    for (int qb = 0; qb < count; qb += QC) {
      const int nq = min(QC, count - qb);
      __syncthreads();
      for (int e = threadIdx.x; e < QC * D; e += blockDim.x) {
        int qq = e / D, c = e % D;
        float qv = 0.f, dv = 0.f;
        if (qq < nq) {
          int z, y, x;
          tile_coord(tg, qb + qq, z, y, x);
          int i = ix.perm[(int64_t)b * g.N + toff + qb + qq];
          int64_t row = (((int64_t)b * g.N + i) * g.H + h) * D;
          qv = rot_channel(q + row, ix.rope, g, c, z, y, x, i, false);
          dv = to_f32(dout[row + c]);
          if (c == 0) {
            sqc[qq][0] = z;
            sqc[qq][1] = y;
            sqc[qq][2] = x;
            slse[qq] = lse[lbase + i];
            sdel[qq] = delta[lbase + i];
          }
        }
        sq[qq][c] = qv;
        sdo[qq][c] = dv;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < QC * BC; e += blockDim.x) {
        int qq = e / BC, kk = e % BC;
        float P = 0.f, dS = 0.f;
        if (qq < nq && kk < nbc) {
          int B = B0 + kk;
          int bz0 = (B / (g.nby * g.nbx)) * g.bz, by0 = ((B / g.nbx) % g.nby) * g.by,
              bx0 = (B % g.nbx) * g.bx;
          int cz = sqc[qq][0], cy = sqc[qq][1], cx = sqc[qq][2];
          bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                       by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                       bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
          if (!meets) {
            float s = 0.f, dp = 0.f;
            for (int c = 0; c < D; ++c) {
              s += sq[qq][c] * skb[kk][c];
              dp += sdo[qq][c] * svb[kk][c];
            }
            P = expf(g.tau * s - slse[qq]);
            dS = P * (dp - sdel[qq]);
          }
        }
        sP[qq][kk] = P;
        sdS[qq][kk] = dS;
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        int e = threadIdx.x + r * 256;
        if (e < NOUT) {
          int which = e / (BC * D), kk = (e / D) % BC, c = e % D;
          float a = acc[r];
          if (which == 0)
            for (int qq = 0; qq < nq; ++qq) a += sdS[qq][kk] * sq[qq][c];
          else
            for (int qq = 0; qq < nq; ++qq) a += sP[qq][kk] * sdo[qq][c];
          acc[r] = a;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    int e = threadIdx.x + r * 256;
    if (e < NOUT) {
      int which = e / (BC * D), kk = (e / D) % BC, c = e % D;
      if (kk < nbc) {
        if (which == 0)
          dks[(sbase + B0 + kk) * D + c] = g.tau * acc[r];
        else
          dvs[(sbase + B0 + kk) * D + c] = acc[r];
      }
    }
  }
}

// Summary gradients for d = 96, register-tiled.  One CTA owns a chunk of
// S96_NB summaries of one (batch item, head) and a contiguous range of query
// tiles (a split); it keeps k̄, v̄ of its summaries in shared memory and walks
// its queries in chunks of S96_QC:
//   phase 1: S = q~ k̄^T and dP = dO v̄^T for the chunk (each warp a 16 x 16
//            piece, each thread 2 x 4 of both, float4 operand reads);
//            P = exp(tau S - lse) where the query's window misses the block
//            (0 where it meets it), dS = P (dP - delta), both to shared memory;
//   phase 2: dk̄ += dS^T q~ and dv̄ += P^T dO, each thread 4 summaries x 6
//            channels of both in registers.
// Partial sums per split go to a workspace and are added in split order by
// k_bwd_summary_reduce, so the result does not depend on scheduling.
constexpr int S96_NB = 64, S96_QC = 32, S96_LD = 100, S96_LDP = 68, S96_THREADS = 256;

struct Sum96Smem {
  float ks[S96_NB][S96_LD];
  float vs[S96_NB][S96_LD];
  float q[S96_QC][S96_LD];
  float dout[S96_QC][S96_LD];
  float p[S96_QC][S96_LDP];
  float ds[S96_QC][S96_LDP];
  float lse[S96_QC], del[S96_QC];
  int qz[S96_QC], qy[S96_QC], qx[S96_QC], tok[S96_QC];
  int bz0[S96_NB], by0[S96_NB], bx0[S96_NB];
};

template <typename T>
__global__ void __launch_bounds__(S96_THREADS, 2) k_bwd_summary96(
    Geo g, pack3d_index ix, const T* __restrict__ q, const T* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ delta,
    const float* __restrict__ ksum, const float* __restrict__ vsum, int nsplit,
    float* __restrict__ part) {
  constexpr int D = 96;
  if (ix.err[0]) return;
  extern __shared__ __align__(16) unsigned char s96_raw[];
  Sum96Smem& sm = *reinterpret_cast<Sum96Smem*>(s96_raw);
  const int nbc = (g.nb + S96_NB - 1) / S96_NB;
  const int bc = blockIdx.x % nbc, split = blockIdx.x / nbc;
  const int b = blockIdx.y, h = blockIdx.z, B0 = bc * S96_NB;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
  for (int e = tid; e < S96_NB * D; e += S96_THREADS) {
    int r = e / D, c = e % D;
    bool ok = B0 + r < g.nb;
    sm.ks[r][c] = ok ? ksum[(sbase + B0 + r) * D + c] : 0.f;
    sm.vs[r][c] = ok ? vsum[(sbase + B0 + r) * D + c] : 0.f;
    if (c == 0) {
      int Bk = B0 + r;
      sm.bz0[r] = (Bk / (g.nby * g.nbx)) * g.bz;
      sm.by0[r] = ((Bk / g.nbx) % g.nby) * g.by;
      sm.bx0[r] = (Bk % g.nbx) * g.bx;
    }
  }
  // phase-1 roles: warp piece (wq, wb) of 16 queries x 16 summaries; lane
  // (lq, lb) takes queries wq*16 + lq + 8i and summaries wb*16 + lb + 4j
  const int wq = warp / 4, wb = warp % 4, lq = lane / 4, lb = lane % 4;
  // phase-2 roles: summaries 4*tb .. 4*tb+3, channels 6*tc .. 6*tc+5
  const int tb = tid / 16, tc = tid % 16;
  float dk[4][6], dv[4][6];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int u = 0; u < 6; ++u) dk[j][u] = dv[j][u] = 0.f;

  const int t0 = (int)((int64_t)split * g.nT / nsplit);
  const int t1 = (int)((int64_t)(split + 1) * g.nT / nsplit);
  const int64_t lbase = ((int64_t)b * g.H + h) * g.N;
  for (int t = t0; t < t1; ++t) {
    const TileGeo tg = tile_geo(g, t);
    const int count = tg.lz * tg.ly * tg.lx;
    const int toff = ix.tile_off[(int64_t)b * (g.nT + 1) + t];
    for (int qb = 0; qb < count; qb += S96_QC) {
      const int nq = min(S96_QC, count - qb);
      __syncthreads();
      if (tid < nq) {
        tile_coord(tg, qb + tid, sm.qz[tid], sm.qy[tid], sm.qx[tid]);
        const int i = ix.perm[(int64_t)b * g.N + toff + qb + tid];
        sm.tok[tid] = i;
        sm.lse[tid] = lse[lbase + i];
        sm.del[tid] = delta[lbase + i];
      }
      __syncthreads();
      stage_rows<T, D, S96_QC, S96_THREADS>(g, ix.rope, q, dout, b, h, sm.tok, sm.qz, sm.qy,
                                            sm.qx, nq, &sm.q[0][0], &sm.dout[0][0], S96_LD);
      __syncthreads();
      // ---- phase 1 ----
      {
        float s[2][4], dp[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) s[i][j] = dp[i][j] = 0.f;
        const int qr0 = wq * 16 + lq, br0 = wb * 16 + lb;
#pragma unroll 1
        for (int k = 0; k < D; k += 4) {
          float4 a[2], w[4];
#pragma unroll
          for (int i = 0; i < 2; ++i) a[i] = *reinterpret_cast<const float4*>(&sm.q[qr0 + 8 * i][k]);
#pragma unroll
          for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const float4*>(&sm.ks[br0 + 4 * j][k]);
#pragma unroll
          for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              s[i][j] += a[i].x * w[j].x + a[i].y * w[j].y + a[i].z * w[j].z + a[i].w * w[j].w;
#pragma unroll
          for (int i = 0; i < 2; ++i)
            a[i] = *reinterpret_cast<const float4*>(&sm.dout[qr0 + 8 * i][k]);
#pragma unroll
          for (int j = 0; j < 4; ++j) w[j] = *reinterpret_cast<const float4*>(&sm.vs[br0 + 4 * j][k]);
#pragma unroll
          for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dp[i][j] += a[i].x * w[j].x + a[i].y * w[j].y + a[i].z * w[j].z + a[i].w * w[j].w;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int qq = qr0 + 8 * i;
          const int cz = sm.qz[qq], cy = sm.qy[qq], cx = sm.qx[qq];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int bb = br0 + 4 * j;
            const int bz0 = sm.bz0[bb], by0 = sm.by0[bb], bx0 = sm.bx0[bb];
            const bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                               by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                               bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
            const bool in = qq < nq && B0 + bb < g.nb && !meets;
            const float P = in ? expf(g.tau * s[i][j] - sm.lse[qq]) : 0.f;
            sm.p[qq][bb] = P;
            sm.ds[qq][bb] = P * (dp[i][j] - sm.del[qq]);
          }
        }
      }
      __syncthreads();
      // ---- phase 2 ----
      for (int qq = 0; qq < nq; ++qq) {
        const float4 pv = *reinterpret_cast<const float4*>(&sm.p[qq][4 * tb]);
        const float4 dsv = *reinterpret_cast<const float4*>(&sm.ds[qq][4 * tb]);
        float xq[6], xo[6];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          float2 a = *reinterpret_cast<const float2*>(&sm.q[qq][6 * tc + 2 * m]);
          float2 o = *reinterpret_cast<const float2*>(&sm.dout[qq][6 * tc + 2 * m]);
          xq[2 * m] = a.x;
          xq[2 * m + 1] = a.y;
          xo[2 * m] = o.x;
          xo[2 * m + 1] = o.y;
        }
        const float pj[4] = {pv.x, pv.y, pv.z, pv.w};
        const float dj[4] = {dsv.x, dsv.y, dsv.z, dsv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int u = 0; u < 6; ++u) {
            dk[j][u] += dj[j] * xq[u];
            dv[j][u] += pj[j] * xo[u];
          }
      }
    }
  }
  // partials: part[split][b][h][summary][2][D]
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int Bk = B0 + 4 * tb + j;
    if (Bk < g.nb) {
      float* dst = part + ((((int64_t)split * g.B + b) * g.H + h) * g.nb + Bk) * 2 * D;
#pragma unroll
      for (int u = 0; u < 6; ++u) {
        dst[6 * tc + u] = dk[j][u];
        dst[D + 6 * tc + u] = dv[j][u];
      }
    }
  }
}

// dks = tau * sum over splits of the dk̄ partials, dvs = the same for dv̄
// (fixed split order).
__global__ void k_bwd_summary_reduce(Geo g, const int32_t* __restrict__ err, int nsplit,
                                     const float* __restrict__ part, float* __restrict__ dks,
                                     float* __restrict__ dvs) {
  if (err[0]) return;
  const int64_t per = (int64_t)g.B * g.H * g.nb * g.d;
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= per) return;
  const int64_t row = e / g.d;
  const int c = (int)(e % g.d);
  float sk = 0.f, sv = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float* src = part + ((int64_t)s * per / g.d + row) * 2 * g.d;
    sk += src[c];
    sv += src[g.d + c];
  }
  dks[e] = g.tau * sk;
  dvs[e] = sv;
}

// dq: query-major, the forward's structure.
template <typename T, int D, bool SUMMARY>
__global__ void __launch_bounds__(TILE * Split<D>::G) k_bwd_dq(
    Geo g, pack3d_index ix, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const T* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ delta, const float* __restrict__ ksum,
    const float* __restrict__ vsum, T* __restrict__ dq) {
  constexpr int G = Split<D>::G, CPT = Split<D>::CPT;
  if (ix.err[0]) return;
  // dynamic: staged keys and values, 2 * CAPK rows of D floats
  extern __shared__ __align__(16) float bwd_dyn[];
  float* const sbuf = bwd_dyn;
  float(*sk)[D] = reinterpret_cast<float(*)[D]>(bwd_dyn);
  float(*sv)[D] = reinterpret_cast<float(*)[D]>(bwd_dyn + CAPK * D);
  __shared__ ChunkCoords cc;
  __shared__ PlaneMeta pm;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int qs = threadIdx.x / G, lane = threadIdx.x % G;
  const TileGeo tg = tile_geo(g, t);
  int cz = 0, cy = 0, cx = 0, qe = 0, qi = 0;
  const bool active = box_slot(tg, qs, cz, cy, cx, qe);
  if (active) qi = ix.perm[(int64_t)b * g.N + ix.tile_off[(int64_t)b * (g.nT + 1) + t] + qe];
  const int64_t qrow = (((int64_t)b * g.N + qi) * g.H + h) * D;
  float qr[CPT], dO[CPT], dqr[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    int c = lane * CPT + u;
    qr[u] = active ? rot_channel(q + qrow, ix.rope, g, c, cz, cy, cx, qi, false) : 0.f;
    dO[u] = active ? to_f32(dout[qrow + c]) : 0.f;
    dqr[u] = 0.f;
  }
  const int64_t lrow = ((int64_t)b * g.H + h) * g.N + qi;
  const float lse_i = active ? lse[lrow] : 0.f;
  const float del_i = active ? delta[lrow] : 0.f;

  const int32_t* hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
  const WarpBox wb = warp_box(active, cz, cy);
  const int rpc = min(tg.hy, CAPK / tg.hx);  // halo rows per chunk
  for (int pz = 0; pz < tg.hz; ++pz) {
    const int zk = tg.hz0 + pz;
    const bool zneed = zk >= wb.zlo - g.rz && zk <= wb.zhi + g.rz;  // warp-uniform
    for (int ry0 = 0; ry0 < tg.hy; ry0 += rpc) {
      const int nr = min(rpc, tg.hy - ry0), nk = nr * tg.hx;
      const int base = (pz * tg.hy + ry0) * tg.hx;
      __syncthreads();
      for (int e = threadIdx.x; e < nk; e += blockDim.x) {
        halo_coord(tg, base + e, pm.z[e], pm.y[e], pm.x[e]);
        pm.tok[e] = hl[base + e];
      }
      __syncthreads();
      stage_rows_n<T, D, TILE * G>(g, ix.rope, k, v, b, h, pm.tok, pm.z, pm.y, pm.x, nk,
                                   &sk[0][0], &sv[0][0]);
      __syncthreads();
      if (!zneed) continue;
      for (int r = 0; r < nr; ++r) {
        const int yk = tg.hy0 + ry0 + r;
        if (yk < wb.ylo - g.ry || yk > wb.yhi + g.ry) continue;  // warp-uniform
        const bool rowin = active && abs(zk - cz) <= g.rz && abs(yk - cy) <= g.ry;
        const int k0 = r * tg.hx, k1 = k0 + tg.hx;
        // keys in pairs (two independent dot-product chains per thread); at an
        // odd row end the second key repeats the first with weight 0.  A pair
        // outside every window of the warp's queries is skipped.
        for (int ka = k0; ka < k1; ka += 2) {
          const int kb = min(ka + 1, k1 - 1);
          const bool in0 = rowin && abs(pm.x[ka] - cx) <= g.rx;
          const bool in1 = rowin && ka + 1 < k1 && abs(pm.x[kb] - cx) <= g.rx;
          if (!__any_sync(0xffffffffu, in0 || in1)) continue;
          const float ps0 = dot_row(qr, &sk[ka][lane * CPT]);
          const float ps1 = dot_row(qr, &sk[kb][lane * CPT]);
          const float pd0 = dot_row(dO, &sv[ka][lane * CPT]);
          const float pd1 = dot_row(dO, &sv[kb][lane * CPT]);
          const float s0 = group_sum<G>(ps0), s1 = group_sum<G>(ps1);
          const float dp0 = group_sum<G>(pd0), dp1 = group_sum<G>(pd1);
          // re-read the staged rows below instead of holding them in registers
          __syncwarp();
          const float P0 = in0 ? expf(g.tau * s0 - lse_i) : 0.f;
          const float P1 = in1 ? expf(g.tau * s1 - lse_i) : 0.f;
          const float dS0 = P0 * (dp0 - del_i), dS1 = P1 * (dp1 - del_i);
          axpy_row(dqr, g.tau * dS0, &sk[ka][lane * CPT]);
          axpy_row(dqr, g.tau * dS1, &sk[kb][lane * CPT]);
        }
      }
    }
  }
  if (SUMMARY) {
    const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;
    for (int base = 0; base < g.nb; base += KC) {
      const int nk = min(KC, g.nb - base);
      __syncthreads();
      for (int e = threadIdx.x; e < KC * D; e += blockDim.x) {
        int kk = e / D, c = e % D;
        float kv = 0.f, vv = 0.f;
        if (kk < nk) {
          kv = ksum[(sbase + base + kk) * D + c];
          vv = vsum[(sbase + base + kk) * D + c];
          if (c == 0) {
            int B = base + kk;
            cc.z[kk] = B / (g.nby * g.nbx);
            cc.y[kk] = (B / g.nbx) % g.nby;
            cc.x[kk] = B % g.nbx;
          }
        }
        sk[kk][c] = kv;
        sv[kk][c] = vv;
      }
      __syncthreads();
      for (int kk = 0; kk < KC; ++kk) {
        const float ps = dot_row(qr, &sk[kk][lane * CPT]);
        const float pd = dot_row(dO, &sv[kk][lane * CPT]);
        float s = group_sum<G>(ps), dp = group_sum<G>(pd);
        int bz0 = cc.z[kk] * g.bz, by0 = cc.y[kk] * g.by, bx0 = cc.x[kk] * g.bx;
        bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                     by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                     bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
        bool in = active && kk < nk && !meets;
        float P = in ? expf(g.tau * s - lse_i) : 0.f;
        float dS = P * (dp - del_i);
        axpy_row(dqr, g.tau * dS, &sk[kk][lane * CPT]);
      }
    }
  }
  // rotate back: dq = R(c)^T dq~ (pairs may straddle the group's lanes), through
  // shared memory in passes of 2 * KC rows
  for (int pass = 0; pass < TILE / (2 * KC); ++pass) {
    const int r = qs - pass * 2 * KC;
    const bool mine = r >= 0 && r < 2 * KC;
    __syncthreads();
    if (mine) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) sbuf[r * D + lane * CPT + u] = dqr[u];
    }
    __syncthreads();
    if (mine && active) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        int c = lane * CPT + u;
        dq[qrow + c] = from_f32<T>(rot_channel_smem(sbuf + r * D, ix.rope, g, c, cz, cy, cx, qi, true));
      }
    }
  }
}

// dk, dv: key-major.  The queries whose window holds key j are those within the
// window radius of j (the box is symmetric), i.e. the halo of j's tile.
template <typename T, int D, bool SUMMARY>
__global__ void __launch_bounds__(TILE * Split<D>::G) k_bwd_dkdv(
    Geo g, pack3d_index ix, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const T* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ delta, const float* __restrict__ dks,
    const float* __restrict__ dvs, T* __restrict__ dk, T* __restrict__ dv) {
  constexpr int G = Split<D>::G, CPT = Split<D>::CPT;
  if (ix.err[0]) return;
  // dynamic: staged queries and dO rows, 2 * CAPK rows of D floats
  extern __shared__ __align__(16) float bwd_dyn[];
  float* const sbuf = bwd_dyn;
  float(*sq)[D] = reinterpret_cast<float(*)[D]>(bwd_dyn);
  float(*sdo)[D] = reinterpret_cast<float(*)[D]>(bwd_dyn + CAPK * D);
  __shared__ float slse[CAPK], sdel[CAPK];
  __shared__ PlaneMeta pm;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int ks = threadIdx.x / G, lane = threadIdx.x % G;
  const TileGeo tg = tile_geo(g, t);
  int cz = 0, cy = 0, cx = 0, ke = 0, kj = 0;
  const bool active = box_slot(tg, ks, cz, cy, cx, ke);
  if (active) kj = ix.perm[(int64_t)b * g.N + ix.tile_off[(int64_t)b * (g.nT + 1) + t] + ke];
  const int64_t krow = (((int64_t)b * g.N + kj) * g.H + h) * D;
  float kr[CPT], vr[CPT], dkr[CPT], dvr[CPT];
#pragma unroll
  for (int u = 0; u < CPT; ++u) {
    int c = lane * CPT + u;
    kr[u] = active ? rot_channel(k + krow, ix.rope, g, c, cz, cy, cx, kj, false) : 0.f;
    vr[u] = active ? to_f32(v[krow + c]) : 0.f;
    dkr[u] = 0.f;
    dvr[u] = 0.f;
  }
  const int64_t lbase = ((int64_t)b * g.H + h) * g.N;
  const int32_t* hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
  const WarpBox wb = warp_box(active, cz, cy);
  const int rpc = min(tg.hy, CAPK / tg.hx);  // halo rows per chunk
  for (int pz = 0; pz < tg.hz; ++pz) {
    const int zq = tg.hz0 + pz;
    const bool zneed = zq >= wb.zlo - g.rz && zq <= wb.zhi + g.rz;  // warp-uniform
    for (int ry0 = 0; ry0 < tg.hy; ry0 += rpc) {
      const int nr = min(rpc, tg.hy - ry0), nq = nr * tg.hx;
      const int base = (pz * tg.hy + ry0) * tg.hx;
      __syncthreads();
      for (int e = threadIdx.x; e < nq; e += blockDim.x) {
        halo_coord(tg, base + e, pm.z[e], pm.y[e], pm.x[e]);
        const int i = hl[base + e];
        pm.tok[e] = i;
        slse[e] = lse[lbase + i];
        sdel[e] = delta[lbase + i];
      }
      __syncthreads();
      stage_rows_n<T, D, TILE * G>(g, ix.rope, q, dout, b, h, pm.tok, pm.z, pm.y, pm.x, nq,
                                   &sq[0][0], &sdo[0][0]);
      __syncthreads();
      if (!zneed) continue;
      for (int r = 0; r < nr; ++r) {
        const int yq = tg.hy0 + ry0 + r;
        if (yq < wb.ylo - g.ry || yq > wb.yhi + g.ry) continue;  // warp-uniform
        const bool rowin = active && abs(zq - cz) <= g.rz && abs(yq - cy) <= g.ry;
        const int q0 = r * tg.hx, q1 = q0 + tg.hx;
        // queries in pairs (two independent dot-product chains per thread); at
        // an odd row end the second query repeats the first with weight 0.  A
        // pair whose windows miss every key of the warp is skipped.
        for (int qa = q0; qa < q1; qa += 2) {
          const int qb = min(qa + 1, q1 - 1);
          const bool in0 = rowin && abs(pm.x[qa] - cx) <= g.rx;
          const bool in1 = rowin && qa + 1 < q1 && abs(pm.x[qb] - cx) <= g.rx;
          if (!__any_sync(0xffffffffu, in0 || in1)) continue;
          const float ps0 = dot_row(kr, &sq[qa][lane * CPT]);
          const float ps1 = dot_row(kr, &sq[qb][lane * CPT]);
          const float pd0 = dot_row(vr, &sdo[qa][lane * CPT]);
          const float pd1 = dot_row(vr, &sdo[qb][lane * CPT]);
          const float s0 = group_sum<G>(ps0), s1 = group_sum<G>(ps1);
          const float dp0 = group_sum<G>(pd0), dp1 = group_sum<G>(pd1);
          // re-read the staged rows below instead of holding them in registers
          __syncwarp();
          const float P0 = in0 ? expf(g.tau * s0 - slse[qa]) : 0.f;
          const float P1 = in1 ? expf(g.tau * s1 - slse[qb]) : 0.f;
          const float dS0 = P0 * (dp0 - sdel[qa]), dS1 = P1 * (dp1 - sdel[qb]);
          axpy_row(dkr, g.tau * dS0, &sq[qa][lane * CPT]);
          axpy_row(dkr, g.tau * dS1, &sq[qb][lane * CPT]);
          axpy_row(dvr, P0, &sdo[qa][lane * CPT]);
          axpy_row(dvr, P1, &sdo[qb][lane * CPT]);
        }
      }
    }
  }
  if (SUMMARY && active) {
    int B = ((cz / g.bz) * g.nby + cy / g.by) * g.nbx + cx / g.bx;
    const int64_t srow = (((int64_t)b * g.H + h) * g.nb + B) * D;
    const BlockExt be = block_ext(g, cz / g.bz, cy / g.by, cx / g.bx);
    const float inv = 1.f / (float)(be.ez * be.ey * be.ex);
#pragma unroll
    for (int u = 0; u < CPT; ++u) {
      int c = lane * CPT + u;
      dkr[u] += dks[srow + c] * inv;
      dvr[u] += dvs[srow + c] * inv;
    }
  }
  for (int pass = 0; pass < TILE / (2 * KC); ++pass) {
    const int r = ks - pass * 2 * KC;
    const bool mine = r >= 0 && r < 2 * KC;
    __syncthreads();
    if (mine) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) sbuf[r * D + lane * CPT + u] = dkr[u];
    }
    __syncthreads();
    if (mine && active) {
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        int c = lane * CPT + u;
        dk[krow + c] = from_f32<T>(rot_channel_smem(sbuf + r * D, ix.rope, g, c, cz, cy, cx, kj, true));
        dv[krow + c] = from_f32<T>(dvr[u]);
      }
    }
  }
}

template <typename T, typename TO, int D>
int forward_launch(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                   const void* v, const float* ksum, const float* vsum, void* out, float* lse,
                   bool summaries, cudaStream_t s) {
  dim3 grid(g.nT, g.H, g.B);
  dim3 block(TILE * Split<D>::G);
  if (summaries)
    k_forward_simt<T, TO, D, true><<<grid, block, 0, s>>>(
        g, *idx, (const T*)q, (const T*)k, (const T*)v, ksum, vsum, (TO*)out, lse);
  else
    k_forward_simt<T, TO, D, false><<<grid, block, 0, s>>>(
        g, *idx, (const T*)q, (const T*)k, (const T*)v, ksum, vsum, (TO*)out, lse);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

template <typename T, int D>
int forward_dispatch_sum(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                         const void* v, const float* ksum, const float* vsum, void* out,
                         float* lse, bool summaries, cudaStream_t s) {
  if (g.out_fp32)
    return forward_launch<T, float, D>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
  return forward_launch<T, T, D>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
}

template <typename T>
int forward_dispatch(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                     const void* v, const float* ksum, const float* vsum, void* out, float* lse,
                     bool summaries, cudaStream_t s) {
  switch (g.d) {
    case 12: return forward_dispatch_sum<T, 12>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
    case 24: return forward_dispatch_sum<T, 24>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
    case 48: return forward_dispatch_sum<T, 48>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
    case 96: return forward_dispatch_sum<T, 96>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
    default: return PACK3D_ERR_UNSUPPORTED;
  }
}

struct BwdWs {
  float *delta, *ksum, *vsum, *dks, *dvs, *part;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Query splits of the d = 96 summary-gradient kernel: as many CTAs as fit in
// one wave of two CTAs per SM, at most one split per query tile, at most 32.
inline int summary96_splits(const Geo& g) {
  if (g.d != 96) return 0;
  const int nbc = (g.nb + S96_NB - 1) / S96_NB;
  const int64_t groups = (int64_t)g.B * g.H * nbc;
  int64_t s = (2 * 148) / groups;
  s = std::min<int64_t>(s, std::min(g.nT, 32));
  return (int)std::max<int64_t>(s, 1);
}

BwdWs carve(const Geo& g, void* ws) {
  char* p = (char*)ws;
  BwdWs w;
  size_t nd = sizeof(float) * (size_t)g.B * g.H * g.N;
  size_t ns = sizeof(float) * (size_t)g.B * g.H * g.nb * g.d;
  w.delta = (float*)p;
  p += align256(nd);
  w.ksum = (float*)p;
  p += align256(ns);
  w.vsum = (float*)p;
  p += align256(ns);
  w.dks = (float*)p;
  p += align256(ns);
  w.dvs = (float*)p;
  p += align256(ns);
  w.part = (float*)p;
  return w;
}

template <typename T, int D>
int backward_typed(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                   const void* v, const void* out, const float* lse, const void* dout, void* dq,
                   void* dk, void* dv, void* workspace, cudaStream_t s) {
  BwdWs w = carve(g, workspace);
  int64_t rows = (int64_t)g.B * g.N * g.H;
  if (g.out_fp32)
    k_bwd_delta<T, float><<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(
        g, idx->err, (const float*)out, (const T*)dout, w.delta);
  else
    k_bwd_delta<T, T><<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(
        g, idx->err, (const T*)out, (const T*)dout, w.delta);
  count_launches(1);
  int rc = launch_block_summaries(g, idx, k, v, w.ksum, w.vsum, s);
  if (rc) return rc;
  if constexpr (D == 96) {
    const int nsplit = summary96_splits(g);
    const int nbc = (g.nb + S96_NB - 1) / S96_NB;
    // set on every call: the attributes belong to the current device
    cudaError_t e = cudaFuncSetAttribute(k_bwd_summary96<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(Sum96Smem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_bwd_summary96<T>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 sgrid(nbc * nsplit, g.B, g.H);
    k_bwd_summary96<T><<<sgrid, S96_THREADS, sizeof(Sum96Smem), s>>>(
        g, *idx, (const T*)q, (const T*)dout, lse, w.delta, w.ksum, w.vsum, nsplit, w.part);
    const int64_t per = (int64_t)g.B * g.H * g.nb * g.d;
    k_bwd_summary_reduce<<<(unsigned)((per + 255) / 256), 256, 0, s>>>(g, idx->err, nsplit,
                                                                       w.part, w.dks, w.dvs);
    count_launches(2);
  } else {
    dim3 sgrid((g.nb + BC - 1) / BC, g.B, g.H);
    k_bwd_summary<T, D><<<sgrid, 256, 0, s>>>(g, *idx, (const T*)q, (const T*)dout, lse,
                                              w.delta, w.ksum, w.vsum, w.dks, w.dvs);
    count_launches(1);
  }
  const size_t dyn = 2 * (size_t)CAPK * D * sizeof(float);
  {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_dq<T, D, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_bwd_dkdv<T, D, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return cuda_status(e);
  }
  dim3 grid(g.nT, g.H, g.B);
  dim3 block(TILE * Split<D>::G);
  k_bwd_dq<T, D, true><<<grid, block, dyn, s>>>(g, *idx, (const T*)q, (const T*)k, (const T*)v,
                                                (const T*)dout, lse, w.delta, w.ksum, w.vsum,
                                                (T*)dq);
  k_bwd_dkdv<T, D, true><<<grid, block, dyn, s>>>(g, *idx, (const T*)q, (const T*)k,
                                                  (const T*)v, (const T*)dout, lse, w.delta,
                                                  w.dks, w.dvs, (T*)dk, (T*)dv);
  count_launches(2);
  return cuda_status(cudaGetLastError());
}

template <typename T>
int backward_dispatch(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                      const void* v, const void* out, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, void* ws, cudaStream_t s) {
  switch (g.d) {
    case 12: return backward_typed<T, 12>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, ws, s);
    case 24: return backward_typed<T, 24>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, ws, s);
    case 48: return backward_typed<T, 48>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, ws, s);
    case 96: return backward_typed<T, 96>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, ws, s);
    default: return PACK3D_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_forward_simt(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                        const void* v, const float* ksum, const float* vsum, void* out,
                        float* lse, bool summaries, cudaStream_t s) {
  if (g.dtype == PACK3D_BF16)
    return forward_dispatch<__nv_bfloat16>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
  return forward_dispatch<float>(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
}

int backward_simt_supported(const Geo& g) {
  // dense volumes only; one halo row (the tile's 8 columns widened by the
  // window radius on both sides, clipped to the volume) must fit in a staged
  // chunk
  if (g.partial || g.sharded) return PACK3D_ERR_UNSUPPORTED;
  return std::min(g.X, TX + 2 * g.rx) <= CAPK ? PACK3D_OK : PACK3D_ERR_UNSUPPORTED;
}

size_t backward_simt_workspace_bytes(const Geo& g) {
  size_t nd = sizeof(float) * (size_t)g.B * g.H * g.N;
  size_t ns = sizeof(float) * (size_t)g.B * g.H * g.nb * g.d;
  return align256(nd) + 4 * align256(ns) + 2 * (size_t)summary96_splits(g) * ns;
}

int launch_backward_simt(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                         const void* v, const void* out, const float* lse, const void* dout,
                         void* dq, void* dk, void* dv, void* workspace, cudaStream_t s) {
  if (g.dtype == PACK3D_BF16)
    return backward_dispatch<__nv_bfloat16>(g, idx, q, k, v, out, lse, dout, dq, dk, dv,
                                            workspace, s);
  return backward_dispatch<float>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, workspace, s);
}

}  // namespace p3d
