// PACK3D attention on the CUDA cores in fp32: the forward used for the fp32
// mode (and for head dims the tensor-core kernel is not built for), and the
// full backward.
//
// Operator ("Geometry Matters in Packed 3D Attention", abstract): exact
// attention over each query's clipped 3D window plus the summaries of the
// blocks that do not meet the window, one softmax, axial RoPE on grid
// coordinates.  One CTA serves one query tile of one (batch item, head);
// G = d / 24 threads (at least 1) share a query, each owning CPT = d / G
// channels, and dot products are finished with warp shuffles inside the
// group.  Keys are staged per chunk of KC tokens in shared memory, already
// rotated, as fp32.  Every reduction runs in a fixed order; key coordinates are
// derived from the halo box, query coordinates from the tile box, so no
// coordinate array is read.
#include <math.h>

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
  int z[KC], y[KC], x[KC];
};

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
  __shared__ float sq[QC][D];
  __shared__ float sdo[QC][D];
  __shared__ float skb[BC][D];
  __shared__ float svb[BC][D];
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

// dq: query-major, the forward's structure.
template <typename T, int D, bool SUMMARY>
__global__ void __launch_bounds__(TILE * Split<D>::G) k_bwd_dq(
    Geo g, pack3d_index ix, const T* __restrict__ q, const T* __restrict__ k,
    const T* __restrict__ v, const T* __restrict__ dout, const float* __restrict__ lse,
    const float* __restrict__ delta, const float* __restrict__ ksum,
    const float* __restrict__ vsum, T* __restrict__ dq) {
  constexpr int G = Split<D>::G, CPT = Split<D>::CPT;
  if (ix.err[0]) return;
  __shared__ float sbuf[2 * KC * D];
  float(*sk)[D] = reinterpret_cast<float(*)[D]>(sbuf);
  float(*sv)[D] = reinterpret_cast<float(*)[D]>(sbuf + KC * D);
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
    for (int kk = 0; kk < KC; ++kk) {
      float ps = 0.f, pd = 0.f;
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        ps += qr[u] * sk[kk][lane * CPT + u];
        pd += dO[u] * sv[kk][lane * CPT + u];
      }
      float s = group_sum<G>(ps), dp = group_sum<G>(pd);
      bool in = active && kk < nk && abs(cc.z[kk] - cz) <= g.rz && abs(cc.y[kk] - cy) <= g.ry &&
                abs(cc.x[kk] - cx) <= g.rx;
      float P = in ? expf(g.tau * s - lse_i) : 0.f;
      float dS = P * (dp - del_i);
#pragma unroll
      for (int u = 0; u < CPT; ++u) dqr[u] += g.tau * dS * sk[kk][lane * CPT + u];
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
        float ps = 0.f, pd = 0.f;
#pragma unroll
        for (int u = 0; u < CPT; ++u) {
          ps += qr[u] * sk[kk][lane * CPT + u];
          pd += dO[u] * sv[kk][lane * CPT + u];
        }
        float s = group_sum<G>(ps), dp = group_sum<G>(pd);
        int bz0 = cc.z[kk] * g.bz, by0 = cc.y[kk] * g.by, bx0 = cc.x[kk] * g.bx;
        bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                     by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                     bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
        bool in = active && kk < nk && !meets;
        float P = in ? expf(g.tau * s - lse_i) : 0.f;
        float dS = P * (dp - del_i);
#pragma unroll
        for (int u = 0; u < CPT; ++u) dqr[u] += g.tau * dS * sk[kk][lane * CPT + u];
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
  __shared__ float sbuf[2 * KC * D];
  float(*sq)[D] = reinterpret_cast<float(*)[D]>(sbuf);
  float(*sdo)[D] = reinterpret_cast<float(*)[D]>(sbuf + KC * D);
  __shared__ float slse[KC], sdel[KC];
  __shared__ ChunkCoords cc;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int ks = threadIdx.x / G, lane = threadIdx.x % G;
  const TileGeo tg = tile_geo(g, t);
  const int count = tg.lz * tg.ly * tg.lx;
  const bool active = ks < count;
  int cz = 0, cy = 0, cx = 0, kj = 0;
  if (active) {
    tile_coord(tg, ks, cz, cy, cx);
    kj = ix.perm[(int64_t)b * g.N + ix.tile_off[(int64_t)b * (g.nT + 1) + t] + ks];
  }
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
  const int nh = tg.hz * tg.hy * tg.hx;
  const int32_t* hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
  for (int base = 0; base < nh; base += KC) {
    const int nq = min(KC, nh - base);
    __syncthreads();
    for (int e = threadIdx.x; e < KC * D; e += blockDim.x) {
      int qq = e / D, c = e % D;
      float qv = 0.f, dov = 0.f;
      if (qq < nq) {
        int z, y, x;
        halo_coord(tg, base + qq, z, y, x);
        int i = hl[base + qq];
        int64_t row = (((int64_t)b * g.N + i) * g.H + h) * D;
        qv = rot_channel(q + row, ix.rope, g, c, z, y, x, i, false);
        dov = to_f32(dout[row + c]);
        if (c == 0) {
          cc.z[qq] = z;
          cc.y[qq] = y;
          cc.x[qq] = x;
          slse[qq] = lse[lbase + i];
          sdel[qq] = delta[lbase + i];
        }
      }
      sq[qq][c] = qv;
      sdo[qq][c] = dov;
    }
    __syncthreads();
    for (int qq = 0; qq < KC; ++qq) {
      float ps = 0.f, pd = 0.f;
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        ps += kr[u] * sq[qq][lane * CPT + u];
        pd += vr[u] * sdo[qq][lane * CPT + u];
      }
      float s = group_sum<G>(ps), dp = group_sum<G>(pd);
      bool in = active && qq < nq && abs(cc.z[qq] - cz) <= g.rz && abs(cc.y[qq] - cy) <= g.ry &&
                abs(cc.x[qq] - cx) <= g.rx;
      float P = in ? expf(g.tau * s - slse[qq]) : 0.f;
      float dS = P * (dp - sdel[qq]);
#pragma unroll
      for (int u = 0; u < CPT; ++u) {
        dkr[u] += g.tau * dS * sq[qq][lane * CPT + u];
        dvr[u] += P * sdo[qq][lane * CPT + u];
      }
    }
  }
  if (SUMMARY && active) {
    int B = ((cz / g.bz) * g.nby + cy / g.by) * g.nbx + cx / g.bx;
    const int64_t srow = (((int64_t)b * g.H + h) * g.nb + B) * D;
    const float inv = 1.f / (float)(g.bz * g.by * g.bx);
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
  float *delta, *ksum, *vsum, *dks, *dvs;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

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
  int rc = launch_block_summaries(g, idx, k, v, w.ksum, w.vsum, s);
  if (rc) return rc;
  dim3 sgrid((g.nb + BC - 1) / BC, g.B, g.H);
  k_bwd_summary<T, D><<<sgrid, 256, 0, s>>>(g, *idx, (const T*)q, (const T*)dout, lse, w.delta,
                                            w.ksum, w.vsum, w.dks, w.dvs);
  dim3 grid(g.nT, g.H, g.B);
  dim3 block(TILE * Split<D>::G);
  k_bwd_dq<T, D, true><<<grid, block, 0, s>>>(g, *idx, (const T*)q, (const T*)k, (const T*)v,
                                              (const T*)dout, lse, w.delta, w.ksum, w.vsum,
                                              (T*)dq);
  k_bwd_dkdv<T, D, true><<<grid, block, 0, s>>>(g, *idx, (const T*)q, (const T*)k, (const T*)v,
                                                (const T*)dout, lse, w.delta, w.dks, w.dvs,
                                                (T*)dk, (T*)dv);
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

size_t backward_workspace_bytes(const Geo& g) {
  size_t nd = sizeof(float) * (size_t)g.B * g.H * g.N;
  size_t ns = sizeof(float) * (size_t)g.B * g.H * g.nb * g.d;
  return align256(nd) + 4 * align256(ns);
}

int launch_backward(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                    const void* v, const void* out, const float* lse, const void* dout, void* dq,
                    void* dk, void* dv, void* workspace, cudaStream_t s) {
  if (g.dtype == PACK3D_BF16)
    return backward_dispatch<__nv_bfloat16>(g, idx, q, k, v, out, lse, dout, dq, dk, dv,
                                            workspace, s);
  return backward_dispatch<float>(g, idx, q, k, v, out, lse, dout, dq, dk, dv, workspace, s);
}

}  // namespace p3d
