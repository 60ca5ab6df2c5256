// PACK3D forward on the Blackwell tensor cores (bf16 in, fp32 accumulate).
//
// "Geometry Matters in Packed 3D Attention" (abstract): each query attends
// exactly to its clipped 3D window and to the summaries of the blocks its
// window misses, in one softmax, with axial RoPE on grid coordinates.
//
// One CTA computes one 4 x 4 x 8 query tile (M = 128 rows) of one
// (batch item, head):
//   * the tile's queries are gathered through the tile permutation, rotated
//     in registers and stored to shared memory in the 64-byte-swizzled K-major
//     layout (head_dim 96 = three 32-channel segments, one per axis, so each
//     rotation segment is exactly one swizzle atom column);
//   * the tile's halo (the union of its windows) is streamed in chunks of 128
//     keys through the halo list; each key row is rotated on the way into
//     shared memory and each value row is stored as the MN-major B operand of
//     the PV product;
//   * S = Q K^T runs as six tcgen05.mma (K = 16) into TMEM; the four softmax
//     warps (one row per thread) read S, apply the 3D window mask, keep the
//     online max and sum, and write P (bf16) back over S in TMEM;
//   * O += P V runs as eight tcgen05.mma with A = P read from TMEM;
//   * after the local chunks, the block summaries are streamed the same way,
//     with the mask "block box does not meet the window box", into the same
//     softmax state (no count bias);
//   * the epilogue divides by the row sum, writes out in packed order and the
//     natural-log LSE.
// The running max is only moved when a row's new maximum exceeds it by more
// than 8 (log2 units), so O is rescaled in TMEM rarely; the result is the same
// softmax.  Two CTAs share an SM (256 TMEM columns each), so one CTA's gather
// overlaps the other's MMAs and softmax.
#include <math.h>

#include "pack3d_internal.cuh"
#include "tc_primitives.cuh"

namespace p3d {

namespace {

using namespace tc;

constexpr int D = 96;                 // head dim handled by this kernel
constexpr int KCH = 128;              // keys per chunk (N of the S MMA)
constexpr int SEG_BYTES = 128 * 64;   // one 32-channel segment of 128 rows
constexpr int OPND_BYTES = 3 * SEG_BYTES;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_O = 0;         // O accumulator: columns [0, 96)
constexpr uint32_t COL_S = 128;       // S / P: columns [128, 256)
constexpr int NTHREADS = 128;
constexpr uint32_t WAIT_LIMIT = 1u << 26;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr int ERR_TIMEOUT_BIT = 4;

struct Smem {
  uint8_t q[OPND_BYTES];     // A of S = Q K^T
  uint8_t k[OPND_BYTES];     // B of S = Q K^T (K-major)
  uint8_t v[OPND_BYTES];     // B of O = P V (MN-major)
  int32_t kz[KCH], ky[KCH], kx[KCH];  // key coordinates (local chunk) or block coordinates
  uint64_t bar_s, bar_o;
  uint32_t tmem_base;
  int32_t abort;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;  // + alignment slack
// Request enough shared memory that at most two CTAs share an SM (their TMEM
// allocations of 256 columns then always fit).
constexpr size_t SMEM_REQUEST = SMEM_BYTES > 80 * 1024 ? SMEM_BYTES : 80 * 1024;

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

// Load a 96-channel bf16 row (192 bytes) as 12 x 16 bytes.
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, uint4 (&r)[12]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 12; ++i) r[i] = __ldg(s + i);
}

// Axial rotation of a loaded row in place.  Word w of the row holds channels
// 2w, 2w+1; segment a covers words [16a, 16a + 16); channel j of a segment
// pairs with j + 16, i.e. word w with word w + 8.
__device__ __forceinline__ void rotate_row(uint4 (&r)[12], const float2* __restrict__ tab,
                                           const Geo& g, int cz, int cy, int cx) {
  uint32_t* w = reinterpret_cast<uint32_t*>(r);
#pragma unroll
  for (int a = 0; a < 3; ++a) {
    int c = a == 0 ? cz : (a == 1 ? cy : cx);
    int off = a == 0 ? 0 : (a == 1 ? g.Z : g.Z + g.Y);
    const float2* t = tab + (off + c) * 16;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float2 x1 = unpack_bf16x2(w[16 * a + u]);
      float2 x2 = unpack_bf16x2(w[16 * a + u + 8]);
      float2 c0 = __ldg(t + 2 * u), c1 = __ldg(t + 2 * u + 1);
      w[16 * a + u] = pack_bf16x2(x1.x * c0.x - x2.x * c0.y, x1.y * c1.x - x2.y * c1.y);
      w[16 * a + u + 8] = pack_bf16x2(x1.x * c0.y + x2.x * c0.x, x1.y * c1.y + x2.y * c1.x);
    }
  }
}

// Store a 96-channel row into an operand region (three 32-channel segments of
// 128 rows x 64 bytes, 64-byte swizzle).  The same bytes serve as a K-major
// operand (rows = M or N) and as an MN-major operand (rows = K).
__device__ __forceinline__ void store_row(uint8_t* region, int row, const uint4 (&r)[12]) {
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(region + a * SEG_BYTES + sw64_off(row, c)) = r[4 * a + c];
}

__device__ __forceinline__ void zero_row(uint4 (&r)[12]) {
#pragma unroll
  for (int i = 0; i < 12; ++i) r[i] = make_uint4(0, 0, 0, 0);
}

__device__ __forceinline__ void fp32_row_to_bf16(const float* __restrict__ src, uint4 (&r)[12]) {
  const float4* s = reinterpret_cast<const float4*>(src);
  uint32_t* w = reinterpret_cast<uint32_t*>(r);
#pragma unroll
  for (int i = 0; i < 24; ++i) {
    float4 f = __ldg(s + i);
    w[2 * i] = pack_bf16x2(f.x, f.y);
    w[2 * i + 1] = pack_bf16x2(f.z, f.w);
  }
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
  const int tid = threadIdx.x, warp = tid / 32;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const TileBox tb = tile_box(g, t);
  const int count = tb.lz * tb.ly * tb.lx;
  const float2* __restrict__ tab = reinterpret_cast<const float2*>(ix.rope);

  if (tid == 0) {
    mbar_init(&sm.bar_s, 1);
    mbar_init(&sm.bar_o, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }

  // ---- query row of this thread: gather, rotate, stage ----
  const bool active = tid < count;
  int cz = 0, cy = 0, cx = 0, qi = 0;
  {
    uint4 r[12];
    if (active) {
      cx = tb.x0 + tid % tb.lx;
      cy = tb.y0 + (tid / tb.lx) % tb.ly;
      cz = tb.z0 + tid / (tb.lx * tb.ly);
      qi = ix.perm[(int64_t)b * g.N + ix.tile_off[(int64_t)b * (g.nT + 1) + t] + tid];
      load_row(q + (((int64_t)b * g.N + qi) * g.H + h) * D, r);
      rotate_row(r, tab, g, cz, cy, cx);
    } else {
      zero_row(r);
    }
    store_row(sm.q, tid, r);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const uint32_t tS = tbase + lane_base + COL_S;
  const uint32_t tO = tbase + lane_base + COL_O;

  // O starts at zero so every PV MMA can accumulate.
  {
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
    tmem_st32(tO + 0, z);
    tmem_st32(tO + 32, z);
    tmem_st32(tO + 64, z);
    tmem_wait_st();
  }

  const float c2 = g.tau * LOG2E;  // logits -> log2 units
  float m_run = -INFINITY, l_run = 0.f;
  uint32_t phase = 0;
  bool ok = true;

  const int nh = tb.hz * tb.hy * tb.hx;
  const int n_local = (nh + KCH - 1) / KCH;
  const int n_sum = SUMMARY ? (g.nb + KCH - 1) / KCH : 0;
  const int32_t* __restrict__ hl = ix.nbr + (int64_t)b * ix.n_halo + ix.nbr_off[t];
  const int64_t sbase = ((int64_t)b * g.H + h) * g.nb;

  for (int ch = 0; ch < n_local + n_sum; ++ch) {
    const bool local = ch < n_local;
    // ---- stage chunk: thread tid loads key row tid ----
    {
      uint4 kr[12], vr[12];
      if (local) {
        const int e = ch * KCH + tid;
        if (e < nh) {
          int x = tb.hx0 + e % tb.hx, y = tb.hy0 + (e / tb.hx) % tb.hy,
              z = tb.hz0 + e / (tb.hx * tb.hy);
          int j = hl[e];
          int64_t row = (((int64_t)b * g.N + j) * g.H + h) * D;
          load_row(k + row, kr);
          load_row(v + row, vr);
          rotate_row(kr, tab, g, z, y, x);
          sm.kz[tid] = z;
          sm.ky[tid] = y;
          sm.kx[tid] = x;
        } else {
          zero_row(kr);
          zero_row(vr);
          sm.kz[tid] = -0x40000000;  // never within a window
          sm.ky[tid] = 0;
          sm.kx[tid] = 0;
        }
      } else {
        const int B = (ch - n_local) * KCH + tid;
        if (B < g.nb) {
          fp32_row_to_bf16(ksum + (sbase + B) * D, kr);
          fp32_row_to_bf16(vsum + (sbase + B) * D, vr);
          sm.kz[tid] = B / (g.nby * g.nbx);
          sm.ky[tid] = (B / g.nbx) % g.nby;
          sm.kx[tid] = B % g.nbx;
        } else {
          zero_row(kr);
          zero_row(vr);
          sm.kz[tid] = -1;  // marks padding
          sm.ky[tid] = 0;
          sm.kx[tid] = 0;
        }
      }
      store_row(sm.k, tid, kr);
      store_row(sm.v, tid, vr);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- S = Q K^T ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t qa = smem_u32(sm.q), ka = smem_u32(sm.k);
      constexpr uint32_t idesc = idesc_bf16(128, KCH, false);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        uint32_t off = (s >> 1) * SEG_BYTES + (s & 1) * 32;
        mma_ss(tbase + COL_S, sdesc_sw64(qa + off, 16, 512), sdesc_sw64(ka + off, 16, 512),
               idesc, s > 0);
      }
      mma_commit(&sm.bar_s);
    }
    if (!mbar_wait(&sm.bar_s, phase, WAIT_LIMIT)) ok = false;
    tc_fence_after();

    // ---- softmax on this thread's row ----
    uint32_t mask[4];
    float cmax = -INFINITY;
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      uint32_t r[32];
      tmem_ld32(tS + seg * 32, r);
      tmem_wait_ld();
      uint32_t mbits = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int kk = seg * 32 + i;
        bool in;
        if (local) {
          in = abs(sm.kz[kk] - cz) <= g.rz && abs(sm.ky[kk] - cy) <= g.ry &&
               abs(sm.kx[kk] - cx) <= g.rx;
        } else {
          int bz0 = sm.kz[kk] * g.bz, by0 = sm.ky[kk] * g.by, bx0 = sm.kx[kk] * g.bx;
          bool meets = bz0 + g.bz - 1 >= cz - g.rz && bz0 <= cz + g.rz &&
                       by0 + g.by - 1 >= cy - g.ry && by0 <= cy + g.ry &&
                       bx0 + g.bx - 1 >= cx - g.rx && bx0 <= cx + g.rx;
          in = sm.kz[kk] >= 0 && !meets;
        }
        in = in && active;
        mbits |= (in ? 1u : 0u) << i;
        if (in) cmax = fmaxf(cmax, __uint_as_float(r[i]));
      }
      mask[seg] = mbits;
    }
    // Move the running max only when the chunk max exceeds it by the threshold.
    const float cmax2 = cmax * c2;  // -inf stays -inf
    bool bump = cmax2 > m_run + RESCALE_THRESHOLD || (m_run == -INFINITY && cmax2 > -INFINITY);
    float corr = 1.f;
    if (bump) {
      corr = m_run == -INFINITY ? 1.f : exp2f(m_run - cmax2);
      l_run *= corr;
      m_run = cmax2;
    }
    if (__any_sync(0xffffffffu, corr != 1.f)) {
      // O is not being written: the previous PV MMA completed before this chunk.
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        uint32_t r[32];
        tmem_ld32(tO + part * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
        tmem_st32(tO + part * 32, r);
      }
    }
    const float mneg = m_run == -INFINITY ? 0.f : -m_run;
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      uint32_t r[32];
      tmem_ld32(tS + seg * 32, r);
      tmem_wait_ld();
      uint32_t p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        bool in0 = (mask[seg] >> (2 * i)) & 1u, in1 = (mask[seg] >> (2 * i + 1)) & 1u;
        float p0 = in0 ? exp2f(fmaf(__uint_as_float(r[2 * i]), c2, mneg)) : 0.f;
        float p1 = in1 ? exp2f(fmaf(__uint_as_float(r[2 * i + 1]), c2, mneg)) : 0.f;
        l_run += p0 + p1;
        p[i] = pack_bf16x2(p0, p1);
      }
      // P for keys [32 seg, 32 seg + 32) goes to columns [16 seg, 16 seg + 16)
      // of the S region, which hold S values already read.
      tmem_st16(tS + seg * 16, p);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t va = smem_u32(sm.v);
      constexpr uint32_t idesc = idesc_bf16(128, D, true);
#pragma unroll
      for (int s = 0; s < KCH / 16; ++s) {
        mma_ts(tbase + COL_O, tbase + COL_S + s * 8,
               sdesc_sw64(va + s * 16 * 64, SEG_BYTES, 512), idesc, 1);
      }
      mma_commit(&sm.bar_o);
    }
    if (!mbar_wait(&sm.bar_o, phase, WAIT_LIMIT)) ok = false;
    tc_fence_after();
    phase ^= 1;
    if (!ok) sm.abort = 1;
    __syncthreads();
    if (sm.abort) break;
  }

  // ---- epilogue ----
  if (!sm.abort) {
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const int64_t orow_off = (((int64_t)b * g.N + qi) * g.H + h) * D;
    if (!g.out_fp32) {
      uint4 orow[12];
      uint32_t* ow = reinterpret_cast<uint32_t*>(orow);
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        uint32_t r[32];
        tmem_ld32(tO + part * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          ow[part * 16 + i] =
              pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
      }
      if (active) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out_raw) + orow_off);
#pragma unroll
        for (int i = 0; i < 12; ++i) dst[i] = orow[i];
      }
    } else {
      float* dstf = reinterpret_cast<float*>(out_raw) + orow_off;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        uint32_t r[32];
        tmem_ld32(tO + part * 32, r);
        tmem_wait_ld();
        if (active) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(dstf + part * 32)[i] = make_float4(
                __uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
        }
      }
    }
    if (active) lse[((int64_t)b * g.H + h) * g.N + qi] = (m_run + log2f(l_run)) * LN2;
  } else if (tid == 0) {
    atomicOr(&ix.err[0], ERR_TIMEOUT_BIT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
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
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_REQUEST);
  if (e != cudaSuccess) return PACK3D_ERR_CUDA;
  kern<<<grid, NTHREADS, SMEM_REQUEST, s>>>(g, *idx, (const __nv_bfloat16*)q,
                                             (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                             ksum, vsum, out, lse);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
