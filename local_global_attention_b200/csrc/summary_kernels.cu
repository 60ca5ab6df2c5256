// Block summaries: per (batch item, head, block) the mean of the rotated keys
// and the mean of the values over the block's tokens, fp32 accumulation.
//
// "Geometry Matters in Packed 3D Attention" (abstract): distant context is
// compressed "into contiguous 3D block summaries", and "the rotation is
// applied before a block is summarized", so the key summary is the mean of
// R(c_j) k_j, not R(.) of a mean.
//
// HBM-bound: every k and v row is read once.  One CTA per (block, batch item,
// head).  In the general kernel the threads form TG token groups of d/4 lanes,
// each lane owning two adjacent rotation pairs (four output channels): a lane
// reads 2 x 4 bytes of k (the pair members sit da/2 channels apart) and 2 x 4
// bytes of v per token, and the d/4 lanes of a token group read one 2d-byte
// row contiguously.  The bf16 head_dim-96 kernel reads 16-byte chunks instead.
// Tokens are visited through the coordinate volume in block raster order, so
// the accumulation order, and the result, do not depend on the packing.
#include "pack3d_internal.cuh"
#include "tc_primitives.cuh"

namespace p3d {

namespace {

constexpr int TG = 8;  // token groups per CTA

template <typename T>
struct Pair2;
template <>
struct Pair2<float> {
  using type = float2;
  static __device__ __forceinline__ float2 f(float2 x) { return x; }
};
template <>
struct Pair2<__nv_bfloat16> {
  using type = __nv_bfloat162;
  static __device__ __forceinline__ float2 f(__nv_bfloat162 x) { return __bfloat1622float2(x); }
};

template <typename T>
__global__ void __launch_bounds__(256) k_block_summaries(Geo g, const int32_t* __restrict__ vol,
                                                         const float* __restrict__ rope,
                                                         const int32_t* __restrict__ err,
                                                         const int32_t* __restrict__ bcount,
                                                         const T* __restrict__ k,
                                                         const T* __restrict__ v, float* ksum,
                                                         float* vsum) {
  if (err[0]) return;
  using P2 = typename Pair2<T>::type;
  extern __shared__ float red[];  // [TG][2][d]
  const int lanes = g.d / 4;
  const int lane = threadIdx.x % lanes, grp = threadIdx.x / lanes;
  const int blk = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int Bz = blk / (g.nby * g.nbx), By = (blk / g.nbx) % g.nby, Bx = blk % g.nbx;
  // Lane -> axis a and first pair j (pairs j, j+1 of that axis); packed mode:
  // pairs j, j + 1 of the whole row, partners d/2 channels on.
  const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
  const int pairs_per_axis = g.half / 2;  // lanes per axis
  const int a = packed ? 0 : lane / pairs_per_axis;
  const int j = packed ? lane * 2 : (lane % pairs_per_axis) * 2;
  const int c1 = packed ? j : a * g.da + j;  // channels of x1 (and +1)
  const int c2 = c1 + g.rope_len;            // channels of x2 (and +1)
  float kx1a = 0.f, kx1b = 0.f, kx2a = 0.f, kx2b = 0.f;
  float vx1a = 0.f, vx1b = 0.f, vx2a = 0.f, vx2b = 0.f;
  const BlockExt be = block_ext(g, Bz, By, Bx);  // cut at the volume's edge
  int bz0, bz1;  // local planes walked
  bool own;      // the block's summary is this call's to give
  block_planes(g, Bz, bz0, bz1, own);
  const int cnt = (bz1 - bz0) * be.ey * be.ex;
  const int32_t* vb = vol + (int64_t)b * g.V;
  if (grp < TG) {
#pragma unroll 4
    for (int e = grp; e < cnt; e += TG) {
      int x = e % be.ex, y = (e / be.ex) % be.ey, z = e / (be.ex * be.ey);
      int cz = bz0 + z, cy = By * g.by + y, cx = Bx * g.bx + x;
      int tok = vb[(cz * g.Y + cy) * g.X + cx];
      if (tok < 0) continue;  // an empty voxel (partly occupied volume)
      int64_t row = (((int64_t)b * g.N + tok) * g.H + h) * g.d;
      float2 k1 = Pair2<T>::f(*reinterpret_cast<const P2*>(k + row + c1));
      float2 k2 = Pair2<T>::f(*reinterpret_cast<const P2*>(k + row + c2));
      float2 v1 = Pair2<T>::f(*reinterpret_cast<const P2*>(v + row + c1));
      float2 v2 = Pair2<T>::f(*reinterpret_cast<const P2*>(v + row + c2));
      int ca = a == 0 ? cz : (a == 1 ? cy : cx);
      float2 csa = rope_cs(rope, g, a, ca, tok, j), csb = rope_cs(rope, g, a, ca, tok, j + 1);
      kx1a += k1.x * csa.x - k2.x * csa.y;
      kx2a += k1.x * csa.y + k2.x * csa.x;
      kx1b += k1.y * csb.x - k2.y * csb.y;
      kx2b += k1.y * csb.y + k2.y * csb.x;
      vx1a += v1.x;
      vx1b += v1.y;
      vx2a += v2.x;
      vx2b += v2.y;
    }
    float* rk = red + (grp * 2 + 0) * g.d;
    float* rv = red + (grp * 2 + 1) * g.d;
    rk[c1] = kx1a;
    rk[c1 + 1] = kx1b;
    rk[c2] = kx2a;
    rk[c2 + 1] = kx2b;
    rv[c1] = vx1a;
    rv[c1 + 1] = vx1b;
    rv[c2] = vx2a;
    rv[c2 + 1] = vx2b;
  }
  __syncthreads();
  // mean over the tokens the block holds (0 for an empty block, and for a
  // block a z-slab does not own)
  const int held = g.partial ? bcount[(int64_t)b * g.nb + blk] : cnt;
  const float inv = held > 0 && own ? 1.0f / (float)held : 0.f;
  int64_t base = (((int64_t)b * g.H + h) * g.nb + blk) * g.d;
  for (int c = threadIdx.x; c < 2 * g.d; c += blockDim.x) {
    int which = c / g.d, ch = c % g.d;
    float s = 0.f;
    for (int t = 0; t < TG; ++t) s += red[(t * 2 + which) * g.d + ch];
    (which ? vsum : ksum)[base + ch] = s * inv;
  }
}

// bf16, head_dim 96: 16-byte loads, two heads per CTA so that a token group
// reads 384 contiguous bytes of k and of v.  Lane u (12 per token) serves head
// u / 6 and owns chunk c1 = 4 (w / 2) + w % 2 (w = u % 6) and its rotation
// partner c2 = c1 + 2 (segment w / 2, pairs 8 (w % 2) .. 8 (w % 2) + 7).  The
// voxel -> token lookups of the next tokens are issued before the current
// tokens' arithmetic.  Partial sums of the 16 token groups are combined in a
// fixed order.
//
// STAGE: the same pass also writes what the tensor-core forward reads - the
// rotated key rows and the value rows in grid order ([b][h][z][y][x][96] bf16,
// kg and vg) and bf16 copies of the summaries (ksb, vsb) - so k and v are read
// from HBM once per step.  The rotated values written are the ones summed
// (rounded to bf16 once), and the fp32 summaries are the same bits as without
// STAGE.
struct StageOut {
  __nv_bfloat16 *kg, *vg, *ksb, *vsb;
};

constexpr int HG96 = 2, LANES96 = 6 * HG96, TG96 = 16, TAB96 = 48;
constexpr int TABS96 = 18;  // staged row stride in float2 (16 + padding against bank conflicts)

template <bool STAGE>
__global__ void __launch_bounds__(TG96 * LANES96) k_block_summaries_bf16_d96(
    Geo g, const int32_t* __restrict__ vol, const float* __restrict__ rope,
    const int32_t* __restrict__ err, const int32_t* __restrict__ bcount,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, float* ksum,
    float* vsum, StageOut so) {
  if (err[0]) return;
  __shared__ float red[TG96][HG96][2][96];
  __shared__ float2 tab_s[TAB96 * TABS96];
  const int u = threadIdx.x % LANES96, grp = threadIdx.x / LANES96;
  const int hh = u / 6, w = u % 6;
  const int blk = blockIdx.x, b = blockIdx.y, h = blockIdx.z * HG96 + hh;
  const bool live = h < g.H;
  const int Bz = blk / (g.nby * g.nbx), By = (blk / g.nbx) % g.nby, Bx = blk % g.nbx;
  const Item96 item = item96(g, w);
  const int a = item.a, c1 = item.c1, c2 = item.c2, j0 = item.j0;
  const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
  // rotation-table rows of this block's coordinates (z, then y, then x rows),
  // staged in shared memory when they fit (packed mode: the rows of the tokens'
  // positions, read from the table)
  const float2* gtab = reinterpret_cast<const float2*>(rope);
  const float2* tab;  // row of coordinate c on this lane's axis: tab + (c - base) * stride
  int base, stride;
  const bool staged = !packed && g.bz + g.by + g.bx <= TAB96;
  if (staged) {
    const int rows = g.bz + g.by + g.bx;
    for (int e = threadIdx.x; e < rows * 16; e += blockDim.x) {
      const int r = e / 16, jj = e % 16;
      // coordinate of table row r on its axis (rows past the volume's edge, in a
      // cut block, are not needed)
      // (local planes of a z-slab: the block row starts at Bz bz - z_origin)
      const int c = r < g.bz ? Bz * g.bz - g.zo + r
                             : (r < g.bz + g.by ? By * g.by + r - g.bz : Bx * g.bx + r - g.bz - g.by);
      const int ext = r < g.bz ? g.Z : (r < g.bz + g.by ? g.Y : g.X);
      const int off = r < g.bz ? 0 : (r < g.bz + g.by ? g.Z : g.Z + g.Y);
      if (c >= 0 && c < ext) tab_s[r * TABS96 + jj] = gtab[(off + c) * 16 + jj];
    }
    __syncthreads();
    tab = a == 0 ? tab_s : (a == 1 ? tab_s + g.bz * TABS96 : tab_s + (g.bz + g.by) * TABS96);
    base = a == 0 ? Bz * g.bz - g.zo : (a == 1 ? By * g.by : Bx * g.bx);
    stride = TABS96;
  } else {
    tab = a == 0 ? gtab : (a == 1 ? gtab + g.Z * 16 : gtab + (g.Z + g.Y) * 16);
    base = 0;
    stride = 16;
  }
  float kx1[8], kx2[8], vx1[8], vx2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) kx1[i] = kx2[i] = vx1[i] = vx2[i] = 0.f;
  const BlockExt be = block_ext(g, Bz, By, Bx);  // cut at the volume's edge
  int bz0, bz1;  // local planes walked
  bool own;      // the block's summary is this call's to give
  block_planes(g, Bz, bz0, bz1, own);
  const int cnt = (bz1 - bz0) * be.ey * be.ex;
  const int32_t* vb = vol + (int64_t)b * g.V;
  auto voxel = [&](int e, int& cz, int& cy, int& cx) {
    cx = Bx * g.bx + e % be.ex;
    cy = By * g.by + (e / be.ex) % be.ey;
    cz = bz0 + e / (be.ex * be.ey);
  };
  // One token's rows (already loaded): rotate, accumulate, and with STAGE
  // write the grid-order copies.
  auto consume = [&](const uint4& ka, const uint4& kb, const uint4& va, const uint4& vb2, int cz,
                     int cy, int cx, int tok_of_consume) {
    const int ca = a == 0 ? cz : (a == 1 ? cy : cx);
    // (an empty voxel's rows are zeros: any table row rotates them to zeros)
    const float2* t = packed ? rope_row96(rope, g, 0, 0, max(tok_of_consume, 0)) + j0
                             : tab + (ca - base) * stride + j0;
    const uint32_t* kaw = reinterpret_cast<const uint32_t*>(&ka);
    const uint32_t* kbw = reinterpret_cast<const uint32_t*>(&kb);
    const uint32_t* vaw = reinterpret_cast<const uint32_t*>(&va);
    const uint32_t* vbw = reinterpret_cast<const uint32_t*>(&vb2);
    uint4 ra, rb;  // rotated chunks c1, c2 (bf16), for the grid-order copy
    uint32_t* raw = reinterpret_cast<uint32_t*>(&ra);
    uint32_t* rbw = reinterpret_cast<uint32_t*>(&rb);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kaw + q));
      float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kbw + q));
      const float4 cs = *reinterpret_cast<const float4*>(t + 2 * q);  // pairs j, j + 1
      const float r1a = x1.x * cs.x - x2.x * cs.y, r2a = x1.x * cs.y + x2.x * cs.x;
      const float r1b = x1.y * cs.z - x2.y * cs.w, r2b = x1.y * cs.w + x2.y * cs.z;
      kx1[2 * q] += r1a;
      kx2[2 * q] += r2a;
      kx1[2 * q + 1] += r1b;
      kx2[2 * q + 1] += r2b;
      if (STAGE) {
        __nv_bfloat162 pa = __floats2bfloat162_rn(r1a, r1b), pb = __floats2bfloat162_rn(r2a, r2b);
        raw[q] = *reinterpret_cast<uint32_t*>(&pa);
        rbw[q] = *reinterpret_cast<uint32_t*>(&pb);
      }
      float2 y1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vaw + q));
      float2 y2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vbw + q));
      vx1[2 * q] += y1.x;
      vx1[2 * q + 1] += y1.y;
      vx2[2 * q] += y2.x;
      vx2[2 * q + 1] += y2.y;
    }
    if (STAGE) {
      const int64_t grow = ((((int64_t)b * g.H + h) * g.Z + cz) * g.Y + cy) * g.X + cx;
      uint4* kd = reinterpret_cast<uint4*>(so.kg + grow * 96);
      uint4* vd = reinterpret_cast<uint4*>(so.vg + grow * 96);
      kd[c1] = ra;
      kd[c2] = rb;
      vd[c1] = va;
      vd[c2] = vb2;
    }
  };
  auto lookup = [&](int e, int& cz, int& cy, int& cx) -> int {
    if (e >= cnt) return 0;
    voxel(e, cz, cy, cx);
    return live ? vb[(cz * g.Y + cy) * g.X + cx] : 0;
  };
  // Tokens e and e + TG96 per iteration (their loads in flight together), the
  // next pair's lookups issued first; each thread still adds its tokens in
  // the order e, e + TG96, e + 2 TG96, ...
  int az = 0, ay = 0, ax = 0, bz2 = 0, by2 = 0, bx2 = 0;
  int ta = lookup(grp, az, ay, ax), tb2 = lookup(grp + TG96, bz2, by2, bx2);
  for (int e = grp; e < cnt; e += 2 * TG96) {
    const bool has_b = e + TG96 < cnt;
    int naz = 0, nay = 0, nax = 0, nbz = 0, nby = 0, nbx = 0;
    const int nta = lookup(e + 2 * TG96, naz, nay, nax);
    const int ntb = lookup(e + 3 * TG96, nbz, nby, nbx);
    if (live) {
      // an empty voxel (token -1) contributes zero rows: nothing to the sums,
      // zeros to the grid-order copies
      uint4 ka = make_uint4(0, 0, 0, 0), kb = ka, va = ka, vb2 = ka;
      if (ta >= 0) {
        const uint4* kra = reinterpret_cast<const uint4*>(k + (((int64_t)b * g.N + ta) * g.H + h) * 96);
        const uint4* vra = reinterpret_cast<const uint4*>(v + (((int64_t)b * g.N + ta) * g.H + h) * 96);
        ka = __ldg(kra + c1);
        kb = __ldg(kra + c2);
        va = __ldg(vra + c1);
        vb2 = __ldg(vra + c2);
      }
      uint4 kbA = make_uint4(0, 0, 0, 0), kbB = kbA, vbA = kbA, vbB = kbA;
      if (has_b && tb2 >= 0) {
        const uint4* krb =
            reinterpret_cast<const uint4*>(k + (((int64_t)b * g.N + tb2) * g.H + h) * 96);
        const uint4* vrb =
            reinterpret_cast<const uint4*>(v + (((int64_t)b * g.N + tb2) * g.H + h) * 96);
        kbA = __ldg(krb + c1);
        kbB = __ldg(krb + c2);
        vbA = __ldg(vrb + c1);
        vbB = __ldg(vrb + c2);
      }
      consume(ka, kb, va, vb2, az, ay, ax, ta);
      if (has_b) consume(kbA, kbB, vbA, vbB, bz2, by2, bx2, tb2);
    }
    ta = nta;
    tb2 = ntb;
    az = naz; ay = nay; ax = nax;
    bz2 = nbz; by2 = nby; bx2 = nbx;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    red[grp][hh][0][8 * c1 + i] = kx1[i];
    red[grp][hh][0][8 * c2 + i] = kx2[i];
    red[grp][hh][1][8 * c1 + i] = vx1[i];
    red[grp][hh][1][8 * c2 + i] = vx2[i];
  }
  __syncthreads();
  for (int o = threadIdx.x; o < HG96 * 2 * 96; o += TG96 * LANES96) {
    const int oh = o / 192, which = (o / 96) % 2, ch = o % 96;
    const int hout = blockIdx.z * HG96 + oh;
    if (hout >= g.H) continue;
    float acc = 0.f;
    for (int q = 0; q < TG96; ++q) acc += red[q][oh][which][ch];
    const int64_t idx = (((int64_t)b * g.H + hout) * g.nb + blk) * 96 + ch;
    const int held = g.partial ? bcount[(int64_t)b * g.nb + blk] : cnt;
    const float mean = held > 0 && own ? acc / (float)held : 0.f;
    (which ? vsum : ksum)[idx] = mean;
    if (STAGE) (which ? so.vsb : so.ksb)[idx] = __float2bfloat16_rn(mean);
  }
}

}  // namespace

// bf16, head_dim 96, up to 8 heads: the block's token rows (all heads, k and
// v: 2 x H x 192 bytes per token) are gathered through the volume with bulk
// asynchronous copies into a shared-memory ring (BS_STAGES stages of BS_TPS
// tokens) by one producer warp, so 32 tokens per CTA are in flight; twelve
// consumer warps take thread (group g, item c): token g of each stage, item
// c = (head, segment, half) - 8 channels of k and their 8 rotation partners,
// and the same channels of v.  A thread adds its tokens in block-raster order
// (g, g + 8, ...), the 8 groups are then summed in order, so the result does
// not depend on the packing.  With STAGE the rotated key rows and the value
// rows are also written in grid order with bf16 copies of the summaries.  Null
// summary pointers skip those outputs (staging alone).
constexpr int BS_TPS = 8, BS_STAGES = 4, BS_MAXH = 8;
constexpr int BS_ITEMS = BS_MAXH * 6;                       // (head, segment, half)
constexpr int BS_CONSUMERS = BS_ITEMS * BS_TPS;             // 384 threads
constexpr int BS_THREADS = BS_CONSUMERS + 32;               // + the producer warp
constexpr int BS_ROW = BS_MAXH * 96 * 2;                    // bytes of one token's k (or v)
constexpr uint32_t BS_WAIT = 1u << 22;
struct BulkSmem {
  uint8_t ring[BS_STAGES][BS_TPS][2][BS_ROW];  // reused for the final reduction
  float2 tab[TAB96 * TABS96];
  int32_t tok[BS_STAGES][BS_TPS];  // packed index of each slot's token
  int4 crd[BS_STAGES][BS_TPS];     // (z, y, x) of each slot's voxel
  uint64_t full[BS_STAGES], empty[BS_STAGES];
  int32_t abort;
};
static_assert(sizeof(float) * BS_TPS * BS_ITEMS * 32 <= sizeof(uint8_t) * BS_STAGES * BS_TPS * 2 * BS_ROW,
              "reduction buffer must fit the ring");

// PARTIAL: a partly occupied volume (empty voxels skipped; compiled out of the
// dense kernels).
template <bool STAGE, bool PARTIAL>
__global__ void __launch_bounds__(BS_THREADS, 2) k_summaries_bulk(
    Geo g, const int32_t* __restrict__ vol, const float* __restrict__ rope,
    int32_t* __restrict__ err, const int32_t* __restrict__ bcount,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, float* ksum,
    float* vsum, StageOut so) {
  using namespace tc;
  if (err[0]) return;
  extern __shared__ uint8_t bs_raw[];
  BulkSmem& sm = *reinterpret_cast<BulkSmem*>((reinterpret_cast<uintptr_t>(bs_raw) + 127) &
                                              ~(uintptr_t)127);
  const int tid = threadIdx.x;
  const int blk = blockIdx.x, b = blockIdx.y;
  const int Bz = blk / (g.nby * g.nbx), By = (blk / g.nbx) % g.nby, Bx = blk % g.nbx;
  const BlockExt be = block_ext(g, Bz, By, Bx);  // cut at the volume's edge
  int bz0, bz1;  // local planes walked
  bool own;      // the block's summary is this call's to give
  block_planes(g, Bz, bz0, bz1, own);
  const int cnt = (bz1 - bz0) * be.ey * be.ex;
  const int n_stage_rounds = (cnt + BS_TPS - 1) / BS_TPS;
  const uint32_t row_bytes = (uint32_t)g.H * 96 * 2;
  volatile int32_t* abort_flag = &sm.abort;
  if (tid == 0) {
    for (int s = 0; s < BS_STAGES; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], BS_CONSUMERS / 32);
    }
    sm.abort = 0;
    fence_barrier_init();
  }
  // rotation-table rows of this block's coordinates (z rows, y rows, x rows)
  const float2* gtab = reinterpret_cast<const float2*>(rope);
  const int tab_rows = g.rope_mode == PACK3D_ROPE_PACKED ? 0 : g.bz + g.by + g.bx;
  for (int e = tid; e < tab_rows * 16; e += BS_THREADS) {
    const int r = e / 16, jj = e % 16;
    // coordinate of table row r on its axis (rows past the volume's edge, in a
    // cut block, are not needed)
    // (local planes of a z-slab: the block row starts at Bz bz - z_origin)
    const int c = r < g.bz ? Bz * g.bz - g.zo + r
                           : (r < g.bz + g.by ? By * g.by + r - g.bz : Bx * g.bx + r - g.bz - g.by);
    const int ext = r < g.bz ? g.Z : (r < g.bz + g.by ? g.Y : g.X);
    const int off = r < g.bz ? 0 : (r < g.bz + g.by ? g.Z : g.Z + g.Y);
    if (c >= 0 && c < ext) sm.tab[r * TABS96 + jj] = gtab[(off + c) * 16 + jj];
  }
  __syncthreads();
  auto voxel = [&](int e, int& cz, int& cy, int& cx) {
    cx = Bx * g.bx + e % be.ex;
    cy = By * g.by + (e / be.ex) % be.ey;
    cz = bz0 + e / (be.ex * be.ey);
  };
  // consumer item and partial sums (8 channels of k and their partners, same of v)
  const int grp = tid / BS_ITEMS, c = tid % BS_ITEMS;
  float kx1[8], kx2[8], vx1[8], vx2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) kx1[i] = kx2[i] = vx1[i] = vx2[i] = 0.f;
  if (tid >= BS_CONSUMERS) {
    // ---- producer warp: lane i copies token i of each stage ----
    // The voxel -> token lookups run ahead of the copies: lane 8 q + i holds
    // token i of round 4 n + q for the batch n of four rounds being issued
    // (cur) and for the next batch (nxt), so no round waits on a lookup.
    static_assert(BS_TPS == 8, "four rounds of token lookups per warp");
    const int lane = tid - BS_CONSUMERS;
    const int32_t* vb = vol + (int64_t)b * g.V;
    auto lookup = [&](int rr) -> int32_t {
      const int e = rr * BS_TPS + (lane & 7);
      if (rr >= n_stage_rounds || e >= cnt) return 0;
      int cz, cy, cx;
      voxel(e, cz, cy, cx);
      return vb[(cz * g.Y + cy) * g.X + cx];
    };
    int32_t cur = lookup(lane >> 3), nxt = lookup(4 + (lane >> 3));
    for (int r = 0; r < n_stage_rounds; ++r) {
      const int s = r % BS_STAGES;
      if (r > 0 && (r & 3) == 0) {
        cur = nxt;
        nxt = lookup(r + 4 + (lane >> 3));
      }
      bool ok = true;
      if (lane == 0 && r >= BS_STAGES)
        ok = mbar_wait_or_abort(&sm.empty[s], ((r / BS_STAGES) - 1) & 1, BS_WAIT, abort_flag);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int ntok = min(BS_TPS, cnt - r * BS_TPS);
      const int64_t tok = __shfl_sync(0xffffffffu, cur, 8 * (r & 3) + (lane & 7));
      if (lane < ntok) {
        // published by the arrive below: the slot's token and voxel, so the
        // consumers need no division to find the voxel
        sm.tok[s][lane] = (int32_t)tok;
        int cz, cy, cx;
        voxel(r * BS_TPS + lane, cz, cy, cx);
        sm.crd[s][lane] = make_int4(cz, cy, cx, 0);
      }
      // empty voxels (token -1, partly occupied volumes) are not copied
      const int nload = PARTIAL ? __popc(__ballot_sync(0xffffffffu, lane < ntok && tok >= 0)) : ntok;
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], (uint32_t)nload * 2 * row_bytes);
      __syncwarp();
      if (lane < ntok && (!PARTIAL || tok >= 0)) {
        bulk_load(sm.ring[s][lane][0], k + (((int64_t)b * g.N + tok) * g.H) * 96, row_bytes,
                  &sm.full[s]);
        bulk_load(sm.ring[s][lane][1], v + (((int64_t)b * g.N + tok) * g.H) * 96, row_bytes,
                  &sm.full[s]);
      }
    }
    // every copy issued has been waited for by the consumers unless they gave up
    if (lane == 0)
      for (int r = max(0, n_stage_rounds - BS_STAGES); r < n_stage_rounds; ++r)
        mbar_wait(&sm.full[r % BS_STAGES], (r / BS_STAGES) & 1, BS_WAIT);
    __syncwarp();
  } else {
    // ---- consumers ----
    const int h = c / 6, w = c % 6;
    const bool live = h < g.H;
    const Item96 item = item96(g, w);
    const int a = item.a, c1 = item.c1, c2 = item.c2, j0 = item.j0;
    const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
    const float2* tab = a == 0 ? sm.tab : (a == 1 ? sm.tab + g.bz * TABS96 : sm.tab + (g.bz + g.by) * TABS96);
    const int base = a == 0 ? Bz * g.bz - g.zo : (a == 1 ? By * g.by : Bx * g.bx);
    for (int r = 0; r < n_stage_rounds; ++r) {
      const int s = r % BS_STAGES;
      if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&sm.full[s], (r / BS_STAGES) & 1, BS_WAIT,
                                                       abort_flag)))
        break;
      const int e = r * BS_TPS + grp;
      if (live && e < cnt) {
        const int4 cc = sm.crd[s][grp];
        const int cz = cc.x, cy = cc.y, cx = cc.z;
        const uint4* kr = reinterpret_cast<const uint4*>(sm.ring[s][grp][0] + h * 192);
        const uint4* vr = reinterpret_cast<const uint4*>(sm.ring[s][grp][1] + h * 192);
        // an empty voxel (token -1, not copied) contributes zero rows: nothing
        // to the sums, zeros to the grid-order copies
        const int tk = PARTIAL || packed ? sm.tok[s][grp] : 0;
        const bool held_tok = !PARTIAL || tk >= 0;
        const uint4 z4 = make_uint4(0, 0, 0, 0);
        const uint4 ka = held_tok ? kr[c1] : z4, kb = held_tok ? kr[c2] : z4;
        const uint4 va = held_tok ? vr[c1] : z4, vb2 = held_tok ? vr[c2] : z4;
        const int ca = a == 0 ? cz : (a == 1 ? cy : cx);
        const float2* t = packed ? rope_row96(rope, g, 0, 0, max(tk, 0)) + j0
                                 : tab + (ca - base) * TABS96 + j0;
        const uint32_t* kaw = reinterpret_cast<const uint32_t*>(&ka);
        const uint32_t* kbw = reinterpret_cast<const uint32_t*>(&kb);
        const uint32_t* vaw = reinterpret_cast<const uint32_t*>(&va);
        const uint32_t* vbw = reinterpret_cast<const uint32_t*>(&vb2);
        uint4 ra, rb;
        uint32_t* raw = reinterpret_cast<uint32_t*>(&ra);
        uint32_t* rbw = reinterpret_cast<uint32_t*>(&rb);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kaw + q));
          float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kbw + q));
          const float4 cs = *reinterpret_cast<const float4*>(t + 2 * q);  // pairs j, j + 1
          const float r1a = x1.x * cs.x - x2.x * cs.y, r2a = x1.x * cs.y + x2.x * cs.x;
          const float r1b = x1.y * cs.z - x2.y * cs.w, r2b = x1.y * cs.w + x2.y * cs.z;
          kx1[2 * q] += r1a;
          kx2[2 * q] += r2a;
          kx1[2 * q + 1] += r1b;
          kx2[2 * q + 1] += r2b;
          if (STAGE) {
            __nv_bfloat162 pa = __floats2bfloat162_rn(r1a, r1b), pb = __floats2bfloat162_rn(r2a, r2b);
            raw[q] = *reinterpret_cast<uint32_t*>(&pa);
            rbw[q] = *reinterpret_cast<uint32_t*>(&pb);
          }
          float2 y1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vaw + q));
          float2 y2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vbw + q));
          vx1[2 * q] += y1.x;
          vx1[2 * q + 1] += y1.y;
          vx2[2 * q] += y2.x;
          vx2[2 * q + 1] += y2.y;
        }
        if (STAGE) {
          const int64_t grow = ((((int64_t)b * g.H + h) * g.Z + cz) * g.Y + cy) * g.X + cx;
          uint4* kd = reinterpret_cast<uint4*>(so.kg + grow * 96);
          uint4* vd = reinterpret_cast<uint4*>(so.vg + grow * 96);
          kd[c1] = ra;
          kd[c2] = rb;
          vd[c1] = va;
          vd[c2] = vb2;
        }
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&sm.empty[s]);
    }
  }
  // every stage is consumed (or abandoned): the ring takes the partial sums
  // [group][item][32]
  __syncthreads();
  if (sm.abort) {
    if (tid == 0) atomicOr(&err[0], 4);
    return;
  }
  if (tid < BS_CONSUMERS) {
    float* red = reinterpret_cast<float*>(&sm.ring[0][0][0][0]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      red[(grp * BS_ITEMS + c) * 32 + i] = kx1[i];
      red[(grp * BS_ITEMS + c) * 32 + 8 + i] = kx2[i];
      red[(grp * BS_ITEMS + c) * 32 + 16 + i] = vx1[i];
      red[(grp * BS_ITEMS + c) * 32 + 24 + i] = vx2[i];
    }
  }
  __syncthreads();
  // sums over the groups in order, means, outputs
  const float* red = reinterpret_cast<const float*>(&sm.ring[0][0][0][0]);
  // mean over the tokens the block holds (0 for an empty block, and for a
  // block a z-slab does not own)
  const int held = PARTIAL ? bcount[(int64_t)b * g.nb + blk] : cnt;
  const float inv_cnt = held > 0 && own ? 1.f / (float)held : 0.f;
  for (int o = tid; o < g.H * 2 * 96; o += BS_THREADS) {
    const int h = o / 192, which = (o / 96) % 2, ch = o % 96;
    // channel ch of head h: 16-byte chunk ch / 8 is chunk c1 (slots 0-7) or c2
    // (slots 8-15) of one item w of item96; values at slots 16-31
    const int chunk = ch / 8, i = ch % 8;
    int w, hi;
    if (g.rope_mode == PACK3D_ROPE_PACKED) {
      hi = chunk >= 6;
      w = chunk % 6;
    } else {
      hi = (chunk & 3) >= 2;
      w = 2 * (chunk >> 2) + (chunk & 1);
    }
    const int slot = (which ? 16 : 0) + (hi ? 8 : 0) + i;
    float acc = 0.f;
    for (int q = 0; q < BS_TPS; ++q) acc += red[(q * BS_ITEMS + h * 6 + w) * 32 + slot];
    const int64_t idx = (((int64_t)b * g.H + h) * g.nb + blk) * 96 + ch;
    const float mean = acc * inv_cnt;
    if (ksum) (which ? vsum : ksum)[idx] = mean;
    if (STAGE && so.ksb) (which ? so.vsb : so.ksb)[idx] = __float2bfloat16_rn(mean);
  }
}

// The bulk-copy kernel: up to 8 heads; the block's rotation-table rows staged.
bool bulk_supported(const Geo& g) {
  return g.H <= BS_MAXH && g.bz + g.by + g.bx <= TAB96;
}

template <bool STAGE>
int launch_bulk(const Geo& g, const pack3d_index* idx, const void* k, const void* v, float* ksum,
                float* vsum, StageOut so, cudaStream_t s) {
  const size_t smem = sizeof(BulkSmem) + 128;
  auto kern = g.partial ? k_summaries_bulk<STAGE, true> : k_summaries_bulk<STAGE, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return PACK3D_ERR_CUDA;
  kern<<<dim3(g.nb, g.B), BS_THREADS, smem, s>>>(g, idx->vol, idx->rope, idx->err, idx->bcount,
                                                  (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                                  ksum, vsum, so);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

int launch_block_summaries(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                           float* ksum, float* vsum, cudaStream_t s) {
  dim3 grid(g.nb, g.B, g.H);
  if (g.dtype == PACK3D_BF16 && g.d == 96) {
    if (bulk_supported(g)) return launch_bulk<false>(g, idx, k, v, ksum, vsum, StageOut{}, s);
    dim3 grid96(g.nb, g.B, (g.H + HG96 - 1) / HG96);
    k_block_summaries_bf16_d96<false><<<grid96, TG96 * LANES96, 0, s>>>(
        g, idx->vol, idx->rope, idx->err, idx->bcount, (const __nv_bfloat16*)k,
        (const __nv_bfloat16*)v, ksum, vsum, StageOut{});
    count_launches(1);
    return cuda_status(cudaGetLastError());
  }
  int threads = TG * (g.d / 4);
  size_t smem = sizeof(float) * TG * 2 * g.d;
  if (g.dtype == PACK3D_BF16)
    k_block_summaries<__nv_bfloat16><<<grid, threads, smem, s>>>(
        g, idx->vol, idx->rope, idx->err, idx->bcount, (const __nv_bfloat16*)k,
        (const __nv_bfloat16*)v, ksum, vsum);
  else
    k_block_summaries<float><<<grid, threads, smem, s>>>(g, idx->vol, idx->rope, idx->err,
                                                         idx->bcount, (const float*)k,
                                                         (const float*)v, ksum,
                                                         vsum);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

int launch_stage_bulk(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                      void* kg, void* vg, cudaStream_t s) {
  if (g.dtype != PACK3D_BF16 || g.d != 96 || !bulk_supported(g)) return PACK3D_ERR_UNSUPPORTED;
  StageOut so{(__nv_bfloat16*)kg, (__nv_bfloat16*)vg, nullptr, nullptr};
  return launch_bulk<true>(g, idx, k, v, nullptr, nullptr, so, s);
}

int launch_block_summaries_staged(const Geo& g, const pack3d_index* idx, const void* k,
                                  const void* v, float* ksum, float* vsum, void* kg, void* vg,
                                  void* ksb, void* vsb, cudaStream_t s) {
  if (g.dtype != PACK3D_BF16 || g.d != 96) return PACK3D_ERR_UNSUPPORTED;
  dim3 grid96(g.nb, g.B, (g.H + HG96 - 1) / HG96);
  StageOut so{(__nv_bfloat16*)kg, (__nv_bfloat16*)vg, (__nv_bfloat16*)ksb, (__nv_bfloat16*)vsb};
  if (bulk_supported(g)) return launch_bulk<true>(g, idx, k, v, ksum, vsum, so, s);
  k_block_summaries_bf16_d96<true><<<grid96, TG96 * LANES96, 0, s>>>(
      g, idx->vol, idx->rope, idx->err, idx->bcount, (const __nv_bfloat16*)k,
      (const __nv_bfloat16*)v, ksum, vsum, so);
  count_launches(1);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
