// Index build of one packing: coordinate volume, tile permutation by counting
// sort, halo lists and the rotation table.
//
// "Geometry Matters in Packed 3D Attention" (abstract) indexes attention by
// true token-grid coordinates rather than packed positions; these kernels turn
// the per-token coordinates into the lookup structures the attention kernels
// gather through, so no token data is ever permuted in memory.
#include "pack3d_internal.cuh"

namespace p3d {

namespace {

constexpr int ERR_RANGE = 1, ERR_DUP = 2;

// cos and sin of c * base^(-2j/da) (axial: c a coordinate value of an axis)
// or of p * base^(-2j/d) (packed mode: p a packed position), evaluated in
// double precision.
__device__ __forceinline__ void rope_entry(const Geo& g, float base, float* tab, int64_t e) {
  const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
  int64_t rows = packed ? g.N : g.Z + g.Y + g.X;
  if (e >= rows * g.rope_len) return;
  int row = (int)(e / g.rope_len), j = (int)(e % g.rope_len);
  // axial rows: the z rows of a z-slab turn by the global plane z + z_origin
  int c = packed ? row : (row < g.Z ? row + g.zo : (row < g.Z + g.Y ? row - g.Z : row - g.Z - g.Y));
  double theta = pow((double)base, -2.0 * (double)j / (double)(packed ? g.d : g.da));
  double sn, cs;
  sincos((double)c * theta, &sn, &cs);
  tab[2 * e + 0] = (float)cs;
  tab[2 * e + 1] = (float)sn;
}

// Scatter packed index -> voxel, detect out-of-range and duplicated voxels,
// count tokens per query tile (histogram of the counting sort) and per block.
// Blocks past the tokens' (blockIdx.x >= nblk) fill the rotation table, which
// depends on the geometry only, alongside.
__global__ void k_scatter_coords(Geo g, const int16_t* __restrict__ coords, int32_t* vol,
                                 int32_t* cnt, int32_t* bcount, int32_t* err, unsigned nblk,
                                 float rope_base, float* rope) {
  if (blockIdx.x >= nblk) {
    rope_entry(g, rope_base, rope, (blockIdx.x - nblk) * (int64_t)blockDim.x + threadIdx.x);
    return;
  }
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= (int64_t)g.B * g.N) return;
  int b = (int)(t / g.N);
  int i = (int)(t % g.N);
  int z = coords[t * 3 + 0], y = coords[t * 3 + 1], x = coords[t * 3 + 2];
  if (z < 0 || z >= g.Z || y < 0 || y >= g.Y || x < 0 || x >= g.X) {
    atomicOr(&err[0], ERR_RANGE);
    atomicMin(&err[1], (int32_t)t);
    return;
  }
  int v = (z * g.Y + y) * g.X + x;
  int old = atomicCAS(&vol[(int64_t)b * g.V + v], -1, i);
  if (old != -1) {
    atomicOr(&err[0], ERR_DUP);
    atomicMin(&err[1], (int32_t)t);
    return;
  }
  int tile = ((z / TZ) * g.nTy + (y / TY)) * g.nTx + (x / TX);
  atomicAdd(&cnt[(int64_t)b * g.nT + tile], 1);
  if (g.partial) {  // block counts: only partly occupied volumes need them
    int blk = (((z + g.zo) / g.bz) * g.nby + (y / g.by)) * g.nbx + (x / g.bx);
    atomicAdd(&bcount[(int64_t)b * g.nb + blk], 1);
  }
}

// Exclusive scan of n ints per row (one CTA per row), writes n + 1 values.
// Used for the tile histogram (per batch item) and for the halo sizes.
template <int NT>
__global__ void k_exclusive_scan(const int32_t* __restrict__ in, int32_t* out, int n,
                                 int64_t in_stride, int64_t out_stride) {
  __shared__ int32_t part[NT];
  const int32_t* src = in + blockIdx.x * in_stride;
  int32_t* dst = out + blockIdx.x * out_stride;
  int per = (n + NT - 1) / NT;
  int lo = threadIdx.x * per, hi = min(n, lo + per);
  int32_t s = 0;
  for (int i = lo; i < hi; ++i) s += src[i];
  part[threadIdx.x] = s;
  __syncthreads();
  // Hillis-Steele inclusive scan of the per-thread sums.
  for (int off = 1; off < NT; off <<= 1) {
    int32_t add = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += add;
    __syncthreads();
  }
  int32_t run = threadIdx.x == 0 ? 0 : part[threadIdx.x - 1];
  for (int i = lo; i < hi; ++i) {
    dst[i] = run;
    run += src[i];
  }
  if (threadIdx.x == NT - 1) dst[n] = part[NT - 1];
}

__device__ __forceinline__ void tile_box(const Geo& g, int t, int& z0, int& y0, int& x0, int& lz,
                                         int& ly, int& lx) {
  int Tx = t % g.nTx, Ty = (t / g.nTx) % g.nTy, Tz = t / (g.nTx * g.nTy);
  z0 = Tz * TZ;
  y0 = Ty * TY;
  x0 = Tx * TX;
  lz = min(TZ, g.Z - z0);
  ly = min(TY, g.Y - y0);
  lx = min(TX, g.X - x0);
}

// Counting-sort scatter.  A token's slot is its tile's offset plus its
// raster rank inside the tile (the volume is dense, so the rank follows from
// the coordinate).
__global__ void k_tile_scatter(Geo g, const int16_t* __restrict__ coords,
                               const int32_t* __restrict__ tile_off, int32_t* perm,
                               const int32_t* __restrict__ err) {
  if (err[0]) return;
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= (int64_t)g.B * g.N) return;
  int b = (int)(t / g.N);
  int i = (int)(t % g.N);
  int z = coords[t * 3 + 0], y = coords[t * 3 + 1], x = coords[t * 3 + 2];
  int tile = ((z / TZ) * g.nTy + (y / TY)) * g.nTx + (x / TX);
  int z0, y0, x0, lz, ly, lx;
  tile_box(g, tile, z0, y0, x0, lz, ly, lx);
  int rank = ((z - z0) * ly + (y - y0)) * lx + (x - x0);
  int slot = tile_off[(int64_t)b * (g.nT + 1) + tile] + rank;
  if (slot < g.N) perm[(int64_t)b * g.N + slot] = i;
}

// Counting-sort scatter of a partly occupied volume: one warp per tile walks
// its voxels in raster order and gives each token present the next slot (a
// ballot prefix count), so perm holds the tile's tokens in raster order.
__global__ void k_tile_perm(Geo g, const int32_t* __restrict__ vol,
                            const int32_t* __restrict__ tile_off, int32_t* perm,
                            const int32_t* __restrict__ err) {
  if (err[0]) return;
  const int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32, b = blockIdx.y;
  const int lane = threadIdx.x % 32;
  if (t >= g.nT) return;
  int z0, y0, x0, lz, ly, lx;
  tile_box(g, t, z0, y0, x0, lz, ly, lx);
  const int n = lz * ly * lx;
  const int base = tile_off[(int64_t)b * (g.nT + 1) + t];
  const int32_t* vb = vol + (int64_t)b * g.V;
  int run = 0;
  for (int e0 = 0; e0 < n; e0 += 32) {
    const int e = e0 + lane;
    int tok = -1;
    if (e < n) {
      const int x = x0 + e % lx, y = y0 + (e / lx) % ly, z = z0 + e / (lx * ly);
      tok = vb[(z * g.Y + y) * g.X + x];
    }
    const uint32_t present = __ballot_sync(0xffffffffu, tok >= 0);
    const int pos = run + __popc(present & ((1u << lane) - 1u));
    if (tok >= 0 && base + pos < g.N) perm[(int64_t)b * g.N + base + pos] = tok;
    run += __popc(present);
  }
}

// Occupancy mask of the blocks: bit B % 32 of word B / 32 set when block B
// holds a token.
__global__ void k_block_occ(Geo g, const int32_t* __restrict__ bcount, uint32_t* bocc) {
  const int nw = (g.nb + 31) / 32;
  const int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (w >= (int64_t)g.B * nw) return;
  const int b = (int)(w / nw), w0 = (int)(w % nw) * 32;
  uint32_t bits = 0;
  for (int i = 0; i < 32 && w0 + i < g.nb; ++i)
    if (bcount[(int64_t)b * g.nb + w0 + i] > 0) bits |= 1u << i;
  bocc[w] = bits;
}

__device__ __forceinline__ void halo_box(const Geo& g, int t, int& hz0, int& hy0, int& hx0,
                                         int& hz, int& hy, int& hx) {
  int z0, y0, x0, lz, ly, lx;
  tile_box(g, t, z0, y0, x0, lz, ly, lx);
  hz0 = max(0, z0 - g.rz);
  hy0 = max(0, y0 - g.ry);
  hx0 = max(0, x0 - g.rx);
  hz = min(g.Z, z0 + lz + g.rz) - hz0;
  hy = min(g.Y, y0 + ly + g.ry) - hy0;
  hx = min(g.X, x0 + lx + g.rx) - hx0;
}

// Offsets of the tiles' halo lists (exclusive scan of the halo box sizes, a
// pure function of the geometry), one CTA of NT threads.
template <int NT>
__global__ void k_halo_offsets(Geo g, int32_t* off) {
  __shared__ int32_t part[NT];
  const int n = g.nT;
  const int per = (n + NT - 1) / NT;
  const int lo = threadIdx.x * per, hi = min(n, lo + per);
  auto size = [&](int t) {
    int hz0, hy0, hx0, hz, hy, hx;
    halo_box(g, t, hz0, hy0, hx0, hz, hy, hx);
    return hz * hy * hx;
  };
  int32_t s = 0;
  for (int i = lo; i < hi; ++i) s += size(i);
  part[threadIdx.x] = s;
  __syncthreads();
  // Hillis-Steele inclusive scan of the per-thread sums.
  for (int d = 1; d < NT; d <<= 1) {
    int32_t add = threadIdx.x >= d ? part[threadIdx.x - d] : 0;
    __syncthreads();
    part[threadIdx.x] += add;
    __syncthreads();
  }
  int32_t run = threadIdx.x == 0 ? 0 : part[threadIdx.x - 1];
  for (int i = lo; i < hi; ++i) {
    off[i] = run;
    run += size(i);
  }
  if (threadIdx.x == NT - 1) off[n] = part[NT - 1];
}

// Halo lists, one CTA per (tile, batch item), raster order over the halo box.
__global__ void k_halo_lists(Geo g, const int32_t* __restrict__ vol,
                             const int32_t* __restrict__ nbr_off, int32_t* nbr,
                             const int32_t* __restrict__ err) {
  if (err[0]) return;
  int t = blockIdx.x, b = blockIdx.y;
  int hz0, hy0, hx0, hz, hy, hx;
  halo_box(g, t, hz0, hy0, hx0, hz, hy, hx);
  int n = hz * hy * hx;
  const int32_t* vb = vol + (int64_t)b * g.V;
  int32_t* dst = nbr + (int64_t)b * g.n_halo + nbr_off[t];
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int x = e % hx, y = (e / hx) % hy, z = e / (hx * hy);
    dst[e] = vb[((hz0 + z) * g.Y + (hy0 + y)) * g.X + (hx0 + x)];
  }
}

__global__ void k_init_err(int32_t* err) {
  err[0] = 0;
  err[1] = 0x7fffffff;
}

}  // namespace

int launch_build_index(const Geo& g, const int16_t* coords, const pack3d_index* idx,
                       float rope_base, cudaStream_t s) {
  int64_t tokens = (int64_t)g.B * g.N;
  int32_t* cnt = idx->nbr;  // the halo lists are written last; their space holds the histogram
  if (cudaMemsetAsync(idx->vol, 0xff, sizeof(int32_t) * (size_t)g.B * g.V, s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (size_t)g.B * g.nT, s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (g.partial &&
      cudaMemsetAsync(idx->bcount, 0, sizeof(int32_t) * (size_t)g.B * g.nb, s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  k_init_err<<<1, 1, 0, s>>>(idx->err);
  int nthr = 256;
  unsigned nblk = (unsigned)((tokens + nthr - 1) / nthr);
  const int64_t entries =
      (g.rope_mode == PACK3D_ROPE_PACKED ? (int64_t)g.N : (int64_t)(g.Z + g.Y + g.X)) *
      g.rope_len;
  const unsigned rope_blk = (unsigned)((entries + nthr - 1) / nthr);
  k_scatter_coords<<<nblk + rope_blk, nthr, 0, s>>>(g, coords, idx->vol, cnt, idx->bcount,
                                                    idx->err, nblk, rope_base, idx->rope);
  k_exclusive_scan<1024><<<g.B, 1024, 0, s>>>(cnt, idx->tile_off, g.nT, g.nT, g.nT + 1);
  if (g.partial) {
    k_tile_perm<<<dim3((g.nT + 3) / 4, g.B), 128, 0, s>>>(g, idx->vol, idx->tile_off, idx->perm,
                                                          idx->err);
    const int64_t words = (int64_t)g.B * ((g.nb + 31) / 32);
    k_block_occ<<<(unsigned)((words + 255) / 256), 256, 0, s>>>(g, idx->bcount, idx->bocc);
    count_launches(1);
  } else {
    k_tile_scatter<<<nblk, nthr, 0, s>>>(g, coords, idx->tile_off, idx->perm, idx->err);
  }
  k_halo_offsets<1024><<<1, 1024, 0, s>>>(g, idx->nbr_off);
  k_halo_lists<<<dim3(g.nT, g.B), 256, 0, s>>>(g, idx->vol, idx->nbr_off, idx->nbr, idx->err);
  count_launches(6);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
