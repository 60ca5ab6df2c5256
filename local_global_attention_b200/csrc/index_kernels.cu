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

// Scatter packed index -> voxel, detect out-of-range and duplicated voxels,
// count tokens per query tile (histogram of the counting sort).
__global__ void k_scatter_coords(Geo g, const int16_t* __restrict__ coords, int32_t* vol,
                                 int32_t* cnt, int32_t* err) {
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
  int old = atomicCAS(&vol[(int64_t)b * g.N + v], -1, i);
  if (old != -1) {
    atomicOr(&err[0], ERR_DUP);
    atomicMin(&err[1], (int32_t)t);
    return;
  }
  int tile = ((z / TZ) * g.nTy + (y / TY)) * g.nTx + (x / TX);
  atomicAdd(&cnt[(int64_t)b * g.nT + tile], 1);
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

__global__ void k_halo_sizes(Geo g, int32_t* sizes) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= g.nT) return;
  int hz0, hy0, hx0, hz, hy, hx;
  halo_box(g, t, hz0, hy0, hx0, hz, hy, hx);
  sizes[t] = hz * hy * hx;
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
  const int32_t* vb = vol + (int64_t)b * g.N;
  int32_t* dst = nbr + (int64_t)b * g.n_halo + nbr_off[t];
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    int x = e % hx, y = (e / hx) % hy, z = e / (hx * hy);
    dst[e] = vb[((hz0 + z) * g.Y + (hy0 + y)) * g.X + (hx0 + x)];
  }
}

// cos and sin of c * base^(-2j/da) (axial: c a coordinate value of an axis)
// or of p * base^(-2j/d) (packed mode: p a packed position), evaluated in
// double precision.
__global__ void k_rope_table(Geo g, float base, float* tab) {
  int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const bool packed = g.rope_mode == PACK3D_ROPE_PACKED;
  int64_t rows = packed ? g.N : g.Z + g.Y + g.X;
  if (e >= rows * g.rope_len) return;
  int row = (int)(e / g.rope_len), j = (int)(e % g.rope_len);
  int c = packed ? row : (row < g.Z ? row : (row < g.Z + g.Y ? row - g.Z : row - g.Z - g.Y));
  double theta = pow((double)base, -2.0 * (double)j / (double)(packed ? g.d : g.da));
  double sn, cs;
  sincos((double)c * theta, &sn, &cs);
  tab[2 * e + 0] = (float)cs;
  tab[2 * e + 1] = (float)sn;
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
  if (cudaMemsetAsync(idx->vol, 0xff, sizeof(int32_t) * tokens, s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (cudaMemsetAsync(cnt, 0, sizeof(int32_t) * (size_t)g.B * g.nT, s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  k_init_err<<<1, 1, 0, s>>>(idx->err);
  int nthr = 256;
  unsigned nblk = (unsigned)((tokens + nthr - 1) / nthr);
  k_scatter_coords<<<nblk, nthr, 0, s>>>(g, coords, idx->vol, cnt, idx->err);
  k_exclusive_scan<1024><<<g.B, 1024, 0, s>>>(cnt, idx->tile_off, g.nT, g.nT, g.nT + 1);
  k_tile_scatter<<<nblk, nthr, 0, s>>>(g, coords, idx->tile_off, idx->perm, idx->err);
  // Halo sizes reuse the histogram space (tile_off already holds the scan).
  k_halo_sizes<<<(g.nT + 255) / 256, 256, 0, s>>>(g, cnt);
  k_exclusive_scan<1024><<<1, 1024, 0, s>>>(cnt, idx->nbr_off, g.nT, 0, 0);
  k_halo_lists<<<dim3(g.nT, g.B), 256, 0, s>>>(g, idx->vol, idx->nbr_off, idx->nbr, idx->err);
  const int64_t entries =
      (g.rope_mode == PACK3D_ROPE_PACKED ? (int64_t)g.N : (int64_t)(g.Z + g.Y + g.X)) *
      g.rope_len;
  k_rope_table<<<(unsigned)((entries + 255) / 256), 256, 0, s>>>(g, rope_base, idx->rope);
  count_launches(8);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
