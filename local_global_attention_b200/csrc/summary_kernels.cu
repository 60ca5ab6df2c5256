// Block summaries: per (batch item, head, block) the mean of the rotated keys
// and the mean of the values over the block's tokens, fp32 accumulation.
//
// "Geometry Matters in Packed 3D Attention" (abstract): distant context is
// compressed "into contiguous 3D block summaries", and "the rotation is
// applied before a block is summarized", so the key summary is the mean of
// R(c_j) k_j, not R(.) of a mean.
//
// HBM-bound: every k and v row is read once.  One CTA per (block, batch item,
// head); its threads form TG token groups of d/4 lanes, each lane owning two
// adjacent rotation pairs (four output channels).  A lane reads 2 x 4 bytes of
// k (the pair members sit da/2 channels apart) and 2 x 4 bytes of v per token;
// the d/4 lanes of a token group read one 2d-byte row contiguously.  Tokens
// are visited through the coordinate volume in block raster order, so the
// accumulation order, and the result, do not depend on the packing.
#include "pack3d_internal.cuh"

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
  // Lane -> axis a and first pair j (pairs j, j+1 of that axis).
  const int pairs_per_axis = g.half / 2;  // lanes per axis
  const int a = lane / pairs_per_axis, j = (lane % pairs_per_axis) * 2;
  const int c1 = a * g.da + j, c2 = c1 + g.half;  // channels of x1 (and +1), x2 (and +1)
  float kx1a = 0.f, kx1b = 0.f, kx2a = 0.f, kx2b = 0.f;
  float vx1a = 0.f, vx1b = 0.f, vx2a = 0.f, vx2b = 0.f;
  const int cnt = g.bz * g.by * g.bx;
  const int32_t* vb = vol + (int64_t)b * g.N;
  if (grp < TG) {
#pragma unroll 4
    for (int e = grp; e < cnt; e += TG) {
      int x = e % g.bx, y = (e / g.bx) % g.by, z = e / (g.bx * g.by);
      int cz = Bz * g.bz + z, cy = By * g.by + y, cx = Bx * g.bx + x;
      int tok = vb[(cz * g.Y + cy) * g.X + cx];
      int64_t row = (((int64_t)b * g.N + tok) * g.H + h) * g.d;
      float2 k1 = Pair2<T>::f(*reinterpret_cast<const P2*>(k + row + c1));
      float2 k2 = Pair2<T>::f(*reinterpret_cast<const P2*>(k + row + c2));
      float2 v1 = Pair2<T>::f(*reinterpret_cast<const P2*>(v + row + c1));
      float2 v2 = Pair2<T>::f(*reinterpret_cast<const P2*>(v + row + c2));
      int ca = a == 0 ? cz : (a == 1 ? cy : cx);
      float2 csa = rope_cs(rope, g, a, ca, j), csb = rope_cs(rope, g, a, ca, j + 1);
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
  const float inv = 1.0f / (float)cnt;
  int64_t base = (((int64_t)b * g.H + h) * g.nb + blk) * g.d;
  for (int c = threadIdx.x; c < 2 * g.d; c += blockDim.x) {
    int which = c / g.d, ch = c % g.d;
    float s = 0.f;
    for (int t = 0; t < TG; ++t) s += red[(t * 2 + which) * g.d + ch];
    (which ? vsum : ksum)[base + ch] = s * inv;
  }
}

}  // namespace

int launch_block_summaries(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                           float* ksum, float* vsum, cudaStream_t s) {
  dim3 grid(g.nb, g.B, g.H);
  int threads = TG * (g.d / 4);
  size_t smem = sizeof(float) * TG * 2 * g.d;
  if (g.dtype == PACK3D_BF16)
    k_block_summaries<__nv_bfloat16><<<grid, threads, smem, s>>>(
        g, idx->vol, idx->rope, idx->err, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
        ksum, vsum);
  else
    k_block_summaries<float><<<grid, threads, smem, s>>>(g, idx->vol, idx->rope, idx->err,
                                                         (const float*)k, (const float*)v, ksum,
                                                         vsum);
  return cuda_status(cudaGetLastError());
}

}  // namespace p3d
