// Internal declarations shared by the PACK3D CUDA translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pack3d.h"

namespace p3d {

// Query tile (z, y, x): 128 queries, the M of one tcgen05 MMA.
constexpr int TZ = 4, TY = 4, TX = 8, TILE = TZ * TY * TX;

// Geometry derived once on the host from pack3d_params and passed by value.
struct Geo {
  int B, H, d, da, half;      // half = da / 2 rotation pairs per axis
  int Z, Y, X;
  int N;                      // tokens per batch item
  int V;                      // voxels per batch item (Z * Y * X)
  int partial;                // N < V: a partly occupied volume
  int sharded;                // a z-slab of a larger volume (Z_total > 0)
  int Zt, zo;                 // global planes, global plane of local plane 0
  int own_lo, own_hi;         // owned local planes (all planes when not sharded)
  int rz, ry, rx;             // window radii
  int bz, by, bx;             // block extents
  int nbz, nby, nbx, nb;      // block counts
  int nTz, nTy, nTx, nT;      // query-tile counts
  int64_t n_halo;             // halo list length per batch item
  float tau;                  // softmax scale
  int dtype;                  // PACK3D_BF16 / PACK3D_FP32
  int out_fp32;               // out is fp32 (also when dtype is bf16)
  int rope_mode;              // PACK3D_ROPE_AXIAL / PACK3D_ROPE_PACKED
  int rope_len;               // (cos, sin) pairs per rotation-table row
};

int make_geo(const pack3d_params* p, Geo* g);  // PACK3D_OK or PACK3D_ERR_*

// Halo extent of query tiles along one axis: sum over tiles of the clipped
// length of [t*T - r, t*T + T - 1 + r].
int64_t halo_axis_total(int extent, int tile, int r);

// ---- small device helpers ------------------------------------------------

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Whether voxel (z, y, x) of batch item b holds a token: always in a dense
// volume; else the coordinate volume has its token or -1.
__device__ __forceinline__ bool occupied(const Geo& g, const int32_t* vol, int b, int z, int y,
                                         int x) {
  return !g.partial || vol[(((int64_t)b * g.Z + z) * g.Y + y) * g.X + x] >= 0;
}

// Extents of block (Bz, By, Bx) cut at the volume's edge (a block that
// does not fit holds only its voxels inside the volume); the global volume's
// edge when the call is a z-slab.
struct BlockExt {
  int ez, ey, ex;
};
__device__ __forceinline__ BlockExt block_ext(const Geo& g, int Bz, int By, int Bx) {
  return {min(g.bz, g.Zt - Bz * g.bz), min(g.by, g.Y - By * g.by), min(g.bx, g.X - Bx * g.bx)};
}

// The local planes [z0, z1) of block row Bz inside this call's volume (the
// block cut at the volume's edge; a z-slab holds part of the block grid), and
// whether the block's summary is this call's to give: always, except in a
// z-slab, where only blocks lying wholly in the owned planes count (the
// others get zero summaries, so that a sum over the ranks gives every block).
// The staging passes walk the planes either way.
__device__ __forceinline__ void block_planes(const Geo& g, int Bz, int& z0, int& z1, bool& own) {
  const int gz0 = Bz * g.bz, gz1 = min(gz0 + g.bz, g.Zt);
  z0 = max(gz0 - g.zo, 0);
  z1 = max(min(gz1 - g.zo, g.Z), z0);
  own = !g.sharded || (gz0 - g.zo >= g.own_lo && gz1 - g.zo <= g.own_hi);
}

// Rotation table entry (cos, sin) of pair j for a token: axial mode, the row of
// coordinate c on axis a (rows: Z values, then Y, then X); packed mode, the row
// of the token's packed index pos.
__device__ __forceinline__ float2 rope_cs(const float* tab, const Geo& g, int a, int c, int pos,
                                          int j) {
  const float2* t = reinterpret_cast<const float2*>(tab);
  if (g.rope_mode == PACK3D_ROPE_PACKED) return t[(int64_t)pos * g.rope_len + j];
  int off = a == 0 ? 0 : (a == 1 ? g.Z : g.Z + g.Y);
  return t[(off + c) * g.rope_len + j];
}

// First (cos, sin) of a row of the rotation table used by the 16-byte-chunk
// kernels (head_dim 96): axial mode, axis a's row of coordinate c; packed mode,
// the row of position pos.
__device__ __forceinline__ const float2* rope_row96(const float* tab, const Geo& g, int a, int c,
                                                    int pos) {
  const float2* t = reinterpret_cast<const float2*>(tab);
  if (g.rope_mode == PACK3D_ROPE_PACKED) return t + (int64_t)pos * 48;
  return t + ((a == 0 ? 0 : (a == 1 ? g.Z : g.Z + g.Y)) + c) * 16;
}

// Item w (0..5) of a head-dim-96 row for the chunk kernels: 16-byte chunk c1
// (8 channels, the first members of 8 rotation pairs), its partner chunk c2,
// the first pair index j0 in the table row, and the axis whose coordinate
// selects the row.  Axial: segment a = w / 2 (32 channels), pairs (j, j + 16);
// packed: pairs (j, j + 48) over the whole row.
struct Item96 {
  int c1, c2, j0, a;
};
__device__ __forceinline__ Item96 item96(const Geo& g, int w) {
  Item96 it;
  if (g.rope_mode == PACK3D_ROPE_PACKED) {
    it.c1 = w;
    it.c2 = w + 6;
    it.j0 = 8 * w;
    it.a = 0;
  } else {
    it.a = w / 2;
    it.c1 = 4 * it.a + (w & 1);
    it.c2 = it.c1 + 2;
    it.j0 = 8 * (w & 1);
  }
  return it;
}

// ---- launchers (defined in the .cu files) --------------------------------

int launch_build_index(const Geo& g, const int16_t* coords, const pack3d_index* idx,
                       float rope_base, cudaStream_t s);
int launch_block_summaries(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                           float* ksum, float* vsum, cudaStream_t s);
int launch_forward_simt(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                        const void* v, const float* ksum, const float* vsum, void* out,
                        float* lse, bool summaries, cudaStream_t s);
bool forward_tc_supported(const Geo& g);
size_t forward_tc_workspace_bytes(const Geo& g);  // 0 when the path does not apply
// Block summaries (bf16, head_dim 96) computed in the pass that also writes
// the grid-order rotated keys and values and bf16 summary copies.
int launch_block_summaries_staged(const Geo& g, const pack3d_index* idx, const void* k,
                                  const void* v, float* ksum, float* vsum, void* kg, void* vg,
                                  void* ksb, void* vsb, cudaStream_t s);
// Grid-order rotated keys and values alone (bf16, head_dim 96, up to 8
// heads: PACK3D_ERR_UNSUPPORTED otherwise), by the summary kernel's gather.
int launch_stage_bulk(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                      void* kg, void* vg, cudaStream_t s);
// Staging of the tensor-core forward's workspace: grid-order rotated keys and
// values, and the summaries' bf16 copies - converted from given summaries
// (STAGE_CONVERT), computed in the same pass (STAGE_COMPUTE: ksum, vsum are
// outputs), or left out (STAGE_NO_SUMMARIES).  Then the attention kernel.
enum StageMode { STAGE_NO_SUMMARIES = 0, STAGE_CONVERT = 1, STAGE_COMPUTE = 2 };
int launch_stage_kv(const Geo& g, const pack3d_index* idx, const void* k, const void* v,
                    const float* ksum, const float* vsum, void* ws, StageMode mode,
                    cudaStream_t s);
int launch_attention_tc(const Geo& g, const pack3d_index* idx, const void* q, void* ws,
                        void* out, float* lse, bool summaries, cudaStream_t s);
// Backward on the CUDA cores (fp32 arithmetic; every dtype and head dim):
// PACK3D_OK when its kernels are built for this shape, else
// PACK3D_ERR_UNSUPPORTED (checked before anything is launched); its
// workspace; its launch.
int backward_simt_supported(const Geo& g);
size_t backward_simt_workspace_bytes(const Geo& g);
int launch_backward_simt(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                         const void* v, const void* out, const float* lse, const void* dout,
                         void* dq, void* dk, void* dv, void* workspace, cudaStream_t s);
// Backward on the tensor cores (bf16, head_dim 96): whether it applies, its
// workspace (0 when it does not apply), its launch.
bool backward_tc_supported(const Geo& g);
size_t backward_tc_workspace_bytes(const Geo& g);
int launch_backward_tc(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                       const void* v, const void* out, const float* lse, const void* dout,
                       void* dq, void* dk, void* dv, void* workspace, cudaStream_t s);
// The two halves of the tensor-core backward: staging and the summary
// gradients over the call's (owned) queries (ksum, vsum: given summaries of the
// whole volume to use, or null for the ones computed from the call's tokens),
// then dq and dk/dv from the same workspace and the given summary gradients.
int backward_tc_summary_grads(const Geo& g, const pack3d_index* idx, const void* q, const void* k,
                              const void* v, const void* out, const float* lse, const void* dout,
                              const float* ksum, const float* vsum, float* dks, float* dvs,
                              void* workspace, cudaStream_t s);
int backward_tc_from_summary_grads(const Geo& g, const pack3d_index* idx, const float* dks,
                                   const float* dvs, void* dq, void* dk, void* dv,
                                   void* workspace, cudaStream_t s);
// The backward pack3d_backward runs: the tensor-core one where it applies,
// else the CUDA-core one (or, with simt, always the CUDA-core one).
size_t backward_workspace_bytes(const Geo& g, bool simt = false);
// Argument checks and launch of the backward with a workspace of ws_bytes.
int backward_call(const pack3d_params* p, const pack3d_index* idx, const void* q, const void* k,
                  const void* v, const void* out, const float* lse, const void* dout, void* dq,
                  void* dk, void* dv, void* workspace, size_t ws_bytes, bool simt,
                  cudaStream_t s);

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? PACK3D_OK : PACK3D_ERR_CUDA; }

// Adds n to the process-wide count of kernel launches this library has issued
// (read by pack3d_kernel_launches); every launcher calls it for its kernels.
void count_launches(int n);

}  // namespace p3d
