// C ABI of the PACK3D operator: argument checks, buffer sizing and launches.
// Every entry point returns a status code and never throws; nothing here
// allocates or frees device memory.
#include <math.h>
#include <string.h>

#include <atomic>

#include "pack3d_internal.cuh"

namespace p3d {

namespace {
std::atomic<uint64_t> g_kernel_launches{0};
}

void count_launches(int n) { g_kernel_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int64_t halo_axis_total(int extent, int tile, int r) {
  int64_t s = 0;
  for (int t0 = 0; t0 < extent; t0 += tile) {
    int lo = t0 - r < 0 ? 0 : t0 - r;
    int end = t0 + tile < extent ? t0 + tile : extent;
    int hi = end + r < extent ? end + r : extent;
    s += hi - lo;
  }
  return s;
}

int make_geo(const pack3d_params* p, Geo* g) {
  if (!p || !g) return PACK3D_ERR_ARG;
  if (p->B < 1 || p->H < 1 || p->head_dim < 6 || p->head_dim % 6) return PACK3D_ERR_ARG;
  if (p->Z < 1 || p->Y < 1 || p->X < 1 || p->Z > 32767 || p->Y > 32767 || p->X > 32767)
    return PACK3D_ERR_ARG;
  if (p->wz < 1 || p->wy < 1 || p->wx < 1 || !(p->wz & 1) || !(p->wy & 1) || !(p->wx & 1))
    return PACK3D_ERR_ARG;
  if (p->bz < 1 || p->by < 1 || p->bx < 1) return PACK3D_ERR_ARG;
  if (!(p->rope_base > 0.f) || !isfinite(p->rope_base) || !isfinite(p->scale))
    return PACK3D_ERR_ARG;
  if (p->dtype != PACK3D_BF16 && p->dtype != PACK3D_FP32) return PACK3D_ERR_ARG;
  if (p->rope_mode != PACK3D_ROPE_AXIAL && p->rope_mode != PACK3D_ROPE_PACKED)
    return PACK3D_ERR_ARG;
  const int64_t V = (int64_t)p->Z * p->Y * p->X;
  if (p->n_tokens < 0 || p->n_tokens > V) return PACK3D_ERR_ARG;
  const int64_t N = p->n_tokens > 0 ? p->n_tokens : V;
  if ((int64_t)p->B * V * p->H * p->head_dim >= (int64_t)1 << 31) return PACK3D_ERR_ARG;
  if (p->head_dim != 12 && p->head_dim != 24 && p->head_dim != 48 && p->head_dim != 96)
    return PACK3D_ERR_UNSUPPORTED;
  g->B = p->B;
  g->H = p->H;
  g->d = p->head_dim;
  g->da = p->head_dim / 3;
  g->half = g->da / 2;
  g->Z = p->Z;
  g->Y = p->Y;
  g->X = p->X;
  g->N = (int)N;
  g->V = (int)V;
  g->partial = N < V ? 1 : 0;
  // spatial sharding along z: this call's volume is planes
  // [z_origin, z_origin + Z) of a volume of Z_total planes
  if (p->Z_total < 0) return PACK3D_ERR_ARG;
  g->sharded = p->Z_total > 0 ? 1 : 0;
  g->Zt = g->sharded ? p->Z_total : p->Z;
  g->zo = g->sharded ? p->z_origin : 0;
  g->own_lo = g->sharded ? p->own_lo : 0;
  g->own_hi = g->sharded ? p->own_hi : p->Z;
  if (g->sharded && (p->z_origin < 0 || p->z_origin + p->Z > p->Z_total || p->own_lo < 0 ||
                     p->own_lo >= p->own_hi || p->own_hi > p->Z || p->Z_total > 32767))
    return PACK3D_ERR_ARG;
  g->rz = (p->wz - 1) / 2;
  g->ry = (p->wy - 1) / 2;
  g->rx = (p->wx - 1) / 2;
  g->bz = p->bz;
  g->by = p->by;
  g->bx = p->bx;
  // blocks that do not divide the volume are cut at its edge: counts round
  // up; a z-slab uses the block grid of the whole volume
  g->nbz = (g->Zt + p->bz - 1) / p->bz;
  g->nby = (p->Y + p->by - 1) / p->by;
  g->nbx = (p->X + p->bx - 1) / p->bx;
  g->nb = g->nbz * g->nby * g->nbx;
  g->nTz = (p->Z + TZ - 1) / TZ;
  g->nTy = (p->Y + TY - 1) / TY;
  g->nTx = (p->X + TX - 1) / TX;
  g->nT = g->nTz * g->nTy * g->nTx;
  g->n_halo = halo_axis_total(p->Z, TZ, g->rz) * halo_axis_total(p->Y, TY, g->ry) *
              halo_axis_total(p->X, TX, g->rx);
  if (g->n_halo * p->B >= (int64_t)1 << 31) return PACK3D_ERR_ARG;
  g->tau = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->head_dim);
  g->dtype = p->dtype;
  g->out_fp32 = (p->out_fp32 != 0 || p->dtype == PACK3D_FP32) ? 1 : 0;
  g->rope_mode = p->rope_mode;
  g->rope_len = p->rope_mode == PACK3D_ROPE_PACKED ? p->head_dim / 2 : g->half;
  return PACK3D_OK;
}

size_t backward_workspace_bytes(const Geo& g, bool simt) {
  if (!simt && backward_tc_supported(g)) return backward_tc_workspace_bytes(g);
  return backward_simt_workspace_bytes(g);
}

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// z-slabs (spatial sharding) are built for dense volumes with axial RoPE.
int shard_supported(const Geo& g) {
  return g.sharded && (g.partial || g.rope_mode != PACK3D_ROPE_AXIAL) ? PACK3D_ERR_UNSUPPORTED
                                                                      : PACK3D_OK;
}

struct IndexLayout {
  size_t vol, perm, tile_off, nbr_off, nbr, rope, err, bcount, bocc, total;
};

IndexLayout index_layout(const Geo& g) {
  IndexLayout L;
  size_t o = 0;
  L.vol = o;
  o += align256(sizeof(int32_t) * (size_t)g.B * g.V);
  L.perm = o;
  o += align256(sizeof(int32_t) * (size_t)g.B * g.N);
  L.tile_off = o;
  o += align256(sizeof(int32_t) * (size_t)g.B * (g.nT + 1));
  L.nbr_off = o;
  o += align256(sizeof(int32_t) * (size_t)(g.nT + 1));
  L.nbr = o;
  o += align256(sizeof(int32_t) * (size_t)g.B * g.n_halo);
  L.rope = o;
  // rotation table: a row per coordinate value of each axis (axial) or per
  // packed position (packed mode)
  const size_t rope_rows = g.rope_mode == PACK3D_ROPE_PACKED ? (size_t)g.N
                                                             : (size_t)(g.Z + g.Y + g.X);
  o += align256(sizeof(float) * 2 * rope_rows * g.rope_len);
  L.err = o;
  o += 256;
  L.bcount = o;
  o += align256(sizeof(int32_t) * (size_t)g.B * g.nb);
  L.bocc = o;
  o += align256(sizeof(uint32_t) * (size_t)g.B * ((g.nb + 31) / 32));
  L.total = o;
  return L;
}

int check_index(const Geo& g, const pack3d_index* ix) {
  if (!ix || !ix->vol || !ix->perm || !ix->tile_off || !ix->nbr_off || !ix->nbr || !ix->rope ||
      !ix->err || !ix->bcount || !ix->bocc)
    return PACK3D_ERR_ARG;
  if (ix->tile[0] != TZ || ix->tile[1] != TY || ix->tile[2] != TX || ix->n_tiles != g.nT ||
      ix->n_halo != g.n_halo)
    return PACK3D_ERR_ARG;
  return PACK3D_OK;
}

}  // namespace

int backward_call(const pack3d_params* p, const pack3d_index* idx, const void* q, const void* k,
                  const void* v, const void* out, const float* lse, const void* dout, void* dq,
                  void* dk, void* dv, void* workspace, size_t ws_bytes, bool simt,
                  cudaStream_t s) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace)
    return PACK3D_ERR_ARG;
  // z-slabs: the summary gradients need an exchange (the two-call form)
  if (g.sharded) return PACK3D_ERR_UNSUPPORTED;
  if (((uintptr_t)workspace & 255) || ws_bytes < backward_workspace_bytes(g, simt))
    return PACK3D_ERR_ARG;
  if (!simt && backward_tc_supported(g))
    return launch_backward_tc(g, idx, q, k, v, out, lse, dout, dq, dk, dv, workspace, s);
  if ((rc = backward_simt_supported(g))) return rc;
  return launch_backward_simt(g, idx, q, k, v, out, lse, dout, dq, dk, dv, workspace, s);
}

}  // namespace p3d

using namespace p3d;

extern "C" {

size_t pack3d_index_bytes(const pack3d_params* p) {
  Geo g;
  if (make_geo(p, &g)) return 0;
  return index_layout(g).total;
}

int pack3d_index_init(const pack3d_params* p, void* buffer, size_t bytes, pack3d_index* out) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if (!buffer || !out || ((uintptr_t)buffer & 255)) return PACK3D_ERR_ARG;
  IndexLayout L = index_layout(g);
  if (bytes < L.total) return PACK3D_ERR_ARG;
  char* base = (char*)buffer;
  out->vol = (int32_t*)(base + L.vol);
  out->perm = (int32_t*)(base + L.perm);
  out->tile_off = (int32_t*)(base + L.tile_off);
  out->nbr_off = (int32_t*)(base + L.nbr_off);
  out->nbr = (int32_t*)(base + L.nbr);
  out->rope = (float*)(base + L.rope);
  out->err = (int32_t*)(base + L.err);
  out->bcount = (int32_t*)(base + L.bcount);
  out->bocc = (uint32_t*)(base + L.bocc);
  out->tile[0] = TZ;
  out->tile[1] = TY;
  out->tile[2] = TX;
  out->n_tiles = g.nT;
  out->n_halo = g.n_halo;
  return PACK3D_OK;
}

int pack3d_build_index(const pack3d_params* p, const int16_t* coords, pack3d_index* idx,
                       pack3d_stream_t stream) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if (!coords || (rc = check_index(g, idx))) return rc ? rc : PACK3D_ERR_ARG;
  return launch_build_index(g, coords, idx, p->rope_base, (cudaStream_t)stream);
}

int pack3d_index_check(const pack3d_index* idx, pack3d_stream_t stream) {
  if (!idx || !idx->err) return PACK3D_ERR_ARG;
  int32_t err[2] = {0, 0};
  if (cudaMemcpyAsync(err, idx->err, sizeof(err), cudaMemcpyDeviceToHost,
                      (cudaStream_t)stream) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PACK3D_ERR_CUDA;
  if (err[0] & 3) return PACK3D_ERR_COORDS;
  return err[0] ? PACK3D_ERR_TIMEOUT : PACK3D_OK;
}

int pack3d_block_summaries(const pack3d_params* p, const pack3d_index* idx, const void* k,
                           const void* v, float* ksum, float* vsum, pack3d_stream_t stream) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  if (!k || !v || !ksum || !vsum) return PACK3D_ERR_ARG;
  return launch_block_summaries(g, idx, k, v, ksum, vsum, (cudaStream_t)stream);
}

size_t pack3d_forward_workspace_bytes(const pack3d_params* p) {
  Geo g;
  if (make_geo(p, &g)) return 0;
  return forward_tc_workspace_bytes(g);
}

static int forward_common(const pack3d_params* p, const pack3d_index* idx, const void* q,
                          const void* k, const void* v, const float* ksum, const float* vsum,
                          void* ws, size_t ws_bytes, void* out, float* lse, bool summaries,
                          cudaStream_t s) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  if (!q || !k || !v || !out || !lse || (summaries && (!ksum || !vsum))) return PACK3D_ERR_ARG;
  if ((rc = shard_supported(g))) return rc;
  const size_t need = forward_tc_workspace_bytes(g);
  if (need) {
    if (!ws || ((uintptr_t)ws & 255) || ws_bytes < need) return PACK3D_ERR_ARG;
    if ((rc = launch_stage_kv(g, idx, k, v, ksum, vsum, ws,
                              summaries ? STAGE_CONVERT : STAGE_NO_SUMMARIES, s)))
      return rc;
    return launch_attention_tc(g, idx, q, ws, out, lse, summaries, s);
  }
  // partly occupied volumes and z-slabs run on the tensor-core path only
  if (g.partial || g.sharded) return PACK3D_ERR_UNSUPPORTED;
  return launch_forward_simt(g, idx, q, k, v, ksum, vsum, out, lse, summaries, s);
}

int pack3d_stage_kv(const pack3d_params* p, const pack3d_index* idx, const void* k, const void* v,
                    float* ksum, float* vsum, void* workspace, size_t workspace_bytes,
                    pack3d_stream_t stream) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  const size_t need = forward_tc_workspace_bytes(g);
  if (!need) return PACK3D_ERR_UNSUPPORTED;
  if ((rc = shard_supported(g))) return rc;
  if (!k || !v || (!ksum != !vsum) || !workspace || ((uintptr_t)workspace & 255) ||
      workspace_bytes < need)
    return PACK3D_ERR_ARG;
  return launch_stage_kv(g, idx, k, v, ksum, vsum, workspace,
                         ksum ? STAGE_COMPUTE : STAGE_NO_SUMMARIES, (cudaStream_t)stream);
}

int pack3d_forward_staged(const pack3d_params* p, const pack3d_index* idx, const void* q,
                          const void* workspace, size_t workspace_bytes, int with_summaries,
                          void* out, float* lse, pack3d_stream_t stream) {
  Geo g;
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  const size_t need = forward_tc_workspace_bytes(g);
  if (!need) return PACK3D_ERR_UNSUPPORTED;
  if ((rc = shard_supported(g))) return rc;
  if (!q || !out || !lse || !workspace || ((uintptr_t)workspace & 255) || workspace_bytes < need)
    return PACK3D_ERR_ARG;
  return launch_attention_tc(g, idx, q, const_cast<void*>(workspace), out, lse,
                             with_summaries != 0, (cudaStream_t)stream);
}

int pack3d_forward(const pack3d_params* p, const pack3d_index* idx, const void* q, const void* k,
                   const void* v, const float* ksum, const float* vsum, void* workspace,
                   size_t workspace_bytes, void* out, float* lse, pack3d_stream_t stream) {
  return forward_common(p, idx, q, k, v, ksum, vsum, workspace, workspace_bytes, out, lse, true,
                        (cudaStream_t)stream);
}

int pack3d_window_forward(const pack3d_params* p, const pack3d_index* idx, const void* q,
                          const void* k, const void* v, void* workspace, size_t workspace_bytes,
                          void* out, float* lse, pack3d_stream_t stream) {
  return forward_common(p, idx, q, k, v, nullptr, nullptr, workspace, workspace_bytes, out, lse,
                        false, (cudaStream_t)stream);
}

size_t pack3d_backward_workspace_bytes(const pack3d_params* p) {
  Geo g;
  if (make_geo(p, &g)) return 0;
  return backward_workspace_bytes(g);
}

int pack3d_backward(const pack3d_params* p, const pack3d_index* idx, const void* q, const void* k,
                    const void* v, const void* out, const float* lse, const void* dout, void* dq,
                    void* dk, void* dv, void* workspace, size_t workspace_bytes,
                    pack3d_stream_t stream) {
  return backward_call(p, idx, q, k, v, out, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                       false, (cudaStream_t)stream);
}

namespace {

int backward_phase_check(const pack3d_params* p, const pack3d_index* idx, void* workspace,
                         size_t workspace_bytes, Geo& g) {
  int rc = make_geo(p, &g);
  if (rc) return rc;
  if ((rc = check_index(g, idx))) return rc;
  if (!workspace || ((uintptr_t)workspace & 255)) return PACK3D_ERR_ARG;
  if (!backward_tc_supported(g)) return PACK3D_ERR_UNSUPPORTED;
  if ((rc = shard_supported(g))) return rc;
  if (workspace_bytes < backward_tc_workspace_bytes(g)) return PACK3D_ERR_ARG;
  return PACK3D_OK;
}

}  // namespace

int pack3d_backward_summary_grads(const pack3d_params* p, const pack3d_index* idx, const void* q,
                                  const void* k, const void* v, const void* out, const float* lse,
                                  const void* dout, const float* ksum, const float* vsum,
                                  float* dks, float* dvs, void* workspace, size_t workspace_bytes,
                                  pack3d_stream_t stream) {
  Geo g;
  int rc = backward_phase_check(p, idx, workspace, workspace_bytes, g);
  if (rc) return rc;
  if (!q || !k || !v || !out || !lse || !dout || !dks || !dvs || (!ksum) != (!vsum) ||
      (g.sharded && !ksum))
    return PACK3D_ERR_ARG;
  return backward_tc_summary_grads(g, idx, q, k, v, out, lse, dout, ksum, vsum, dks, dvs,
                                   workspace, (cudaStream_t)stream);
}

int pack3d_backward_from_summary_grads(const pack3d_params* p, const pack3d_index* idx,
                                       const float* dks, const float* dvs, void* workspace,
                                       size_t workspace_bytes, void* dq, void* dk, void* dv,
                                       pack3d_stream_t stream) {
  Geo g;
  int rc = backward_phase_check(p, idx, workspace, workspace_bytes, g);
  if (rc) return rc;
  if (!dks || !dvs || !dq || !dk || !dv) return PACK3D_ERR_ARG;
  return backward_tc_from_summary_grads(g, idx, dks, dvs, dq, dk, dv, workspace,
                                        (cudaStream_t)stream);
}

uint64_t pack3d_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

const char* pack3d_strerror(int status) {
  switch (status) {
    case PACK3D_OK: return "ok";
    case PACK3D_ERR_ARG: return "invalid argument";
    case PACK3D_ERR_COORDS: return "coordinates out of range or not a bijection onto the grid";
    case PACK3D_ERR_CUDA: return "CUDA launch or runtime error";
    case PACK3D_ERR_TIMEOUT: return "bounded device-side wait timed out";
    case PACK3D_ERR_UNSUPPORTED: return "shape not built into this library";
    default: return "unknown status";
  }
}

}  // extern "C"
