/*
 * pack3d.h - C ABI of the PACK3D local-global attention operator on NVIDIA
 * B200 (sm_100a).
 *
 * The operator is the one introduced in "Geometry Matters in Packed 3D
 * Attention" (abstract): a 3D volume is packed into a token sequence in an
 * arbitrary memory order; each query attends, in one softmax, exactly to the
 * tokens of its local 3D neighbourhood and to summaries of the contiguous 3D
 * blocks that lie outside that neighbourhood; every query-key and
 * query-summary interaction is indexed by axial RoPE on the tokens' true grid
 * coordinates, never on their packed position, and keys are rotated before a
 * block is summarised.  The conventions the abstract leaves open are fixed
 * here:
 *
 *   - head_dim d = 3 * da; channels [0, da) rotate with z, [da, 2da) with y,
 *     [2da, 3da) with x; inside a segment channel j pairs with j + da/2 and
 *     turns by the angle c * rope_base^(-2j/da) (c = the token's coordinate
 *     on that axis); v is not rotated.
 *   - window (wz, wy, wx), all odd: the box of half-widths (w - 1) / 2
 *     centred on the query, clipped at the volume edge (never shifted).
 *   - blocks (bz, by, bx) tile the volume in raster order; where an extent
 *     does not divide the volume, the last block along that axis is cut at the
 *     volume's edge and holds only the tokens inside it; a block's summary is
 *     the mean of its tokens' rotated keys and the mean of their values; a
 *     query sees the summary of every block whose box does not intersect its
 *     window box, with logit scale * q~ . kbar and no count bias.
 *   - scale defaults to 1 / sqrt(head_dim); lse is the natural log of the
 *     softmax normaliser, summaries included.
 *   - occupancy: by default (n_tokens = 0) the coordinates are a bijection
 *     onto the Z x Y x X grid per batch item (a dense volume).  With
 *     n_tokens > 0 every batch item holds n_tokens tokens at distinct voxels
 *     and the other voxels are empty: windows and blocks hold only the tokens
 *     present, a block's summary averages over its tokens, and a block
 *     holding none has no summary.  Each batch item may use its own packing.
 *
 * Memory: every buffer is allocated and owned by the caller; the library
 * never allocates or frees device memory.  Its only global state is a count of
 * the kernels it has launched (pack3d_kernel_launches) and the static scratch
 * array of pack3d_backward_noalloc.  All
 * pointers except the params and index structs are DEVICE pointers.  Layouts:
 *   q, k, v, out, dout, dq, dk, dv : [B][N][H][head_dim], packed order,
 *                                    bf16 (dtype PACK3D_BF16) or fp32
 *                                    (out is fp32 when out_fp32 is set);
 *   coords                        : int16 [B][N][3] as (z, y, x);
 *   ksum, vsum                    : fp32 [B][H][nb][head_dim], blocks in
 *                                    raster order (nb = ceil(Z/bz) *
 *                                    ceil(Y/by) * ceil(X/bx)); 0 for an
 *                                    empty block;
 *   lse                           : fp32 [B][H][N].
 * N = n_tokens if n_tokens > 0, else Z * Y * X.  Every call is asynchronous on the given stream (a
 * cudaStream_t; 0 is the legacy default stream) and returns a status code
 * (0 on success, a negative PACK3D_ERR_* otherwise); no call synchronises
 * except pack3d_index_check.  Errors found on the host (bad arguments) are
 * returned before anything is launched; launch failures return
 * PACK3D_ERR_CUDA.
 */
#ifndef PACK3D_H
#define PACK3D_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PACK3D_API __attribute__((visibility("default")))
#else
#define PACK3D_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pack3d_stream_t; /* the same type as cudaStream_t */

enum { PACK3D_BF16 = 0, PACK3D_FP32 = 1 };
enum { PACK3D_ROPE_AXIAL = 0, PACK3D_ROPE_PACKED = 1 };

enum {
  PACK3D_OK = 0,
  PACK3D_ERR_ARG = -1,         /* null pointer, inconsistent sizes, even window, ... */
  PACK3D_ERR_COORDS = -2,      /* coordinates out of range or not a bijection */
  PACK3D_ERR_CUDA = -3,        /* a CUDA launch or runtime call failed */
  PACK3D_ERR_TIMEOUT = -4,     /* a bounded device-side wait gave up */
  PACK3D_ERR_UNSUPPORTED = -5  /* valid operator, shape not built into this library */
};

/* Operator shape and conventions.  head_dim must be a multiple of 12 and at
 * most 96 (12, 24, 48, 96 are built), windows odd and positive, block extents
 * positive (any size: blocks that do not divide the volume are cut at its
 * edge), 1 <= Z, Y, X <= 32767 and B * N * H * head_dim < 2^31. */
typedef struct {
  int32_t B, H, head_dim;
  int32_t Z, Y, X;
  int32_t wz, wy, wx;
  int32_t bz, by, bx;
  float rope_base; /* > 0 */
  float scale;     /* softmax scale; <= 0 selects 1 / sqrt(head_dim) */
  int32_t dtype;   /* PACK3D_BF16 or PACK3D_FP32 (inputs, outputs, gradients) */
  int32_t out_fp32; /* nonzero: the forward's out (and the backward's out argument) is
                       fp32 even when dtype is PACK3D_BF16 */
  int32_t rope_mode; /* PACK3D_ROPE_AXIAL (0, the operator): axial RoPE on grid
                        coordinates; PACK3D_ROPE_PACKED (1, the comparison mode):
                        one-dimensional RoPE on the token's packed index (pairs
                        j, j + head_dim/2, theta_j = rope_base^(-2j/head_dim));
                        windows, blocks and summaries stay geometric */
  int32_t n_tokens;  /* 0: a dense volume, N = Z * Y * X tokens per batch item;
                        1 .. Z*Y*X: a partly occupied volume of N = n_tokens
                        tokens per batch item at distinct voxels (the forward
                        and backward run it on the tensor-core path, bf16 at
                        head_dim 96; other dtypes and head dims report
                        PACK3D_ERR_UNSUPPORTED for it) */
  int32_t Z_total;   /* 0: the volume is the whole problem.  > 0: spatial sharding
                        along z.  The call's volume holds planes
                        [z_origin, z_origin + Z) of a volume of Z_total planes
                        (one rank's z-slab with its halo planes): coordinates
                        stay local (0 .. Z-1), RoPE angles and the block grid
                        follow the global plane z + z_origin (nb counts the
                        blocks of the whole volume), and only the local planes
                        [own_lo, own_hi) are owned.  Outputs (out, lse) are
                        written for tokens in owned planes only, and
                        pack3d_block_summaries computes the blocks lying wholly
                        in owned planes and writes zeros for the others, so
                        that a sum over the ranks (an all-reduce) gives every
                        block's summary.  A query's window must lie inside the
                        call's volume: rz halo planes on each side of the owned
                        planes where the whole volume continues.  The
                        tensor-core path only (bf16, head_dim 96), dense
                        volumes, axial RoPE; others report
                        PACK3D_ERR_UNSUPPORTED.  The backward of a slab runs
                        as the two calls of pack3d_backward_summary_grads
                        with an all-reduce between them (pack3d_backward
                        reports PACK3D_ERR_UNSUPPORTED for a slab). */
  int32_t z_origin;  /* global plane of local plane 0 (sharding; 0 otherwise) */
  int32_t own_lo, own_hi; /* owned local planes (sharding; both 0 otherwise) */
} pack3d_params;

/* Geometry index of one packing, built by pack3d_build_index into one
 * caller-allocated device buffer (see pack3d_index_init).  Query tiles are
 * tile[0] x tile[1] x tile[2] boxes (z, y, x) in raster order, cut by the
 * volume edge where the extents do not divide.
 *   vol      int32 [B][Z*Y*X]   packed index of the token at each voxel, -1 for
 *                               an empty voxel
 *   perm     int32 [B][N]       tile-ordered permutation: tile by tile, raster
 *                               order inside a tile, the packed index of each
 *                               token (a counting sort by tile)
 *   tile_off int32 [B][T+1]     start of tile t in perm
 *   nbr_off  int32 [T+1]        start of tile t's halo list (same for every
 *                               batch item)
 *   nbr      int32 [B][n_halo]  halo lists: for each tile, the packed indices
 *                               of the voxels in the tile box widened by the
 *                               window radius and clipped to the volume, in
 *                               raster order (-1 for an empty voxel)
 *   rope     float [(Z+Y+X)][head_dim/6][2]  cos and sin of c * theta_j per
 *                               axis (z rows, then y, then x), computed in fp64
 *   err      int32 [2]          [0]: 0 or a bit set of 1 = coordinate out of
 *                               range, 2 = voxel held twice, 4 = a kernel
 *                               gave up a bounded device-side wait; [1]:
 *                               smallest offending flat token index b * N + i
 *   bcount   int32 [B][nb]      tokens held by each block (built for partly
 *                               occupied volumes only)
 *   bocc     uint32 [B][ceil(nb/32)]  bit B % 32 of word B / 32: block B holds
 *                               at least one token (built for partly occupied
 *                               volumes only)
 */
typedef struct {
  int32_t* vol;
  int32_t* perm;
  int32_t* tile_off;
  int32_t* nbr_off;
  int32_t* nbr;
  float* rope;
  int32_t* err;
  int32_t* bcount;
  uint32_t* bocc;
  int32_t tile[3];
  int32_t n_tiles;
  int64_t n_halo;
} pack3d_index;

/* Bytes of device memory an index needs for these params (0 if the params
 * are invalid).  Host-only; no CUDA call. */
PACK3D_API size_t pack3d_index_bytes(const pack3d_params* p);

/* Carve an index out of a caller-allocated device buffer of at least
 * pack3d_index_bytes(p) bytes, aligned to 256 bytes.  Fills *out; no CUDA
 * call.  The buffer stays owned by the caller and must outlive every use of
 * the index. */
PACK3D_API int pack3d_index_init(const pack3d_params* p, void* buffer, size_t bytes, pack3d_index* out);

/* Build the index of one packing from its coordinates: the coordinate volume,
 * the tile permutation by counting sort, the halo lists and the rotation
 * table.  This is what lets attention follow the true grid coordinates instead
 * of the packed order ("Geometry Matters in Packed 3D Attention", abstract).  Asynchronous: coordinate errors are recorded in idx->err on
 * the device and make every later kernel using this index return without
 * writing; call pack3d_index_check to read them. */
PACK3D_API int pack3d_build_index(const pack3d_params* p, const int16_t* coords, pack3d_index* idx,
                       pack3d_stream_t stream);

/* Synchronise the stream and report the index's error word: PACK3D_OK,
 * PACK3D_ERR_COORDS (bits 1 or 2), PACK3D_ERR_TIMEOUT (bit 4: a kernel that
 * used this index gave up a bounded wait) or PACK3D_ERR_CUDA.  The only
 * blocking call of the library. */
PACK3D_API int pack3d_index_check(const pack3d_index* idx, pack3d_stream_t stream);

/* Block summaries ("compresses only distant context into contiguous 3D block
 * summaries"; "the rotation is applied before a block is summarized",
 * abstract): ksum[b][h][B] = mean over the tokens of block B of R(c_j) k_j,
 * vsum[b][h][B] = mean of v_j, accumulated in fp32 in grid order (the result
 * does not depend on the packing). */
PACK3D_API int pack3d_block_summaries(const pack3d_params* p, const pack3d_index* idx, const void* k,
                           const void* v, float* ksum, float* vsum, pack3d_stream_t stream);

/* Bytes of device workspace pack3d_forward and pack3d_window_forward need for
 * these params; 0 when the call needs none (fp32, or a head_dim other than 96,
 * which run on the CUDA cores).  At the 65,536-token, batch 2, 8-head, d = 96
 * shape: 403 MB (grid-order copies of the rotated keys and of the values, and
 * bf16 copies of the summaries). */
PACK3D_API size_t pack3d_forward_workspace_bytes(const pack3d_params* p);

/* Full PACK3D forward (abstract: exact local neighbourhood attention plus
 * the block summaries, axial RoPE on grid coordinates, one softmax): out and
 * lse for every query, from the local window keys and the summaries (from
 * pack3d_block_summaries; they may be reused across calls with the same k, v
 * and index).  workspace: caller-allocated device memory of at least
 * pack3d_forward_workspace_bytes(p) bytes, 256-byte aligned (may be NULL when
 * that size is 0); its contents on entry do not matter and it holds no result
 * afterwards.  PACK3D_ERR_ARG if it is missing, short or misaligned. */
PACK3D_API int pack3d_forward(const pack3d_params* p, const pack3d_index* idx, const void* q,
                              const void* k, const void* v, const float* ksum, const float* vsum,
                              void* workspace, size_t workspace_bytes, void* out, float* lse,
                              pack3d_stream_t stream);

/* Window-only forward: the same operator without summaries (windowed
 * attention with axial RoPE, the latency comparator the abstract names);
 * lse covers the local keys only.  workspace as for pack3d_forward. */
PACK3D_API int pack3d_window_forward(const pack3d_params* p, const pack3d_index* idx,
                                     const void* q, const void* k, const void* v, void* workspace,
                                     size_t workspace_bytes, void* out, float* lse,
                                     pack3d_stream_t stream);

/* The two halves of the tensor-core forward, for callers that run several
 * forwards against the same keys and values, or that want the block
 * summaries and the staging in one pass over k and v.
 * pack3d_stage_kv writes into the workspace the rotated keys and the values in
 * grid order.  When ksum and vsum are given (both or neither) it also computes
 * the block summaries in the same pass - OUTPUTS, the same values
 * pack3d_block_summaries writes - and stages their bf16 copies.
 * pack3d_forward_staged then computes out and lse from q and a workspace
 * staged with the same params, k, v and index (with_summaries != 0: the full
 * operator, which needs a staging with summaries; 0: window only).
 * pack3d_forward = pack3d_stage_kv without summaries + staging of the given
 * summaries + pack3d_forward_staged.  Both return PACK3D_ERR_UNSUPPORTED where
 * pack3d_forward_workspace_bytes is 0, and PACK3D_ERR_ARG for a missing,
 * short or misaligned workspace. */
PACK3D_API int pack3d_stage_kv(const pack3d_params* p, const pack3d_index* idx, const void* k,
                               const void* v, float* ksum, float* vsum, void* workspace,
                               size_t workspace_bytes, pack3d_stream_t stream);
PACK3D_API int pack3d_forward_staged(const pack3d_params* p, const pack3d_index* idx,
                                     const void* q, const void* workspace, size_t workspace_bytes,
                                     int with_summaries, void* out, float* lse,
                                     pack3d_stream_t stream);

/* Bytes of device workspace pack3d_backward needs for these params. */
PACK3D_API size_t pack3d_backward_workspace_bytes(const pack3d_params* p);

/* Backward of the full operator (the abstract calls the operator "trainable
 * at scale"): gradients of sum(dout * out) with
 * respect to q, k, v, through the rotation and through the block means, from
 * the forward's out and lse.  workspace: caller-allocated, at least
 * pack3d_backward_workspace_bytes(p) bytes, 256-byte aligned; its contents on
 * entry do not matter.  Reductions run in a fixed order (deterministic, no
 * floating-point atomics). */
PACK3D_API int pack3d_backward(const pack3d_params* p, const pack3d_index* idx, const void* q, const void* k,
                    const void* v, const void* out, const float* lse, const void* dout, void* dq,
                    void* dk, void* dv, void* workspace, size_t workspace_bytes,
                    pack3d_stream_t stream);

/* The backward of pack3d_backward in two calls, for a volume cut into
 * z-slabs (params with Z_total > 0).  The gradient of a block summary is a sum
 * over every query of the volume whose window misses the block, so on a slab it
 * is a partial sum: the caller adds the ranks' partial sums (an all-reduce)
 * between the two calls.  The operator is the one the paper's abstract
 * describes (each query also attends to the mean-pooled keys and values of the
 * blocks its window misses); the split into two calls is this library's.
 *
 * pack3d_backward_summary_grads stages q, k, v, out, lse and dout into the
 * workspace and writes dks, dvs [B, H, nb, head_dim] fp32 (nb blocks of the
 * whole volume in block-raster order, as pack3d_block_summaries writes the
 * summaries): the gradients of sum(dout * out)
 * with respect to the block summaries, over the call's owned queries (all
 * queries unless the call is a slab).  ksum, vsum [B, H, nb, head_dim] fp32:
 * the summaries the forward used - for a slab the all-reduced summaries of the
 * whole volume, required; otherwise NULL (both) to compute them from k and v
 * here.  A slab's call needs q, k, v, out, lse and dout of its halo planes too
 * (the neighbours' tokens: their queries reach the owned keys).
 *
 * pack3d_backward_from_summary_grads then writes dq, dk, dv for the call's
 * owned tokens (other rows are left untouched), from the workspace left by
 * the first call (same params, index and workspace, unmodified in between)
 * and the summary gradients of the whole volume (for a slab, the sum over
 * ranks).  The two calls with no exchange between them give exactly
 * pack3d_backward's results.
 *
 * workspace: at least pack3d_backward_workspace_bytes(p) bytes, 256-byte
 * aligned (PACK3D_ERR_ARG otherwise).  Built on the tensor-core path only (bf16,
 * head_dim 96); other shapes and slabs of partly occupied volumes or of the
 * packed RoPE mode report PACK3D_ERR_UNSUPPORTED.  Fixed-order reductions, no
 * floating-point atomics. */
PACK3D_API int pack3d_backward_summary_grads(const pack3d_params* p, const pack3d_index* idx,
                                             const void* q, const void* k, const void* v,
                                             const void* out, const float* lse, const void* dout,
                                             const float* ksum, const float* vsum, float* dks,
                                             float* dvs, void* workspace, size_t workspace_bytes,
                                             pack3d_stream_t stream);
PACK3D_API int pack3d_backward_from_summary_grads(const pack3d_params* p, const pack3d_index* idx,
                                                  const float* dks, const float* dvs,
                                                  void* workspace, size_t workspace_bytes,
                                                  void* dq, void* dk, void* dv,
                                                  pack3d_stream_t stream);

/* Size of the device scratch array behind pack3d_backward_noalloc. */
#define PACK3D_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* The backward of pack3d_backward for callers that cannot allocate device
 * memory: code that is handed its input and output buffers by a host
 * framework that owns every allocation (a plugin, an embedded runtime), or
 * code that must not allocate once running (cudaMalloc may synchronise the
 * device and take unbounded time).  The paper has no counterpart; this is a
 * deployment variant of the same backward, with the same arguments minus the
 * workspace.
 *
 * The workspace lives in a static device array of
 * PACK3D_NOALLOC_SCRATCH_BYTES (32 MiB) inside this library; every GPU on
 * which the library is used holds that array until the process exits.  Every
 * call looks up the array's device address on the current device
 * (cudaGetSymbolAddress); on the first call on a device that lookup also loads
 * the library's device code there, so make that first call before any stream
 * capture.  Shapes whose workspace (pack3d_backward_workspace_bytes) exceeds
 * the array are rejected with PACK3D_ERR_UNSUPPORTED before anything is
 * launched (the 65k-token, 8-head training shape needs 20.5 MiB).  Nothing is
 * allocated or freed.  Every call on every stream shares the one array: calls
 * whose executions overlap on the GPU race and give wrong results, so issue
 * them on one stream or serialise them.  Each call writes every scratch byte it
 * reads, so what an earlier call left there does not matter. */
PACK3D_API int pack3d_backward_noalloc(const pack3d_params* p, const pack3d_index* idx,
                                       const void* q, const void* k, const void* v,
                                       const void* out, const float* lse, const void* dout,
                                       void* dq, void* dk, void* dv, pack3d_stream_t stream);

/* Number of kernels this library has launched in this process, over every
 * call, device and stream (a host-side counter, incremented when a launch is
 * issued; no CUDA call).  The difference of two readings counts the launches
 * of the calls made in between, e.g. inside a timed region.  No counterpart in
 * the paper: an instrumentation aid. */
PACK3D_API uint64_t pack3d_kernel_launches(void);

/* Diagnostic of the bounded device-side waits (no counterpart in the paper).
 * Every wait in the library's kernels polls an mbarrier at most a fixed number
 * of times; a CTA that runs out sets the timeout bit of the index error word
 * (reported as PACK3D_ERR_TIMEOUT by pack3d_index_check), lets its own copies
 * and tensor-core products land and returns.  This call launches one warp
 * that waits, with at most `polls` polls (1 .. 2^24), on a barrier phase that
 * nothing completes, then synchronises the stream and returns
 * PACK3D_ERR_TIMEOUT - the status a timed-out wait produces; PACK3D_ERR_ARG
 * for a poll count out of range. */
PACK3D_API int pack3d_wait_selftest(uint32_t polls, pack3d_stream_t stream);

/* Human-readable text of a status code (static storage). */
PACK3D_API const char* pack3d_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* PACK3D_H */
