/*
 * PACK3D oracle: a plain, slow, fp64 CPU implementation of the PACK3D
 * local-global attention operator.
 *
 * TEST INFRASTRUCTURE ONLY.  It exists to check the CUDA library.  Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg load it; the
 * CUDA library neither links, includes nor calls anything here, and nothing here
 * uses the CUDA library.
 *
 * What is computed (from "Geometry Matters in Packed 3D Attention", abstract:
 * "keeps local neighborhood attention exact, compresses only distant context
 * into contiguous 3D block summaries, and indexes every query-key interaction
 * with axial RoPE on true token-grid coordinates"; "the rotation is applied
 * before a block is summarized").  For batch item b, head h and the query token
 * i with grid coordinate c_i = (z, y, x):
 *
 *   1. q~_i = R(c_i) q_i and k~_j = R(c_j) k_j, the axial rotation: channel
 *      segment a in {z, y, x} is [a*da, (a+1)*da) with da = d/3; inside a
 *      segment channel j pairs with j + da/2, theta_j = base^(-2j/da), and the
 *      pair (x1, x2) turns by the angle c_a * theta_j.  v is not rotated.
 *   2. W(i): the tokens j whose coordinate lies in the box
 *      [c_i - r, c_i + r] (r = (w - 1) / 2 per axis) clipped to the volume.
 *   3. Blocks: the volume cut into contiguous bz x by x bx boxes, in raster
 *      order; where an extent does not divide the volume, the last box along
 *      that axis is cut at the volume's edge.  kbar_B = mean over the block's
 *      tokens of k~_j, vbar_B = mean of v_j (over the tokens the block actually
 *      holds), summed in raster order inside the block.
 *   4. S(i): the blocks whose box does not intersect the window box of i.
 *   5. Logits tau * q~_i . k~_j (j in W(i)) and tau * q~_i . kbar_B (B in
 *      S(i)), with no count bias; one softmax over both sets.
 *   6. o_i = softmax-weighted sum of v_j and vbar_B; lse_i = m + ln(l).
 *
 * Packed-sequence comparison mode (rope_mode = 1): the same operator with the
 * rotation of step 1 replaced by the standard one-dimensional RoPE on the
 * token's position p in the packed sequence (its index in memory order): the
 * whole head is one segment, channel j pairs with j + d/2, theta_j =
 * base^(-2j/d), angle p * theta_j.  Windows, blocks and summaries stay
 * geometric.  This is the positional encoding the abstract contrasts with
 * axial RoPE on grid coordinates; with it the result depends on the packing.
 *
 * Every loop runs in grid order (never in packed order), so results do not
 * depend on the memory order of the tokens.  Inputs are read as fp64, fp32 or
 * bf16 bit patterns and widened exactly to fp64; all arithmetic is fp64 with
 * libm's cos, sin, exp and log.
 *
 * Layouts: q, k, v, dout, dq, dk, dv are [B][N][H][d] in packed order; coords
 * is int16 [B][N][3] as (z, y, x); summaries are [B][H][nb][d] in block raster
 * order; lse is [B][H][N].
 *
 * Occupancy: by default (n_tokens = 0) the tokens fill the volume, N = Z*Y*X,
 * one token per voxel.  With n_tokens > 0 every batch item holds N = n_tokens
 * tokens at distinct voxels and the other voxels are empty: windows and blocks
 * then hold only the tokens present, a block's summary averages over its
 * present tokens, and a block holding none has no summary (it is in no S(i)).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t B, H, d, Z, Y, X;
  int32_t wz, wy, wx;
  int32_t bz, by, bx;
  double base;
  double scale;      /* tau; <= 0 means 1/sqrt(d) */
  int32_t rope_mode; /* 0: axial on grid coordinates; 1: 1-D on the packed position */
  int32_t n_tokens;  /* 0: dense volume (N = Z*Y*X); > 0: N tokens at distinct voxels */
} orc_params;

enum { ORC_OK = 0, ORC_ERR_ARG = -1, ORC_ERR_COORDS = -2, ORC_ERR_MEM = -3 };
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

/* ---- small helpers ---------------------------------------------------- */

static double widen(const void* base, int dtype, size_t idx) {
  if (dtype == ORC_F64) return ((const double*)base)[idx];
  if (dtype == ORC_F32) return (double)((const float*)base)[idx];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &bits, 4);
  return (double)f;
}

static int check_params(const orc_params* p) {
  if (p->B < 1 || p->H < 1 || p->Z < 1 || p->Y < 1 || p->X < 1) return ORC_ERR_ARG;
  if (p->d < 6 || p->d % 6 != 0) return ORC_ERR_ARG;
  if (p->wz < 1 || p->wy < 1 || p->wx < 1) return ORC_ERR_ARG;
  if (p->wz % 2 == 0 || p->wy % 2 == 0 || p->wx % 2 == 0) return ORC_ERR_ARG;
  if (p->bz < 1 || p->by < 1 || p->bx < 1) return ORC_ERR_ARG;
  if (!(p->base > 0.0)) return ORC_ERR_ARG;
  if (p->rope_mode != 0 && p->rope_mode != 1) return ORC_ERR_ARG;
  if (p->n_tokens < 0 || (int64_t)p->n_tokens > (int64_t)p->Z * p->Y * p->X) return ORC_ERR_ARG;
  return ORC_OK;
}

static double tau_of(const orc_params* p) {
  return p->scale > 0.0 ? p->scale : 1.0 / sqrt((double)p->d);
}

static size_t nvox(const orc_params* p) { return (size_t)p->Z * p->Y * p->X; }

/* Tokens per batch item. */
static size_t ntok(const orc_params* p) { return p->n_tokens > 0 ? (size_t)p->n_tokens : nvox(p); }

static size_t vox_id(const orc_params* p, int z, int y, int x) {
  return ((size_t)z * p->Y + y) * p->X + x;
}

/* Blocks along each axis (the last one cut at the volume's edge when the
 * extent does not divide the volume). */
static int nb_axis(int dim, int ext) { return (dim + ext - 1) / ext; }

static int nblocks(const orc_params* p) {
  return nb_axis(p->Z, p->bz) * nb_axis(p->Y, p->by) * nb_axis(p->X, p->bx);
}

/* Tokens held by every block of one batch item (vb: its volume, -1 where a
 * voxel is empty): cnt[B] for B in block raster order. */
static void block_members(const orc_params* p, const int32_t* vb, int32_t* cnt) {
  int nby = nb_axis(p->Y, p->by), nbx = nb_axis(p->X, p->bx), nb = nblocks(p);
  for (int B = 0; B < nb; ++B) cnt[B] = 0;
  for (int z = 0; z < p->Z; ++z)
    for (int y = 0; y < p->Y; ++y)
      for (int x = 0; x < p->X; ++x)
        if (vb[vox_id(p, z, y, x)] >= 0) ++cnt[((z / p->bz) * nby + y / p->by) * nbx + x / p->bx];
}

/* Axial mode: cos and sin of c * theta_j for every axis, coordinate value and
 * pair j: tab[((axis_offset + c) * (da/2) + j) * 2 + {0,1}], axis offsets 0, Z,
 * Z+Y.  Packed mode: cos and sin of p * theta_j for every packed position p < N
 * and pair j < d/2: tab[(p * (d/2) + j) * 2 + {0,1}]. */
static double* rope_table(const orc_params* p) {
  if (p->rope_mode == 1) {
    size_t N = ntok(p);
    int half = p->d / 2;
    double* tab = (double*)malloc(N * half * 2 * sizeof(double));
    if (!tab) return NULL;
    for (size_t pos = 0; pos < N; ++pos)
      for (int j = 0; j < half; ++j) {
        double theta = pow(p->base, -2.0 * j / (double)p->d);
        tab[(pos * half + j) * 2 + 0] = cos((double)pos * theta);
        tab[(pos * half + j) * 2 + 1] = sin((double)pos * theta);
      }
    return tab;
  }
  int da = p->d / 3, half = da / 2;
  int ext[3] = {p->Z, p->Y, p->X};
  size_t rows = (size_t)p->Z + p->Y + p->X;
  double* tab = (double*)malloc(rows * half * 2 * sizeof(double));
  if (!tab) return NULL;
  size_t r = 0;
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < ext[a]; ++c, ++r)
      for (int j = 0; j < half; ++j) {
        double theta = pow(p->base, -2.0 * j / (double)da);
        tab[(r * half + j) * 2 + 0] = cos((double)c * theta);
        tab[(r * half + j) * 2 + 1] = sin((double)c * theta);
      }
  return tab;
}

/* out = R in (transpose = 0) or R^T in (transpose = 1), R the rotation of the
 * token with grid coordinate c and packed position pos. */
static void rope_apply(const orc_params* p, const double* tab, const double* in,
                       const int c[3], size_t pos, int transpose, double* out) {
  if (p->rope_mode == 1) {
    int half = p->d / 2;
    const double* t = tab + pos * half * 2;
    for (int j = 0; j < half; ++j) {
      double x1 = in[j], x2 = in[j + half];
      double cs = t[2 * j], sn = transpose ? -t[2 * j + 1] : t[2 * j + 1];
      out[j] = x1 * cs - x2 * sn;
      out[j + half] = x1 * sn + x2 * cs;
    }
    return;
  }
  int da = p->d / 3, half = da / 2;
  int off[3] = {0, p->Z, p->Z + p->Y};
  for (int a = 0; a < 3; ++a) {
    const double* t = tab + (size_t)(off[a] + c[a]) * half * 2;
    for (int j = 0; j < half; ++j) {
      double x1 = in[a * da + j], x2 = in[a * da + j + half];
      double cs = t[2 * j], sn = transpose ? -t[2 * j + 1] : t[2 * j + 1];
      out[a * da + j] = x1 * cs - x2 * sn;
      out[a * da + j + half] = x1 * sn + x2 * cs;
    }
  }
}

static void load_row(const void* base, int dtype, const orc_params* p, int b, size_t i, int h,
                     double* row) {
  size_t o = (((size_t)b * ntok(p) + i) * p->H + h) * p->d;
  for (int c = 0; c < p->d; ++c) row[c] = widen(base, dtype, o + c);
}

static void coord_of(const int16_t* coords, const orc_params* p, int b, size_t i, int c[3]) {
  const int16_t* t = coords + ((size_t)b * ntok(p) + i) * 3;
  c[0] = t[0];
  c[1] = t[1];
  c[2] = t[2];
}

/* ---- coordinate volume ------------------------------------------------ */

/* vol[b][voxel] = packed index of the token at that voxel, -1 where empty.
 * No voxel may hold two tokens (with n_tokens = 0 there are Z*Y*X tokens, so
 * every voxel holds exactly one). */
int oracle_volume(const orc_params* p, const int16_t* coords, int32_t* vol) {
  if (check_params(p)) return ORC_ERR_ARG;
  size_t N = nvox(p), NT = ntok(p);
  for (int b = 0; b < p->B; ++b) {
    int32_t* vb = vol + (size_t)b * N;
    for (size_t v = 0; v < N; ++v) vb[v] = -1;
    for (size_t i = 0; i < NT; ++i) {
      int c[3];
      coord_of(coords, p, b, i, c);
      if (c[0] < 0 || c[0] >= p->Z || c[1] < 0 || c[1] >= p->Y || c[2] < 0 || c[2] >= p->X)
        return ORC_ERR_COORDS;
      size_t v = vox_id(p, c[0], c[1], c[2]);
      if (vb[v] != -1) return ORC_ERR_COORDS;
      vb[v] = (int32_t)i;
    }
  }
  return ORC_OK;
}

/* ---- index: tile permutation and halo lists --------------------------- */

/* Query tiles are tz x ty x tx boxes in raster order (the last ones along an
 * axis may be cut by the volume edge).  perm lists, tile by tile and in raster
 * order inside a tile, the packed index of each token; tile_off[b][t] is where
 * tile t starts.  The halo of tile t is the tile box widened by r per axis and
 * clipped to the volume; nbr lists what the coordinate volume holds at each of
 * its voxels (a packed index, or -1 for an empty voxel of a partly occupied
 * volume), in raster order, starting at nbr_off[b][t] within batch item b's
 * list (the lists of item b start at b * nbr_off[0][nT]).  In a partly
 * occupied volume perm lists only the tokens present, so a tile's stretch of
 * perm is as long as the tokens it holds. */
int oracle_build_index(const orc_params* p, const int16_t* coords, int tz, int ty, int tx,
                       int32_t* vol, int32_t* perm, int32_t* tile_off, int64_t* nbr_off,
                       int32_t* nbr) {
  int rc = oracle_volume(p, coords, vol);
  if (rc) return rc;
  if (tz < 1 || ty < 1 || tx < 1) return ORC_ERR_ARG;
  int nTz = (p->Z + tz - 1) / tz, nTy = (p->Y + ty - 1) / ty, nTx = (p->X + tx - 1) / tx;
  int nT = nTz * nTy * nTx;
  int rz = (p->wz - 1) / 2, ry = (p->wy - 1) / 2, rx = (p->wx - 1) / 2;
  size_t V = nvox(p), N = ntok(p);
  int64_t per_item = 0; /* halo list length of one batch item (geometry only) */
  for (int b = 0; b < p->B; ++b) {
    const int32_t* vb = vol + (size_t)b * V;
    int32_t* pb = perm + (size_t)b * N;
    int32_t* tob = tile_off + (size_t)b * (nT + 1);
    int64_t* nob = nbr_off + (size_t)b * (nT + 1);
    int32_t* nbb = nbr ? nbr + (size_t)b * per_item : NULL;
    int64_t nfill = nob[0] = 0;
    int32_t fill = 0;
    int t = 0;
    for (int Tz = 0; Tz < nTz; ++Tz)
      for (int Ty = 0; Ty < nTy; ++Ty)
        for (int Tx = 0; Tx < nTx; ++Tx, ++t) {
          int z0 = Tz * tz, y0 = Ty * ty, x0 = Tx * tx;
          int z1 = z0 + tz < p->Z ? z0 + tz : p->Z;
          int y1 = y0 + ty < p->Y ? y0 + ty : p->Y;
          int x1 = x0 + tx < p->X ? x0 + tx : p->X;
          tob[t] = fill;
          for (int z = z0; z < z1; ++z)
            for (int y = y0; y < y1; ++y)
              for (int x = x0; x < x1; ++x)
                if (vb[vox_id(p, z, y, x)] >= 0) pb[fill++] = vb[vox_id(p, z, y, x)];
          int hz0 = z0 - rz < 0 ? 0 : z0 - rz, hz1 = z1 + rz < p->Z ? z1 + rz : p->Z;
          int hy0 = y0 - ry < 0 ? 0 : y0 - ry, hy1 = y1 + ry < p->Y ? y1 + ry : p->Y;
          int hx0 = x0 - rx < 0 ? 0 : x0 - rx, hx1 = x1 + rx < p->X ? x1 + rx : p->X;
          nob[t] = nfill;
          for (int z = hz0; z < hz1; ++z)
            for (int y = hy0; y < hy1; ++y)
              for (int x = hx0; x < hx1; ++x) {
                if (nbb) nbb[nfill] = vb[vox_id(p, z, y, x)];
                ++nfill;
              }
        }
    tob[nT] = fill;
    nob[nT] = nfill;
    per_item = nfill;
  }
  return ORC_OK;
}

/* ---- rotation (exported for the property tests) ----------------------- */

/* out[B][N][H][d] = R(c_i) x_i (transpose = 0) or R(c_i)^T x_i. */
int oracle_rope(const orc_params* p, const int16_t* coords, const void* x, int dtype,
                int transpose, double* out) {
  if (check_params(p)) return ORC_ERR_ARG;
  double* tab = rope_table(p);
  if (!tab) return ORC_ERR_MEM;
  size_t N = ntok(p);
  double* row = (double*)malloc(sizeof(double) * p->d);
  for (int b = 0; b < p->B; ++b)
    for (size_t i = 0; i < N; ++i) {
      int c[3];
      coord_of(coords, p, b, i, c);
      for (int h = 0; h < p->H; ++h) {
        load_row(x, dtype, p, b, i, h, row);
        rope_apply(p, tab, row, c, i, transpose, out + (((size_t)b * N + i) * p->H + h) * p->d);
      }
    }
  free(row);
  free(tab);
  return ORC_OK;
}

/* ---- block summaries -------------------------------------------------- */

static void summaries_bh(const orc_params* p, const double* tab, const int32_t* vb,
                         const int16_t* coords, const void* k, const void* v, int dtype, int b,
                         int h, double* ks, double* vs) {
  int nby = nb_axis(p->Y, p->by), nbx = nb_axis(p->X, p->bx);
  int nb = nblocks(p), d = p->d;
  double* row = (double*)malloc(sizeof(double) * d);
  double* rot = (double*)malloc(sizeof(double) * d);
  for (int B = 0; B < nb; ++B) {
    int Bz = B / (nby * nbx), By = (B / nbx) % nby, Bx = B % nbx;
    double* kd = ks + (size_t)B * d;
    double* vd = vs + (size_t)B * d;
    double cnt = 0.0;
    for (int c = 0; c < d; ++c) kd[c] = vd[c] = 0.0;
    for (int z = Bz * p->bz; z < (Bz + 1) * p->bz && z < p->Z; ++z)
      for (int y = By * p->by; y < (By + 1) * p->by && y < p->Y; ++y)
        for (int x = Bx * p->bx; x < (Bx + 1) * p->bx && x < p->X; ++x) {
          if (vb[vox_id(p, z, y, x)] < 0) continue;
          size_t j = (size_t)vb[vox_id(p, z, y, x)];
          cnt += 1.0;
          int cj[3];
          coord_of(coords, p, b, j, cj);
          load_row(k, dtype, p, b, j, h, row);
          rope_apply(p, tab, row, cj, j, 0, rot);
          for (int c = 0; c < d; ++c) kd[c] += rot[c];
          load_row(v, dtype, p, b, j, h, row);
          for (int c = 0; c < d; ++c) vd[c] += row[c];
        }
    if (cnt > 0.0) /* an empty block keeps zero means and gets no summary term */
      for (int c = 0; c < d; ++c) {
        kd[c] /= cnt;
        vd[c] /= cnt;
      }
  }
  free(row);
  free(rot);
}

/* ksum, vsum: [B][H][nb][d]. */
int oracle_block_summaries(const orc_params* p, const int16_t* coords, const void* k,
                           const void* v, int dtype, double* ksum, double* vsum) {
  if (check_params(p)) return ORC_ERR_ARG;
  size_t N = nvox(p);
  int32_t* vol = (int32_t*)malloc(sizeof(int32_t) * N * p->B);
  double* tab = rope_table(p);
  if (!vol || !tab) return ORC_ERR_MEM;
  int rc = oracle_volume(p, coords, vol);
  if (rc) {
    free(vol);
    free(tab);
    return rc;
  }
  size_t per = (size_t)nblocks(p) * p->d;
  int BH = p->B * p->H;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int b = bh / p->H, h = bh % p->H;
    summaries_bh(p, tab, vol + (size_t)b * N, coords, k, v, dtype, b, h, ksum + bh * per,
                 vsum + bh * per);
  }
  free(vol);
  free(tab);
  return ORC_OK;
}

/* ---- forward ------------------------------------------------------------ */

/* Whether block B (block coordinates Bc) intersects the window box of a query
 * at coordinate c: the intervals must overlap on every axis. */
static int block_meets_window(const orc_params* p, const int Bc[3], const int c[3]) {
  int w[3] = {p->wz, p->wy, p->wx}, bs[3] = {p->bz, p->by, p->bx};
  for (int a = 0; a < 3; ++a) {
    int r = (w[a] - 1) / 2;
    int lo = Bc[a] * bs[a], hi = lo + bs[a] - 1;
    if (hi < c[a] - r || lo > c[a] + r) return 0;
  }
  return 1;
}

typedef struct {
  double* qrot; /* d */
  double* row;  /* d */
  double* krot; /* d */
  double* logit;
  int64_t* src; /* >= 0: key token; < 0: -(block+1) */
} orc_scratch;

/* Logits of one query (grid-order list), returns how many. */
static int query_logits(const orc_params* p, const double* tab, const int32_t* vb,
                        const int32_t* bcnt, const int16_t* coords, const void* q,
                        const void* k, int dtype, const double* ks, int b, int h, size_t i,
                        int window_only, orc_scratch* s) {
  int d = p->d;
  double tau = tau_of(p);
  int c[3];
  coord_of(coords, p, b, i, c);
  load_row(q, dtype, p, b, i, h, s->row);
  rope_apply(p, tab, s->row, c, i, 0, s->qrot);
  int rz = (p->wz - 1) / 2, ry = (p->wy - 1) / 2, rx = (p->wx - 1) / 2;
  int n = 0;
  for (int z = c[0] - rz; z <= c[0] + rz; ++z) {
    if (z < 0 || z >= p->Z) continue;
    for (int y = c[1] - ry; y <= c[1] + ry; ++y) {
      if (y < 0 || y >= p->Y) continue;
      for (int x = c[2] - rx; x <= c[2] + rx; ++x) {
        if (x < 0 || x >= p->X || vb[vox_id(p, z, y, x)] < 0) continue;
        size_t j = (size_t)vb[vox_id(p, z, y, x)];
        int cj[3] = {z, y, x};
        load_row(k, dtype, p, b, j, h, s->row);
        rope_apply(p, tab, s->row, cj, j, 0, s->krot);
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += s->qrot[e] * s->krot[e];
        s->logit[n] = tau * acc;
        s->src[n] = (int64_t)j;
        ++n;
      }
    }
  }
  if (!window_only) {
    int nby = nb_axis(p->Y, p->by), nbx = nb_axis(p->X, p->bx), nb = nblocks(p);
    for (int B = 0; B < nb; ++B) {
      int Bc[3] = {B / (nby * nbx), (B / nbx) % nby, B % nbx};
      if (bcnt[B] == 0 || block_meets_window(p, Bc, c)) continue;
      const double* kb = ks + (size_t)B * d;
      double acc = 0.0;
      for (int e = 0; e < d; ++e) acc += s->qrot[e] * kb[e];
      s->logit[n] = tau * acc;
      s->src[n] = -(int64_t)(B + 1);
      ++n;
    }
  }
  return n;
}

static int max_terms(const orc_params* p) {
  return p->wz * p->wy * p->wx + nblocks(p);
}

static void scratch_alloc(const orc_params* p, orc_scratch* s) {
  int d = p->d, m = max_terms(p);
  s->qrot = (double*)malloc(sizeof(double) * d);
  s->row = (double*)malloc(sizeof(double) * d);
  s->krot = (double*)malloc(sizeof(double) * d);
  s->logit = (double*)malloc(sizeof(double) * m);
  s->src = (int64_t*)malloc(sizeof(int64_t) * m);
}

static void scratch_free(orc_scratch* s) {
  free(s->qrot);
  free(s->row);
  free(s->krot);
  free(s->logit);
  free(s->src);
}

/* Forward for a list of queries.  sel[n] = (b * H + h) * N + i names query token
 * i (packed index) of batch item b, head h; out is [nsel][d] and lse [nsel].
 * ksum, vsum: summaries [B][H][nb][d] (ignored when window_only). */
int oracle_forward(const orc_params* p, const int16_t* coords, const void* q, const void* k,
                   const void* v, int dtype, const double* ksum, const double* vsum,
                   int window_only, const int64_t* sel, int64_t nsel, double* out,
                   double* lse) {
  if (check_params(p)) return ORC_ERR_ARG;
  size_t N = nvox(p);
  int32_t* vol = (int32_t*)malloc(sizeof(int32_t) * N * p->B);
  double* tab = rope_table(p);
  if (!vol || !tab) return ORC_ERR_MEM;
  int rc = oracle_volume(p, coords, vol);
  if (rc) {
    free(vol);
    free(tab);
    return rc;
  }
  size_t per = (size_t)nblocks(p) * p->d, NT = ntok(p);
  int d = p->d, nb = nblocks(p);
  int32_t* bcnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)nb * p->B);
  if (!bcnt) {
    free(vol);
    free(tab);
    return ORC_ERR_MEM;
  }
  for (int b = 0; b < p->B; ++b) block_members(p, vol + (size_t)b * N, bcnt + (size_t)b * nb);
#pragma omp parallel
  {
    orc_scratch s;
    scratch_alloc(p, &s);
    double* row = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 64)
    for (int64_t n = 0; n < nsel; ++n) {
      int64_t f = sel[n];
      size_t i = (size_t)(f % (int64_t)NT);
      int bh = (int)(f / (int64_t)NT), b = bh / p->H, h = bh % p->H;
      const double* ks = window_only ? NULL : ksum + bh * per;
      const double* vs = window_only ? NULL : vsum + bh * per;
      int nt = query_logits(p, tab, vol + (size_t)b * N, bcnt + (size_t)b * nb, coords, q, k,
                            dtype, ks, b, h, i, window_only, &s);
      double m = -INFINITY;
      for (int t = 0; t < nt; ++t)
        if (s.logit[t] > m) m = s.logit[t];
      double l = 0.0;
      double* o = out + n * d;
      for (int e = 0; e < d; ++e) o[e] = 0.0;
      for (int t = 0; t < nt; ++t) {
        double w = exp(s.logit[t] - m);
        l += w;
        if (s.src[t] >= 0) {
          load_row(v, dtype, p, b, (size_t)s.src[t], h, row);
          for (int e = 0; e < d; ++e) o[e] += w * row[e];
        } else {
          const double* vb = vs + (size_t)(-s.src[t] - 1) * d;
          for (int e = 0; e < d; ++e) o[e] += w * vb[e];
        }
      }
      for (int e = 0; e < d; ++e) o[e] /= l;
      lse[n] = m + log(l);
    }
    free(row);
    scratch_free(&s);
  }
  free(bcnt);
  free(vol);
  free(tab);
  return ORC_OK;
}

/* ---- backward ----------------------------------------------------------- */

/* Gradients of sum(dout * out) with respect to q, k, v for the full operator
 * (or the window-only operator), all queries.  dq, dk, dv: [B][N][H][d] fp64,
 * packed order.  The gradient reaches k and v through the local terms and
 * through the block means: every token of block B receives dkbar_B / |B| (and
 * dvbar_B / |B|), rotated back by R(c_j)^T for k. */
int oracle_backward(const orc_params* p, const int16_t* coords, const void* q, const void* k,
                    const void* v, const void* dout, int dtype, int window_only, double* dq,
                    double* dk, double* dv) {
  if (check_params(p)) return ORC_ERR_ARG;
  size_t N = nvox(p);
  int d = p->d, nb = nblocks(p);
  int32_t* vol = (int32_t*)malloc(sizeof(int32_t) * N * p->B);
  double* tab = rope_table(p);
  if (!vol || !tab) return ORC_ERR_MEM;
  int rc = oracle_volume(p, coords, vol);
  if (rc) {
    free(vol);
    free(tab);
    return rc;
  }
  double tau = tau_of(p);
  int nby = nb_axis(p->Y, p->by), nbx = nb_axis(p->X, p->bx);
  size_t NT = ntok(p);
  int BH = p->B * p->H;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int b = bh / p->H, h = bh % p->H;
    const int32_t* vb = vol + (size_t)b * N;
    int32_t* bcnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)nb);
    block_members(p, vb, bcnt);
    double* ks = (double*)calloc((size_t)nb * d, sizeof(double));
    double* vs = (double*)calloc((size_t)nb * d, sizeof(double));
    double* dks = (double*)calloc((size_t)nb * d, sizeof(double));
    double* dvs = (double*)calloc((size_t)nb * d, sizeof(double));
    double* dkrot = (double*)calloc(NT * d, sizeof(double)); /* d/dk~ in packed order */
    double* dvacc = (double*)calloc(NT * d, sizeof(double));
    double* dO = (double*)malloc(sizeof(double) * d);
    double* vrow = (double*)malloc(sizeof(double) * d);
    double* dqr = (double*)malloc(sizeof(double) * d);
    double* tmp = (double*)malloc(sizeof(double) * d);
    orc_scratch s;
    scratch_alloc(p, &s);
    double* P = (double*)malloc(sizeof(double) * max_terms(p));
    double* dP = (double*)malloc(sizeof(double) * max_terms(p));
    if (!window_only) summaries_bh(p, tab, vb, coords, k, v, dtype, b, h, ks, vs);
    for (int z = 0; z < p->Z; ++z)
      for (int y = 0; y < p->Y; ++y)
        for (int x = 0; x < p->X; ++x) {
          if (vb[vox_id(p, z, y, x)] < 0) continue;
          size_t i = (size_t)vb[vox_id(p, z, y, x)];
          int nt = query_logits(p, tab, vb, bcnt, coords, q, k, dtype, ks, b, h, i, window_only,
                                &s);
          double m = -INFINITY;
          for (int t = 0; t < nt; ++t)
            if (s.logit[t] > m) m = s.logit[t];
          double l = 0.0;
          for (int t = 0; t < nt; ++t) l += exp(s.logit[t] - m);
          double lse_i = m + log(l);
          load_row(dout, dtype, p, b, i, h, dO);
          double D = 0.0;
          for (int t = 0; t < nt; ++t) {
            P[t] = exp(s.logit[t] - lse_i);
            const double* vv;
            if (s.src[t] >= 0) {
              load_row(v, dtype, p, b, (size_t)s.src[t], h, vrow);
              vv = vrow;
            } else {
              vv = vs + (size_t)(-s.src[t] - 1) * d;
            }
            double acc = 0.0;
            for (int e = 0; e < d; ++e) acc += dO[e] * vv[e];
            dP[t] = acc;
            D += P[t] * acc;
          }
          for (int e = 0; e < d; ++e) dqr[e] = 0.0;
          for (int t = 0; t < nt; ++t) {
            double dS = P[t] * (dP[t] - D);
            if (s.src[t] >= 0) {
              size_t j = (size_t)s.src[t];
              int cj[3];
              coord_of(coords, p, b, j, cj);
              load_row(k, dtype, p, b, j, h, s.row);
              rope_apply(p, tab, s.row, cj, j, 0, s.krot);
              for (int e = 0; e < d; ++e) {
                dqr[e] += tau * dS * s.krot[e];
                dkrot[j * d + e] += tau * dS * s.qrot[e];
                dvacc[j * d + e] += P[t] * dO[e];
              }
            } else {
              size_t B = (size_t)(-s.src[t] - 1);
              for (int e = 0; e < d; ++e) {
                dqr[e] += tau * dS * ks[B * d + e];
                dks[B * d + e] += tau * dS * s.qrot[e];
                dvs[B * d + e] += P[t] * dO[e];
              }
            }
          }
          int ci[3] = {z, y, x};
          rope_apply(p, tab, dqr, ci, i, 1, dq + (((size_t)b * NT + i) * p->H + h) * d);
        }
    /* Spread the summary gradients over the block members, rotate back. */
    for (int z = 0; z < p->Z; ++z)
      for (int y = 0; y < p->Y; ++y)
        for (int x = 0; x < p->X; ++x) {
          if (vb[vox_id(p, z, y, x)] < 0) continue;
          size_t j = (size_t)vb[vox_id(p, z, y, x)];
          if (!window_only) {
            size_t B = ((size_t)(z / p->bz) * nby + (size_t)(y / p->by)) * nbx + (x / p->bx);
            double cnt = (double)bcnt[B];
            for (int e = 0; e < d; ++e) {
              dkrot[j * d + e] += dks[B * d + e] / cnt;
              dvacc[j * d + e] += dvs[B * d + e] / cnt;
            }
          }
          int cj[3] = {z, y, x};
          for (int e = 0; e < d; ++e) tmp[e] = dkrot[j * d + e];
          rope_apply(p, tab, tmp, cj, j, 1, dk + (((size_t)b * NT + j) * p->H + h) * d);
          for (int e = 0; e < d; ++e) dv[(((size_t)b * NT + j) * p->H + h) * d + e] = dvacc[j * d + e];
        }
    free(bcnt);
    free(P);
    free(dP);
    scratch_free(&s);
    free(ks);
    free(vs);
    free(dks);
    free(dvs);
    free(dkrot);
    free(dvacc);
    free(dO);
    free(vrow);
    free(dqr);
    free(tmp);
  }
  free(vol);
  free(tab);
  return ORC_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
