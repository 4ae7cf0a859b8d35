/*
 * CPU oracle for one 3D Gaussian Splatting training step -- TEST
 * INFRASTRUCTURE ONLY.  Nothing on the product path includes, links or
 * calls this code; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code with the CUDA library.
 *
 * Everything is computed in fp64 from fp64 inputs (the fp32 scene values,
 * promoted exactly), in the plain order the stage definitions give:
 * cull + EWA projection, per-tile lists sorted by (depth bits, index),
 * front-to-back compositing, the reverse blend, projection backward, Leaf
 * partition.  See gs_oracle.cpp for the citation of each stage.
 *
 * Camera array (16 doubles): R[9] (world->camera, row-major), t[3],
 * fx, fy, cx, cy.
 *
 * Record array (OR_REC doubles per Gaussian), indices below.
 */
#ifndef GS_ORACLE_H
#define GS_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  OR_U = 0, OR_V = 1, OR_DEPTH = 2, OR_RADIUS = 3,
  OR_A = 4, OR_B = 5, OR_C = 6, OR_OPAC = 7,
  OR_R = 8, OR_G = 9, OR_BL = 10,
  OR_S00 = 11, OR_S01 = 12, OR_S11 = 13,
  OR_SQUARE = 14,  /* tiles of the plain 3-sigma square (clamped) */
  OR_REC = 16
};

/* projection flags (per Gaussian) */
enum { OR_F_RADIUS_NEAR = 1, OR_F_CLAMP_NEAR = 2, OR_F_NONFINITE = 4 };
/* pixel flags */
enum { OR_P_NEAR = 1, OR_P_INVALID = 0x80 };

int32_t or_version(void);
int32_t or_num_threads(void);

/* Cull + project every Gaussian.  params: [P][n_pad] fp64, P = 11+3(D+1)^2.
 * Outputs per Gaussian i < n: is_cand, rec[i*OR_REC..], rect[i*4..]
 * (x0,y0,x1,y1 half-open tiles), depth_key (bits of fp32(t_z)), flags.
 * Returns the number of candidates. */
int64_t or_project(const double* params, int64_t n, int64_t n_pad, int32_t D,
                   const double* cam, int32_t W, int32_t H, uint8_t* is_cand,
                   double* rec, int32_t* rect, uint32_t* depth_key,
                   uint8_t* flags);

/* The same with the rect chosen by `tight`: 1 = the tiles of the 3-sigma
 * square whose pixel-centre box meets the inflated alpha >= 1/255 box (and
 * Gaussians that cannot reach 1/255 culled), as or_project; 0 = the plain
 * closed 3-sigma square clamped to the grid. */
int64_t or_project_rects(const double* params, int64_t n, int64_t n_pad,
                         int32_t D, const double* cam, int32_t W, int32_t H,
                         int32_t tight, uint8_t* is_cand, double* rec,
                         int32_t* rect, uint32_t* depth_key, uint8_t* flags);

/* Real SH basis (degree <= 3, 16 values) and its gradient (16 x 3) at a unit
 * direction d. */
void or_sh_basis(const double* d, double* Y, double* dY);

/* Per-tile lists by brute force: for each requested tile, every candidate
 * whose rect contains it, ordered by (key, candidate position).  rect/key
 * are per candidate (C entries).  offsets: n_tiles+1.  vals may be NULL
 * (count only).  Returns the total count. */
int64_t or_tile_lists_scan(int64_t C, const int32_t* rect, const uint32_t* key,
                           int32_t TW, const int32_t* tiles, int64_t n_tiles,
                           int64_t* offsets, int32_t* vals);

/* Same lists for ALL tiles of the grid by scattering each candidate into
 * the tiles of its rect, then a stable sort per tile. */
int64_t or_tile_lists_scatter(int64_t C, const int32_t* rect,
                              const uint32_t* key, int32_t TW, int32_t TH,
                              int64_t* offsets, int32_t* vals);

/* Front-to-back compositing of requested tiles.  Per tile k outputs are
 * compact: img[k][3][256], T_final[k][256], last[k][256], pflags[k][256],
 * n_eval[k][256] (list entries visited), sig[k][256] (hash of every
 * discrete decision taken for the pixel), T_err[k][256] (optional: bound of
 * the relative error of an fp32 evaluation of T_final). */
int32_t or_raster_fwd(int64_t C, const double* rec, int32_t TW, int32_t W,
                      int32_t H, const int32_t* tiles, int64_t n_tiles,
                      const int64_t* offsets, const int32_t* vals, double* img,
                      double* T_final, int32_t* last, uint8_t* pflags,
                      int32_t* n_eval, uint64_t* sig, double* T_err);

/* Reverse blend: accumulates dL/d{u,v,a,b,c,o,R,G,B} per candidate into
 * g2d[C][9] given dL/dpixel[k][3][256] for the requested tiles. */
int32_t or_raster_bwd(int64_t C, const double* rec, int32_t TW, int32_t W,
                      int32_t H, const int32_t* tiles, int64_t n_tiles,
                      const int64_t* offsets, const int32_t* vals,
                      const double* dL_dpix, double* g2d);

/* Projection backward for the C candidates cand_idx[] given g2d[C][9];
 * writes g3d[P][C]. */
int32_t or_project_bwd(const double* params, int64_t n_pad, int32_t D,
                       const double* cam, int64_t C, const int32_t* cand_idx,
                       const double* g2d, double* g3d);

/* Recursive Leaf partition of the tile grid.  sat: (TH+1)x(TW+1) summed-area
 * table of per-tile intersection counts.  lm: {bytes_per_isect,
 * bytes_per_pixel, bytes_per_tile, fixed_bytes, align}.  Returns the number
 * of Leaves (or -1 if max_leaves is too small). */
int32_t or_leaf_partition(const int64_t* sat, int32_t TW, int32_t TH,
                          int32_t W, int32_t H, const int64_t* lm,
                          int64_t budget, int32_t* leaves, int64_t* leaf_isect,
                          int64_t* leaf_bytes, uint8_t* over_budget,
                          int32_t max_leaves);

#ifdef __cplusplus
}
#endif
#endif
