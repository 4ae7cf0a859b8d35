"""CPU oracle for one 3DGS training step -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this module.  It loads ``liboracle.so`` (plain fp64
C++, ``gs_oracle.cpp``) through ctypes and composes the step from it; the L1
loss and Adam, which are one line of elementwise arithmetic each, are
written here in numpy (fp64).  It imports nothing from the CUDA package.

Stages and their sources (page title, section):

* cull + EWA projection, SH colour          -- SkipGS paper notes, "loss
  function / training strategy" (gradients through the projected 2D
  covariance to means, quaternions, scales, opacities, SH); constants are
  readings (0.3 px^2 low-pass, 3-sigma radius, near 0.2, guard band 1.3).
* per-tile lists ordered by (depth, index)  -- the sort that the tile
  rasteriser's duplicated tile|depth keys realise; the oracle states it
  as its plain definition and uses std::stable_sort.
* compositing, reverse blend                 -- SkipGS notes, "loss
  function" (transmittance accumulation) and "key design 2" (backward:
  gradient back-propagation, atomic accumulation).
* L1 loss over the whole view                -- BoundedGS, section 01: every
  Leaf keeps full-view supervision; the normaliser is the full image.
* composite loss (1 - lambda) L1 + lambda (1 - SSIM), lambda = 0.2
                                             -- SkipGS notes, "loss function
  / training strategy".  SSIM is the structural similarity index of Wang,
  Bovik, Sheikh and Simoncelli (IEEE TIP 2004) with its Gaussian window
  (11 x 11, sigma 1.5) and constants C1 = (0.01)^2, C2 = (0.03)^2 for a
  data range of 1 (readings: the pages name SSIM only).  Windows are
  local to each Leaf's pixel rectangle, zero outside it (BoundedGS,
  section 02: local SSIM windows differ from full-image ones at the
  boundary); one Leaf covering the view is the full-image SSIM.
* Leaf partition                             -- BoundedGS, section 01 (load
  from overlaps, pixels and buffer layout) and section 02, B -> C (split
  over-budget regions again).
* one Adam update per view                   -- BoundedGS, section 01 (sum
  the gradients of the whole view, then update once).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "gs_oracle.cpp")
TILE = 16

REC = 16
U, V, DEPTH, RADIUS, A, B, Cc, OPAC, RED, GREEN, BLUE = range(11)
P_NEAR, P_INVALID = 1, 0x80

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with g++ (OpenMP, no FP contraction)."""
    if force or not os.path.exists(LIB_PATH) or \
            os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC):
        tmp = LIB_PATH + ".tmp"
        subprocess.check_call(["g++", "-O2", "-fopenmp", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, SRC])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB_PATH)
        p = C.c_void_p
        i64, i32 = C.c_int64, C.c_int32
        L.or_project.restype = i64
        L.or_project.argtypes = [p, i64, i64, i32, p, i32, i32, p, p, p, p, p]
        L.or_project_rects.restype = i64
        L.or_project_rects.argtypes = [p, i64, i64, i32, p, i32, i32, i32, p,
                                       p, p, p, p]
        L.or_sh_basis.argtypes = [p, p, p]
        L.or_tile_lists_scan.restype = i64
        L.or_tile_lists_scan.argtypes = [i64, p, p, i32, p, i64, p, p]
        L.or_tile_lists_scatter.restype = i64
        L.or_tile_lists_scatter.argtypes = [i64, p, p, i32, i32, p, p]
        L.or_raster_fwd.argtypes = [i64, p, i32, i32, i32, p, i64, p, p,
                                    p, p, p, p, p, p, p]
        L.or_raster_bwd.argtypes = [i64, p, i32, i32, i32, p, i64, p, p, p, p]
        L.or_project_bwd.argtypes = [p, i64, i32, p, i64, p, p, p]
        L.or_leaf_partition.restype = i32
        L.or_leaf_partition.argtypes = [p, i32, i32, i32, i32, p, i64, p, p,
                                        p, p, i32]
        L.or_num_threads.restype = i32
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def num_threads() -> int:
    return int(lib().or_num_threads())


def cam_array(cam) -> np.ndarray:
    a = np.zeros(16, np.float64)
    a[0:9] = np.asarray(cam.R, np.float32).reshape(-1)
    a[9:12] = np.asarray(cam.t, np.float32).reshape(-1)
    a[12:16] = np.float32([cam.fx, cam.fy, cam.cx, cam.cy])
    return a


def grid(cam):
    return (cam.width + TILE - 1) // TILE, (cam.height + TILE - 1) // TILE


# ---------------------------------------------------------------------------
# stage wrappers
# ---------------------------------------------------------------------------

def project(params: np.ndarray, n: int, sh_degree: int, cam, tight=True):
    """Cull + project all Gaussians.  Returns per-Gaussian arrays and the
    candidate view (ascending Gaussian index).  `tight` selects the tile
    rect: the tiles of the 3-sigma square that meet the alpha >= 1/255 box
    (the binning the library uses), or with False the plain closed 3-sigma
    square, in which case a Gaussian that can never reach 1/255 is still a
    candidate."""
    par = np.ascontiguousarray(params, np.float64)
    n_pad = par.shape[1]
    is_c = np.zeros(n, np.uint8)
    rec = np.zeros((n, REC), np.float64)
    rect = np.zeros((n, 4), np.int32)
    key = np.zeros(n, np.uint32)
    flags = np.zeros(n, np.uint8)
    ca = cam_array(cam)
    lib().or_project_rects(_p(par), n, n_pad, sh_degree, _p(ca), cam.width,
                           cam.height, 1 if tight else 0, _p(is_c), _p(rec),
                           _p(rect), _p(key), _p(flags))
    cand = np.nonzero(is_c)[0].astype(np.int32)
    return dict(is_cand=is_c.astype(bool), rec_all=rec, rect_all=rect,
                key_all=key, flags_all=flags, cand_idx=cand, rec=rec[cand],
                rect=rect[cand], key=key[cand], flags=flags[cand])


def sh_basis(d):
    d = np.ascontiguousarray(d, np.float64)
    Y = np.zeros(16)
    dY = np.zeros(48)
    lib().or_sh_basis(_p(d), _p(Y), _p(dY))
    return Y, dY.reshape(16, 3)


def tile_lists(rect_c, key_c, TW, tiles):
    """Lists of the requested tiles (brute force over candidates)."""
    rect_c = np.ascontiguousarray(rect_c, np.int32)
    key_c = np.ascontiguousarray(key_c, np.uint32)
    tiles = np.ascontiguousarray(tiles, np.int32)
    off = np.zeros(len(tiles) + 1, np.int64)
    total = lib().or_tile_lists_scan(len(rect_c), _p(rect_c), _p(key_c), TW,
                                     _p(tiles), len(tiles), _p(off), None)
    vals = np.zeros(max(total, 1), np.int32)
    lib().or_tile_lists_scan(len(rect_c), _p(rect_c), _p(key_c), TW, _p(tiles),
                             len(tiles), _p(off), _p(vals))
    return off, vals[:total]


def tile_lists_all(rect_c, key_c, TW, TH):
    """Lists of every tile (scatter + stable sort per tile)."""
    rect_c = np.ascontiguousarray(rect_c, np.int32)
    key_c = np.ascontiguousarray(key_c, np.uint32)
    off = np.zeros(TW * TH + 1, np.int64)
    total = lib().or_tile_lists_scatter(len(rect_c), _p(rect_c), _p(key_c), TW,
                                        TH, _p(off), None)
    vals = np.zeros(max(total, 1), np.int32)
    lib().or_tile_lists_scatter(len(rect_c), _p(rect_c), _p(key_c), TW, TH,
                                _p(off), _p(vals))
    return off, vals[:total]


def raster_fwd(rec_c, TW, W, H, tiles, off, vals):
    rec_c = np.ascontiguousarray(rec_c, np.float64)
    tiles = np.ascontiguousarray(tiles, np.int32)
    k = len(tiles)
    img = np.zeros((k, 3, 256))
    T = np.zeros((k, 256))
    last = np.zeros((k, 256), np.int32)
    fl = np.zeros((k, 256), np.uint8)
    ne = np.zeros((k, 256), np.int32)
    sig = np.zeros((k, 256), np.uint64)
    terr = np.zeros((k, 256))
    vals = np.ascontiguousarray(vals, np.int32)
    if len(vals) == 0:
        vals = np.zeros(1, np.int32)
    lib().or_raster_fwd(len(rec_c), _p(rec_c), TW, W, H, _p(tiles), k,
                        _p(np.ascontiguousarray(off, np.int64)), _p(vals),
                        _p(img), _p(T), _p(last), _p(fl), _p(ne), _p(sig), _p(terr))
    return dict(img=img, T=T, last=last, flags=fl, n_eval=ne, sig=sig, T_err=terr)


def raster_bwd(rec_c, TW, W, H, tiles, off, vals, dL_dpix, g2d=None):
    rec_c = np.ascontiguousarray(rec_c, np.float64)
    if g2d is None:
        g2d = np.zeros((len(rec_c), 9))
    vals = np.ascontiguousarray(vals, np.int32)
    if len(vals) == 0:
        vals = np.zeros(1, np.int32)
    d = np.ascontiguousarray(dL_dpix, np.float64)
    lib().or_raster_bwd(len(rec_c), _p(rec_c), TW, W, H,
                        _p(np.ascontiguousarray(tiles, np.int32)), len(tiles),
                        _p(np.ascontiguousarray(off, np.int64)), _p(vals),
                        _p(d), _p(g2d))
    return g2d


def project_bwd(params, sh_degree, cam, cand_idx, g2d):
    par = np.ascontiguousarray(params, np.float64)
    Cn = len(cand_idx)
    P = par.shape[0]
    g3d = np.zeros((P, max(Cn, 1)))
    lib().or_project_bwd(_p(par), par.shape[1], sh_degree, _p(cam_array(cam)),
                         Cn, _p(np.ascontiguousarray(cand_idx, np.int32)),
                         _p(np.ascontiguousarray(g2d, np.float64)), _p(g3d))
    return g3d[:, :Cn]


def tile_counts(rect_c, TW, TH):
    """Per-tile intersection counts by direct enumeration of rects."""
    cnt = np.zeros((TH, TW), np.int64)
    for x0, y0, x1, y1 in np.asarray(rect_c):
        cnt[y0:y1, x0:x1] += 1
    return cnt


def tile_counts_fast(rect_c, TW, TH):
    """Same counts via the 2D difference grid (used for large scenes)."""
    r = np.asarray(rect_c, np.int64)
    d = np.zeros((TH + 1, TW + 1), np.int64)
    np.add.at(d, (r[:, 1], r[:, 0]), 1)
    np.add.at(d, (r[:, 1], r[:, 2]), -1)
    np.add.at(d, (r[:, 3], r[:, 0]), -1)
    np.add.at(d, (r[:, 3], r[:, 2]), 1)
    return d.cumsum(0).cumsum(1)[:TH, :TW]


def sat(counts):
    """(TH+1) x (TW+1) summed-area table with a zero first row / column."""
    TH, TW = counts.shape
    s = np.zeros((TH + 1, TW + 1), np.int64)
    s[1:, 1:] = counts.cumsum(0).cumsum(1)
    return s


def leaf_partition(sat_tab, TW, TH, W, H, lm, budget, max_leaves=1 << 20):
    s = np.ascontiguousarray(sat_tab, np.int64)
    lm = np.ascontiguousarray(lm, np.int64)
    leaves = np.zeros((max_leaves, 4), np.int32)
    li = np.zeros(max_leaves, np.int64)
    lb = np.zeros(max_leaves, np.int64)
    ov = np.zeros(max_leaves, np.uint8)
    n = lib().or_leaf_partition(_p(s), TW, TH, W, H, _p(lm), int(budget),
                                _p(leaves), _p(li), _p(lb), _p(ov), max_leaves)
    if n < 0:
        raise RuntimeError("too many leaves")
    return leaves[:n].copy(), li[:n].copy(), lb[:n].copy(), ov[:n].astype(bool)


def loss_l1(img, target, norm_count):
    """L = sum |r - t| / norm_count; dL/dr = sign(r - t) / norm_count."""
    d = np.asarray(img, np.float64) - np.asarray(target, np.float64)
    return float(np.abs(d).sum() / norm_count), np.sign(d) / norm_count


SSIM_RADIUS = 5
SSIM_SIGMA = 1.5
SSIM_C1 = 0.01 ** 2
SSIM_C2 = 0.03 ** 2
SSIM_LAMBDA = 0.2


def ssim_window():
    """The 1D factor g of the 11 x 11 Gaussian window w(i, j) = g(i) g(j):
    g(k) proportional to exp(-k^2 / (2 sigma^2)), k = -5..5, sum 1."""
    k = np.arange(-SSIM_RADIUS, SSIM_RADIUS + 1, dtype=np.float64)
    g = np.exp(-k * k / (2.0 * SSIM_SIGMA ** 2))
    return g / g.sum()


def window_sum(img):
    """Gaussian-weighted local sum of a [h][w] plane with zero outside it:
    out[y, x] = sum_{i, j} w(i, j) img[y + i, x + j], i, j = -5..5, written
    out as the 121 shifted, weighted copies of the plane."""
    g = ssim_window()
    R = SSIM_RADIUS
    h, w = img.shape
    pad = np.zeros((h + 2 * R, w + 2 * R))
    pad[R:R + h, R:R + w] = img
    out = np.zeros((h, w))
    for i in range(2 * R + 1):
        for j in range(2 * R + 1):
            out += g[i] * g[j] * pad[i:i + h, j:j + w]
    return out


def ssim_moments(x, y):
    """Local statistics of one channel pair: mu_x, mu_y, sigma_x^2,
    sigma_y^2, sigma_xy (Wang et al. 2004, eq. 14-16 with the Gaussian
    window)."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    mx, my = window_sum(x), window_sum(y)
    sxx = window_sum(x * x) - mx * mx
    syy = window_sum(y * y) - my * my
    sxy = window_sum(x * y) - mx * my
    return mx, my, sxx, syy, sxy


def ssim_map(x, y):
    """Per-pixel SSIM of [C][h][w] images (eq. 13 of Wang et al. with
    C3 = C2 / 2): luminance (2 mu_x mu_y + C1) / (mu_x^2 + mu_y^2 + C1)
    times contrast-structure (2 sigma_xy + C2) / (sigma_x^2 + sigma_y^2 + C2)."""
    out = np.zeros(np.shape(x))
    for c in range(out.shape[0]):
        mx, my, sxx, syy, sxy = ssim_moments(x[c], y[c])
        out[c] = ((2 * mx * my + SSIM_C1) * (2 * sxy + SSIM_C2)) / \
                 ((mx * mx + my * my + SSIM_C1) * (sxx + syy + SSIM_C2))
    return out


def ssim_map_grad(x, y):
    """d (sum of ssim_map(x, y)) / d x for [C][h][w] images.  S at pixel q
    depends on x through the window sums m = W[x], e = W[x^2], f = W[x y];
    with the partials of S in those (sigma_x^2 = e - m^2, sigma_xy =
    f - m mu_y), the chain rule gives
      dS_sum/dx_p = W[dS/dm](p) + 2 x_p W[dS/de](p) + y_p W[dS/df](p)
    (the window is symmetric and zero outside the image, so the transposed
    window sum is the window sum)."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    out = np.zeros(x.shape)
    for c in range(x.shape[0]):
        mx, my, sxx, syy, sxy = ssim_moments(x[c], y[c])
        a = 2 * mx * my + SSIM_C1
        b = 2 * sxy + SSIM_C2
        cc = mx * mx + my * my + SSIM_C1
        d = sxx + syy + SSIM_C2
        S = a * b / (cc * d)
        # total partials of S = a b / (cc d) in (m, e, f)
        dS_dm = S * (2 * my / a - 2 * my / b - 2 * mx / cc + 2 * mx / d)
        dS_de = -S / d
        dS_df = 2 * S / b
        out[c] = window_sum(dS_dm) + 2 * x[c] * window_sum(dS_de) + y[c] * window_sum(dS_df)
    return out


def loss_ssim(img, target, norm_count):
    """SSIM term of one pixel rectangle (windows local to it):
    L = sum (1 - S) / norm_count, and dL/dimg."""
    img = np.asarray(img, np.float64)
    target = np.asarray(target, np.float64)
    S = ssim_map(img, target)
    return float((1.0 - S).sum() / norm_count), -ssim_map_grad(img, target) / norm_count


def adam(p, m, v, g, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, step=1):
    """One Adam step (bias-corrected), fp64; returns new (p, m, v)."""
    p = np.asarray(p, np.float64)
    m = b1 * np.asarray(m, np.float64) + (1 - b1) * g
    v = b2 * np.asarray(v, np.float64) + (1 - b2) * g * g
    mh = m / (1 - b1 ** step)
    vh = v / (1 - b2 ** step)
    return p - lr * mh / (np.sqrt(vh) + eps), m, v


# ---------------------------------------------------------------------------
# composition
# ---------------------------------------------------------------------------

def tiles_of_rect(x0, y0, x1, y1, TW):
    ys, xs = np.mgrid[y0:y1, x0:x1]
    return (ys * TW + xs).reshape(-1).astype(np.int32)


def scatter_tiles(per_tile, tiles, TW, TH, W, H, channels=None):
    """Place compact per-tile pixel data into a full image array."""
    k = len(tiles)
    if channels is None:
        out = np.zeros((TH * 16, TW * 16), per_tile.dtype)
        blk = per_tile.reshape(k, 16, 16)
    else:
        out = np.zeros((channels, TH * 16, TW * 16), per_tile.dtype)
        blk = per_tile.reshape(k, channels, 16, 16)
    for j, t in enumerate(tiles):
        ty, tx = divmod(int(t), TW)
        if channels is None:
            out[ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = blk[j]
        else:
            out[:, ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = blk[j]
    return out[..., :H, :W]


def gather_tiles(img, tiles, TW, channels):
    """Inverse of scatter_tiles for a [3][H][W] image: compact [k][3][256]."""
    Cc_, H, W = img.shape
    TH = (H + 15) // 16
    pad = np.zeros((channels, TH * 16, TW * 16), img.dtype)
    pad[:, :H, :W] = img
    out = np.zeros((len(tiles), channels, 256), img.dtype)
    for j, t in enumerate(tiles):
        ty, tx = divmod(int(t), TW)
        out[j] = pad[:, ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16].reshape(channels, 256)
    return out


def render(params, n, sh_degree, cam):
    """Full-image forward only: image [3][H][W], T, last, flags, proj, lists."""
    pr = project(params, n, sh_degree, cam)
    TW, TH = grid(cam)
    tiles = np.arange(TW * TH, dtype=np.int32)
    off, vals = tile_lists_all(pr["rect"], pr["key"], TW, TH)
    fw = raster_fwd(pr["rec"], TW, cam.width, cam.height, tiles, off, vals)
    img = scatter_tiles(fw["img"], tiles, TW, TH, cam.width, cam.height, 3)
    return dict(img=img, proj=pr, off=off, vals=vals, fwd=fw, tiles=tiles)


def step(params, n, sh_degree, cam, target, leaves=None, m=None, v=None,
         lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, t=1, ssim_lambda=None,
         tight=True):
    """One training step for one view: project, per-Leaf raster forward +
    loss + raster backward (summed over Leaves), projection backward, one
    Adam update.  `leaves` is a list of tile rects; None = whole image.
    The loss is L1, or with `ssim_lambda` the composite
    (1 - lambda) L1 + lambda (1 - SSIM), SSIM over each Leaf's pixel
    rectangle (loss_ssim), both normalised by 3 W H.  `tight` is passed to
    `project`.  Besides the list position `last`, the result holds
    `last_id`: the Gaussian index of each pixel's last composited entry
    (-1 if none), which does not depend on which skipped entries a list
    holds; `n_eval_px`: the list entries each pixel visits (up to and
    including the one it stops at, else its whole list), `list_len`: the
    length of each pixel's tile list."""
    W, H = cam.width, cam.height
    TW, TH = grid(cam)
    pr = project(params, n, sh_degree, cam, tight=tight)
    if leaves is None:
        leaves = [(0, 0, TW, TH)]
    Cn = len(pr["cand_idx"])
    g2d = np.zeros((Cn, 9))
    norm = 3.0 * W * H
    loss = 0.0
    img = np.zeros((3, TH * 16, TW * 16))
    Tfin = np.ones((TH * 16, TW * 16))
    last = np.zeros((TH * 16, TW * 16), np.int32)
    last_id = np.full((TH * 16, TW * 16), -1, np.int64)
    n_eval_px = np.zeros((TH * 16, TW * 16), np.int64)
    list_len = np.zeros((TH * 16, TW * 16), np.int64)
    pflags = np.zeros((TH * 16, TW * 16), np.uint8)
    n_eval = 0
    n_isect = 0
    tpad = np.zeros((3, TH * 16, TW * 16))
    tpad[:, :H, :W] = target
    for (x0, y0, x1, y1) in leaves:
        tiles = tiles_of_rect(x0, y0, x1, y1, TW)
        off, vals = tile_lists(pr["rect"], pr["key"], TW, tiles)
        n_isect += len(vals)
        fw = raster_fwd(pr["rec"], TW, W, H, tiles, off, vals)
        valid = (fw["flags"] & P_INVALID) == 0
        tg = gather_tiles(tpad, tiles, TW, 3)
        d = np.where(valid[:, None, :], fw["img"] - tg, 0.0)
        if ssim_lambda is None:
            loss += float(np.abs(d).sum() / norm)
            dL = np.sign(d) / norm
        else:
            lam = float(ssim_lambda)
            loss += (1.0 - lam) * float(np.abs(d).sum() / norm)
            dL = (1.0 - lam) * np.sign(d) / norm
            # the Leaf's pixel rectangle, clipped to the image
            px0, py0 = x0 * 16, y0 * 16
            px1, py1 = min(x1 * 16, W), min(y1 * 16, H)
            fimg = scatter_tiles(fw["img"], tiles, TW, TH, TW * 16, TH * 16, 3)
            r_img = fimg[:, py0:py1, px0:px1]
            r_tg = tpad[:, py0:py1, px0:px1]
            ls, gs = loss_ssim(r_img, r_tg, norm)
            loss += lam * ls
            gpad = np.zeros((3, TH * 16, TW * 16))
            gpad[:, py0:py1, px0:px1] = lam * gs
            dL = dL + gather_tiles(gpad, tiles, TW, 3)
        raster_bwd(pr["rec"], TW, W, H, tiles, off, vals, dL, g2d)
        n_eval += int(fw["n_eval"][valid].sum())
        for j, tt in enumerate(tiles):
            ty, tx = divmod(int(tt), TW)
            sl = (slice(ty * 16, ty * 16 + 16), slice(tx * 16, tx * 16 + 16))
            img[(slice(None),) + sl] = fw["img"][j].reshape(3, 16, 16)
            Tfin[sl] = fw["T"][j].reshape(16, 16)
            last[sl] = fw["last"][j].reshape(16, 16)
            lj = fw["last"][j].astype(np.int64)
            lid = np.full(256, -1, np.int64)
            hit = lj > 0
            lid[hit] = pr["cand_idx"][vals[off[j] + lj[hit] - 1]]
            last_id[sl] = lid.reshape(16, 16)
            n_eval_px[sl] = fw["n_eval"][j].reshape(16, 16)
            list_len[sl] = off[j + 1] - off[j]
            pflags[sl] = fw["flags"][j].reshape(16, 16)
    g3d = project_bwd(params, sh_degree, cam, pr["cand_idx"], g2d)
    P, n_pad = params.shape
    grad = np.zeros((P, n_pad))
    grad[:, pr["cand_idx"]] = g3d
    if m is None:
        m = np.zeros((P, n_pad))
    if v is None:
        v = np.zeros((P, n_pad))
    p_new, m_new, v_new = adam(params, m, v, grad, lr, b1, b2, eps, t)
    p_new[:, n:] = params[:, n:]
    m_new[:, n:] = 0
    v_new[:, n:] = 0
    return dict(proj=pr, g2d=g2d, grad=grad, loss=loss, img=img[:, :H, :W],
                T=Tfin[:H, :W], last=last[:H, :W], last_id=last_id[:H, :W],
                n_eval_px=n_eval_px[:H, :W], list_len=list_len[:H, :W],
                pflags=pflags[:H, :W],
                params=p_new, m=m_new, v=v_new, n_eval=n_eval,
                n_isect=n_isect)


def decision_signature(params, n, sh_degree, cam, target):
    """Hash of every discrete decision of the forward + loss (cull, rects,
    lists, per-pixel skip/stop/clamp, residual signs)."""
    r = render(params, n, sh_degree, cam)
    pr = r["proj"]
    h = hash((pr["is_cand"].tobytes(), pr["rect_all"].tobytes(),
              r["vals"].tobytes(), r["fwd"]["sig"].tobytes(),
              np.signbit(r["img"] - target).tobytes(),
              ((r["img"] - target) == 0).tobytes()))
    return h


def loss_only(params, n, sh_degree, cam, target, ssim_lambda=None, leaves=None):
    """The view's loss from a full-image render: L1, or the composite loss
    with SSIM windows local to each Leaf's pixel rectangle (as step)."""
    r = render(params, n, sh_degree, cam)
    norm = 3.0 * cam.width * cam.height
    l1 = float(np.abs(r["img"] - target).sum() / norm)
    if ssim_lambda is None:
        return l1
    TW, TH = grid(cam)
    if leaves is None:
        leaves = [(0, 0, TW, TH)]
    ls = 0.0
    for (x0, y0, x1, y1) in leaves:
        sl = (slice(None), slice(y0 * 16, min(y1 * 16, cam.height)),
              slice(x0 * 16, min(x1 * 16, cam.width)))
        ls += loss_ssim(r["img"][sl], np.asarray(target)[sl], norm)[0]
    return (1.0 - ssim_lambda) * l1 + ssim_lambda * ls
