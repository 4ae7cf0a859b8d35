"""Pins of the CPU oracle against things other than itself: closed forms,
library routines (scipy SH and rotations, numpy stable sorts, torch Adam),
brute force on tiny inputs, central finite differences and the Leaf
invariants.  CPU only."""
import math

import numpy as np
import pytest

from gaussian_splatting_differentiable_dgs_b200 import synth
from gaussian_splatting_differentiable_dgs_b200.synth import Camera, Scene


def make_cam(W, H, f=100.0, cx=None, cy=None, R=None, t=None):
    return Camera(np.eye(3, dtype=np.float32) if R is None else np.float32(R),
                  np.zeros(3, np.float32) if t is None else np.float32(t),
                  f, f, W / 2 if cx is None else cx, H / 2 if cy is None else cy,
                  W, H)


def one_gaussian(mean, log_scale, quat, logit, colour, D=0):
    p = np.zeros((synth.n_params(D), 64), np.float32)
    p[0:3, 0] = mean
    p[3:6, 0] = log_scale
    p[6:10, 0] = quat
    p[10, 0] = logit
    p[11:14, 0] = (np.asarray(colour) - 0.5) / (0.5 / math.sqrt(math.pi))
    return p


def stack_gaussians(cols):
    P = cols[0].shape[0]
    p = np.zeros((P, 64), np.float32)
    for i, c in enumerate(cols):
        p[:, i] = c[:, 0]
    return p


# ---------------------------------------------------------------------------
# spherical harmonics
# ---------------------------------------------------------------------------

def test_sh_orthonormal(oracle_mod):
    # Gauss-Legendre in cos(theta) x uniform phi integrates products of
    # degree <= 3 harmonics (degree <= 6 polynomials) exactly.
    xs, ws = np.polynomial.legendre.leggauss(8)
    nphi = 16
    G = np.zeros((16, 16))
    for ct, w in zip(xs, ws):
        st = math.sqrt(1 - ct * ct)
        for k in range(nphi):
            ph = 2 * math.pi * k / nphi
            d = np.array([st * math.cos(ph), st * math.sin(ph), ct])
            Y, _ = oracle_mod.sh_basis(d)
            G += w * (2 * math.pi / nphi) * np.outer(Y, Y)
    assert np.abs(G - np.eye(16)).max() < 1e-12


def test_sh_matches_scipy(oracle_mod):
    from scipy.special import sph_harm_y
    rng = np.random.default_rng(3)
    for _ in range(50):
        d = rng.normal(size=3)
        d /= np.linalg.norm(d)
        theta = math.acos(d[2])
        phi = math.atan2(d[1], d[0])
        Y, _ = oracle_mod.sh_basis(d)
        k = 0
        for l in range(4):
            for m in range(-l, l + 1):
                yc = sph_harm_y(l, abs(m), theta, phi)  # includes Condon-Shortley
                if m < 0:
                    ref = math.sqrt(2) * yc.imag
                elif m == 0:
                    ref = yc.real
                else:
                    ref = math.sqrt(2) * yc.real
                assert abs(Y[k] - ref) < 1e-12, (l, m)
                k += 1


def test_sh_gradient_fd(oracle_mod):
    rng = np.random.default_rng(4)
    for _ in range(10):
        d = rng.normal(size=3)
        _, dY = oracle_mod.sh_basis(d)
        for a in range(3):
            h = 1e-6
            e = np.zeros(3)
            e[a] = h
            fd = (oracle_mod.sh_basis(d + e)[0] - oracle_mod.sh_basis(d - e)[0]) / (2 * h)
            assert np.abs(fd - dY[:, a]).max() < 1e-7


# ---------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------

def test_isotropic_on_axis_closed_form(oracle_mod):
    W = H = 64
    f, z, s = 100.0, 3.0, 0.05
    cam = make_cam(W, H, f)
    p = one_gaussian([0, 0, z], [math.log(s)] * 3, [1, 0, 0, 0], 0.0, [0.3, 0.6, 0.9])
    pr = oracle_mod.project(p, 1, 0, cam)
    assert pr["is_cand"][0]
    r = pr["rec_all"][0]
    s32 = math.exp(float(np.float32(math.log(s))))
    var = (f * s32 / z) ** 2 + 0.3
    assert abs(r[oracle_mod.U] - W / 2) < 1e-12 and abs(r[oracle_mod.V] - H / 2) < 1e-12
    assert abs(r[11] - var) < 1e-9 * var and abs(r[12]) < 1e-15 and abs(r[13] - var) < 1e-9 * var
    assert abs(r[oracle_mod.A] - 1 / var) < 1e-9 / var and abs(r[oracle_mod.B]) < 1e-15
    assert r[oracle_mod.RADIUS] == math.ceil(3 * math.sqrt(var))
    assert abs(r[oracle_mod.DEPTH] - z) < 1e-12
    np.testing.assert_allclose(r[8:11], [0.3, 0.6, 0.9], atol=1e-7)
    assert abs(r[oracle_mod.OPAC] - 0.5) < 1e-15


def _pinhole(t, f, cx, cy):
    return np.array([f * t[0] / t[2] + cx, f * t[1] / t[2] + cy])


def test_projected_covariance_matches_scipy_rotation(oracle_mod):
    from scipy.spatial.transform import Rotation
    rng = np.random.default_rng(5)
    W, H, f = 200, 160, 150.0
    # a non-trivial camera pose
    Rc = Rotation.from_euler("xyz", [0.1, -0.2, 0.05]).as_matrix().astype(np.float32)
    tc = np.float32([0.1, -0.05, 0.2])
    cam = make_cam(W, H, f, R=Rc, t=tc)
    for _ in range(20):
        x = np.float32(rng.uniform(-0.4, 0.4, 3) + [0, 0, 3])
        ls = np.float32(rng.normal(-2.5, 0.4, 3))
        q = np.float32(rng.normal(size=4))
        p = one_gaussian(x, ls, q, 0.3, [0.5, 0.5, 0.5])
        pr = oracle_mod.project(p, 1, 0, cam)
        if not pr["is_cand"][0]:
            continue
        qd = q.astype(np.float64)
        Rg = Rotation.from_quat([qd[1], qd[2], qd[3], qd[0]]).as_matrix()
        S = np.diag(np.exp(ls.astype(np.float64)))
        Sigma = Rg @ S @ S @ Rg.T
        Rd, td = Rc.astype(np.float64), tc.astype(np.float64)
        t = Rd @ x.astype(np.float64) + td
        J = np.zeros((2, 3))
        for a in range(3):
            e = np.zeros(3)
            e[a] = 1e-5 * abs(t[2])
            J[:, a] = (_pinhole(t + e, f, W / 2, H / 2) - _pinhole(t - e, f, W / 2, H / 2)) / (2 * e[a])
        Sp = J @ Rd @ Sigma @ Rd.T @ J.T + 0.3 * np.eye(2)
        r = pr["rec_all"][0]
        got = np.array([[r[11], r[12]], [r[12], r[13]]])
        assert np.abs(got - Sp).max() < 1e-6 * np.abs(Sp).max()
        np.testing.assert_allclose(r[[0, 1]], _pinhole(t, f, W / 2, H / 2), rtol=1e-12)
        inv = np.linalg.inv(Sp)
        np.testing.assert_allclose(r[[4, 5, 6]], [inv[0, 0], inv[0, 1], inv[1, 1]], rtol=1e-6)
        lam = np.linalg.eigvalsh(Sp).max()
        assert r[oracle_mod.RADIUS] == math.ceil(3 * math.sqrt(lam))


def test_quaternion_90deg_swaps_scale_axes(oracle_mod):
    W = H = 128
    cam = make_cam(W, H, 100.0)
    a = one_gaussian([0, 0, 3], [math.log(0.05), math.log(0.02), -3], [1, 0, 0, 0], 0, [0.5] * 3)
    c, s = math.cos(math.pi / 4), math.sin(math.pi / 4)
    b = one_gaussian([0, 0, 3], [math.log(0.02), math.log(0.05), -3], [c, 0, 0, s], 0, [0.5] * 3)
    ra = oracle_mod.project(a, 1, 0, cam)["rec_all"][0]
    rb = oracle_mod.project(b, 1, 0, cam)["rec_all"][0]
    np.testing.assert_allclose(ra[11:14], rb[11:14], rtol=1e-6, atol=1e-9)
    assert ra[11] > ra[13]  # x axis is the long one


def test_degree0_colour_and_clamp(oracle_mod):
    cam = make_cam(64, 64)
    y0 = 0.5 / math.sqrt(math.pi)
    for col in [0.0, 0.25, 1.0, 1.7]:
        p = one_gaussian([0, 0, 3], [-3] * 3, [1, 0, 0, 0], 0, [col] * 3)
        r = oracle_mod.project(p, 1, 0, cam)["rec_all"][0]
        sh0 = np.float32((col - 0.5) / y0)
        assert abs(r[8] - max(0.0, y0 * float(sh0) + 0.5)) < 1e-15
    p = one_gaussian([0, 0, 3], [-3] * 3, [1, 0, 0, 0], 0, [-0.2] * 3)
    r = oracle_mod.project(p, 1, 0, cam)["rec_all"][0]
    assert r[8] == 0.0 and r[9] == 0.0


def test_cull_rules(oracle_mod):
    W, H, f = 64, 48, 50.0
    cam = make_cam(W, H, f)
    lim = 1.3 * (W / 2) / f
    cases = [
        ([0, 0, -1], False),                    # behind the camera
        ([0, 0, 0.19], False),                  # in front of the near plane
        ([0, 0, 0.25], True),
        ([3 * (lim + 0.01), 0, 3], False),      # outside the guard band
        ([3 * (lim - 0.01), 0, 3], False),      # inside the band, rect off-image
        ([0, 0, 3], True),
    ]
    for mean, expect in cases:
        p = one_gaussian(mean, [-4] * 3, [1, 0, 0, 0], 0, [0.5] * 3)
        assert oracle_mod.project(p, 1, 0, cam)["is_cand"][0] == expect, mean


def _square_bruteforce(u, v, r, TW, TH):
    """Tiles (tx, ty) of the grid that meet the closed square [u-r, u+r] x
    [v-r, v+r], by enumeration."""
    return {(tx, ty) for ty in range(TH) for tx in range(TW)
            if tx * 16 <= u + r and (tx + 1) * 16 > u - r
            and ty * 16 <= v + r and (ty + 1) * 16 > v - r}


def _alpha_at_centres(rec, tiles, W, H):
    """alpha = min(0.99, o exp(-q)) of one record at every in-image pixel
    centre of the given tiles, with q = (a dx^2 + c dy^2)/2 + b dx dy,
    d = mean - centre (the compositing definition, evaluated directly)."""
    out = []
    for tx, ty in tiles:
        ys, xs = np.mgrid[ty * 16:ty * 16 + 16, tx * 16:tx * 16 + 16]
        keep = (xs < W) & (ys < H)
        dx = rec[0] - (xs[keep] + 0.5)
        dy = rec[1] - (ys[keep] + 0.5)
        q = 0.5 * (rec[4] * dx * dx + rec[6] * dy * dy) + rec[5] * dx * dy
        out.append(np.minimum(0.99, rec[7] * np.exp(-q)))
    return np.concatenate(out) if out else np.zeros(0)


def _rect_tiles(r):
    return {(tx, ty) for ty in range(r[1], r[3]) for tx in range(r[0], r[2])}


def _pin_scenes():
    """Seeded scenes for the rect pins: SH degree 3 spread, large splats,
    opacities near the 0.99 clamp, opacities around 1/255, needle-thin
    Gaussians across the image border, and the 2,000-Gaussian scene."""
    return {
        "sh3_spread": synth.tiny_scene(n=60, width=96, height=80, sh_degree=3, seed=0,
                                       scale_px=(1.0, 9.0), opacity=(0.01, 0.99)),
        "sh3_large": synth.tiny_scene(n=40, width=80, height=64, sh_degree=3, seed=1,
                                      scale_px=(3.0, 14.0), opacity=(0.05, 0.95)),
        "near_clamp": synth.tiny_scene(n=60, width=80, height=64, sh_degree=3, seed=2,
                                       scale_px=(3.0, 10.0), opacity=(0.97, 0.9999)),
        "near_skip": synth.tiny_scene(n=80, width=80, height=64, sh_degree=0, seed=3,
                                      scale_px=(1.0, 8.0), opacity=(0.0025, 0.008)),
        "needles_edge": synth.edge_needle_scene(n=48, width=96, height=80, seed=4),
        "needles_edge_faint": synth.edge_needle_scene(n=48, width=96, height=80, seed=5,
                                                      opacity=(0.003, 0.05)),
        "tiny_2k": synth.tiny_oracle_scene(0),
    }


@pytest.mark.parametrize("name", list(_pin_scenes()))
def test_rects_and_removed_tiles_bruteforce(oracle_mod, name):
    """The plain rect is the 3-sigma square by enumeration; the tight rect
    lies inside it; every tile the tight rect drops (all of the square for a
    Gaussian the tight projection culls) has alpha below 1/255 at every
    in-image pixel centre, with a margin far above fp32 rounding.  The
    depth key is the fp32 bit pattern of t_z; records do not depend on the
    rect mode."""
    sc, cams = _pin_scenes()[name]
    cam = cams[0]
    W, H = cam.width, cam.height
    TW, TH = oracle_mod.grid(cam)
    p = sc.params.astype(np.float64)
    tight = oracle_mod.project(p, sc.n, sc.sh_degree, cam, tight=True)
    sq = oracle_mod.project(p, sc.n, sc.sh_degree, cam, tight=False)
    assert not (tight["is_cand"] & ~sq["is_cand"]).any()
    worst = 0.0
    n_removed = 0
    for g in np.nonzero(sq["is_cand"])[0]:
        rec = sq["rec_all"][g]
        square = _square_bruteforce(rec[0], rec[1], rec[3], TW, TH)
        assert square == _rect_tiles(sq["rect_all"][g])
        assert rec[14] == len(square)
        if tight["is_cand"][g]:
            assert (tight["rec_all"][g] == rec).all()
            assert tight["key_all"][g] == sq["key_all"][g]
            kept = _rect_tiles(tight["rect_all"][g])
            assert kept <= square
        else:
            kept = set()
        removed = square - kept
        n_removed += len(removed)
        a = _alpha_at_centres(rec, sorted(removed), W, H)
        if a.size:
            worst = max(worst, float(a.max()) * 255.0)
    assert n_removed > 0
    # the inflation of the alpha box (1e-4 in q) leaves every removed pixel
    # at least ~1e-4 relative below the threshold
    assert worst < 1.0 - 5e-5, worst
    keys = np.float32(sq["rec"][:, 2]).view(np.uint32)
    assert (keys == sq["key"]).all()
    assert (np.diff(sq["cand_idx"]) > 0).all() and (np.diff(tight["cand_idx"]) > 0).all()


@pytest.mark.parametrize("name", list(_pin_scenes()))
def test_tight_rects_give_the_plain_square_step(oracle_mod, name):
    """Reading (tight tile rects): binning each candidate into only the
    tiles of its 3-sigma square that meet its alpha >= 1/255 box, and culling
    the Gaussians that cannot reach 1/255, gives the step of the plain
    3-sigma-square binning: the same image, transmittance, last composited
    Gaussian per pixel, loss, 2D gradients (zero for every Gaussian the
    tight binning drops), 3D gradients and Adam update.  Checked with two
    Leaves and a non-trivial Adam state (t = 5), so that the update depends
    on the gradient's magnitude."""
    sc, cams = _pin_scenes()[name]
    cam = cams[0]
    W, H = cam.width, cam.height
    TW, TH = oracle_mod.grid(cam)
    p = sc.params.astype(np.float64)
    target = synth.random_image(W, H, seed=11).astype(np.float64)
    rng = np.random.default_rng(12)
    m0 = rng.normal(0, 1e-3, p.shape)
    v0 = rng.uniform(0, 1e-6, p.shape)
    m0[:, sc.n:] = 0
    v0[:, sc.n:] = 0
    leaves = [(0, 0, TW // 2, TH), (TW // 2, 0, TW, TH)]
    a = oracle_mod.step(p, sc.n, sc.sh_degree, cam, target, leaves=leaves,
                        m=m0, v=v0, t=5, tight=True)
    b = oracle_mod.step(p, sc.n, sc.sh_degree, cam, target, leaves=leaves,
                        m=m0, v=v0, t=5, tight=False)
    assert a["n_isect"] < b["n_isect"]
    assert (a["img"] == b["img"]).all() and (a["T"] == b["T"]).all()
    assert (a["last_id"] == b["last_id"]).all()
    assert (a["last_id"] >= 0).any()
    assert abs(a["loss"] - b["loss"]) <= 1e-14 * abs(b["loss"])
    # 2D gradients: per candidate of the tight binning equal, zero elsewhere
    ca, cb = a["proj"]["cand_idx"], b["proj"]["cand_idx"]
    pos = np.searchsorted(cb, ca)
    assert (cb[pos] == ca).all()
    g_sq = b["g2d"]
    scale = np.abs(g_sq).max()
    assert scale > 0
    assert np.abs(a["g2d"] - g_sq[pos]).max() <= 1e-12 * scale
    dropped = np.ones(len(cb), bool)
    dropped[pos] = False
    assert (g_sq[dropped] == 0).all()
    # dense 3D gradients and the Adam update
    gs = np.abs(b["grad"]).max()
    assert np.abs(a["grad"] - b["grad"]).max() <= 1e-12 * gs
    for key in ("params", "m", "v"):
        ref = b[key]
        assert np.abs(a[key] - ref).max() <= 1e-12 * max(np.abs(ref).max(), 1e-30), key


def test_pin_scenes_reach_the_thresholds(oracle_mod):
    """The rect pins' scenes do exercise the decisions the tight rects
    touch: the 0.99 clamp, Gaussians under 1/255 everywhere, the T stop, and
    needles that cross the image border."""
    sc_ = _pin_scenes()
    hit = {}
    for name in ("near_clamp", "near_skip", "needles_edge", "sh3_large"):
        sc, cams = sc_[name]
        cam = cams[0]
        p = sc.params.astype(np.float64)
        tight = oracle_mod.project(p, sc.n, sc.sh_degree, cam, tight=True)
        sq = oracle_mod.project(p, sc.n, sc.sh_degree, cam, tight=False)
        r = oracle_mod.render(p, sc.n, sc.sh_degree, cam)
        o = sq["rec"][:, 7]
        hit[name] = dict(n_faint=int((o < 1 / 255).sum()),
                         n_culled=int(sq["is_cand"].sum() - tight["is_cand"].sum()),
                         clamp=bool((o > 0.99).any()),
                         # a pixel stopped iff it visited fewer entries than its list
                         stop=bool((r["fwd"]["n_eval"] < np.diff(r["off"])[:, None])
                                   [(r["fwd"]["flags"] & oracle_mod.P_INVALID) == 0].any()),
                         cross=int(((sq["rec"][:, 0] < 0) | (sq["rec"][:, 0] > cam.width)
                                    | (sq["rec"][:, 1] < 0) | (sq["rec"][:, 1] > cam.height)).sum()))
    assert hit["near_clamp"]["clamp"]
    assert hit["near_skip"]["n_faint"] > 0 and hit["near_skip"]["n_culled"] > 0
    assert hit["needles_edge"]["cross"] > 0
    assert hit["near_clamp"]["stop"]


# ---------------------------------------------------------------------------
# tile lists (binning + sort)
# ---------------------------------------------------------------------------

def _random_rects(rng, C, TW, TH):
    x0 = rng.integers(0, TW, C)
    y0 = rng.integers(0, TH, C)
    x1 = np.minimum(TW, x0 + rng.integers(1, 4, C))
    y1 = np.minimum(TH, y0 + rng.integers(1, 4, C))
    return np.stack([x0, y0, x1, y1], 1).astype(np.int32)


def test_tile_lists_bruteforce_and_64bit_sort(oracle_mod):
    rng = np.random.default_rng(7)
    TW, TH, C = 7, 5, 300
    rect = _random_rects(rng, C, TW, TH)
    # many equal depths to exercise the index tie-break
    key = np.float32(rng.integers(1, 20, C) * 0.25 + 0.5).view(np.uint32)
    tiles = np.arange(TW * TH, dtype=np.int32)
    off, vals = oracle_mod.tile_lists(rect, key, TW, tiles)
    off2, vals2 = oracle_mod.tile_lists_all(rect, key, TW, TH)
    assert (off == off2).all() and (vals == vals2).all()
    # full 64-bit key sort of the duplicated (tile << 32 | depth) keys
    kk, vv = [], []
    for j in range(C):
        for ty in range(rect[j, 1], rect[j, 3]):
            for tx in range(rect[j, 0], rect[j, 2]):
                kk.append((np.uint64(ty * TW + tx) << np.uint64(32)) | np.uint64(key[j]))
                vv.append(j)
    kk = np.array(kk, np.uint64)
    vv = np.array(vv, np.int32)
    order = np.argsort(kk, kind="stable")
    assert (vv[order] == vals).all()
    tile_of = (kk[order] >> np.uint64(32)).astype(np.int64)
    assert (np.searchsorted(tile_of, tiles, "left") == off[:-1]).all()
    # presort by depth, then a stable sort on the tile bits only
    d_order = np.argsort(key, kind="stable")
    k2, v2 = [], []
    for j in d_order:
        for ty in range(rect[j, 1], rect[j, 3]):
            for tx in range(rect[j, 0], rect[j, 2]):
                k2.append(ty * TW + tx)
                v2.append(j)
    o2 = np.argsort(np.array(k2), kind="stable")
    assert (np.array(v2)[o2] == vals).all()


def test_tile_counts_and_sat(oracle_mod):
    rng = np.random.default_rng(8)
    TW, TH = 9, 6
    rect = _random_rects(rng, 500, TW, TH)
    c1 = oracle_mod.tile_counts(rect, TW, TH)
    c2 = oracle_mod.tile_counts_fast(rect, TW, TH)
    assert (c1 == c2).all()
    s = oracle_mod.sat(c1)
    for _ in range(50):
        x0, x1 = sorted(rng.integers(0, TW + 1, 2))
        y0, y1 = sorted(rng.integers(0, TH + 1, 2))
        got = s[y1, x1] - s[y0, x1] - s[y1, x0] + s[y0, x0]
        assert got == c1[y0:y1, x0:x1].sum()


# ---------------------------------------------------------------------------
# compositing closed forms
# ---------------------------------------------------------------------------

def _render_one_tile_scene(oracle_mod, p, n, cam):
    return oracle_mod.render(p, n, 0, cam)


def test_single_gaussian_peak_and_support(oracle_mod):
    W = H = 32
    cam = make_cam(W, H, 100.0, cx=16.5, cy=16.5)
    col = [0.2, 0.5, 0.8]
    for o, bounded_by_rect in [(0.3, False), (0.9, True), (0.995, True)]:
        p = one_gaussian([0, 0, 4], [math.log(0.1)] * 3, [1, 0, 0, 0],
                         math.log(o / (1 - o)), col)
        r = oracle_mod.render(p, 1, 0, cam)
        img = r["img"]
        rec = r["proj"]["rec"][0]
        # peak value at the pixel whose centre is the mean: min(0.99, o) * rgb
        np.testing.assert_allclose(img[:, 16, 16], rec[8:11] * min(0.99, rec[oracle_mod.OPAC]), rtol=1e-14)
        np.testing.assert_allclose(rec[8:11], col, atol=1e-7)
        var = rec[11]
        rad = rec[3]
        yy, xx = np.mgrid[0:H, 0:W] + 0.5
        q = 0.5 * ((xx - 16.5) ** 2 + (yy - 16.5) ** 2) / var
        inside = q <= math.log(255 * rec[oracle_mod.OPAC])
        rect = r["proj"]["rect"][0]
        in_rect = ((xx >= rect[0] * 16) & (xx < rect[2] * 16) &
                   (yy >= rect[1] * 16) & (yy < rect[3] * 16))
        support = img[0] > 0
        if not bounded_by_rect:
            assert math.log(255 * o) < 4.5  # 1/255 ellipse inside the 3-sigma square
            assert (support == inside).all()
        else:
            assert (support == (inside & in_rect)).all()
        assert rad >= 3 * math.sqrt(var)


def test_two_gaussian_blend(oracle_mod):
    W = H = 16
    cam = make_cam(W, H, 100.0, cx=8.5, cy=8.5)
    c1, c2 = [0.9, 0.1, 0.2], [0.1, 0.7, 0.4]
    o1, o2 = 0.6, 0.5
    g1 = one_gaussian([0, 0, 2], [-3] * 3, [1, 0, 0, 0], math.log(o1 / (1 - o1)), c1)
    g2 = one_gaussian([0, 0, 3], [-3] * 3, [1, 0, 0, 0], math.log(o2 / (1 - o2)), c2)
    p = stack_gaussians([g2, g1])  # index order != depth order
    r = oracle_mod.render(p, 2, 0, cam)
    rec = r["proj"]["rec"]
    # candidate 1 (index 1) is the nearer one
    c1r, o1r, c2r, o2r = rec[1, 8:11], rec[1, 7], rec[0, 8:11], rec[0, 7]
    assert abs(o1r - o1) < 1e-7 and abs(o2r - o2) < 1e-7
    exp = c1r * o1r + c2r * o2r * (1 - o1r)
    np.testing.assert_allclose(r["img"][:, 8, 8], exp, rtol=1e-14)
    assert abs(r["fwd"]["T"][0, 8 * 16 + 8] - (1 - o1r) * (1 - o2r)) < 1e-15


def test_transmittance_stop(oracle_mod):
    W = H = 16
    cam = make_cam(W, H, 100.0, cx=8.5, cy=8.5)
    col = [0.3, 0.6, 0.9]
    gs = [one_gaussian([0, 0, 2 + 0.1 * k], [-3] * 3, [1, 0, 0, 0],
                       math.log(0.95 / 0.05), col) for k in range(6)]
    r = oracle_mod.render(stack_gaussians(gs), 6, 0, cam)
    j = 8 * 16 + 8
    o = r["proj"]["rec"][0, 7]
    assert abs(o - 0.95) < 1e-7
    assert r["fwd"]["last"][0, j] == 3
    # T = 0.05, 2.5e-3, 1.25e-4, then 6.25e-6 < 1e-4 stops
    assert abs(r["fwd"]["T"][0, j] - (1 - o) ** 3) < 1e-15
    assert abs(r["fwd"]["T"][0, j] - 1.25e-4) < 1e-10
    np.testing.assert_allclose(r["img"][:, 8, 8], r["proj"]["rec"][0, 8:11] * (1 - (1 - o) ** 3), rtol=1e-13)
    assert r["fwd"]["n_eval"][0, j] == 4  # the fourth entry triggers the stop


def test_alpha_skip_threshold(oracle_mod):
    W = H = 16
    cam = make_cam(W, H, 100.0, cx=8.5, cy=8.5)
    for o, expect in [(0.003, False), (0.005, True)]:
        p = one_gaussian([0, 0, 2], [-3] * 3, [1, 0, 0, 0], math.log(o / (1 - o)), [1, 1, 1])
        r = oracle_mod.render(p, 1, 0, cam)
        assert (r["img"][0, 8, 8] > 0) == expect


def test_loss_constant_images(oracle_mod):
    img = np.full((3, 5, 7), 0.75)
    tgt = np.full((3, 5, 7), 0.25)
    L, d = oracle_mod.loss_l1(img, tgt, 3 * 5 * 7)
    assert abs(L - 0.5) < 1e-15
    assert np.all(d == 1.0 / 105)
    L, d = oracle_mod.loss_l1(tgt, tgt, 105)
    assert L == 0 and np.all(d == 0)


# ---------------------------------------------------------------------------
# Adam
# ---------------------------------------------------------------------------

def test_adam_step1_closed_form(oracle_mod):
    rng = np.random.default_rng(9)
    p0 = rng.normal(size=1000)
    g = rng.normal(size=1000) * 10.0 ** rng.uniform(-6, 1, 1000)
    p1, m1, v1 = oracle_mod.adam(p0, 0 * p0, 0 * p0, g, lr=1e-3, step=1)
    np.testing.assert_allclose(p1, p0 - 1e-3 * g / (np.abs(g) + 1e-8), rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(m1, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v1, 0.001 * g * g, rtol=1e-13)


def test_adam_matches_torch(oracle_mod):
    import torch
    rng = np.random.default_rng(10)
    p = torch.tensor(rng.normal(size=500), dtype=torch.float64, requires_grad=True)
    opt = torch.optim.Adam([p], lr=1e-3, betas=(0.9, 0.999), eps=1e-8)
    pn = p.detach().numpy().copy()
    m = np.zeros(500)
    v = np.zeros(500)
    for t in range(1, 6):
        g = rng.normal(size=500)
        p.grad = torch.tensor(g)
        opt.step()
        pn, m, v = oracle_mod.adam(pn, m, v, g, step=t)
        np.testing.assert_allclose(pn, p.detach().numpy(), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# gradients by central finite differences (fp64)
# ---------------------------------------------------------------------------

def _raster_loss(oracle_mod, rec, cam, tiles, off, vals, target):
    TW, TH = oracle_mod.grid(cam)
    fw = oracle_mod.raster_fwd(rec, TW, cam.width, cam.height, tiles, off, vals)
    img = oracle_mod.scatter_tiles(fw["img"], tiles, TW, TH, cam.width, cam.height, 3)
    d = img - target
    sig = hash((fw["sig"].tobytes(), np.signbit(d).tobytes(), (d == 0).tobytes()))
    return float(np.abs(d).sum() / (3 * cam.width * cam.height)), sig, fw


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_raster_bwd_finite_differences(oracle_mod, seed):
    sc, cams = synth.tiny_scene(n=10, width=48, height=40, seed=seed)
    cam = cams[0]
    TW, TH = oracle_mod.grid(cam)
    pr = oracle_mod.project(sc.params, sc.n, 0, cam)
    tgt = synth.random_image(cam.width, cam.height, seed + 100).astype(np.float64) * 0.6
    tiles = np.arange(TW * TH, dtype=np.int32)
    off, vals = oracle_mod.tile_lists(pr["rect"], pr["key"], TW, tiles)
    rec = pr["rec"].copy()
    L0, sig0, fw = _raster_loss(oracle_mod, rec, cam, tiles, off, vals, tgt)
    img = oracle_mod.scatter_tiles(fw["img"], tiles, TW, TH, cam.width, cam.height, 3)
    dL = oracle_mod.gather_tiles(np.sign(img - tgt) / (3 * cam.width * cam.height), tiles, TW, 3)
    g2d = oracle_mod.raster_bwd(rec, TW, cam.width, cam.height, tiles, off, vals, dL)
    fields = [0, 1, 4, 5, 6, 7, 8, 9, 10]  # u v a b c o R G B
    checked = skipped = 0
    for j in range(len(rec)):
        for fi, col in enumerate(fields):
            h = 1e-6 * max(abs(rec[j, col]), 1e-2)
            rp, rm = rec.copy(), rec.copy()
            rp[j, col] += h
            rm[j, col] -= h
            Lp, sp, _ = _raster_loss(oracle_mod, rp, cam, tiles, off, vals, tgt)
            Lm, sm, _ = _raster_loss(oracle_mod, rm, cam, tiles, off, vals, tgt)
            if sp != sig0 or sm != sig0:
                skipped += 1
                continue
            fd = (Lp - Lm) / (2 * h)
            an = g2d[j, fi]
            scale = np.abs(g2d[:, fi]).max()
            assert abs(fd - an) <= 1e-3 * abs(an) + 1e-7 * scale + 1e-14, (j, fi, fd, an)
            checked += 1
    assert checked > 0.8 * (checked + skipped)


@pytest.mark.parametrize("D,seed", [(0, 0), (0, 1), (3, 2), (3, 3)])
def test_full_gradient_finite_differences(oracle_mod, D, seed):
    sc, cams = synth.tiny_scene(n=6, width=40, height=36, sh_degree=D, seed=seed)
    cam = cams[0]
    tgt = synth.random_image(cam.width, cam.height, seed + 7).astype(np.float64) * 0.6
    st = oracle_mod.step(sc.params, sc.n, D, cam, tgt)
    grad = st["grad"]
    base = sc.params.astype(np.float64)
    sig0 = oracle_mod.decision_signature(base, sc.n, D, cam, tgt)
    checked = skipped = 0
    groups = [(0, 3), (3, 6), (6, 10), (10, 11), (11, 14), (14, base.shape[0])]
    for (a, b) in groups:
        if b <= a:
            continue
        scale = np.abs(grad[a:b, :sc.n]).max()
        for plane in range(a, b):
            for i in range(sc.n):
                h = 1e-6 * max(abs(base[plane, i]), 1e-1)
                pp, pm = base.copy(), base.copy()
                pp[plane, i] += h
                pm[plane, i] -= h
                if (oracle_mod.decision_signature(pp, sc.n, D, cam, tgt) != sig0 or
                        oracle_mod.decision_signature(pm, sc.n, D, cam, tgt) != sig0):
                    skipped += 1
                    continue
                fd = (oracle_mod.loss_only(pp, sc.n, D, cam, tgt) -
                      oracle_mod.loss_only(pm, sc.n, D, cam, tgt)) / (2 * h)
                an = grad[plane, i]
                assert abs(fd - an) <= 1e-3 * abs(an) + 1e-7 * scale + 1e-13, (plane, i, fd, an)
                checked += 1
    assert checked > 0.8 * (checked + skipped), (checked, skipped)


# ---------------------------------------------------------------------------
# Leaf partition
# ---------------------------------------------------------------------------

LM = [24, 44, 8, 4096, 512]


def _check_partition(leaves, li, lb, ov, sat_tab, TW, TH, W, H, budget):
    cover = np.zeros((TH, TW), np.int32)
    for (x0, y0, x1, y1), I, by, o in zip(leaves, li, lb, ov):
        assert 0 <= x0 < x1 <= TW and 0 <= y0 < y1 <= TH
        cover[y0:y1, x0:x1] += 1
        cnt = sat_tab[y1, x1] - sat_tab[y0, x1] - sat_tab[y1, x0] + sat_tab[y0, x0]
        assert cnt == I
        px = (min(x1 * 16, W) - x0 * 16) * (min(y1 * 16, H) - y0 * 16)
        al = lambda z: (z + 511) // 512 * 512
        est = al(I * LM[0]) + al(px * LM[1]) + al((x1 - x0) * (y1 - y0) * LM[2]) + LM[3]
        assert est == by
        assert (by <= budget) or (x1 - x0 == 1 and y1 - y0 == 1)
        assert o == (by > budget)
    assert (cover == 1).all()


def test_leaf_partition_invariants(oracle_mod):
    sc, cams = synth.tiny_oracle_scene(0)
    cam = cams[0]
    TW, TH = oracle_mod.grid(cam)
    pr = oracle_mod.project(sc.params, sc.n, 0, cam)
    s = oracle_mod.sat(oracle_mod.tile_counts(pr["rect"], TW, TH))
    for budget in [1, 20_000, 60_000, 200_000, 10 ** 9]:
        out = oracle_mod.leaf_partition(s, TW, TH, cam.width, cam.height, LM, budget)
        _check_partition(*out, s, TW, TH, cam.width, cam.height, budget)
        again = oracle_mod.leaf_partition(s, TW, TH, cam.width, cam.height, LM, budget)
        assert all((a == b).all() for a, b in zip(out, again))
    one = oracle_mod.leaf_partition(s, TW, TH, cam.width, cam.height, LM, 10 ** 9)[0]
    assert len(one) == 1 and tuple(one[0]) == (0, 0, TW, TH)
    tiny = oracle_mod.leaf_partition(s, TW, TH, cam.width, cam.height, LM, 1)
    assert len(tiny[0]) == TW * TH and tiny[3].all()


def test_leaf_partition_dense_regions_get_smaller_leaves(oracle_mod):
    TW, TH = 32, 32
    cnt = np.ones((TH, TW), np.int64)
    cnt[:8, :8] = 20_000  # one dense corner (intersections dominate the load)
    s = oracle_mod.sat(cnt)
    leaves = oracle_mod.leaf_partition(s, TW, TH, 512, 512, LM, 2_000_000)[0]
    area = lambda L: (L[2] - L[0]) * (L[3] - L[1])
    dense = [area(L) for L in leaves if L[0] < 8 and L[1] < 8]
    sparse = [area(L) for L in leaves if L[0] >= 16 and L[1] >= 16]
    assert max(dense) < min(sparse)


def test_leaf_invariance_oracle(oracle_mod):
    sc, cams = synth.tiny_scene(n=40, width=96, height=80, sh_degree=3, seed=5)
    cam = cams[0]
    TW, TH = oracle_mod.grid(cam)
    tgt = synth.random_image(cam.width, cam.height, 11).astype(np.float64) * 0.5
    whole = oracle_mod.step(sc.params, sc.n, 3, cam, tgt)
    pr = whole["proj"]
    s = oracle_mod.sat(oracle_mod.tile_counts(pr["rect"], TW, TH))
    rng = np.random.default_rng(0)
    partitions = [oracle_mod.leaf_partition(s, TW, TH, cam.width, cam.height, LM, b)[0]
                  for b in (40_000, 120_000)]
    partitions.append(np.array([[x, y, x + 1, y + 1] for y in range(TH) for x in range(TW)]))
    # a random guillotine partition
    rects, stack = [], [(0, 0, TW, TH)]
    while stack:
        x0, y0, x1, y1 = stack.pop()
        if (x1 - x0) * (y1 - y0) <= 3 or rng.uniform() < 0.2:
            rects.append((x0, y0, x1, y1))
        elif x1 - x0 >= y1 - y0:
            xm = rng.integers(x0 + 1, x1)
            stack += [(x0, y0, xm, y1), (xm, y0, x1, y1)]
        else:
            ym = rng.integers(y0 + 1, y1)
            stack += [(x0, y0, x1, ym), (x0, ym, x1, y1)]
    partitions.append(np.array(rects))
    for leaves in partitions:
        st = oracle_mod.step(sc.params, sc.n, 3, cam, tgt, leaves=[tuple(L) for L in leaves])
        assert (st["img"] == whole["img"]).all()
        assert (st["last"] == whole["last"]).all()
        assert abs(st["loss"] - whole["loss"]) < 1e-14
        for a, b in [(0, 3), (3, 6), (6, 10), (10, 11), (11, st["grad"].shape[0])]:
            ga, gb = st["grad"][a:b], whole["grad"][a:b]
            assert np.linalg.norm(ga - gb) <= 1e-12 * np.linalg.norm(gb) + 1e-300


# ---------------------------------------------------------------------------
# SSIM term of the composite loss (structural similarity of Wang et al. 2004,
# Gaussian window 11 x 11, sigma 1.5, zero outside the pixel rectangle)
# ---------------------------------------------------------------------------
def _interior(a, r=5):
    return a[..., r:-r, r:-r]


def test_ssim_window_sums_match_scipy(oracle_mod):
    """The windowed sums are a zero-padded correlation with the 2D Gaussian
    of sigma 1.5 truncated at radius 5, as scipy.ndimage computes it."""
    from scipy import ndimage
    O = oracle_mod
    rng = np.random.default_rng(3)
    x = rng.random((19, 27))
    out = O.window_sum(x)
    # scipy's own Gaussian filter (truncate = 5 / 1.5 gives radius 5), zero padding
    ref = ndimage.gaussian_filter(x, 1.5, mode="constant", cval=0.0, truncate=5.0 / 1.5)
    assert np.abs(out - ref).max() <= 1e-14
    g = O.ssim_window()
    assert len(g) == 11 and abs(g.sum() - 1.0) <= 1e-15 and np.allclose(g, g[::-1])


def test_ssim_identical_images(oracle_mod):
    O = oracle_mod
    x = np.random.default_rng(4).random((3, 12, 17))
    assert np.abs(O.ssim_map(x, x) - 1.0).max() <= 1e-12
    assert np.abs(O.ssim_map_grad(x, x)).max() <= 1e-10
    L, g = O.loss_ssim(x, x, 3 * 12 * 17)
    assert abs(L) <= 1e-12


def test_ssim_constant_images_closed_form(oracle_mod):
    """Constant planes a, b: wherever the window lies inside the image the
    variances vanish and S is the luminance term alone."""
    O = oracle_mod
    a, b = 0.3, 0.7
    x = np.full((1, 15, 16), a)
    y = np.full((1, 15, 16), b)
    S = _interior(O.ssim_map(x, y))
    assert np.abs(S - (2 * a * b + O.SSIM_C1) / (a * a + b * b + O.SSIM_C1)).max() <= 1e-12


def test_ssim_special_structures(oracle_mod):
    """With library window sums m = W[x], s = W[x^2] - m^2 (scipy), in the
    interior: y = x + delta keeps the structure term at 1; y = 1 - x makes
    sigma_xy = -sigma^2; y = k x scales the variances by k^2."""
    from scipy import ndimage
    O = oracle_mod
    filt = lambda z: ndimage.gaussian_filter(z, 1.5, mode="constant", cval=0.0, truncate=5.0 / 1.5)
    x = np.random.default_rng(5).uniform(0.2, 0.8, (1, 24, 25))
    mu = _interior(filt(x[0]))
    var = _interior(filt(x[0] ** 2)) - mu ** 2
    C1, C2 = O.SSIM_C1, O.SSIM_C2
    lum = lambda m1, m2: (2 * m1 * m2 + C1) / (m1 ** 2 + m2 ** 2 + C1)
    d = 0.05
    S = _interior(O.ssim_map(x, x + d))[0]
    assert np.abs(S - lum(mu, mu + d)).max() <= 1e-10
    S = _interior(O.ssim_map(x, 1.0 - x))[0]
    assert np.abs(S - lum(mu, 1 - mu) * (C2 - 2 * var) / (2 * var + C2)).max() <= 1e-10
    k = 0.6
    S = _interior(O.ssim_map(x, k * x))[0]
    cs = (2 * k * var + C2) / ((1 + k * k) * var + C2)
    assert np.abs(S - lum(mu, k * mu) * cs).max() <= 1e-10


def test_ssim_crop_interior_matches_full_image(oracle_mod):
    """Local windows: SSIM over a crop agrees with the full image's at pixels
    whose window lies inside the crop, and differs at the crop's edge."""
    O = oracle_mod
    rng = np.random.default_rng(6)
    x, y = rng.random((2, 3, 40, 44))
    full = O.ssim_map(x, y)
    crop = O.ssim_map(x[:, 7:30, 9:37], y[:, 7:30, 9:37])
    assert np.abs(_interior(crop) - _interior(full[:, 7:30, 9:37])).max() <= 1e-12
    assert np.abs(crop[:, 0, :] - full[:, 7, 9:37]).max() > 1e-3


def test_ssim_gradient_finite_differences(oracle_mod):
    """The analytic gradient of sum(S) against central differences at every
    pixel (borders included) of a small random pair."""
    O = oracle_mod
    rng = np.random.default_rng(7)
    x, y = rng.uniform(0.1, 0.9, (2, 2, 9, 13))
    g = O.ssim_map_grad(x, y)
    h = 1e-6
    fd = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd[idx] = (O.ssim_map(xp, y).sum() - O.ssim_map(xm, y).sum()) / (2 * h)
    assert np.abs(g - fd).max() <= 1e-7 * max(1.0, np.abs(fd).max())


def test_composite_loss_step_weights(oracle_mod):
    """step(ssim_lambda=0) is the L1 step; for lambda in (0, 1) the loss is
    the weighted sum of the L1 step's loss and the SSIM term computed by
    loss_ssim on the rendered image (one Leaf = the whole image)."""
    O = oracle_mod
    sc, cams = synth.tiny_scene(n=60, width=45, height=37, sh_degree=1, seed=2)
    cam = cams[0]
    p64 = sc.params.astype(np.float64)
    tgt = synth.random_image(cam.width, cam.height, 3).astype(np.float64)
    r1 = O.step(p64, sc.n, sc.sh_degree, cam, tgt)
    r0 = O.step(p64, sc.n, sc.sh_degree, cam, tgt, ssim_lambda=0.0)
    # the oracle's threaded gradient sums vary in their last bits between runs
    assert r0["loss"] == r1["loss"]
    assert np.abs(r0["grad"] - r1["grad"]).max() <= 1e-14 * np.abs(r1["grad"]).max()
    lam = 0.2
    rs = O.step(p64, sc.n, sc.sh_degree, cam, tgt, ssim_lambda=lam)
    ls, _ = O.loss_ssim(r1["img"], tgt, 3.0 * cam.width * cam.height)
    assert abs(rs["loss"] - ((1 - lam) * r1["loss"] + lam * ls)) <= 1e-12
    assert np.abs(rs["grad"] - r1["grad"]).max() > 1e-3 * np.abs(r1["grad"]).max()


@pytest.mark.parametrize("seed", [0, 1])
def test_composite_loss_gradient_finite_differences(oracle_mod, seed):
    """The whole step's gradient of the composite loss, over two Leaves
    (SSIM windows local to each), against central differences of the
    rendered loss."""
    O = oracle_mod
    sc, cams = synth.tiny_scene(n=6, width=40, height=36, sh_degree=1, seed=seed)
    cam = cams[0]
    TW, TH = O.grid(cam)
    leaves = [(0, 0, 1, TH), (1, 0, TW, TH)]
    tgt = synth.random_image(cam.width, cam.height, seed + 9).astype(np.float64) * 0.6
    st = O.step(sc.params, sc.n, 1, cam, tgt, leaves=leaves, ssim_lambda=O.SSIM_LAMBDA)
    assert abs(st["loss"] - O.loss_only(sc.params.astype(np.float64), sc.n, 1, cam, tgt,
                                        O.SSIM_LAMBDA, leaves)) <= 1e-12
    grad = st["grad"]
    base = sc.params.astype(np.float64)
    sig0 = O.decision_signature(base, sc.n, 1, cam, tgt)
    checked = skipped = 0
    scale = np.abs(grad[:, :sc.n]).max()
    for plane in range(base.shape[0]):
        for i in range(sc.n):
            h = 1e-6 * max(abs(base[plane, i]), 1e-1)
            pp, pm = base.copy(), base.copy()
            pp[plane, i] += h
            pm[plane, i] -= h
            if (O.decision_signature(pp, sc.n, 1, cam, tgt) != sig0 or
                    O.decision_signature(pm, sc.n, 1, cam, tgt) != sig0):
                skipped += 1
                continue
            fd = (O.loss_only(pp, sc.n, 1, cam, tgt, O.SSIM_LAMBDA, leaves) -
                  O.loss_only(pm, sc.n, 1, cam, tgt, O.SSIM_LAMBDA, leaves)) / (2 * h)
            an = grad[plane, i]
            assert abs(fd - an) <= 1e-3 * abs(an) + 1e-7 * scale + 1e-13, (plane, i, fd, an)
            checked += 1
    assert checked > 0.8 * (checked + skipped), (checked, skipped)
