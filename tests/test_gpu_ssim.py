"""GPU parity of the SSIM term of the composite loss (gs_loss_ssim) against
the oracle's windowed SSIM, through the C ABI, and of the composite-loss step
end to end.

Tolerances.  The kernels form the window sums of x, y, x^2, y^2, x y in fp32
(two chains of 11 multiply-adds of non-negative terms, fp32 window weights),
then the differences sigma^2 = W[x^2] - mu^2 and sigma_xy = W[x y] - mu_x mu_y.
With u = 2^-24 and gamma = 23 u the relative error of each window sum, first
order error analysis bounds the error of S at each pixel by
  |dS| <= |S| (da/a + dc/c + dd/d + 4u) + |a / (c d)| db,
  dd <= (3 gamma + 2u)(W[x^2] + W[y^2]) + 2u d,
  db <= 2 (3 gamma + 2u)(W[x y] + mu_x mu_y) + 2u |b|,
  da / a, dc / c <= 2 gamma + 3u
(a = 2 mu_x mu_y + C1, b = 2 sigma_xy + C2, c = mu_x^2 + mu_y^2 + C1,
d = sigma_x^2 + sigma_y^2 + C2).  The per-tile loss is checked against the sum
of that bound (times 2 for second-order terms) plus the fp32 summation bound.
The gradient is a window sum of partials with cancellation between its three
terms; it is checked by relative L2 per channel (1e-4) and per pixel against
1e-3 of the gradient's largest magnitude."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_dgs_b200 import synth
from gpu_util import B, need_gpu, rel_err, rel_l2

pytestmark = pytest.mark.gpu

U = 2.0 ** -24
GAMMA = 23 * U
GRAD_L2 = 1e-4
GRAD_MAX = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    torch.cuda.set_device(0)


def s_bound(O, x, y):
    """Per pixel and channel bound of |S_fp32 - S| (first order, see above)."""
    out = np.zeros(x.shape)
    for c in range(x.shape[0]):
        mx, my, vx, vy, cxy = O.ssim_moments(x[c], y[c])
        ex, ey, f = vx + mx * mx, vy + my * my, cxy + mx * my
        a = 2 * mx * my + O.SSIM_C1
        b = 2 * cxy + O.SSIM_C2
        cc = mx * mx + my * my + O.SSIM_C1
        d = vx + vy + O.SSIM_C2
        S = a * b / (cc * d)
        dd = (3 * GAMMA + 2 * U) * (ex + ey) + 2 * U * d
        db = 2 * (3 * GAMMA + 2 * U) * (f + mx * my) + 2 * U * np.abs(b)
        rel_ac = 2 * (2 * GAMMA + 3 * U)
        out[c] = np.abs(S) * (rel_ac + dd / d + 4 * U) + np.abs(a / (cc * d)) * db
    return out


def run_ssim(x_leaf, target, L, W, H, weight, with_grad, dL0, lt0):
    """gs_loss_ssim on a Leaf-local render buffer x_leaf [3][h][w] and the whole
    view's resident target; dL0 / lt0 are the values the kernel adds to."""
    b = B()
    cam = b.camera_struct(synth.axis_camera(50.0, W, H))
    x0, y0 = 16 * L[0], 16 * L[1]
    _, h, w = x_leaf.shape
    img = torch.as_tensor(np.ascontiguousarray(x_leaf, np.float32)).cuda().reshape(-1)
    dL = torch.as_tensor(np.ascontiguousarray(dL0, np.float32)).cuda().reshape(-1)
    tgt = torch.as_tensor(np.ascontiguousarray(target, np.float32)).cuda()
    lt = torch.as_tensor(np.ascontiguousarray(lt0, np.float32)).cuda()
    T = torch.zeros(w * h, dtype=torch.float32, device="cuda")
    last = torch.zeros(w * h, dtype=torch.int32, device="cuda")
    px = b.pixels(x0, y0, w, h, img, T, last, dL, target=tgt, target_origin=(0, 0),
                  target_pitch=W, target_plane=W * H, loss_tiles=lt)
    ws = None
    if with_grad:
        ws = torch.empty(b.gs_ssim_workspace_size(L, cam), dtype=torch.uint8, device="cuda")
    b.gs_loss_ssim(px, L, cam, weight, ws)
    torch.cuda.synchronize()
    return dL.cpu().numpy().reshape(3, h, w), lt.cpu().numpy()


CASES = [
    # (W, H, leaf): whole ragged view, an interior Leaf (its windows stop at
    # its own edges), the ragged corner tile, a view smaller than one window
    (83, 61, (0, 0, 6, 4)),
    (83, 61, (1, 1, 4, 3)),
    (83, 61, (5, 3, 6, 4)),
    (83, 61, (3, 0, 6, 2)),
    (7, 5, (0, 0, 1, 1)),
    (1, 1, (0, 0, 1, 1)),
    (256, 160, (2, 1, 13, 9)),
]


@pytest.mark.parametrize("W,H,L", CASES)
@pytest.mark.parametrize("kind", ["random", "render_like"])
def test_ssim_stagewise(oracle_mod, W, H, L, kind):
    O = oracle_mod
    rng = np.random.default_rng(W * 7 + H + L[0] * 3 + L[2])
    if kind == "random":
        x_full = rng.random((3, H, W)).astype(np.float32)
    else:
        # smooth blobs on a black background, the value mix of a render
        yy, xx = np.mgrid[0:H, 0:W]
        x_full = np.zeros((3, H, W), np.float32)
        for _ in range(6):
            cx, cy, r = rng.uniform(0, W), rng.uniform(0, H), rng.uniform(2, 12)
            x_full += (rng.uniform(0.2, 0.9, (3, 1, 1)) *
                       np.exp(-((xx - cx) ** 2 + (yy - cy) ** 2) / (2 * r * r))).astype(np.float32)
        x_full = np.minimum(x_full, 1.0)
    target = (rng.random((3, H, W)) * 0.6).astype(np.float32)
    X0, Y0 = 16 * L[0], 16 * L[1]
    X1, Y1 = min(16 * L[2], W), min(16 * L[3], H)
    x = x_full[:, Y0:Y1, X0:X1]
    y = target[:, Y0:Y1, X0:X1]
    TW = (W + 15) // 16
    TH = (H + 15) // 16
    weight = 0.2 / (3.0 * W * H)
    dL0 = rng.standard_normal(x.shape).astype(np.float32) * 1e-6
    lt0 = rng.random(TW * TH).astype(np.float32) * 1e-3

    S = O.ssim_map(x.astype(np.float64), y.astype(np.float64))
    grad = -weight * O.ssim_map_grad(x.astype(np.float64), y.astype(np.float64))
    bnd = 2 * s_bound(O, x.astype(np.float64), y.astype(np.float64))

    for with_grad in (True, False):
        dL, lt = run_ssim(x, target, L, W, H, weight, with_grad, dL0, lt0)
        # per-tile loss sums
        for ty in range(L[1], L[3]):
            for tx in range(L[0], L[2]):
                sl = (slice(None), slice(16 * ty - Y0, min(16 * ty + 16, Y1) - Y0),
                      slice(16 * tx - X0, min(16 * tx + 16, X1) - X0))
                t = ty * TW + tx
                exp_add = weight * (1.0 - S[sl]).sum()
                tol = (weight * (bnd[sl].sum() + 770 * U * np.abs(1.0 - S[sl]).sum())
                       + 2 * U * (abs(lt0[t]) + abs(exp_add)))
                assert abs((lt[t] - lt0[t]) - exp_add) <= tol + U * abs(lt0[t]), (t, lt[t], exp_add)
        # tiles outside the Leaf are untouched
        mask = np.ones((TH, TW), bool)
        mask[L[1]:L[3], L[0]:L[2]] = False
        assert (lt.reshape(TH, TW)[mask] == lt0.reshape(TH, TW)[mask]).all()
        if not with_grad:
            assert (dL == dL0).all()
            continue
        got = dL.astype(np.float64) - dL0
        scale = np.abs(grad).max()
        for c in range(3):
            assert rel_l2(got[c], grad[c]) <= GRAD_L2, c
        assert np.abs(got - grad).max() <= GRAD_MAX * scale + 4 * U * np.abs(dL0).max()


def test_ssim_identical_and_constant(oracle_mod):
    """x = y gives S = 1 within the bound and a gradient near zero; constant
    planes reduce S to the luminance term in the window's interior."""
    O = oracle_mod
    W, H, L = 40, 36, (0, 0, 3, 3)
    x = np.random.default_rng(2).random((3, H, W)).astype(np.float32)
    weight = 1.0 / (3.0 * W * H)
    TW, TH = 3, 3
    dL, lt = run_ssim(x, x, L, W, H, weight, True, np.zeros_like(x), np.zeros(TW * TH, np.float32))
    bnd = 2 * s_bound(O, x.astype(np.float64), x.astype(np.float64))
    assert np.abs(lt).sum() <= weight * (bnd.sum() + 1e-3)
    assert np.abs(dL).max() <= 1e-3 * weight
    a, b = 0.3, 0.7
    xc = np.full((3, H, W), a, np.float32)
    yc = np.full((3, H, W), b, np.float32)
    dL, lt = run_ssim(xc, yc, L, W, H, weight, True, np.zeros_like(xc), np.zeros(TW * TH, np.float32))
    S = O.ssim_map(xc.astype(np.float64), yc.astype(np.float64))
    # sigma = 0: W[x^2] - mu^2 cancels to rounding noise of a^2 against C2
    bnd = 2 * s_bound(O, xc.astype(np.float64), yc.astype(np.float64))
    assert abs(lt.sum() - weight * (1 - S).sum()) <= weight * (bnd.sum() + 1e-3)
    grad = -weight * O.ssim_map_grad(xc.astype(np.float64), yc.astype(np.float64))
    assert rel_l2(dL, grad) <= GRAD_L2


@pytest.mark.parametrize("mode,budget,streams", [("bounded", 60_000, 1), ("bounded", 384 << 20, 1),
                                                 ("original", 384 << 20, 1),
                                                 ("bounded", 60_000, 2)])
def test_composite_loss_step(oracle_mod, mode, budget, streams):
    """One training step with (1 - lambda) L1 + lambda (1 - SSIM) against the
    oracle's step with the same Leaves (SSIM windows local to each)."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    O = oracle_mod
    sc, cams = synth.tiny_scene(n=300, width=160, height=120, sh_degree=3, seed=9,
                                scale_px=(1.0, 12.0))
    cam = cams[0]
    target = synth.random_image(cam.width, cam.height, 12) * 0.6

    class Leaves:
        def on_leaf(self, ctx, lc):
            self.leaves.append(lc["leaf"])

        def on_bwd(self, ctx):
            C = ctx["n_cand"]
            self.g2d = ctx["g2d"][:12 * C].cpu().numpy().reshape(-1, 12)[:, :9]
            self.cand_idx = ctx["cand_idx"][:C].cpu().numpy() if "cand_idx" in ctx else None

        def on_project(self, ctx):
            self.leaves = []

    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=budget, fuse_adam=False, mode=mode, loss="l1_ssim",
                  leaf_streams=streams)
    hk = Leaves()
    stats = stp.run_view(cam, torch.as_tensor(target).cuda(), hooks=hk)
    stp.check()
    if budget < (1 << 20):
        assert stats.n_leaves > 1
    ref = O.step(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam, target.astype(np.float64),
                 leaves=hk.leaves, ssim_lambda=0.2)
    loss = stp.last_loss()
    assert abs(loss - ref["loss"]) <= 1e-5 * ref["loss"]
    if mode == "original":
        live = np.isin(np.arange(sc.n), ref["proj"]["cand_idx"])
        g2d = hk.g2d[:sc.n][live]
    else:
        g2d = hk.g2d[:len(ref["proj"]["cand_idx"])]
    for f in range(9):
        assert rel_l2(g2d[:, f], ref["g2d"][:, f]) <= 1e-4, f
    p = model.params.cpu().numpy()
    g = ref["grad"][:, :sc.n]
    mask = np.abs(g) > 1e-3 * np.abs(g).max(axis=1, keepdims=True)
    d = np.abs(p[:, :sc.n] - ref["params"][:, :sc.n])
    assert d[mask].max() <= 1e-5
    assert d.max() <= 2.1e-3


def test_composite_loss_gated_step():
    """A gated step with the composite loss (loss-only forward pass, then the
    Leaves again with the gradient) takes the same update as the plain step
    when the gate says yes."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cams = synth.tiny_scene(n=200, width=96, height=80, sh_degree=1, seed=3)
    cam = cams[0]
    target = torch.as_tensor(synth.random_image(cam.width, cam.height, 4) * 0.6).cuda()
    outs = []
    for loss, gate in (("l1_ssim", None), ("l1_ssim", lambda l: True)):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=40_000, loss=loss)
        stp.run_view(cam, target, gate=gate)
        stp.check()
        outs.append((stp.last_loss(), model.params.cpu().numpy()))
    assert outs[0][0] == outs[1][0]
    assert np.abs(outs[0][1] - outs[1][1]).max() <= 2.1e-3
