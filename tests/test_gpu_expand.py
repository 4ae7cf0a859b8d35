"""Two-level binning (per-block candidate lists, then per-Leaf expansion into
per-tile segments) against the oracle's per-tile lists: vals and ranges must
be bit-identical to the lists sorted by (depth bits, candidate position),
the front-to-back order the tile rasteriser composites in (SkipGS paper
notes, "loss function / training strategy": the rasterisation pipeline is
the standard one).  The block-level intermediates are checked against their
plain definitions."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_dgs_b200 import synth
from gpu_util import B, ProjBuffers, need_gpu

pytestmark = pytest.mark.gpu

BLK = 8


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    torch.cuda.set_device(0)


def _block_rects(rect):
    r = np.asarray(rect, np.int64)
    return np.stack([r[:, 0] // BLK, r[:, 1] // BLK, (r[:, 2] - 1) // BLK + 1,
                     (r[:, 3] - 1) // BLK + 1], 1)


def _leaf_tiles(L, TW):
    x0, y0, x1, y1 = L
    return np.array([ty * TW + tx for ty in range(y0, y1) for tx in range(x0, x1)], np.int32)


class Case:
    """Candidate rects/keys (oracle projection or synthetic) on the device."""

    def __init__(self, oracle_mod, rect, key, TW, TH):
        self.O = oracle_mod
        self.rect = np.asarray(rect, np.int32).reshape(-1, 4)
        self.key = np.asarray(key, np.uint32)
        self.C = C = len(self.rect)
        self.TW, self.TH = TW, TH
        self.BW, self.BH = (TW + BLK - 1) // BLK, (TH + BLK - 1) // BLK
        rec = np.zeros((C, 16))
        rec[:, 4] = rec[:, 6] = rec[:, 11] = rec[:, 13] = 1.0  # unit conic (unused here)
        rec[:, 7] = 0.5
        pr = dict(cand_idx=np.arange(C, dtype=np.int32), rect=self.rect, key=self.key, rec=rec)
        self.pb = ProjBuffers.from_oracle(pr, max(C, 1))
        self.order = np.argsort(self.key, kind="stable").astype(np.int32)
        self.order_d = torch.as_tensor(self.order if C else np.zeros(1, np.int32)).cuda()
        dr = self.rect[self.order].astype(np.int16).reshape(-1)
        self.drect_d = torch.as_tensor(dr if C else np.zeros(4, np.int16)).cuda()
        self.sat = oracle_mod.sat(oracle_mod.tile_counts_fast(self.rect, TW, TH)) if C else \
            np.zeros((TH + 1, TW + 1), np.int64)
        self.sat_d = torch.as_tensor(self.sat.reshape(-1)).cuda()
        self.st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def block_sat(self):
        b = B()
        bs = torch.full(((self.BH + 1) * (self.BW + 1),), -7, dtype=torch.int64, device="cuda")
        ws = torch.empty(b.gs_block_sat_workspace_size(self.TW, self.TH), dtype=torch.uint8,
                         device="cuda")
        b.gs_block_sat(self.pb.struct, self.TW, self.TH, bs, ws, self.st)
        assert b.gs_check(self.st) == 0
        self.bsat_d = bs
        self.bsat = bs.cpu().numpy().reshape(self.BH + 1, self.BW + 1)
        return self.bsat

    def bin_blocks(self):
        b = B()
        n = int(self.bsat[self.BH, self.BW])
        self.bvals = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
        self.branges = torch.full((2 * self.BW * self.BH,), -1, dtype=torch.int64, device="cuda")
        ws = torch.empty(max(b.gs_bin_blocks_workspace_size(self.C, n, self.TW, self.TH), 256),
                         dtype=torch.uint8, device="cuda")
        b.gs_bin_blocks(self.pb.struct, self.C, self.order_d, self.drect_d, self.TW, self.TH,
                        self.bsat_d, n, self.bvals, max(n, 1), self.branges, ws, self.st)
        assert b.gs_check(self.st) == 0
        return n

    def expand(self, L):
        b = B()
        x0, y0, x1, y1 = L
        S = self.sat
        I = int(S[y1, x1] - S[y0, x1] - S[y1, x0] + S[y0, x0])
        vals = torch.full((max(I, 1),), -1, dtype=torch.int32, device="cuda")
        ranges = torch.full((2 * (x1 - x0) * (y1 - y0),), -1, dtype=torch.int64, device="cuda")
        be = b.block_entries(self.bsat, L)
        ws = torch.empty(max(b.gs_expand_workspace_size(L, be), 256), dtype=torch.uint8,
                         device="cuda")
        b.gs_expand_tiles(self.pb.struct, self.bvals, self.branges, be, L, self.TW, self.TH,
                          self.sat_d, I, vals, max(I, 1), ranges, ws, self.st)
        assert b.gs_check(self.st) == 0
        return I, vals.cpu().numpy()[:I], ranges.cpu().numpy().reshape(-1, 2)

    def check_blocks(self):
        bsat = self.block_sat()
        br = _block_rects(self.rect) if self.C else np.zeros((0, 4), np.int64)
        cnt = np.zeros((self.BH, self.BW), np.int64)
        for x0, y0, x1, y1 in br:
            cnt[y0:y1, x0:x1] += 1
        assert (bsat == self.O.sat(cnt)).all()
        n = self.bin_blocks()
        assert n == cnt.sum()
        bv = self.bvals.cpu().numpy()[:n]
        rg = self.branges.cpu().numpy().reshape(-1, 2)
        ob = br[self.order] if self.C else br
        pos = 0
        for blk in range(self.BW * self.BH):
            bx, by = blk % self.BW, blk // self.BW
            hit = (ob[:, 0] <= bx) & (bx < ob[:, 2]) & (ob[:, 1] <= by) & (by < ob[:, 3])
            exp = self.order[hit]
            assert rg[blk, 0] == pos and rg[blk, 1] == pos + len(exp)
            assert (bv[pos:pos + len(exp)] == exp).all()
            pos += len(exp)

    def check_leaf(self, L):
        I, vals, rg = self.expand(L)
        tiles = _leaf_tiles(L, self.TW)
        off, vals_o = self.O.tile_lists(self.rect, self.key, self.TW, tiles)
        assert I == off[-1]
        assert (rg[:, 0] == off[:-1]).all() and (rg[:, 1] == off[1:]).all()
        assert (vals == vals_o).all()


def _proj_case(oracle_mod, name):
    if name == "tiny":
        sc, cams = synth.tiny_oracle_scene(0)
    elif name == "hd":
        sc, cams = synth.hd_cluster_scene(0)
    else:
        sc, cams = synth.tiny_scene(n=80, width=83, height=61, sh_degree=3, seed=4)
    cam = cams[0]
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    TW, TH = oracle_mod.grid(cam)
    return Case(oracle_mod, pr["rect"], pr["key"], TW, TH), cam


@pytest.mark.parametrize("name", ["tiny", "ragged", "hd"])
def test_two_level_binning_on_projection(oracle_mod, name):
    case, cam = _proj_case(oracle_mod, name)
    case.check_blocks()
    TW, TH = case.TW, case.TH
    lm = [4, 44, 16, 2048, 512]
    budget = {"tiny": 150_000, "ragged": 40_000, "hd": 8_000_000}[name]
    leaves = oracle_mod.leaf_partition(case.sat, TW, TH, cam.width, cam.height, lm, budget)[0]
    assert len(leaves) > 1
    rng = np.random.default_rng(1)
    picks = [tuple(int(v) for v in L) for L in leaves[rng.permutation(len(leaves))[:10]]]
    # the whole grid, one tile, and rects that cut blocks at odd offsets
    picks += [(0, 0, TW, TH), (TW - 1, TH - 1, TW, TH),
              (min(3, TW - 1), min(5, TH - 1), TW, TH),
              (1, 1, max(2, TW // 2 + 3), max(2, TH // 3 + 1))]
    for L in picks:
        case.check_leaf(L)


@pytest.mark.parametrize("seed,C,TW,TH,wmax", [(0, 1, 1, 1, 1), (1, 3000, 9, 17, 9),
                                                (2, 200_000, 100, 80, 24),
                                                (3, 60_000, 333, 7, 40)])
def test_two_level_binning_synthetic(oracle_mod, seed, C, TW, TH, wmax):
    """Rects and depth keys drawn directly: many chunks per block (a block
    list far longer than one chunk), ties of the depth key, edge blocks."""
    rng = np.random.default_rng(seed)
    x0 = rng.integers(0, TW, C)
    y0 = rng.integers(0, TH, C)
    x1 = np.minimum(x0 + rng.integers(1, wmax + 1, C), TW)
    y1 = np.minimum(y0 + rng.integers(1, wmax + 1, C), TH)
    key = rng.integers(0, 1 << 20, C).astype(np.uint32) << np.uint32(10)  # many ties
    key[: C // 7] = key[0]
    case = Case(oracle_mod, np.stack([x0, y0, x1, y1], 1), key, TW, TH)
    case.check_blocks()
    leaves = [(0, 0, TW, TH), (0, 0, 1, 1), (TW // 3, TH // 4, TW, TH),
              (TW // 2, 0, max(TW // 2 + 1, TW - 3), TH)]
    for L in leaves:
        case.check_leaf(L)


def test_two_level_binning_leaf_without_entries(oracle_mod):
    # every candidate in the left half: a Leaf on the right gets no entries
    rect = np.array([[0, 0, 3, 3], [1, 2, 4, 9], [0, 5, 2, 6]], np.int32)
    case = Case(oracle_mod, rect, np.array([5, 3, 4], np.uint32), 20, 10)
    case.check_blocks()
    case.check_leaf((10, 0, 20, 10))
    case.check_leaf((0, 0, 20, 10))


@pytest.mark.parametrize("name", ["tiny", "ragged", "hd"])
@pytest.mark.parametrize("flags", [0, 4, 0x20, 0x20 | 4])
def test_fused_forward_matches_oracle(oracle_mod, name, flags):
    """gs_raster_fwd_blocks: image, T, last and loss as the oracle's
    compositing of the full lists; vals holds an exact prefix of each tile's
    list that covers every position the backward reads (< last).  Both forms:
    all threads filling, staging and compositing in turn (default), and a
    producer warp filling and staging for the compositing warps (0x20); 2 or
    4 pixels per thread."""
    sc, cams = {"tiny": synth.tiny_oracle_scene, "hd": synth.hd_cluster_scene}.get(
        name, lambda s: synth.tiny_scene(n=80, width=83, height=61, sh_degree=3, seed=4))(0)
    cam = cams[0]
    b = B()
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    TW, TH = oracle_mod.grid(cam)
    W, H = cam.width, cam.height
    case = Case(oracle_mod, pr["rect"], pr["key"], TW, TH)
    case.pb = ProjBuffers.from_oracle(pr, sc.n)  # the real records
    case.block_sat()
    case.bin_blocks()
    target = synth.random_image(W, H, 3) * 0.6
    tgt = torch.as_tensor(target.astype(np.float32)).cuda()
    leaves = [(0, 0, TW, TH), (1, 0, max(2, TW // 2 + 1), max(1, TH - 1))]
    for L in leaves:
        x0, y0, x1, y1 = L
        tiles = _leaf_tiles(L, TW)
        off, vals_o = oracle_mod.tile_lists(pr["rect"], pr["key"], TW, tiles)
        I = int(off[-1])
        px0, py0 = 16 * x0, 16 * y0
        pw, ph = min(16 * x1, W) - px0, min(16 * y1, H) - py0
        npx = pw * ph
        img = torch.zeros(3 * npx, device="cuda")
        Tf = torch.zeros(npx, device="cuda")
        last = torch.zeros(npx, dtype=torch.int32, device="cuda")
        dL = torch.zeros(3 * npx, device="cuda")
        loss_tiles = torch.zeros(TW * TH, device="cuda")
        px = b.pixels(px0, py0, pw, ph, img, Tf, last, dL, target=tgt, target_origin=(0, 0),
                      target_pitch=W, target_plane=W * H, loss_tiles=loss_tiles,
                      norm=1.0 / (3.0 * W * H))
        vals = torch.full((max(I, 1),), -1, dtype=torch.int32, device="cuda")
        ranges = torch.zeros(2 * len(tiles), dtype=torch.int64, device="cuda")
        b.gs_tile_ranges(case.sat_d, TW, TH, L, ranges)
        b.gs_raster_fwd_blocks(case.pb.struct, case.bvals, case.branges, L, b.camera_struct(cam),
                               px, vals, max(I, 1), I, ranges, case.st, flags=flags)
        assert b.gs_check(case.st) == 0
        # the same outputs as the full-list forward on the oracle's lists
        ref_img = torch.zeros_like(img)
        ref_T = torch.zeros_like(Tf)
        ref_last = torch.zeros_like(last)
        ref_dL = torch.zeros_like(dL)
        ref_lt = torch.zeros_like(loss_tiles)
        pxr = b.pixels(px0, py0, pw, ph, ref_img, ref_T, ref_last, ref_dL, target=tgt,
                       target_origin=(0, 0), target_pitch=W, target_plane=W * H,
                       loss_tiles=ref_lt, norm=1.0 / (3.0 * W * H))
        vals_full = torch.as_tensor(vals_o if I else np.zeros(1, np.int32)).cuda()
        rg_full = torch.as_tensor(np.stack([off[:-1], off[1:]], 1).astype(np.int64).reshape(-1)).cuda()
        # the same pixels per thread: the per-tile loss partial's fp32 sum
        # runs over the tile's warps in order
        b.gs_raster_fwd(case.pb.struct, vals_full, rg_full, L, b.camera_struct(cam), pxr, case.st,
                        flags & 7)
        assert b.gs_check(case.st) == 0
        assert torch.equal(img, ref_img) and torch.equal(Tf, ref_T) and torch.equal(last, ref_last)
        assert torch.equal(dL, ref_dL) and torch.equal(loss_tiles, ref_lt)
        # vals: the exact prefix of each oracle list that the backward reads
        rg = ranges.cpu().numpy().reshape(-1, 2)
        v = vals.cpu().numpy()
        lst = last.cpu().numpy().reshape(ph, pw)
        for k, tile in enumerate(tiles):
            tx, ty = tile % TW, tile // TW
            a, e = int(rg[k, 0]), int(rg[k, 1])
            assert a == off[k] and off[k] <= e <= off[k + 1]
            assert (v[a:e] == vals_o[off[k]:off[k] + (e - a)]).all()
            ys, xs = 16 * ty - py0, 16 * tx - px0
            need = lst[max(ys, 0):ys + 16, max(xs, 0):xs + 16]
            assert need.size == 0 or need.max() <= e - a


def test_step_paths_agree(oracle_mod):
    """The step with the two-level binning and with bin + tile sort: the same
    image, loss and Leaf plan inputs; gradients equal up to atomic order."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cams = synth.hd_cluster_scene(0)
    cam = cams[0]
    target = torch.as_tensor(synth.random_image(cam.width, cam.height, 2) * 0.5).cuda()
    outs = []
    for binning in ("fused", "expand", "sort"):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=6 << 20, binning=binning)
        seen = {}

        class Hooks:
            def on_bwd(self, ctx):
                seen["g2d"] = ctx["g2d"].clone()

        stats = stp.run_view(cam, target, hooks=Hooks(), update=False)
        stp.check()
        outs.append((stats, seen, stp.last_loss()))
    (s0, h0, l0) = outs[-1]
    g0 = h0["g2d"].cpu().numpy().reshape(-1, 12)
    for s1, h1, l1 in outs[:-1]:
        assert s0.n_isect == s1.n_isect and s1.n_leaves <= s0.n_leaves
        assert l0 == l1
        g1 = h1["g2d"].cpu().numpy().reshape(-1, 12)
        for f in range(9):
            d = np.linalg.norm(g0[:, f] - g1[:, f])
            assert d <= 1e-5 * max(np.linalg.norm(g0[:, f]), 1e-30), f
