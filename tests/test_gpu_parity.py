"""GPU parity of every stage against the CPU oracle, through the C ABI.

Stagewise tests feed both sides the same inputs (seeded generators or the
oracle's own outputs), so integer stages must match bit-exactly and fp32
stages within the stated tolerances:
  image / loss: max relative error <= 1e-5 (floor 1e-3), pixels with a
                decision within the oracle's margin of a threshold excluded
                and counted;
  gradients:    relative L2 <= 1e-4 per tensor.
"""
import math

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_dgs_b200 import synth
from gpu_util import (B, ProjBuffers, decode_records, encode_records, need_gpu, rel_err,
                      rel_l2)

pytestmark = pytest.mark.gpu

IMG_TOL = 1e-5
GRAD_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()
    torch.cuda.set_device(0)


_SCENES = {}


def scene(name):
    if name not in _SCENES:
        if name == "tiny":
            s, cams = synth.tiny_oracle_scene(0)
        elif name == "hd":
            s, cams = synth.hd_cluster_scene(0)
        elif name == "ragged":
            s, cams = synth.tiny_scene(n=80, width=83, height=61, sh_degree=3, seed=4)
        elif name == "small3":
            s, cams = synth.tiny_scene(n=300, width=160, height=120, sh_degree=3, seed=9,
                                       scale_px=(1.0, 12.0))
        else:
            raise KeyError(name)
        _SCENES[name] = (s, cams[0])
    return _SCENES[name]


def run_project(sc, cam):
    b = B()
    n = sc.n
    pb = ProjBuffers(n)
    params = torch.as_tensor(sc.params).cuda()
    model = b.gs_model(n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
    TW, TH = (cam.width + 15) // 16, (cam.height + 15) // 16
    sat = torch.zeros((TH + 1) * (TW + 1), dtype=torch.int64, device="cuda")
    ws = torch.empty(b.gs_project_workspace_size(n, cam.width, cam.height), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_project(model, b.camera_struct(cam), pb.struct, sat, ws, st)
    assert b.gs_check(st) == 0
    return pb, sat.cpu().numpy().reshape(TH + 1, TW + 1), params


# ---------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "ragged", "small3", "hd"])
def test_project_parity(oracle_mod, name):
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    pb, sat, _ = run_project(sc, cam)
    C = int(pb.n_cand.item())
    Co = len(pr["cand_idx"])
    assert C == Co
    assert (pb.cand_idx[:C].cpu().numpy() == pr["cand_idx"]).all()
    slot = pb.slot[:sc.n].cpu().numpy()
    exp_slot = np.full(sc.n, -1)
    exp_slot[pr["cand_idx"]] = np.arange(Co)
    assert (slot == exp_slot).all()
    rect = pb.rect[:4 * C].cpu().numpy().reshape(-1, 4).astype(np.int32)
    near = (pr["flags"] & 1) != 0
    assert (rect[~near] == pr["rect"][~near]).all()
    assert near.sum() <= max(1, C // 10000)
    key = pb.depth_key[:C].cpu().numpy().view(np.uint32)
    assert (key == pr["key"]).all()
    got = pb.rec[:12 * C].cpu().numpy().reshape(-1, 12)
    exp = encode_records(pr["rec"])
    d = decode_records(got)
    ro = pr["rec"]
    # u, v: fp32 + fp16 correction, exact to ~2e-7 px
    assert np.abs(d["u"] - ro[:, 0]).max() <= 2.5e-7 + 1e-12 * np.abs(ro[:, 0]).max()
    assert np.abs(d["v"] - ro[:, 1]).max() <= 2.5e-7 + 1e-12 * np.abs(ro[:, 1]).max()
    # the fp32 coefficient fields are the correctly rounded fp64 values
    for col in (4, 5, 6, 7, 8, 9, 10, 11):
        assert rel_err(got[:, col], exp[:, col], floor=1e-30).max() <= 2.4e-7, col
    # alpha box half extents: the reading's bound, rounded up to fp16
    de = decode_records(exp)
    assert (np.abs(d["hx"] - de["hx"]) <= 1e-3 * de["hx"]).all()
    assert (np.abs(d["hy"] - de["hy"]) <= 1e-3 * de["hy"]).all()
    TW, TH = (cam.width + 15) // 16, (cam.height + 15) // 16
    exp_sat = oracle_mod.sat(oracle_mod.tile_counts_fast(pr["rect"], TW, TH))
    assert (sat == exp_sat).all()
    assert int(pb.square.item()) == int(pr["rec"][:, 14].sum())


def test_project_edge_cases(oracle_mod):
    b = B()
    sc, cam = scene("tiny")
    # everything behind the camera: no candidates, zero SAT
    s2 = sc.copy()
    s2.params[2, :s2.n] = -3.0
    pb, sat, _ = run_project(s2, cam)
    assert int(pb.n_cand.item()) == 0 and (sat == 0).all()
    assert (pb.slot[:s2.n].cpu().numpy() == -1).all()
    # n = 0
    params = torch.zeros((sc.P, 64), device="cuda")
    pb0 = ProjBuffers(1)
    TW, TH = 16, 16
    satt = torch.ones((TH + 1) * (TW + 1), dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(b.gs_project_workspace_size(0, 256, 256), 256), dtype=torch.uint8,
                     device="cuda")
    b.gs_project(b.gs_model(0, 64, 0, 0, params.data_ptr()), b.camera_struct(cam), pb0.struct,
                 satt, ws, st)
    assert b.gs_check(st) == 0
    assert int(pb0.n_cand.item()) == 0 and (satt.cpu() == 0).all()
    # a NaN parameter is culled and flagged
    s3 = sc.copy()
    s3.params[4, 7] = np.nan
    pb3, _, _ = run_project(s3, cam)
    assert pb3.slot[7].item() == -1
    # bad arguments are rejected on the host
    with pytest.raises(b.GsError):
        b.gs_project(b.gs_model(10, 63, 0, 0, params.data_ptr()), b.camera_struct(cam),
                     pb0.struct, satt, ws, st)


# ---------------------------------------------------------------------------
# radix sorts
# ---------------------------------------------------------------------------

def _sort_ws(n, kb, lo, hi):
    return torch.empty(max(B().gs_sort_workspace_size(n, kb, lo, hi), 256), dtype=torch.uint8,
                       device="cuda")


def test_project_dense_layout(oracle_mod):
    """GS_PROJ_DENSE: slot i for every Gaussian; candidates' records, rects and
    keys equal the compact projection's, culled ones are marked; same SAT."""
    sc, cam = scene("hd")
    b = B()
    pb, sat, params = run_project(sc, cam)
    C = int(pb.n_cand.item())
    n = sc.n
    pd = ProjBuffers(n)
    model = b.gs_model(n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
    TW, TH = (cam.width + 15) // 16, (cam.height + 15) // 16
    sat_d = torch.zeros((TH + 1) * (TW + 1), dtype=torch.int64, device="cuda")
    ws = torch.empty(b.gs_project_workspace_size(n, cam.width, cam.height), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_project(model, b.camera_struct(cam), pd.struct, sat_d, ws, st, flags=b.GS_PROJ_DENSE)
    assert b.gs_check(st) == 0
    assert int(pd.n_cand.item()) == n and C < n
    assert (sat_d.cpu().numpy().reshape(TH + 1, TW + 1) == sat).all()
    assert (pd.cand_idx.cpu().numpy() == np.arange(n)).all()
    ci = pb.cand_idx[:C].cpu().numpy()
    live = np.zeros(n, bool)
    live[ci] = True
    rec_d = pd.rec.cpu().numpy().reshape(n, 12)
    rec_c = pb.rec[:12 * C].cpu().numpy().reshape(C, 12)
    assert (rec_d[ci].view(np.uint32) == rec_c.view(np.uint32)).all()
    assert (pd.rect.cpu().numpy().reshape(n, 4)[ci] == pb.rect[:4 * C].cpu().numpy().reshape(C, 4)).all()
    assert (pd.depth_key.cpu().numpy()[ci] == pb.depth_key[:C].cpu().numpy()).all()
    assert (rec_d[~live, 11] == -1).all()
    assert (pd.rect.cpu().numpy().reshape(n, 4)[~live] == 0).all()
    assert (pd.depth_key.cpu().numpy()[~live].view(np.uint32) == 0xffffffff).all()


@pytest.mark.parametrize("n", [1, 100, 4095, 4096, 4097, 50_000, 1_000_003])
@pytest.mark.parametrize("bits", [(0, 32), (0, 13), (7, 23), (3, 3)])
@pytest.mark.parametrize("onesweep", [False, True])
def test_sort32_stable(n, bits, onesweep):
    b = B()
    rng = np.random.default_rng(n + bits[0])
    keys = (rng.integers(0, 1 << 32, n, dtype=np.uint64) & np.uint64(0xFFFF00F0)).astype(np.uint32)
    keys[::3] = keys[0]  # ties
    lo, hi = bits
    kin = torch.as_tensor(keys.view(np.int32)).cuda()
    kout = torch.empty_like(kin)
    vals = torch.empty(n, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fl = b.GS_SORT_IOTA | (b.GS_SORT_ONESWEEP if onesweep else 0)
    b.gs_sort_keys32(kin, kout, vals, n, lo, hi, fl, _sort_ws(n, 4, lo, hi), st)
    assert b.gs_check(st) == 0
    dig = (keys.astype(np.uint64) >> np.uint64(lo)) & np.uint64((1 << (hi - lo)) - 1)
    order = np.argsort(dig, kind="stable")
    assert (vals.cpu().numpy() == order).all()
    assert (kout.cpu().numpy().view(np.uint32) == keys[order]).all()
    assert (kin.cpu().numpy().view(np.uint32) == keys).all()  # input untouched


@pytest.mark.parametrize("n,tile_bits", [(5000, 8), (300_001, 13), (2_000_000, 16), (70_000, 20)])
def test_sort64_tile_bits(n, tile_bits):
    b = B()
    rng = np.random.default_rng(tile_bits)
    tiles = rng.integers(0, 1 << tile_bits, n).astype(np.uint64)
    depth = np.float32(rng.uniform(0.3, 50, n)).view(np.uint32).astype(np.uint64)
    keys = (tiles << np.uint64(32)) | depth
    vals = rng.integers(0, 1 << 30, n).astype(np.int32)
    kd = torch.as_tensor(keys.view(np.int64)).cuda()
    vd = torch.as_tensor(vals).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_sort_keys(kd, vd, n, 32, 32 + tile_bits, _sort_ws(n, 8, 32, 32 + tile_bits), st)
    assert b.gs_check(st) == 0
    order = np.argsort(tiles, kind="stable")
    assert (kd.cpu().numpy().view(np.uint64) == keys[order]).all()
    assert (vd.cpu().numpy() == vals[order]).all()


@pytest.mark.parametrize("n,n_tiles", [(1, 1), (9000, 3), (777_777, 5000), (3_000_000, 65536),
                                       (100_000, 200_000)])
def test_sort_tiles_from_ranges(n, n_tiles):
    b = B()
    rng = np.random.default_rng(n_tiles)
    keys = rng.integers(0, n_tiles, n).astype(np.uint32)
    vals = rng.integers(0, 1 << 31, n).astype(np.int32)
    counts = np.bincount(keys, minlength=n_tiles)
    off = np.concatenate([[0], np.cumsum(counts)])
    ranges = torch.as_tensor(np.stack([off[:-1], off[1:]], 1).reshape(-1).astype(np.int64)).cuda()
    kd = torch.as_tensor(keys.view(np.int32)).cuda()
    vd = torch.as_tensor(vals).cuda()
    bits = (n_tiles - 1).bit_length() if n_tiles > 1 else 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_sort_tiles(kd, vd, n, ranges, n_tiles, _sort_ws(n, 4, 0, bits), st)
    assert b.gs_check(st) == 0
    order = np.argsort(keys, kind="stable")
    assert (kd.cpu().numpy().view(np.uint32) == keys[order]).all()
    assert (vd.cpu().numpy() == vals[order]).all()


def test_sort_bounded_wait_reports_timeout():
    """The look-back wait gives up and reports instead of hanging: tile 0
    of the first pass is told (test flag) never to publish its counts."""
    b = B()
    n = 3 * 4096
    keys = np.arange(n, dtype=np.uint32)[::-1].copy()
    kin = torch.as_tensor(keys.view(np.int32)).cuda()
    kout = torch.empty_like(kin)
    vals = torch.empty(n, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_sort_keys32(kin, kout, vals, n, 0, 16, b.GS_SORT_IOTA | b.GS_SORT_TEST_STALL,
                     _sort_ws(n, 4, 0, 16), st)
    assert b.gs_check(st) == b.GS_ERR_TIMEOUT
    # the context stays usable and the status word was cleared
    b.gs_sort_keys32(kin, kout, vals, n, 0, 16, b.GS_SORT_IOTA, _sort_ws(n, 4, 0, 16), st)
    assert b.gs_check(st) == 0
    assert (vals.cpu().numpy() == np.argsort(keys & 0xFFFF, kind="stable")).all()


# ---------------------------------------------------------------------------
# binning + sort + ranges from the oracle's projection
# ---------------------------------------------------------------------------

def _leaf_tiles(L, TW):
    x0, y0, x1, y1 = L
    return np.array([ty * TW + tx for ty in range(y0, y1) for tx in range(x0, x1)], np.int32)


def _bin_leaf(pb, C, order_d, drect_d, L, TW, TH, sat_d, I, tile_bits):
    """Bin one Leaf (with the 64-bit keys), then sort it two ways: the
    product path (32-bit local tile keys) and the 64-bit keys on their tile
    bits.  Returns the emitted keys64 and both sorted results."""
    b = B()
    n = max(I, 1)
    tkeys = torch.zeros(n, dtype=torch.int32, device="cuda")
    vals = torch.zeros(n, dtype=torch.int32, device="cuda")
    keys64 = torch.zeros(n, dtype=torch.int64, device="cuda")
    nt = (L[2] - L[0]) * (L[3] - L[1])
    ranges = torch.zeros(2 * nt, dtype=torch.int64, device="cuda")
    ws = torch.empty(max(b.gs_bin_workspace_size(C), 256), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_bin_tiles(pb.struct, C, order_d, drect_d, L, TW, TH, sat_d, I, tkeys, vals, n, ranges, ws,
                   st, keys64=keys64)
    assert b.gs_check(st) == 0
    emitted = (keys64.cpu().numpy().view(np.uint64)[:I].copy(), tkeys.cpu().numpy()[:I].copy(),
               vals.cpu().numpy()[:I].copy())
    k64, v64 = keys64.clone(), vals.clone()
    t2, v2 = tkeys.clone(), vals.clone()
    lb = b.local_tile_bits(L)
    if I and lb:
        b.gs_sort_keys32(None, tkeys, vals, I, 0, lb, 0, _sort_ws(I, 4, 0, lb), st)
        b.gs_sort_keys(k64, v64, I, 32, 32 + tile_bits, _sort_ws(I, 8, 32, 32 + tile_bits), st)
        b.gs_sort_tiles(t2, v2, I, ranges, nt, _sort_ws(I, 4, 0, lb), st)
    assert b.gs_check(st) == 0
    assert (v2.cpu().numpy()[:I] == vals.cpu().numpy()[:I]).all()
    assert (t2.cpu().numpy()[:I] == tkeys.cpu().numpy()[:I]).all()
    return emitted, tkeys, vals, k64, v64, ranges


@pytest.mark.parametrize("name,on_device", [("hd", False), ("hd", True), ("tiny", True)])
def test_depth_order(oracle_mod, name, on_device):
    """gs_depth_order against numpy's stable argsort of the oracle's depth
    keys, with the count given by the host or read on the device
    (GS_COUNT_ON_DEVICE: buffers sized for a capacity above the count)."""
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    C = len(pr["cand_idx"])
    pb = ProjBuffers.from_oracle(pr, sc.n)
    b = B()
    cap = pb.cap if on_device else C
    assert cap >= C
    order = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    drect = torch.zeros(4 * cap, dtype=torch.int16, device="cuda")
    ws = torch.empty(b.gs_depth_order_workspace_size(cap), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_depth_order(pb.struct, b.GS_COUNT_ON_DEVICE if on_device else C, order, drect, ws, st)
    assert b.gs_check(st) == 0
    exp = np.argsort(pr["key"], kind="stable")
    assert (order[:C].cpu().numpy() == exp).all()
    assert (drect[:4 * C].cpu().numpy().reshape(-1, 4) == pr["rect"][exp]).all()


@pytest.mark.parametrize("name", ["tiny", "ragged", "hd"])
def test_bin_sort_ranges_bitexact(oracle_mod, name):
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    TW, TH = oracle_mod.grid(cam)
    C = len(pr["cand_idx"])
    pb = ProjBuffers.from_oracle(pr, sc.n)
    sat = oracle_mod.sat(oracle_mod.tile_counts_fast(pr["rect"], TW, TH))
    sat_d = torch.as_tensor(sat.reshape(-1)).cuda()
    order = np.argsort(pr["key"], kind="stable").astype(np.int32)
    order_d = torch.as_tensor(order).cuda()
    drect_d = torch.as_tensor(pr["rect"][order].astype(np.int16).reshape(-1)).cuda()
    tile_bits = max(1, math.ceil(math.log2(TW * TH)))
    lm = [17, 44, 16, 30000, 512]
    budget = {"tiny": 150_000, "ragged": 40_000, "hd": 8_000_000}[name]
    leaves = oracle_mod.leaf_partition(sat, TW, TH, cam.width, cam.height, lm, budget)[0]
    assert len(leaves) > 1
    rng = np.random.default_rng(0)
    for L in leaves[rng.permutation(len(leaves))[:12]]:
        L = tuple(int(v) for v in L)
        tiles = _leaf_tiles(L, TW)
        off, vals_o = oracle_mod.tile_lists(pr["rect"], pr["key"], TW, tiles)
        I = int(off[-1])
        emitted, tkeys, vals, k64, v64, ranges = _bin_leaf(pb, C, order_d, drect_d, L, TW, TH,
                                                           sat_d, I, tile_bits)
        rg = ranges.cpu().numpy().reshape(-1, 2)
        assert (rg[:, 0] == off[:-1]).all() and (rg[:, 1] == off[1:]).all()
        tile_of = np.repeat(tiles.astype(np.uint64), np.diff(off))
        exp_k = (tile_of << np.uint64(32)) | pr["key"][vals_o].astype(np.uint64)
        # emitted 64-bit keys: the oracle's multiset, in depth order of the candidates
        k_emit, t_emit, v_emit = emitted
        assert (np.sort(k_emit) == np.sort(exp_k)).all()
        depth_rank = np.empty(C, np.int64)
        depth_rank[order] = np.arange(C)
        assert (np.diff(depth_rank[v_emit]) >= 0).all()
        x0, y0, x1, y1 = L
        g_tile = (k_emit >> np.uint64(32)).astype(np.int64)
        loc = (g_tile // TW - y0) * (x1 - x0) + (g_tile % TW - x0)
        assert (t_emit == loc).all()
        # both sorts give the oracle's per-tile lists, bit-exactly
        assert (vals.cpu().numpy()[:I] == vals_o).all()
        assert (v64.cpu().numpy()[:I] == vals_o).all()
        assert (k64.cpu().numpy().view(np.uint64)[:I] == exp_k).all()


# ---------------------------------------------------------------------------
# raster forward / loss / backward on the oracle's records and lists
# ---------------------------------------------------------------------------

class LeafInputs:
    """Oracle-made inputs of one Leaf in the library layout."""

    def __init__(self, oracle_mod, sc, cam, L, target):
        self.O = oracle_mod
        W, H = cam.width, cam.height
        TW, TH = oracle_mod.grid(cam)
        self.TW, self.TH = TW, TH
        self.pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
        self.pb = ProjBuffers.from_oracle(self.pr, sc.n)
        self.L = L
        self.tiles = _leaf_tiles(L, TW)
        self.off, self.vals_o = oracle_mod.tile_lists(self.pr["rect"], self.pr["key"], TW,
                                                      self.tiles)
        self.vals = torch.as_tensor(self.vals_o if len(self.vals_o) else np.zeros(1, np.int32)).cuda()
        rg = np.stack([self.off[:-1], self.off[1:]], 1).astype(np.int64)
        self.ranges = torch.as_tensor(rg.reshape(-1)).cuda()
        self.fw = oracle_mod.raster_fwd(self.pr["rec"], TW, W, H, self.tiles, self.off,
                                        self.vals_o)
        x0, y0, x1, y1 = L
        self.px0, self.py0 = 16 * x0, 16 * y0
        self.pw = min(16 * x1, W) - self.px0
        self.ph = min(16 * y1, H) - self.py0
        self.target = target
        self.cam = cam

    def to_leaf(self, per_tile, channels=None):
        """Compact per-tile oracle data -> Leaf-local image layout."""
        full = self.O.scatter_tiles(per_tile, self.tiles, self.TW, self.TH, self.cam.width,
                                    self.cam.height, channels)
        return full[..., self.py0:self.py0 + self.ph, self.px0:self.px0 + self.pw]

    def buffers(self):
        npx = self.pw * self.ph
        self.img = torch.zeros(3 * npx, device="cuda")
        self.Tf = torch.zeros(npx, device="cuda")
        self.last = torch.zeros(npx, dtype=torch.int32, device="cuda")
        self.dL = torch.zeros(3 * npx, device="cuda")
        self.loss_tiles = torch.zeros(self.TW * self.TH, device="cuda")
        self.tgt = torch.as_tensor(self.target.astype(np.float32)).cuda()
        W, H = self.cam.width, self.cam.height
        return B().pixels(self.px0, self.py0, self.pw, self.ph, self.img, self.Tf, self.last,
                          self.dL, target=self.tgt, target_origin=(0, 0), target_pitch=W,
                          target_plane=W * H, loss_tiles=self.loss_tiles,
                          norm=1.0 / (3.0 * W * H))


def _fwd_case(oracle_mod, name, leaf_frac=None, ppt=0):
    sc, cam = scene(name)
    TW, TH = oracle_mod.grid(cam)
    L = (0, 0, TW, TH) if leaf_frac is None else leaf_frac(TW, TH)
    target = synth.random_image(cam.width, cam.height, 3) * 0.6
    li = LeafInputs(oracle_mod, sc, cam, L, target)
    px = li.buffers()
    b = B()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_raster_fwd(li.pb.struct, li.vals, li.ranges, L, b.camera_struct(cam), px, st, ppt)
    assert b.gs_check(st) == 0
    return li


@pytest.mark.parametrize("name", ["tiny", "ragged", "small3", "hd"])
@pytest.mark.parametrize("ppt", [1, 2, 4])
def test_raster_fwd_and_l1_stagewise(oracle_mod, name, ppt):
    if name == "hd" and ppt != 2:
        pytest.skip("hd case runs once")
    part = None if name != "tiny" else (lambda TW, TH: (3, 2, TW - 1, TH - 5))
    li = _fwd_case(oracle_mod, name, part, ppt)
    ph, pw = li.ph, li.pw
    flags = li.to_leaf(li.fw["flags"])
    ok = (flags & 0x81) == 0
    img_o = li.to_leaf(li.fw["img"], 3)
    img = li.img.cpu().numpy().reshape(3, ph, pw)
    err = rel_err(img, img_o)[:, ok]
    assert err.max() <= IMG_TOL, err.max()
    assert (~ok).sum() <= max(3, ok.size // 500)
    T_o = li.to_leaf(li.fw["T"])
    T = li.Tf.cpu().numpy().reshape(ph, pw)
    last_o = li.to_leaf(li.fw["last"])
    # fp32 transmittance: the oracle's per-pixel bound of the fp32 error
    # (per factor: alpha / (1 - alpha) x alpha's relative error, + 1 ulp)
    T_bound = 1e-6 + 2.0 * li.to_leaf(li.fw["T_err"])
    assert (rel_err(T, T_o, floor=1e-4) <= T_bound)[ok].all()
    assert (li.last.cpu().numpy().reshape(ph, pw)[ok] == last_o[ok]).all()
    # L1 terms: dL = sign(r - t) / (3 W H) and the per-tile loss sums
    W, H = li.cam.width, li.cam.height
    tg = li.target[:, li.py0:li.py0 + ph, li.px0:li.px0 + pw].astype(np.float64)
    diff_o = img_o - tg
    dL = li.dL.cpu().numpy().reshape(3, ph, pw)
    clear = ok[None] & (np.abs(diff_o) > 1e-5)
    assert (np.sign(dL[clear]) == np.sign(diff_o[clear])).all()
    np.testing.assert_allclose(np.abs(dL[clear]), 1.0 / (3 * W * H), rtol=1e-7)
    lt = li.loss_tiles.cpu().numpy()
    for j, t in enumerate(li.tiles[:50]):
        ty, tx = divmod(int(t), li.TW)
        ys = slice(ty * 16 - li.py0, min(ty * 16 + 16, H) - li.py0)
        xs = slice(tx * 16 - li.px0, min(tx * 16 + 16, W) - li.px0)
        if not ok[ys, xs].all():
            continue
        exp = np.abs(diff_o[:, ys, xs]).sum() / (3 * W * H)
        assert abs(lt[t] - exp) <= IMG_TOL * max(exp, 1e-3 / (3 * W * H) * 256)


@pytest.mark.parametrize("name", ["tiny", "ragged", "small3", "hd"])
@pytest.mark.parametrize("ppt", [1, 2, 4])
def test_raster_bwd_stagewise(oracle_mod, name, ppt):
    if name == "hd" and ppt != 2:
        pytest.skip("hd case runs once")
    sc, cam = scene(name)
    TW, TH = oracle_mod.grid(cam)
    L = (0, 0, TW, TH)
    target = synth.random_image(cam.width, cam.height, 3) * 0.6
    li = LeafInputs(oracle_mod, sc, cam, L, target)
    W, H = cam.width, cam.height
    # inputs from the oracle's forward: T_final, last and dL (zeroed on
    # pixels whose decisions sit within the margin of a threshold)
    ok_t = (li.fw["flags"] & 0x81) == 0
    tg = oracle_mod.gather_tiles(np.pad(target, ((0, 0), (0, TH * 16 - H), (0, TW * 16 - W))),
                                 li.tiles, TW, 3)
    dL_t = np.sign(li.fw["img"] - tg) / (3.0 * W * H) * ok_t[:, None, :]
    g2d_o = oracle_mod.raster_bwd(li.pr["rec"], TW, W, H, li.tiles, li.off, li.vals_o, dL_t)
    px = li.buffers()
    li.Tf.copy_(torch.as_tensor(li.to_leaf(li.fw["T"]).astype(np.float32).reshape(-1)))
    li.last.copy_(torch.as_tensor(li.to_leaf(li.fw["last"]).astype(np.int32).reshape(-1)))
    li.dL.copy_(torch.as_tensor(li.to_leaf(dL_t, 3).astype(np.float32).reshape(-1)))
    C = len(li.pr["cand_idx"])
    g2d = torch.zeros(max(C, 1) * 12, device="cuda")
    b = B()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.gs_raster_bwd(li.pb.struct, li.vals, li.ranges, L, b.camera_struct(cam), px, g2d, st, ppt)
    assert b.gs_check(st) == 0
    g = g2d.cpu().numpy().reshape(-1, 12)[:C]
    names = ["du", "dv", "da", "db", "dc", "do", "dR", "dG", "dB"]
    for f in range(9):
        e = rel_l2(g[:, f], g2d_o[:, f])
        assert e <= GRAD_TOL, (names[f], e)
    assert np.all(g[:, 9:] == 0)


def test_raster_fwd_leaf_buffers_and_empty_tiles(oracle_mod):
    """A Leaf over a corner with empty tiles: background 0, T = 1, last = 0."""
    sc, cam = scene("tiny")
    s2 = sc.copy()
    s2.params[0, :s2.n] = np.abs(s2.params[0, :s2.n]) + 0.3  # empty left half
    _SCENES["tiny_right"] = (s2, cam)
    li = _fwd_case(oracle_mod, "tiny_right", lambda TW, TH: (0, 0, 4, TH))
    img = li.img.cpu().numpy().reshape(3, li.ph, li.pw)
    img_o = li.to_leaf(li.fw["img"], 3)
    empty = li.to_leaf(li.fw["n_eval"]) == 0
    assert empty.any()
    assert (img[:, empty] == 0).all()
    assert (li.Tf.cpu().numpy().reshape(li.ph, li.pw)[empty] == 1).all()
    assert rel_err(img, img_o).max() <= IMG_TOL


# ---------------------------------------------------------------------------
# projection backward and Adam on generated gradients
# ---------------------------------------------------------------------------

GROUPS = [("mean", 0, 3), ("log_scale", 3, 6), ("quat", 6, 10), ("logit", 10, 11),
          ("sh_dc", 11, 14), ("sh_rest", 14, None)]


@pytest.mark.parametrize("name", ["tiny", "small3", "hd"])
def test_project_bwd_stagewise(oracle_mod, name):
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    C = len(pr["cand_idx"])
    rng = np.random.default_rng(1)
    g2d = rng.normal(size=(C, 9)) * np.array([1e-3, 1e-3, 1e-1, 1e-1, 1e-1, 1e-3, 1e-3, 1e-3, 1e-3])
    g2d = g2d.astype(np.float32)
    g3d_o = oracle_mod.project_bwd(sc.params.astype(np.float64), sc.sh_degree, cam,
                                   pr["cand_idx"], g2d.astype(np.float64))
    pb = ProjBuffers.from_oracle(pr, sc.n)
    b = B()
    params = torch.as_tensor(sc.params).cuda()
    model = b.gs_model(sc.n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
    g2 = np.zeros((C, 12), np.float32)
    g2[:, :9] = g2d
    g2d_d = torch.as_tensor(g2.reshape(-1)).cuda()
    g3d = torch.zeros(sc.P * C, device="cuda")
    b.gs_project_bwd(model, b.camera_struct(cam), pb.struct, C, g2d_d, g3d=g3d, g3d_stride=C)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert b.gs_check(st) == 0
    g = g3d.cpu().numpy().reshape(sc.P, C)
    for gname, a, e in GROUPS:
        e = sc.P if e is None else e
        if e <= a:
            continue
        assert rel_l2(g[a:e], g3d_o[a:e]) <= 1e-6, gname


def test_adam_dense_and_compact(oracle_mod):
    b = B()
    rng = np.random.default_rng(2)
    P, n, n_pad = 14, 5000, 5056
    p = rng.normal(size=(P, n_pad)).astype(np.float32)
    m = (rng.normal(size=(P, n_pad)) * 1e-3).astype(np.float32)
    v = (rng.uniform(0, 1e-5, size=(P, n_pad))).astype(np.float32)
    g = (rng.normal(size=(P, n_pad)) * 10.0 ** rng.uniform(-7, 0, (P, n_pad))).astype(np.float32)
    def check(pd, md, vd, g_used, step):
        pe, me, ve = oracle_mod.adam(p, m, v, g_used, step=step)
        gm = np.abs(g_used[:, :n])
        # m, v: two terms that can cancel; bound by the terms' magnitude
        m_scale = 0.9 * np.abs(m[:, :n]) + 0.1 * gm
        v_scale = 0.999 * v[:, :n] + 0.001 * gm * gm
        mg, vg, pg = (x.cpu().numpy().astype(np.float64) for x in (md, vd, pd))
        assert (np.abs(mg[:, :n] - me[:, :n]) <= 1e-6 * m_scale + 1e-30).all()
        assert (np.abs(vg[:, :n] - ve[:, :n]) <= 1e-6 * v_scale + 1e-30).all()
        # p: the update formula applied to the kernel's own m and v
        pe2 = p[:, :n] - 1e-3 * (mg[:, :n] / (1 - 0.9 ** step)) / (
            np.sqrt(vg[:, :n] / (1 - 0.999 ** step)) + 1e-8)
        assert (np.abs(pg[:, :n] - pe2) <= 1e-6 * np.abs(p[:, :n]) + 1e-8).all()
        assert (pg[:, n:] == p[:, n:]).all()

    for step in (1, 7):
        args = b.gs_adam_args(1e-3, 0.9, 0.999, 1e-8, step, 0)
        pd, md, vd = (torch.as_tensor(x).cuda() for x in (p, m, v))
        b.gs_adam(pd, md, vd, torch.as_tensor(g).cuda(), n_pad, None, n, n_pad, P, args)
        check(pd, md, vd, g.astype(np.float64), step)
    # compact gradient through a slot map (-1 = no gradient)
    slot = np.where(rng.uniform(size=n) < 0.6, 0, -1).astype(np.int32)
    cand = np.nonzero(slot >= 0)[0]
    slot[cand] = np.arange(len(cand))
    gc = np.ascontiguousarray(g[:, cand])
    pd, md, vd = (torch.as_tensor(x).cuda() for x in (p, m, v))
    args = b.gs_adam_args(1e-3, 0.9, 0.999, 1e-8, 3, 0)
    b.gs_adam(pd, md, vd, torch.as_tensor(gc).cuda(), len(cand), torch.as_tensor(slot).cuda(), n,
              n_pad, P, args)
    gd = np.zeros((P, n_pad))
    gd[:, cand] = gc
    check(pd, md, vd, gd, 3)


@pytest.mark.parametrize("name", ["small3", "hd"])
def test_fused_project_bwd_adam(oracle_mod, name):
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    C = len(pr["cand_idx"])
    rng = np.random.default_rng(3)
    g2d = (rng.normal(size=(C, 9)) * 1e-3).astype(np.float32)
    g3d_o = oracle_mod.project_bwd(sc.params.astype(np.float64), sc.sh_degree, cam,
                                   pr["cand_idx"], g2d.astype(np.float64))
    grad = np.zeros((sc.P, sc.n_pad))
    grad[:, pr["cand_idx"]] = g3d_o
    m0 = (rng.normal(size=sc.params.shape) * 1e-4).astype(np.float32)
    v0 = rng.uniform(0, 1e-7, size=sc.params.shape).astype(np.float32)
    pe, me, ve = oracle_mod.adam(sc.params, m0, v0, grad, step=2)
    b = B()
    pb = ProjBuffers.from_oracle(pr, sc.n)
    params = torch.as_tensor(sc.params).cuda()
    md, vd = torch.as_tensor(m0).cuda(), torch.as_tensor(v0).cuda()
    model = b.gs_model(sc.n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
    g2 = np.zeros((C, 12), np.float32)
    g2[:, :9] = g2d
    geo = torch.zeros(14 * C, device="cuda")
    b.gs_project_bwd(model, b.camera_struct(cam), pb.struct, C, torch.as_tensor(g2.reshape(-1)).cuda(),
                     g3d=geo, g3d_stride=geo.numel(), adam_m=md, adam_v=vd,
                     fused=b.gs_adam_args(1e-3, 0.9, 0.999, 1e-8, 2, 0))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert b.gs_check(st) == 0
    n = sc.n
    ci = pr["cand_idx"]
    md_h, vd_h, pd_h = md.cpu().numpy(), vd.cpu().numpy(), params.cpu().numpy()
    # 1. the candidates' geometric gradients (scratch planes 3..10, fp32
    #    chain) against the oracle: relative L2 per tensor
    raw = geo.cpu().numpy()
    g_rest = raw[6 * C:14 * C].reshape(8, C).astype(np.float64)
    for k in range(8):
        assert rel_l2(g_rest[k], g3d_o[3 + k]) <= GRAD_TOL, 3 + k
    # 2. Adam on those planes: element-wise against the update of the
    #    kernel's own gradients.  m and v are sums of two terms that can
    #    cancel: the bound follows the magnitude of the terms
    own = grad.copy()
    own[3:11, ci] = g_rest
    pe2, me2, ve2 = oracle_mod.adam(sc.params, m0, v0, own, step=2)
    gm = np.abs(own[:, :n])
    m_scale = 0.9 * np.abs(m0[:, :n]) + 0.1 * gm
    v_scale = 0.999 * v0[:, :n] + 0.001 * gm * gm
    rows = np.r_[3:11, 11:sc.P]   # geometric planes (own g) and SH planes (fp64 g)
    assert (np.abs(md_h[rows, :n] - me2[rows, :n]) <= 1e-6 * m_scale[rows] + 1e-30).all()
    assert (np.abs(vd_h[rows, :n] - ve2[rows, :n]) <= 1e-6 * v_scale[rows] + 1e-30).all()
    np.testing.assert_allclose(pd_h[rows, :n], pe2[rows, :n], rtol=1e-6, atol=2e-8)
    # 3. the SH planes' gradients equal the oracle's (the same m as above)
    assert (np.abs(me2[11:, :n] - me[11:, :n]) <= 1e-6 * m_scale[11:] + 1e-30).all()
    # 4. the mean planes (geometric + view-direction terms): the gradient
    #    implied by m against the oracle, relative L2 per tensor
    g_mean = (md_h[0:3, :n].astype(np.float64) - 0.9 * m0[0:3, :n]) / 0.1
    for k in range(3):
        assert rel_l2(g_mean[k, ci], grad[k, ci]) <= GRAD_TOL, k


@pytest.mark.parametrize("name", ["small3", "hd"])
def test_fused_project_bwd_adam_in_stream(oracle_mod, name):
    """g3d = NULL: the geometric chain runs inside the Adam stream.  The
    gradients implied by the updated m (g = (m - 0.9 m0) / 0.1) match the
    oracle's per tensor, and the SH planes match the two-pass form."""
    sc, cam = scene(name)
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    C = len(pr["cand_idx"])
    rng = np.random.default_rng(4)
    g2d = (rng.normal(size=(C, 9)) * 1e-3).astype(np.float32)
    g3d_o = oracle_mod.project_bwd(sc.params.astype(np.float64), sc.sh_degree, cam,
                                   pr["cand_idx"], g2d.astype(np.float64))
    m0 = (rng.normal(size=sc.params.shape) * 1e-4).astype(np.float32)
    v0 = rng.uniform(0, 1e-7, size=sc.params.shape).astype(np.float32)
    b = B()
    pb = ProjBuffers.from_oracle(pr, sc.n)
    g2 = np.zeros((C, 12), np.float32)
    g2[:, :9] = g2d
    g2_d = torch.as_tensor(g2.reshape(-1)).cuda()
    out = []
    for two_pass in (False, True):
        params = torch.as_tensor(sc.params).cuda()
        md, vd = torch.as_tensor(m0).cuda(), torch.as_tensor(v0).cuda()
        model = b.gs_model(sc.n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
        geo = torch.zeros(14 * C, device="cuda") if two_pass else None
        b.gs_project_bwd(model, b.camera_struct(cam), pb.struct, C, g2_d, g3d=geo,
                         g3d_stride=geo.numel() if two_pass else 0, adam_m=md, adam_v=vd,
                         fused=b.gs_adam_args(1e-3, 0.9, 0.999, 1e-8, 2, 0))
        torch.cuda.synchronize()
        out.append((params.cpu().numpy(), md.cpu().numpy(), vd.cpu().numpy()))
    (p1, m1, v1), (p2, m2, v2) = out
    n = sc.n
    ci = pr["cand_idx"]
    g_impl = (m1[:, :n].astype(np.float64) - 0.9 * m0[:, :n]) / 0.1
    for k in range(11):
        assert rel_l2(g_impl[k, ci], g3d_o[k]) <= GRAD_TOL, k
    np.testing.assert_allclose(m1[11:, :n], m2[11:, :n], rtol=1e-6, atol=1e-30)
    np.testing.assert_allclose(p1[11:, :n], p2[11:, :n], rtol=1e-6, atol=2e-8)
    # non-candidates: m, v decay and p moves by the same dense rule in both
    nc = np.setdiff1d(np.arange(n), ci)
    assert np.array_equal(m1[:, nc], m2[:, nc]) and np.array_equal(v1[:, nc], v2[:, nc])


# ---------------------------------------------------------------------------
# end to end through the Step driver
# ---------------------------------------------------------------------------

class Capture:
    def __init__(self, W, H):
        self.img = np.zeros((3, H, W), np.float32)
        self.T = np.zeros((H, W), np.float32)
        self.last = np.zeros((H, W), np.int32)

    def on_leaf(self, ctx, lc):
        x0, y0, w, h = lc["px_rect"]
        self.img[:, y0:y0 + h, x0:x0 + w] = lc["img"][:3 * w * h].view(3, h, w).cpu().numpy()
        self.T[y0:y0 + h, x0:x0 + w] = lc["T_final"][:w * h].view(h, w).cpu().numpy()
        self.last[y0:y0 + h, x0:x0 + w] = lc["last"][:w * h].view(h, w).cpu().numpy()

    def on_bwd(self, ctx):
        self.g2d = ctx["g2d"].cpu().numpy().reshape(-1, 12)
        self.cand_idx = ctx["cand_idx"][:ctx["n_cand"]].cpu().numpy()


def implied_grad(m, beta1=0.9):
    """The gradient of a first Adam step from its first moment: with m0 = 0,
    m1 = (1 - beta1) g (one fp32 rounding), so g = m1 / (1 - beta1) to about
    1e-7 relative.  Unlike the step-1 parameter update, which is about
    p - lr sign(g), it carries the gradient's magnitude."""
    return np.asarray(m, np.float64) / float(np.float32(1.0 - beta1))


def check_grad_groups(g_impl, g_ref, n, P, tol=GRAD_TOL):
    """Relative L2 per parameter group (mean, log-scale, quaternion, logit,
    SH DC, SH rest) over the n Gaussians."""
    for gname, a, e in GROUPS:
        e = P if e is None else e
        if e <= a:
            continue
        err = rel_l2(g_impl[a:e, :n], g_ref[a:e, :n])
        assert err <= tol, (gname, err)


@pytest.mark.parametrize("name,budget,binning,mode,streams,fuse", [
    ("tiny", 384 << 20, "fused", "bounded", 1, False),
    ("tiny", 120_000, "fused", "bounded", 1, False),
    ("tiny", 120_000, "expand", "bounded", 1, False), ("tiny", 120_000, "sort", "bounded", 1, False),
    ("ragged", 30_000, "fused", "bounded", 1, False),
    ("small3", 200_000, "fused", "bounded", 1, False),
    ("small3", 200_000, "sort", "bounded", 1, False),
    ("hd", 384 << 20, "fused", "bounded", 1, False), ("hd", 20 << 20, "fused", "bounded", 1, False),
    ("hd", 20 << 20, "expand", "bounded", 1, False), ("hd", 20 << 20, "sort", "bounded", 1, False),
    ("tiny", 120_000, "fused", "original", 1, False),
    ("ragged", 30_000, "sort", "original", 1, False),
    ("hd", 20 << 20, "fused", "original", 1, False),
    # two Leaves in flight on two streams with two raster arenas
    ("tiny", 120_000, "fused", "bounded", 2, False), ("ragged", 30_000, "fused", "bounded", 2, False),
    ("small3", 200_000, "expand", "bounded", 2, False), ("hd", 20 << 20, "fused", "bounded", 2, False),
    ("hd", 20 << 20, "sort", "bounded", 2, False),
    # projection backward fused with the view's Adam update (the bench's path)
    ("tiny", 120_000, "fused", "bounded", 1, True), ("ragged", 30_000, "fused", "bounded", 2, True),
    ("small3", 200_000, "fused", "bounded", 2, True), ("hd", 384 << 20, "fused", "bounded", 1, True),
    ("hd", 20 << 20, "fused", "bounded", 2, True), ("hd", 20 << 20, "sort", "bounded", 1, "in_stream")])
def test_end_to_end_step(oracle_mod, name, budget, binning, mode, streams, fuse):
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene(name)
    target = synth.random_image(cam.width, cam.height, 12) * 0.6
    ref = oracle_mod.step(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam,
                          target.astype(np.float64))
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=budget, fuse_adam=fuse, binning=binning, mode=mode,
                  leaf_streams=streams)
    cap = Capture(cam.width, cam.height)
    stats = stp.run_view(cam, torch.as_tensor(target).cuda(), hooks=cap)
    stp.check()
    if mode == "original":
        assert stats.n_leaves == 1 and stats.n_cand == sc.n
        live = np.isin(np.arange(sc.n), ref["proj"]["cand_idx"])
        cap.cand_idx = np.arange(sc.n)[live]
        cap.g2d = cap.g2d[:sc.n][live]
    elif budget < (384 << 20):
        assert stats.n_leaves > 1
    assert stats.n_isect == ref["n_isect"]
    ok = (ref["pflags"] & 0x81) == 0
    assert rel_err(cap.img, ref["img"])[:, ok].max() <= IMG_TOL
    assert (cap.last[ok] == ref["last"][ok]).all()
    loss = stp.last_loss()
    assert abs(loss - ref["loss"]) <= IMG_TOL * ref["loss"]
    # gradients through the compact g2d and projection backward
    for f in range(9):
        assert rel_l2(cap.g2d[:len(cap.cand_idx), f], ref["g2d"][:, f]) <= GRAD_TOL, f
    # the 3D gradient with its magnitude, from Adam's first moment
    check_grad_groups(implied_grad(model.m.cpu().numpy()), ref["grad"], sc.n, sc.P)
    # parameters after one Adam step where the gradient is clearly non-zero
    p = model.params.cpu().numpy()
    g = ref["grad"]
    for gname, a, e in GROUPS:
        e = sc.P if e is None else e
        if e <= a:
            continue
        gg = g[a:e, :sc.n]
        mask = np.abs(gg) > 1e-3 * np.abs(gg).max()
        d = np.abs(p[a:e, :sc.n] - ref["params"][a:e, :sc.n])
        assert d[mask].max() <= 1e-5, gname
        assert d.max() <= 2.1e-3, gname  # at most one sign flip of a ~zero gradient


@pytest.mark.parametrize("name,budget,streams", [("small3", 200_000, 1), ("small3", 384 << 20, 2),
                                                 ("hd", 20 << 20, 2), ("tiny", 120_000, 1)])
def test_work_counters_match_oracle(oracle_mod, name, budget, streams):
    """The raster kernels' accounting counters, the numerator of the
    roofline, against the oracle: the forward's [2] is the method's
    evaluations, each pixel's list entries up to and including the one it
    stops at (its whole list if it never stops) = the sum of the oracle's
    per-pixel n_eval; [3] = the sum of last = the backward's evaluations.
    Exact, except that a pixel the oracle flags as within rounding of a
    threshold decision may differ by at most its list length.  The
    backward's pairs differentiated equal the forward's pairs composited."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene(name)
    target = synth.random_image(cam.width, cam.height, 12) * 0.6
    ref = oracle_mod.step(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam,
                          target.astype(np.float64))
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=budget, leaf_streams=streams)
    counters = torch.zeros(6, dtype=torch.int64, device="cuda")
    cap = Capture(cam.width, cam.height)
    stats = stp.run_view(cam, torch.as_tensor(target).cuda(), hooks=cap, counters=counters,
                         update=False)
    stp.check()
    cnt = [int(x) for x in counters.cpu()]
    near = (ref["pflags"] & 1) != 0
    slack = int(ref["list_len"][near].sum())
    # the counter is the sum of the per-pixel last buffer, which matches the
    # oracle pixel by pixel away from threshold decisions
    assert cnt[3] == int(cap.last.astype(np.int64).sum())
    assert (cap.last[~near] == ref["last"][~near]).all()
    e_fwd, e_bwd = int(ref["n_eval_px"].sum()), int(ref["last"].astype(np.int64).sum())
    assert e_fwd == ref["n_eval"]
    assert abs(cnt[2] - e_fwd) <= slack, (cnt[2], e_fwd, slack)
    assert abs(cnt[3] - e_bwd) <= slack, (cnt[3], e_bwd, slack)
    if slack == 0:
        assert cnt[2] == e_fwd and cnt[3] == e_bwd
    # pairs: evaluated >= composited; the backward differentiates exactly
    # the composited pairs, and evaluates at most the entries before last
    assert cnt[0] >= cnt[1] and cnt[5] == cnt[1]
    assert cnt[4] <= cnt[3] and cnt[1] <= cnt[3]
    if name != "tiny":
        assert stats.n_leaves >= 1


@pytest.mark.parametrize("name,part", [("ragged", None), ("tiny", (3, 2, 13, 11)),
                                       ("small3", (0, 3, 5, 8))])
def test_loss_l1_stagewise(oracle_mod, name, part):
    """gs_loss_l1 on its own against the oracle's L1: dL/dimg = sign(r - t) /
    (3 W H) with sign(0) = 0 (some pixels are set equal to the target), the
    per-tile loss sums, and their fixed-order total (gs_loss_total) = the
    loss of the Leaf's pixels."""
    b = B()
    sc, cam = scene(name)
    W, H = cam.width, cam.height
    TW, TH = oracle_mod.grid(cam)
    L = (0, 0, TW, TH) if part is None else part
    x0, y0, x1, y1 = L
    px0, py0 = 16 * x0, 16 * y0
    pw, ph = min(16 * x1, W) - px0, min(16 * y1, H) - py0
    rng = np.random.default_rng(21)
    target = synth.random_image(W, H, 22)
    img = rng.uniform(0, 1, (3, ph, pw)).astype(np.float32)
    eq = rng.uniform(size=(3, ph, pw)) < 0.05
    img[eq] = target[:, py0:py0 + ph, px0:px0 + pw][eq]
    img_d = torch.as_tensor(img.reshape(-1)).cuda()
    Tf = torch.zeros(pw * ph, device="cuda")
    last = torch.zeros(pw * ph, dtype=torch.int32, device="cuda")
    dL = torch.full((3 * pw * ph,), 7.0, device="cuda")
    lt = torch.zeros(TW * TH, device="cuda")
    tgt = torch.as_tensor(target).cuda()
    norm = 1.0 / (3.0 * W * H)
    px = b.pixels(px0, py0, pw, ph, img_d, Tf, last, dL, target=tgt, target_origin=(0, 0),
                  target_pitch=W, target_plane=W * H, loss_tiles=lt, norm=norm)
    b.gs_loss_l1(px, L, b.camera_struct(cam))
    tot = torch.zeros(1, dtype=torch.float64, device="cuda")
    b.gs_loss_total(lt, TW * TH, tot)
    torch.cuda.synchronize()
    tcrop = target[:, py0:py0 + ph, px0:px0 + pw]
    loss_o, dL_o = oracle_mod.loss_l1(img, tcrop, 3.0 * W * H)
    got = dL.cpu().numpy().reshape(3, ph, pw)
    assert (np.sign(got) == np.sign(dL_o)).all()
    assert (got[eq] == 0).all()
    np.testing.assert_allclose(np.abs(got[~eq]), np.float32(norm), rtol=1e-7)
    ltn = lt.cpu().numpy()
    for ty in range(y0, y1):
        for tx in range(x0, x1):
            ys = slice(16 * ty - py0, min(16 * ty + 16, H) - py0)
            xs = slice(16 * tx - px0, min(16 * tx + 16, W) - px0)
            exp = np.abs(img[:, ys, xs].astype(np.float64) - tcrop[:, ys, xs]).sum() * norm
            assert abs(ltn[ty * TW + tx] - exp) <= IMG_TOL * exp + 1e-12
    outside = np.ones((TH, TW), bool)
    outside[y0:y1, x0:x1] = False
    assert (ltn.reshape(TH, TW)[outside] == 0).all()
    assert abs(float(tot.item()) - loss_o) <= IMG_TOL * loss_o


@pytest.mark.parametrize("streams", [1, 2])
def test_host_target_matches_resident_target(streams):
    """The bounded supply of a pinned host target (per-Leaf crops uploaded on a
    copy stream, double-buffered) gives the same loss and last as the
    resident target, and the same gradients up to atomic order; with one or
    two Leaf streams."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    tgt = synth.random_image(cam.width, cam.height, 8) * 0.5
    outs = []
    for host in (False, True):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=6 << 20, leaf_streams=streams)
        t = torch.as_tensor(tgt).pin_memory() if host else torch.as_tensor(tgt).cuda()
        cap = Capture(cam.width, cam.height)
        stats = stp.run_view(cam, t, hooks=cap)
        stp.check()
        assert stats.n_leaves >= 3
        outs.append((stp.last_loss(), cap.last.copy(), cap.g2d.copy(), model.params.cpu().numpy()))
    (l0, last0, g0, p0), (l1, last1, g1, p1) = outs
    assert l0 == l1 and (last0 == last1).all()
    for f in range(9):
        assert rel_l2(g1[:, f], g0[:, f]) <= 1e-5
    # Adam moves a parameter by about lr whatever the gradient's size, so an
    # atomic-order sign flip of a ~zero gradient moves it by up to 2 lr
    assert np.abs(p1 - p0).max() <= 2.1e-3


@pytest.mark.parametrize("bound", [False, True])
def test_target_prefetcher_matches_resident_targets(bound):
    """Views fed by TargetPrefetcher (each target uploaded from pinned host
    memory during the previous view's step, two device buffers) take the same
    steps as views whose targets are resident, over a sequence that reuses
    both buffers; bound: the prefetcher knows the Stepper and issues each
    upload after the current view's projection tables reached the host."""
    from gaussian_splatting_differentiable_dgs_b200.step import (GaussianModel, Stepper,
                                                                  TargetPrefetcher)
    sc, cam = scene("small3")
    tg = [synth.random_image(cam.width, cam.height, 20 + k) * 0.5 for k in range(3)]
    order = [0, 1, 2, 1, 0]
    outs = []
    for prefetch in (False, True):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=100_000, leaf_streams=2)
        losses = []
        if prefetch:
            host = [torch.as_tensor(t).pin_memory() for t in tg]
            supply = TargetPrefetcher(host, stepper=stp if bound else None).iterate(order)
        else:
            dev = [torch.as_tensor(t).cuda() for t in tg]
            supply = ((v, dev[v]) for v in order)
        for v, t in supply:
            stp.run_view(cam, t)
            losses.append(stp.last_loss())
        stp.check()
        outs.append((losses, model.params.cpu().numpy()))
    (l0, p0), (l1, p1) = outs
    # the first loss is bit-identical; later ones follow parameters that differ
    # by the atomic order of the earlier steps' compact gradients
    assert l0[0] == l1[0]
    assert all(abs(a - b) <= 1e-5 * abs(a) for a, b in zip(l0, l1))
    assert np.abs(p1 - p0).max() <= 2.1e-3 * len(order)
    assert np.median(np.abs(p1 - p0)) <= 1e-6


def test_two_leaf_streams_working_set():
    """Two Leaves in flight hold at most one more Leaf arena than one Leaf at
    a time, and both release the raster buffers before projection backward
    (the same loss either way)."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    target = torch.as_tensor(synth.random_image(cam.width, cam.height, 6) * 0.5).cuda()
    out = {}
    for streams in (1, 2):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=6 << 20, leaf_streams=streams)
        stats = stp.run_view(cam, target)
        stp.check()
        assert stats.n_leaves >= 3
        out[streams] = (stats, stp.last_loss())
    (s1, l1), (s2, l2) = out[1], out[2]
    assert l1 == l2
    # a bounded run's arena holds 1/16 headroom over its largest Leaf (at most
    # the Leaf budget, or an over-budget Leaf's size)
    arena = max(min(6 << 20, s1.arena_bytes + s1.arena_bytes // 16), s1.arena_bytes)
    assert s2.peak_ws_bytes <= s1.peak_ws_bytes + arena + (1 << 20)


def test_leaf_invariance_gpu(oracle_mod):
    """Any Leaf partition: bit-identical image and loss, the same summed
    gradients (atomics reorder only)."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("small3")
    target = torch.as_tensor(synth.random_image(cam.width, cam.height, 5) * 0.5).cuda()
    TW, TH = (cam.width + 15) // 16, (cam.height + 15) // 16
    parts = [None, [(0, 0, TW, TH)],
             [(x, y, x + 1, y + 1) for y in range(TH) for x in range(TW)],
             [(0, 0, 3, TH), (3, 0, TW, 4), (3, 4, TW, TH)]]
    outs = []
    # the multi-Leaf partitions also with two Leaves in flight (two streams)
    for leaves, streams in [(q, 1) for q in parts] + [(parts[2], 2), (parts[3], 2)]:
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=100_000, leaf_streams=streams)
        cap = Capture(cam.width, cam.height)
        stp.run_view(cam, target, leaves=leaves, hooks=cap, update=False)
        stp.check()
        outs.append((cap.img.copy(), cap.last.copy(), stp.last_loss(), cap.g2d.copy()))
    img0, last0, loss0, g0 = outs[0]
    for img, last, loss, g in outs[1:]:
        assert (img == img0).all() and (last == last0).all()
        assert loss == loss0
        for f in range(9):
            assert rel_l2(g[:, f], g0[:, f]) <= 1e-5


# ---------------------------------------------------------------------------
# region projection and the grouped / fixed-block schedules
# ---------------------------------------------------------------------------

def test_project_region_matches_oracle(oracle_mod):
    """gs_project_region against the oracle's projection: the candidates whose
    rect meets the region (ascending index), their rects clipped to it, the
    oracle's records, the SAT of the clipped rects, and the 3-sigma count of
    the view's candidates' squares inside the region."""
    sc, cam = scene("hd")
    b = B()
    pr = oracle_mod.project(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam)
    rect = pr["rect"].astype(np.int64)
    near = (pr["flags"] & 1) != 0
    ro = pr["rec"]
    exp_rec = encode_records(ro)
    u, v, rad = ro[:, 0], ro[:, 1], ro[:, 3]
    TW, TH = oracle_mod.grid(cam)
    square = np.stack([np.floor((u - rad) / 16), np.floor((v - rad) / 16),
                       np.floor((u + rad) / 16) + 1, np.floor((v + rad) / 16) + 1], 1)
    square = np.clip(square, 0, [TW, TH, TW, TH]).astype(np.int64)
    params = torch.as_tensor(sc.params).cuda()
    model = b.gs_model(sc.n, sc.n_pad, sc.sh_degree, 0, params.data_ptr())
    for region in [(0, 0, TW, TH), (3, 5, 41, 30), (TW - 7, TH - 3, TW, TH), (10, 10, 11, 11)]:
        x0, y0, x1, y1 = region
        clip = lambda r: np.stack([np.clip(r[:, 0], x0, x1), np.clip(r[:, 1], y0, y1),
                                   np.clip(r[:, 2], x0, x1), np.clip(r[:, 3], y0, y1)], 1)
        cr = clip(rect)
        keep = (cr[:, 2] > cr[:, 0]) & (cr[:, 3] > cr[:, 1])
        pb = ProjBuffers(sc.n)
        sat = torch.zeros((TH + 1) * (TW + 1), dtype=torch.int64, device="cuda")
        ws = torch.empty(b.gs_project_workspace_size(sc.n, cam.width, cam.height),
                         dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        b.gs_project_region(model, b.camera_struct(cam), region, pb.struct, sat, ws, st)
        assert b.gs_check(st) == 0
        Cr = int(pb.n_cand.item())
        assert Cr == keep.sum()
        assert (pb.cand_idx[:Cr].cpu().numpy() == pr["cand_idx"][keep]).all()
        got_rect = pb.rect[:4 * Cr].cpu().numpy().reshape(-1, 4)
        nk = near[keep]
        assert (got_rect[~nk] == cr[keep][~nk]).all()
        got = pb.rec[:12 * Cr].cpu().numpy().reshape(-1, 12)
        d = decode_records(got)
        assert np.abs(d["u"] - u[keep]).max() <= 2.5e-7 + 1e-12 * np.abs(u).max()
        assert np.abs(d["v"] - v[keep]).max() <= 2.5e-7 + 1e-12 * np.abs(v).max()
        for col in (4, 5, 6, 7, 8, 9, 10, 11):
            assert rel_err(got[:, col], exp_rec[keep][:, col], floor=1e-30).max() <= 2.4e-7, col
        if not nk.any():
            exp_sat = oracle_mod.sat(oracle_mod.tile_counts_fast(cr[keep], TW, TH))
            assert (sat.cpu().numpy().reshape(TH + 1, TW + 1) == exp_sat).all()
        sq = clip(square)
        exp_sq = int(((sq[:, 2] - sq[:, 0]) * (sq[:, 3] - sq[:, 1])).sum())
        assert int(pb.square.item()) == exp_sq


def test_grad_accumulate_matches_oracle():
    """gs_grad_accumulate: G[:, cand_idx[j]] += g3d[:, j], one fp32 add per
    element (a Gaussian is at most one candidate of a projection), so the
    result equals numpy's fp32 scatter-add bit for bit; other columns and
    the padding are untouched; repeated calls accumulate."""
    b = B()
    rng = np.random.default_rng(31)
    P, n, n_pad = 59, 5000, 5056
    C, stride = 1234, 1300
    idx = np.sort(rng.choice(n, C, replace=False)).astype(np.int32)
    g3d = rng.normal(size=(P, stride)).astype(np.float32)
    G0 = rng.normal(size=(P, n_pad)).astype(np.float32)
    G = torch.as_tensor(G0.copy()).cuda()
    gd = torch.as_tensor(g3d).cuda()
    idd = torch.as_tensor(idx).cuda()
    exp = G0.copy()
    for _ in range(2):
        b.gs_grad_accumulate(gd, stride, idd, C, P, G, n_pad)
        exp[:, idx] = exp[:, idx] + g3d[:, :C]
    torch.cuda.synchronize()
    assert (G.cpu().numpy().view(np.uint32) == exp.view(np.uint32)).all()
    b.gs_grad_accumulate(gd, stride, idd, 0, P, G, n_pad)  # no candidates: no change
    torch.cuda.synchronize()
    assert (G.cpu().numpy().view(np.uint32) == exp.view(np.uint32)).all()


def test_grouped_step_matches_oracle(oracle_mod):
    """3x3 groups (BoundedGS page, section 02 F), each with its own candidate
    projection and Leaves, their gradients summed into one dense gradient,
    then ONE Adam update: against the oracle's step over the whole view (the
    same lists per pixel, so the same image, last and loss; the summed
    gradient within the gradient tolerance, read from Adam's first moment;
    the update)."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    tgt = synth.random_image(cam.width, cam.height, 9) * 0.5
    ref = oracle_mod.step(sc.params.astype(np.float64), sc.n, sc.sh_degree, cam,
                          tgt.astype(np.float64))
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=2 << 20)
    cap = Capture(cam.width, cam.height)
    stats = stp.run_view_grouped(cam, torch.as_tensor(tgt).cuda(), groups=(3, 3), hooks=cap)
    stp.check()
    assert model.step == 1 and stats.n_leaves > 9
    assert stats.n_isect == ref["n_isect"]
    ok = (ref["pflags"] & 0x81) == 0
    assert rel_err(cap.img, ref["img"])[:, ok].max() <= IMG_TOL
    assert (cap.last[ok] == ref["last"][ok]).all()
    assert abs(stp.last_loss() - ref["loss"]) <= IMG_TOL * ref["loss"]
    check_grad_groups(implied_grad(model.m.cpu().numpy()), ref["grad"], sc.n, sc.P)
    p = model.params.cpu().numpy()
    g = np.abs(ref["grad"][:, :sc.n])
    mask = g > 1e-3 * g.max(axis=1, keepdims=True)
    d = np.abs(p[:, :sc.n] - ref["params"][:, :sc.n])
    assert d[mask].max() <= 1e-5
    assert d.max() <= 2.1e-3  # at most one sign flip of a ~zero gradient


def _oracle_blocks(oracle_mod, sc, cam, tgt, regions, lr):
    """The oracle's fixed-block schedule: its step restricted to each block's
    tiles, block after block from the updated parameters, Adam t = 1 .. B."""
    p = sc.params.astype(np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    loss = 0.0
    for k, r in enumerate(regions):
        ref = oracle_mod.step(p, sc.n, sc.sh_degree, cam, tgt.astype(np.float64),
                              leaves=[r], m=m, v=v, t=k + 1, lr=lr)
        p, m, v, loss = ref["params"], ref["m"], ref["v"], loss + ref["loss"]
    return p, m, v, loss


@pytest.mark.parametrize("blocks", [(2, 2), (3, 3)])
@pytest.mark.parametrize("lr", [0.0, 1e-3])
def test_fixed_block_schedule_matches_oracle(oracle_mod, blocks, lr):
    """The fixed-block schedule (BoundedGS page, Figs. 5-6): the view cut into
    a fixed grid, each block a step of its own (its candidates, the view's
    loss normaliser) with its own Adam update, t = 1 .. B, against the oracle
    composing the same schedule.

    With lr = 0 every block's gradient is taken at the same parameters on
    both sides, so Adam's moments (the decayed sum of the blocks' gradients
    and of their squares) meet the gradient tolerance.  With lr = 1e-3 a
    later block sees parameters that differ from the oracle's by the fp32
    rounding of the earlier updates, which can move a pixel across a
    threshold decision; the moments then get a ten times looser bound, and
    the parameters the per-update bound of the single-step tests."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    tgt = synth.random_image(cam.width, cam.height, 4) * 0.5
    TW, TH = oracle_mod.grid(cam)
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=4 << 20, lr=lr)
    stp.run_view_blocks(cam, torch.as_tensor(tgt).cuda(), blocks=blocks)
    stp.check()
    regions = Stepper.split_regions(TW, TH, *blocks)
    nb = len(regions)
    assert model.step == nb and nb == blocks[0] * blocks[1]
    p, m, v, loss = _oracle_blocks(oracle_mod, sc, cam, tgt, regions, lr)
    assert abs(stp.last_loss() - loss) <= IMG_TOL * loss
    n = sc.n
    tol = GRAD_TOL if lr == 0.0 else 10 * GRAD_TOL
    mg, vg = model.m.cpu().numpy(), model.v.cpu().numpy()
    for gname, a, e in GROUPS:
        e = sc.P if e is None else e
        assert rel_l2(mg[a:e, :n], m[a:e, :n]) <= tol, gname
        assert rel_l2(vg[a:e, :n], v[a:e, :n]) <= 2 * tol, gname
    pg = model.params.cpu().numpy()
    if lr == 0.0:
        assert (pg == sc.params).all()
        return
    dp = np.abs(pg[:, :n] - p[:, :n])
    big = np.abs(m[:, :n]) > 1e-3 * np.abs(m[:, :n]).max(axis=1, keepdims=True)
    assert dp[big].max() <= 1e-5 * nb
    # an element whose every block gradient is ~zero can flip sign per step
    assert dp.max() <= 2.1e-3 * nb


def test_candidate_capacity_retry():
    """Candidate buffers sized from a hint below the view's count: the step
    projects again with the exact count and gives the same result."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    tgt = torch.as_tensor(synth.random_image(cam.width, cam.height, 6) * 0.5).cuda()
    outs = []
    for hint in (None, 1000):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=4 << 20)
        if hint is not None:
            stp._cap_hint[None] = hint
        cap = Capture(cam.width, cam.height)
        stats = stp.run_view(cam, tgt, hooks=cap)
        stp.check()
        outs.append((stats.n_cand, cap.img.copy(), cap.last.copy(), stp.last_loss()))
        # the next view of this region is sized from this count
        assert stp._cap_hint[None] >= stats.n_cand
    (c0, i0, l0, s0), (c1, i1, l1, s1) = outs
    assert c0 == c1 > 1000
    assert (i0 == i1).all() and (l0 == l1).all() and s0 == s1


@pytest.mark.parametrize("streams", [1, 2])
def test_gated_step(streams):
    """run_view with a backward gate: a skipped step leaves the parameters
    and the optimizer untouched and reports the forward loss; an accepted
    step equals the ungated one (the Leaves are rendered twice); with one or
    two Leaf streams."""
    from gaussian_splatting_differentiable_dgs_b200.skipgs import BackwardGate
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("hd")
    tgt = torch.as_tensor(synth.random_image(cam.width, cam.height, 3) * 0.5).cuda()
    runs = {}
    for mode in ("plain", "skip", "take"):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=3 << 20, leaf_streams=streams)
        gate = None if mode == "plain" else (lambda loss, m=mode: m == "take")
        stats = stp.run_view(cam, tgt, gate=gate)
        stp.check()
        runs[mode] = (stp.last_loss(), model.params.cpu().numpy(), model.step, stats.n_leaves)
    lp, pp, sp, nl = runs["plain"]
    ls, ps, ss, _ = runs["skip"]
    lt, pt, st_, _ = runs["take"]
    assert nl > 1
    assert ls == lp and lt == lp
    assert ss == 0 and (ps == sc.params).all()
    assert st_ == sp == 1 and np.abs(pt - pp).max() <= 2.1e-3
    assert np.median(np.abs(pt - pp)) <= 1e-7
    # the SkipGS gate over a few steps: warm-up steps update, the rest follow the rule
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    stp = Stepper(model, budget=3 << 20)
    g = BackwardGate(warmup=2)
    took = []
    for k in range(5):
        before = model.params.clone()
        stp.run_view(cam, tgt, gate=g.decide_for(0))
        stp.check()
        took.append(g.last[3])
        assert bool((model.params != before).any()) == g.last[3]
    assert took[:2] == [True, True] and g.b == sum(took) and model.step == g.b


def test_in_stream_chain_step_matches_two_pass():
    """Stepper(fuse_adam="in_stream") (geometric chain inside the Adam
    stream, no scratch) takes the same step as the default two-pass form up
    to fp32 rounding of the chain, and needs no more working set (less where
    the projection backward sets the peak)."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cam = scene("small3")
    target = torch.as_tensor(synth.random_image(cam.width, cam.height, 6) * 0.5).cuda()
    outs = []
    for fa in (True, "in_stream"):
        model = GaussianModel(sc.params, sc.n, sc.sh_degree)
        stp = Stepper(model, budget=100_000, fuse_adam=fa)
        stats = stp.run_view(cam, target)
        stp.check()
        outs.append((stp.last_loss(), model.params.cpu().numpy(), model.m.cpu().numpy(),
                     stats.peak_ws_bytes))
    (l0, p0, m0, w0), (l1, p1, m1, w1) = outs
    assert l0 == l1
    assert np.abs(p1 - p0).max() <= 2.1e-3
    assert rel_l2(m1, m0) <= 1e-5
    assert w1 <= w0


def test_reserve_sizes_arenas_for_all_views():
    """Stepper.reserve plans every view first (projection and Leaf plan only,
    no update): the parameters stay as they were, and each later step's
    largest Leaf fits the reserved arena size, which keeps 1/16 headroom and
    stays within the Leaf budget."""
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, cams = synth.outdoor_scene(200_000, seed=3, width=960, height=640, n_views=4)
    model = GaussianModel(sc.params, sc.n, sc.sh_degree)
    budget = 3 << 20
    stp = Stepper(model, budget=budget, leaf_streams=2)
    p0 = model.params.clone()
    stp.reserve(cams)
    torch.cuda.synchronize()
    assert torch.equal(model.params, p0) and model.step == 0
    hint = stp._arena_hint
    assert 0 < hint <= budget
    for k, cam in enumerate(cams):
        target = torch.as_tensor(synth.random_image(cam.width, cam.height, 40 + k) * 0.5).cuda()
        st = stp.run_view(cam, target)
        assert st.n_leaves > 1
        assert st.arena_bytes <= hint or st.over_budget.any()
    stp.check()
