"""CPU tests of libgs: the library loads without a GPU, exports every entry
point include/gs.h declares, rejects bad arguments on the host, and its
host-side Leaf planner matches the oracle's partition bit for bit."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def gsb():
    from gaussian_splatting_differentiable_dgs_b200 import build
    build.build()
    from gaussian_splatting_differentiable_dgs_b200 import binding
    return binding


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "gs.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(gs_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(gsb):
    names = declared_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(gsb.LIB_PATH)
    for nm in names:
        assert hasattr(lib, nm), nm
    assert set(names) == set(gsb.SYMBOLS)
    assert gsb.version() == 1
    assert gsb.status_string(gsb.GS_ERR_TIMEOUT) == "bounded device wait expired"


def test_host_argument_checks(gsb):
    b = gsb
    L = b.lib()
    launches0 = b.gs_launch_counter()
    # null structs / sizes are rejected before any device work
    assert L.gs_project(None, None, 0, None, None, None, 0, None, None) == b.GS_ERR_ARG
    assert L.gs_sort_keys(None, None, 5, 0, 70, None, 0, None, None) == b.GS_ERR_ARG
    assert L.gs_sort_keys32(None, None, None, 0, 0, 32, 0, None, 0, None, None) == b.GS_OK
    assert L.gs_loss_total(None, -1, None, None) == b.GS_ERR_ARG
    args = b.gs_adam_args(1e-3, 0.9, 0.999, 1e-8, 0, 0)  # step 0 is invalid
    assert L.gs_adam(None, None, None, None, 0, None, 1, 1, 1, ctypes.byref(args), None) == b.GS_ERR_ARG
    # capacity errors report the needed size
    proj = b.gs_proj(10, 1, 1, 1, 16, 8, 1)
    needed = ctypes.c_int64(0)
    st = L.gs_bin_tiles(ctypes.byref(proj), 10, 8, 8, b.gs_rect(0, 0, 2, 2), 4, 4, 8, 1000, 8, 8,
                        None, 999, 8, ctypes.byref(needed), 256, 1 << 20, None, None)
    assert st == b.GS_ERR_CAPACITY and needed.value == 1000
    # ... and none of the rejected calls launched a kernel
    assert b.gs_launch_counter() == launches0


def test_workspace_sizes(gsb):
    b = gsb
    assert b.gs_project_workspace_size(1000, 256, 256) > 0
    s1 = b.gs_sort_workspace_size(1 << 20, 8, 32, 48)
    s2 = b.gs_sort_workspace_size(1 << 20, 8, 32, 64)
    assert s2 > s1 > 12 << 20
    assert b.gs_bin_workspace_size(1 << 20) >= 8 * (1 << 20) // 1024
    assert b.gs_depth_order_workspace_size(1 << 20) > 12 << 20
    # the allocation-free sort's array holds the plan of its largest size
    # for every bit range (32-bit keys)
    for lo, hi in ((0, 32), (0, 16), (5, 29), (0, 1)):
        need = b.gs_sort_workspace_size(b.SORT_NOALLOC_MAX_N, 4, lo, hi)
        assert 0 < need <= b.SORT_NOALLOC_SCRATCH_BYTES, (lo, hi, need)


def test_load_model_matches_buffers(gsb):
    b = gsb
    for bits in (8, 13, 16, 20):
        lm = b.gs_leaf_load_model(bits, b.GS_BIN_SORT)
        passes = 2 * ((bits + 15) // 16)
        n = 5_000_000
        need = 8 * n + b.gs_sort_workspace_size(n, 4, 0, bits)
        est = lm.bytes_per_isect * n + lm.fixed_bytes
        assert need <= est
        assert lm.bytes_per_pixel == 44 and lm.bytes_per_tile == 16 and lm.align == 512
        assert lm.bytes_per_isect == 16 + (passes + 1) // 2
    # two-level binning: a Leaf holds its 32-bit values, ranges and pixels
    lm = b.gs_leaf_load_model(20, b.GS_BIN_EXPAND)
    assert lm.bytes_per_isect == 4 and lm.bytes_per_pixel == 44 and lm.bytes_per_tile == 16
    assert lm.fixed_bytes >= 8 * 255  # the 256-byte alignment of up to 8 buffers
    with pytest.raises(b.GsError):
        b.gs_leaf_load_model(20, 7)


def _lm_list(lm):
    return [lm.bytes_per_isect, lm.bytes_per_pixel, lm.bytes_per_tile, lm.fixed_bytes, lm.align]


@pytest.mark.parametrize("seed", range(6))
def test_leaf_partition_matches_oracle(gsb, oracle_mod, seed):
    rng = np.random.default_rng(seed)
    TW, TH = int(rng.integers(1, 90)), int(rng.integers(1, 60))
    W, H = TW * 16 - int(rng.integers(0, 16)), TH * 16 - int(rng.integers(0, 16))
    cnt = rng.poisson(rng.uniform(1, 4000), size=(TH, TW)).astype(np.int64)
    cnt[: TH // 3, : TW // 4] *= 40
    sat = oracle_mod.sat(cnt)
    lm = gsb.gs_leaf_load_model(16, gsb.GS_BIN_SORT)
    for budget in (1, 200_000, 5_000_000, 60_000_000, 10 ** 12):
        st, lv, li, lb, ov = gsb.gs_leaf_partition(sat, TW, TH, W, H, lm, budget)
        ol, oi, ob, oo = oracle_mod.leaf_partition(sat, TW, TH, W, H, _lm_list(lm), budget)
        assert (lv == ol).all() and (li == oi).all() and (lb == ob).all() and (ov == oo).all()
        assert st == (gsb.GS_WARN_BUDGET if ov.any() else gsb.GS_OK)


def test_leaf_partition_capacity_retry(gsb, oracle_mod):
    cnt = np.full((40, 50), 3000, np.int64)
    sat = oracle_mod.sat(cnt)
    lm = gsb.gs_leaf_load_model(12, gsb.GS_BIN_SORT)
    st, lv, *_ = gsb.gs_leaf_partition(sat, 50, 40, 800, 640, lm, 300_000, max_leaves=2)
    assert len(lv) > 2  # the wrapper grew the output after GS_ERR_CAPACITY


def test_stepper_rejects_unknown_options():
    """Stepper's options are checked on the host before any device work."""
    import numpy as np
    import pytest
    from gaussian_splatting_differentiable_dgs_b200 import synth
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    sc, _ = synth.tiny_scene(n=4)
    model = GaussianModel(np.asarray(sc.params), sc.n, sc.sh_degree, device="cpu")
    for kw in ({"leaf_streams": 5}, {"leaf_streams": 0}, {"binning": "tiles"},
               {"mode": "whole"}, {"loss": "l2"}):
        with pytest.raises(ValueError):
            Stepper(model, device="cpu", **kw)


def test_step_roofline_properties():
    """bench.step_roofline: each stage takes the larger of its HBM and ALU
    times, the fraction is the roofline over the step time, and it responds
    to the peaks and the step time as a roofline must."""
    import types
    import bench

    a = types.SimpleNamespace(binning="fused", loss="l1")
    model = types.SimpleNamespace(n=1_000_000, P=59)
    st = types.SimpleNamespace(n_cand=800_000, n_isect=50_000_000, n_block_entries=3_000_000,
                               n_block_reads=0, n_leaves=2)
    per_step = {"project": 0.2, "raster_bwd": 0.5, "project_bwd": 0.4}
    peaks = {"hbm_gbs": 6000.0}
    alu = 37e12

    def run(peaks, alu, step_ms, ops_bwd=4e10):
        return bench.step_roofline(a, model, [st], 1e10, ops_bwd, per_step, peaks, alu,
                                   2000, 1000, step_ms)

    r = run(peaks, alu, 2.0)
    s = r["stages"]
    for name, v in s.items():
        t_hbm = v["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e3
        t_alu = v["lane_ops"] / alu * 1e3
        assert abs(v["roofline_ms"] - max(t_hbm, t_alu)) <= 1e-4
        assert v["bound"] == ("alu" if t_alu > t_hbm else "hbm")
    assert s["raster_bwd"]["bound"] == "alu" and s["project_bwd"]["bound"] == "hbm"
    assert abs(r["roofline_ms"] - sum(v["roofline_ms"] for v in s.values())) <= 1e-3
    assert abs(r["frac"] - r["roofline_ms"] / 2.0) <= 1e-4
    assert abs(run(peaks, alu, 4.0)["frac"] - r["frac"] / 2) <= 1e-4
    # twice the bandwidth halves every HBM-bound stage's roofline time
    r2 = run({"hbm_gbs": 12000.0}, alu, 2.0)
    assert abs(r2["stages"]["project_bwd"]["roofline_ms"] * 2
               - s["project_bwd"]["roofline_ms"]) <= 1e-3
    assert r2["stages"]["raster_bwd"]["roofline_ms"] == s["raster_bwd"]["roofline_ms"]
    # the dominant kernel's roofline object and the step roofline's stage take
    # the same lane-ops, so an ALU-bound stage's fraction is the same in both
    k = bench.alu_roofline("k_raster_bwd", 4e10, per_step["raster_bwd"], alu)
    st_b = s["raster_bwd"]
    assert abs(k["frac"] - st_b["roofline_ms"] / st_b["measured_ms"]) <= 1e-3
    assert k["lane_ops_per_step"] == st_b["lane_ops"]


def test_committed_dram_record_matches_its_kernel_source():
    """bench.py reports the dominant kernel's DRAM traffic from the committed
    ncu record only while the kernel's source file is the one the counters
    were taken on (else the traffic is null); the record in profiles/ is
    current, and its scaling to another launch follows the algorithmic
    bytes."""
    import hashlib
    import json
    import bench
    path = os.path.join(ROOT, "profiles", "k_raster_bwd_outdoor_3m_2k5_dram.json")
    rec = json.load(open(path))
    src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    assert hashlib.sha256(src).hexdigest() == rec["source_sha256"]
    t, where = bench.profile_traffic("k_raster_bwd")
    assert t == rec["dram_bytes_per_launch"] and where.endswith("_dram.json")
    half = rec["alg_bytes_per_launch"] // 2
    t2, _ = bench.profile_traffic("k_raster_bwd", half)
    assert abs(t2 - rec["dram_bytes_per_launch"] * half / rec["alg_bytes_per_launch"]) <= 1
    assert bench.raster_bwd_alg_bytes(1000, 100) == 1000 * 96 + 100 * 20
    assert bench.profile_traffic("k_no_such_kernel") == (None, None)
