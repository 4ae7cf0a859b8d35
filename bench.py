"""Benchmark of one 3DGS training step (fwd + L1 + bwd + one Adam update per
view, BoundedGS Leaf schedule) on the outdoor-like synthetic scene:
6,000,000 Gaussians, SH degree 3, 5000x3300, 8 views on a circle, 384 MiB
Leaf budget, two Leaves in flight (--leaf-streams 1: one at a time).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0).  Under torchrun (N > 1) every rank trains an
independent replica of the workload on its own GPU (no data-path
collective); value is the total over ranks divided by the max-over-ranks
device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("fwd+bwd+Adam step ms & Gaussian-tile intersections/s per B200; "
          "peak working set GiB")
UNIT = "intersections/s"
SM_COUNT, LANES_PER_SM = 148, 128
# Algorithmic issue work of the raster stages: E evaluations times k
# lane-ops each.  E is the method's pixel-Gaussian evaluations: in the
# forward, each pixel's tile list up to its stop (the whole list if it never
# stops); in the backward, its entries before last.  The kernels evaluate
# fewer (their exact warp culling skips pairs that cannot reach 1/255); the
# forward's accounting variant counts E itself.  k per evaluation: forward
# 16 (2 sub, 5 fma/mul for q, ex2 and its scale, the clamp, the test, a
# 4-op blend), backward 40 (the forward's evaluation plus the reverse blend
# and the 9 gradient terms).
K_FWD, K_BWD = 16, 40
# SSIM term, lane-ops per pixel and channel with its gradient: the window
# sums of x, y, x^2, y^2, x y (5 maps x 2 separable passes x 11 taps), the
# three products, S and its three partials (about 30 operations, a division
# counted as one), the window sums of the partials (3 x 2 x 11) and their
# combination (4).
K_SSIM = 110 + 3 + 30 + 66 + 4


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=48)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--config", type=int, default=3, choices=[1, 2, 3],
                    help="1: 2,000 Gaussians SH0 256x256; 2: 100,000 Gaussians SH3 1920x1080; "
                         "3: the outdoor scene (--gaussians, --width, --height, --views)")
    ap.add_argument("--gaussians", type=int, default=6_000_000)
    ap.add_argument("--width", type=int, default=5000)
    ap.add_argument("--height", type=int, default=3300)
    ap.add_argument("--views", type=int, default=8)
    ap.add_argument("--budget-mib", type=float, default=384)
    ap.add_argument("--raster-ppt", type=int, default=0)
    # 2: consecutive Leaves alternate between two streams and two raster
    # arenas (one Leaf's kernels fill the SMs the other's tail leaves idle)
    ap.add_argument("--leaf-streams", type=int, default=2, choices=[1, 2, 3, 4])
    # steps of the serialized pass (Leaves on one stream) whose per-stage
    # CUDA-event times give the kernels' own durations when the timed region
    # overlaps Leaves
    ap.add_argument("--stage-steps", type=int, default=8)
    # projection backward: the geometric chain as its own pass ("two_pass")
    # or inside the Adam stream ("in_stream")
    ap.add_argument("--fuse-adam", default="two_pass", choices=["two_pass", "in_stream"])
    ap.add_argument("--binning", default="fused", choices=["fused", "expand", "sort"])
    ap.add_argument("--loss", default="l1", choices=["l1", "l1_ssim"],
                    help="l1: the L1 photometric loss; l1_ssim: (1 - 0.2) L1 + 0.2 (1 - SSIM) "
                         "with SSIM windows local to each Leaf")
    ap.add_argument("--sweep", default=None,
                    help="comma-separated widths: resolution sweep, whole image vs bounded")
    ap.add_argument("--skipgs", type=int, default=0,
                    help="N training steps over the views with and without the SkipGS gate")
    ap.add_argument("--skipgs-warmup", type=int, default=16)
    ap.add_argument("--schedules", action="store_true",
                    help="schedule comparison: Leaves, 3x3 groups at 128 MiB, fixed 8x8 blocks")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-mode", default="prefetch", choices=["prefetch", "crops"],
                    help="how the e2e run supplies the targets from pinned host memory")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-tiles", type=int, default=64)
    return ap.parse_args()


def workload_name(a):
    if a.config == 1:
        return ("tiny_2k_256x256: 2,000 Gaussians SH0, one camera at the origin, f 300, "
                f"{a.budget_mib:g} MiB Leaf budget")
    if a.config == 2:
        return ("hd_100k_1920x1080: 100,000 Gaussians SH3 in 64 clusters, one camera, f 1500, "
                f"{a.budget_mib:g} MiB Leaf budget")
    return (f"outdoor_{a.gaussians / 1e6:g}m_{a.width}x{a.height}: {a.gaussians:,} Gaussians "
            f"SH3, {a.views} views on a radius-4 circle, {a.budget_mib:g} MiB Leaf budget")


def make_workload(a, synth):
    """(scene, cameras) of the selected configuration; the small ones fit in
    L2, so their timed steps are preceded by an L2 flush."""
    if a.config == 1:
        return synth.tiny_oracle_scene(0)
    if a.config == 2:
        return synth.hd_cluster_scene(0)
    return synth.outdoor_scene(a.gaussians, seed=0, width=a.width, height=a.height,
                               n_views=a.views)


def cpu_model():
    """The host CPU's model name (/proc/cpuinfo) and its logical core count."""
    name = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return name or "unknown", os.cpu_count()


def step_roofline(a, model, stats, ops_fwd, ops_bwd, per_step, peaks, alu_peak, W, H,
                  step_ms):
    """Roofline time of the step: for each stage the larger of its compulsory
    HBM bytes / measured copy bandwidth and its lane-ops / ALU issue peak,
    summed; frac = that sum / the measured step time (the timed region's ms
    per step, gaps between kernels included; stages_ms is the sum of the
    stages' own device times).  Bytes per view:
      project      N*12 (means for the cull) + N*4 (slot map)
                   + C*((P-3)*4 + 48 + 8 + 4 + 4) (rest of a candidate's
                   parameters; record, rect, depth key, candidate index)
      sort_depth   4 passes x C x 16 (keys + values in and out) + C*4
                   (histogram read) + C*20 (rect gather)
      bin          C*12 (rects + slots in depth order) + E_blk*4 (the block
                   lists written once: they are built by a counting scatter)
      sort_tiles   2 passes x I x 20 (the bin + sort path only)
      expand       2 passes x R_blk x 12 (block entries + rect gathers) +
                   I*4 (the Leaf lists)
      raster_fwd   C*48 + pixels*(20 + 12 + 12) (records; colour, T, last;
                   target; dL/dcolour; the list entries a tile reads stop where
                   its pixels saturate, so none are counted)
      raster_bwd   C*48 + pixels*20 (T, last, dL/dcolour) + C*48 (gradient
                   atomics)
      ssim         pixels*48 (render and target read, dL/dcolour read and
                   written; with --loss l1_ssim), lane-ops pixels*3*K_SSIM
      project_bwd  N*P*24 (p, m, v read and written) + C*(48 + 48 + 56*2)
                   (g2d, record, fp64 geometric scratch) + N*4 (slot map)
    (E_blk = block-list entries, R_blk = their reads over the Leaves, I =
    tile-list entries, C = candidates, N = Gaussians.)  The raster stages'
    lane-ops are E k (K_FWD, K_BWD), E counted on the same views the stage
    times are averaged over."""
    hbm = peaks["hbm_gbs"] * 1e9
    n, P = model.n, model.P
    k = len(stats)
    C = sum(s.n_cand for s in stats) / k
    I = sum(s.n_isect for s in stats) / k
    E = sum(s.n_block_entries for s in stats) / k
    R = sum(s.n_block_reads for s in stats) / k
    px = W * H
    expand = a.binning in ("expand", "fused")
    byt = {
        "project": n * 12 + n * 4 + C * ((P - 3) * 4 + 64),
        "sort_depth": C * (4 * 16 + 4 + 20),
        "bin": (C * 12 + E * 4) if expand else C * 12 * max(1, stats[0].n_leaves) + I * 8,
        "sort_tiles": 0.0 if expand else I * 40,
        "expand": (R * 24 + I * 4) if a.binning == "expand" else 0.0,
        "raster_fwd": C * 48 + px * 44,
        "raster_bwd": C * 96 + px * 20,
        "project_bwd": n * P * 24 + C * 208 + n * 4,
    }
    ops = {"raster_fwd": ops_fwd, "raster_bwd": ops_bwd}
    if a.loss == "l1_ssim":
        byt["ssim"] = px * 48
        ops["ssim"] = px * 3 * K_SSIM
    stages, total = {}, 0.0
    for s, b in byt.items():
        t_hbm = b / hbm * 1e3
        t_alu = ops.get(s, 0.0) / alu_peak * 1e3
        t = max(t_hbm, t_alu)
        total += t
        stages[s] = {"bound": "alu" if t_alu > t_hbm else "hbm", "roofline_ms": round(t, 4),
                     "measured_ms": round(per_step.get(s, 0.0), 4), "bytes": round(b),
                     "lane_ops": round(ops.get(s, 0.0))}
    measured = sum(per_step.values())
    return {"roofline_ms": round(total, 4), "stages_ms": round(measured, 4),
            "step_ms": round(step_ms, 4),
            "frac": round(total / step_ms, 4) if step_ms > 0 else None, "stages": stages}


def alu_roofline(kernel, lane_ops, stage_ms, alu_peak):
    """Roofline of an issue-bound kernel: achieved = its algorithmic lane-ops
    per step / its device time per step, against the ALU issue peak.  The
    same lane-ops enter the step roofline's stage, so the two agree."""
    ach = lane_ops / (stage_ms / 1e3) / 1e12
    return {"bound": "alu", "kernel": kernel, "achieved": round(ach, 3),
            "peak": round(alu_peak / 1e12, 3), "unit": "Tlane-op/s",
            "frac": round(ach / (alu_peak / 1e12), 4), "lane_ops_per_step": round(lane_ops)}


def profile_traffic(kernel, alg_bytes_per_launch=None):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/<kernel>_*_dram.json), or None when there is none or the
    kernel's source file has changed since it was taken.  A summary taken on
    a smaller case records that case's algorithmic bytes per launch; its
    traffic is then scaled to this workload's launch by the ratio of the
    algorithmic bytes (the kernel's DRAM traffic is its compulsory bytes
    times a waste factor that does not depend on the size)."""
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"{kernel}_*_dram.json"))):
        try:
            with open(path) as f:
                rec = json.load(f)
            src = os.path.join(ROOT, rec["source"])
            with open(src, "rb") as f:
                digest = hashlib.sha256(f.read()).hexdigest()
        except (OSError, KeyError, ValueError):
            continue
        if digest != rec.get("source_sha256"):
            continue
        t = rec["dram_bytes_per_launch"]
        base = rec.get("alg_bytes_per_launch")
        if base and alg_bytes_per_launch:
            return round(t * alg_bytes_per_launch / base), (
                f"{os.path.relpath(path, ROOT)}, scaled by algorithmic bytes per launch "
                f"{alg_bytes_per_launch:.4g} / {base:.4g}")
        return t, os.path.relpath(path, ROOT)
    return None, None


def raster_bwd_alg_bytes(n_cand, pixels):
    """Compulsory DRAM bytes of the raster backward over a region: each
    record fetched once (48 B), the gradient reductions (48 B per candidate),
    and T, last and dL/dcolour per pixel (20 B); as in step_roofline."""
    return n_cand * 96 + pixels * 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling every 100 ms from before the warm-up to the end of
    the timed region; stop(t0, t1) keeps the samples stamped inside [t0, t1]
    (host wall clock), all samples if none is."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        try:
            import tempfile
            self.f = tempfile.NamedTemporaryFile("w", suffix=f"_clocks_gpu{gpu_index}.csv",
                                                 delete=False)
            self.path = self.f.name
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return None
        import datetime
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 10:
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                rows.append([ts] + parts[1:])
        os.unlink(self.path)
        if t0 is not None and t1 is not None:
            inside = [r for r in rows if r[0] is not None and t0 <= r[0] <= t1]
            rows = inside or rows
        if not rows:
            return None
        num = lambda x: x.replace(".", "", 1).isdigit()
        sm = [float(r[2]) for r in rows if num(r[2])]
        mx = [float(r[3]) for r in rows if num(r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[6 + k].lower() == "active"})
        loaded = [x for x in sm if x > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
class OracleSample:
    """Times the oracle's stages on samples of one view and scales each to
    the full step: projection of a 1/8 subset of the Gaussians (x8), tile
    lists (scatter + stable sort) of a 1/16 subset of the candidates (x16),
    raster forward + L1 + raster backward on `n_tiles` uniformly random tiles
    (x tiles / n_tiles), projection backward on a 1/16 subset of the
    candidates (x16) and Adam on a 1/64 subset of the Gaussians (x64)."""

    def __init__(self, scene, cams, target_fn, n_tiles=64, seed=0):
        from oracle import oracle as O
        self.O = O
        O.build()
        self.scene = scene
        self.cams = cams
        self.n_tiles = n_tiles
        self.rng = np.random.default_rng(seed)
        self.target_fn = target_fn
        self.cache = {}

    def _setup(self, v):
        if v in self.cache:
            return self.cache[v]
        O, sc, cam = self.O, self.scene, self.cams[v]
        p64 = sc.params.astype(np.float64)
        pr = O.project(p64, sc.n, sc.sh_degree, cam)
        TW, TH = O.grid(cam)
        counts = O.tile_counts_fast(pr["rect"], TW, TH).reshape(-1)
        self.cache[v] = (p64, pr, counts, TW, TH)
        return self.cache[v]

    def step(self, v):
        O, sc, cam = self.O, self.scene, self.cams[v]
        p64, pr, counts, TW, TH = self._setup(v)
        n = sc.n
        W, H = cam.width, cam.height
        I_total = int(pr["rec"][:, 14].sum())   # tiles of the 3-sigma squares
        # projection of 1/8 of the Gaussians
        sub = np.sort(self.rng.choice(n, n // 8, replace=False))
        ps = np.ascontiguousarray(p64[:, sub])
        measured = 0.0
        t0 = time.perf_counter()
        O.project(ps, len(sub), sc.sh_degree, cam)
        dt = time.perf_counter() - t0
        measured += dt
        t_proj = dt * n / len(sub)
        # tile lists: scatter + per-tile stable sort for 1/16 of the candidates
        C = len(pr["cand_idx"])
        cs = np.sort(self.rng.choice(C, max(C // 16, 1), replace=False))
        t0 = time.perf_counter()
        O.tile_lists_all(pr["rect"][cs], pr["key"][cs], TW, TH)
        dt = time.perf_counter() - t0
        measured += dt
        t_lists = dt * C / len(cs)
        # raster forward + L1 + raster backward on uniformly random tiles
        tiles = np.sort(self.rng.choice(TW * TH, self.n_tiles, replace=False)).astype(np.int32)
        off, vals = O.tile_lists(pr["rect"], pr["key"], TW, tiles)
        target = self.target_fn(v)
        tg = O.gather_tiles(np.pad(target, ((0, 0), (0, TH * 16 - H), (0, TW * 16 - W))),
                            tiles, TW, 3)
        t0 = time.perf_counter()
        fw = O.raster_fwd(pr["rec"], TW, W, H, tiles, off, vals)
        valid = (fw["flags"] & 0x80) == 0
        d = np.where(valid[:, None, :], fw["img"] - tg, 0.0)
        dL = np.sign(d) / (3.0 * W * H)
        O.raster_bwd(pr["rec"], TW, W, H, tiles, off, vals, dL)
        dt = time.perf_counter() - t0
        measured += dt
        t_raster = dt * (TW * TH) / self.n_tiles
        I_s = int(off[-1])
        # projection backward on 1/16 of the candidates
        g2d = self.rng.normal(size=(len(cs), 9)) * 1e-3
        t0 = time.perf_counter()
        O.project_bwd(p64, sc.sh_degree, cam, pr["cand_idx"][cs], g2d)
        dt = time.perf_counter() - t0
        measured += dt
        t_pbwd = dt * C / len(cs)
        # Adam on 1/64 of the Gaussians (all planes)
        k = max(n // 64, 1)
        pa = p64[:, :k]
        g = self.rng.normal(size=pa.shape)
        t0 = time.perf_counter()
        O.adam(pa, np.zeros_like(pa), np.zeros_like(pa), g, step=1)
        dt = time.perf_counter() - t0
        measured += dt
        t_adam = dt * n / k
        est = t_proj + t_lists + t_raster + t_pbwd + t_adam
        return dict(est_step_s=est, measured_s=measured, I_total=I_total, sample_isect=I_s,
                    parts=dict(project=t_proj, lists=t_lists, raster=t_raster,
                               project_bwd=t_pbwd, adam=t_adam))

    def describe(self):
        return (f"per step: oracle projection of 1/8 of the Gaussians (x8), tile lists of 1/16 "
                f"of the candidates (x16), raster fwd + L1 + raster bwd on {self.n_tiles} "
                f"uniformly random tiles (x tiles/{self.n_tiles}), projection bwd on 1/16 of the "
                f"candidates (x16), Adam on 1/64 of the Gaussians (x64); value = the view's "
                f"intersections / estimated step time")


def oracle_full_step(O, scene, cam, target, reps=1):
    """The oracle's whole step of one view (projection, lists, raster forward,
    L1, raster backward, projection backward, one Adam update), timed on the
    host cores: the fastest of `reps` runs."""
    p64 = scene.params.astype(np.float64)
    best, r = None, None
    for _ in range(reps):
        t0 = time.perf_counter()
        r = O.step(p64, scene.n, scene.sh_degree, cam, target)
        dt = time.perf_counter() - t0
        best = dt if best is None else min(best, dt)
    return dict(step_s=best, I_total=int(r["proj"]["rec"][:, 14].sum()), loss=r["loss"])


# ---------------------------------------------------------------------------
# replicas: rank r takes views r, r + 1, ... (mod the view count); the job's
# time is the slowest rank's, its work the sum over ranks
# ---------------------------------------------------------------------------
def rank_view(k, rank, n_views):
    return (k + rank) % n_views


def combine_ranks(ms, units, dist, device):
    """(max over ranks of ms, sum over ranks of units); dist = None for one
    process.  Every rank must call it, in the same order."""
    if dist is None:
        return float(ms), float(units)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([float(units)], dtype=torch.float64, device=device)
    dist.all_reduce(u)
    return float(t.item()), float(u.item())


# ---------------------------------------------------------------------------
def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from gaussian_splatting_differentiable_dgs_b200 import synth

    if a.impl == "reference":
        return run_reference(a, rank, world)
    if a.sweep:
        return run_sweep(a)
    if a.schedules:
        return run_schedules(a)
    if a.skipgs:
        return run_skipgs(a)

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper, STAGES

    scene, cams = make_workload(a, synth)
    W, H = cams[0].width, cams[0].height
    budget = int(a.budget_mib * (1 << 20))
    # a workload that fits in L2 gets it flushed before every timed step
    # (outside the step's events); the outdoor scene's 4.25 GB of parameters
    # and moments stream through HBM every step
    flush = (torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
             if a.config in (1, 2) else None)
    # targets: renders of the jittered copy (means N(0, 0.02), colour N(0, 0.05))
    jit = synth.jittered(scene, seed=1)
    jm = GaussianModel(jit.params, jit.n, jit.sh_degree)
    js = Stepper(jm, budget=budget, raster_flags=a.raster_ppt, binning=a.binning)
    targets = [js.render(c) for c in cams]
    torch.cuda.synchronize()
    del jm, js
    model = GaussianModel(scene.params, scene.n, scene.sh_degree)
    stp = Stepper(model, budget=budget, raster_flags=a.raster_ppt, binning=a.binning,
                  loss=a.loss, leaf_streams=a.leaf_streams,
                  fuse_adam=True if a.fuse_adam == "two_pass" else "in_stream")
    nv = len(cams)
    view_of = lambda k: rank_view(k, rank, nv)

    # the Leaf arenas sized for every view of the run (projection and Leaf
    # planning only, before the warm-up), so that no timed step allocates
    stp.reserve(cams)
    clocks = ClockSampler(local)
    for k in range(a.warmup):
        stp.run_view(cams[view_of(k)], targets[view_of(k)])
    stp.check()

    # ---- timed region (device time, CUDA events on the launching stream) -----
    timing = {}
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stats = []
    if flush is None:
        e0.record()
        for k in range(a.steps):
            v = view_of(a.warmup + k)
            stats.append(stp.run_view(cams[v], targets[v], timing=timing))
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    else:
        ms = 0.0
        for k in range(a.steps):
            v = view_of(a.warmup + k)
            flush.fill_(k & 255)          # evicts the step's inputs from L2
            e0.record()
            stats.append(stp.run_view(cams[v], targets[v], timing=timing))
            e1.record()
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
    if dist:
        dist.barrier()
    clk = clocks.stop(wall0, time.time())
    stp.check()
    isect = sum(s.n_isect_square for s in stats)   # conventional 3-sigma-square count
    entries = sum(s.n_isect for s in stats)         # entries of the tight tile lists
    launches = sum(s.launches for s in stats)
    peak_ws = max(s.peak_ws_bytes for s in stats)
    stage_ms = {name: sum(x.elapsed_time(y) for x, y in timing.get(name, [])) for name in STAGES}
    stage_n = {name: len(timing.get(name, [])) for name in STAGES}
    ms_max, isect_all = combine_ranks(ms, isect, dist, "cuda")
    value = isect_all / (ms_max / 1e3)
    n_steps = a.steps
    stage_src = "timed region"
    stage_views = [view_of(a.warmup + k) for k in range(a.steps)]
    overlapped = None
    if a.leaf_streams > 1:
        # several Leaves in flight: a stage's events span the other streams'
        # kernels too, so the kernels' own durations come from a serialized
        # pass of the same workload (same views, Leaves on one stream)
        overlapped = {s: round(stage_ms[s] / a.steps, 3) for s in STAGES}
        stp.leaf_streams = 1
        timing = {}
        for k in range(a.stage_steps):
            v = view_of(a.warmup + k)
            stp.run_view(cams[v], targets[v], timing=timing)
        torch.cuda.synchronize()
        stp.leaf_streams = a.leaf_streams
        stage_ms = {name: sum(x.elapsed_time(y) for x, y in timing.get(name, []))
                    for name in STAGES}
        stage_n = {name: len(timing.get(name, [])) for name in STAGES}
        n_steps = a.stage_steps
        stage_src = f"serialized pass of {a.stage_steps} steps (Leaves on one stream)"
        stage_views = [view_of(a.warmup + k) for k in range(a.stage_steps)]

    # ---- accounting (untimed): the work counters of every view whose stage
    # times are averaged, so the raster stages' lane-ops per step are the mean
    # over exactly those views (no update: the counts are the views' own) --
    cnt_view = {}
    for v in sorted(set(stage_views)):
        counters = torch.zeros(6, dtype=torch.int64, device="cuda")
        stp.run_view(cams[v], targets[v], counters=counters, update=False)
        torch.cuda.synchronize()
        cnt_view[v] = [int(x) for x in counters.cpu()]
    cnt = [statistics.mean(cnt_view[v][j] for v in stage_views) for j in range(6)]
    ops_fwd = cnt[2] * K_FWD
    ops_bwd = cnt[3] * K_BWD

    peaks, peak_src = load_peaks()
    sm_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    alu_peak = SM_COUNT * LANES_PER_SM * sm_mhz * 1e6  # lane-ops/s
    # dominant kernel over the timed region
    dom = max(STAGES, key=lambda s: stage_ms[s])
    per_step = {s: stage_ms[s] / n_steps for s in STAGES}
    if dom in ("raster_bwd", "raster_fwd"):
        ops = ops_bwd if dom == "raster_bwd" else ops_fwd
        # per launch (one Leaf): the view's compulsory bytes over its Leaves
        leaves = statistics.mean(st.n_leaves for st in stats)
        alg = raster_bwd_alg_bytes(statistics.mean(st.n_cand for st in stats), W * H) / leaves
        traffic, traffic_src = profile_traffic(f"k_{dom}", alg if dom == "raster_bwd" else None)
        roof = alu_roofline(f"k_{dom}", ops, per_step[dom], alu_peak)
        roof.update(traffic=traffic, traffic_source=traffic_src,
                    peak_source=f"{SM_COUNT} SMs x {LANES_PER_SM} lanes x {sm_mhz:g} MHz "
                                f"(sm_max_mhz of {peak_src})")
    else:
        P = model.P
        C = statistics.mean(s.n_cand for s in stats)
        byt = scene.n * P * 24 + C * (48 + 16) + scene.n * 4
        ach = byt / (per_step[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": f"k_{dom}", "achieved": round(ach, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                "traffic": None}

    # ---- step roofline: per stage max(algorithmic bytes / HBM, lane-ops / ALU)
    step_roof = step_roofline(a, model, stats, ops_fwd, ops_bwd, per_step, peaks,
                              alu_peak, W, H, ms_max / a.steps)

    # ---- end to end through host buffers --------------------------------------
    e2e = None
    if not a.no_e2e:
        # the step's public calls with the views' targets in pinned host
        # memory: "prefetch" uploads each view's target during the previous
        # view's step (TargetPrefetcher); "crops" uploads each Leaf's crop on
        # a copy stream during the view's own Leaves (two crops resident)
        from gaussian_splatting_differentiable_dgs_b200.step import TargetPrefetcher
        host_t = [t.cpu().pin_memory() for t in targets]
        feeder = TargetPrefetcher(host_t, stepper=stp) if a.e2e_mode == "prefetch" else None
        loss_h = torch.empty(1, dtype=torch.float64, pin_memory=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record()
        e2e_isect = 0
        order = [view_of(k) for k in range(a.steps)]
        supply = feeder.iterate(order) if feeder else ((v, host_t[v]) for v in order)
        for v, tgt in supply:
            s = stp.run_view(cams[v], tgt)
            loss_h.copy_(stp._last_loss, non_blocking=True)
            e2e_isect += s.n_isect_square
        f1.record()
        torch.cuda.synchronize()
        ems, e2e_isect = combine_ranks(f0.elapsed_time(f1), e2e_isect, dist, "cuda")
        TW, TH = (W + 15) // 16, (H + 15) // 16
        BW, BH = (TW + 7) // 8, (TH + 7) // 8
        # per step: the tile SAT, candidate count, 3-sigma count, block SAT
        # (two-level binning) and the loss
        d2h = (TW + 1) * (TH + 1) * 8 + 4 + 8 + 8
        if a.binning in ("expand", "fused"):
            d2h += (BW + 1) * (BH + 1) * 8
        e2e = {"value": e2e_isect / (ems / 1e3), "unit": UNIT, "ms_per_step": ems / a.steps,
               "h2d_bytes_per_step": 3 * W * H * 4, "d2h_bytes_per_step": d2h,
               "supply": ("prefetch: each view's target uploaded during the previous view's "
                          "step (issued once that step's projection tables reached the host), "
                          "two device targets resident") if feeder else
                         ("crops: each Leaf's crop uploaded during the view's Leaves, "
                          "two crops resident")}

    # ---- CPU baseline (rank 0, one GPU) ---------------------------------------
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu and a.loss == "l1":
        tg_host = {}

        def target_fn(v):
            if v not in tg_host:
                tg_host[v] = targets[v].cpu().numpy().astype(np.float64)
            return tg_host[v]

        from oracle import oracle as O
        model_name, ncpu = cpu_model()
        if a.config in (1, 2):
            # the whole oracle step, measured (no sampling)
            r = oracle_full_step(O, scene, cams[0], target_fn(0), reps=3 if a.config == 1 else 1)
            cpu = {"value": r["I_total"] / r["step_s"], "unit": UNIT, "cores": O.num_threads(),
                   "cpu_model": model_name, "logical_cpus": ncpu, "kind": "oracle",
                   "sample": "the whole step of the view (projection, lists, raster forward, "
                             "L1, raster backward, projection backward, Adam), measured",
                   "estimated": False, "step_s": round(r["step_s"], 4)}
        else:
            osm = OracleSample(scene, cams, target_fn, n_tiles=a.cpu_tiles)
            r = osm.step(0)
            cpu = {"value": r["I_total"] / r["est_step_s"], "unit": UNIT,
                   "cores": O.num_threads(), "cpu_model": model_name, "logical_cpus": ncpu,
                   "kind": "oracle", "sample": osm.describe(),
                   "estimated": True, "est_step_s": round(r["est_step_s"], 2),
                   "measured_s": round(r["measured_s"], 2),
                   "parts_s": {k: round(x, 2) for k, x in r["parts"].items()}}

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_max / a.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded generator; targets = renders of a jittered copy)",
            "config": {"workload": workload_name(a), "gaussians": scene.n,
                       "sh_degree": scene.sh_degree,
                       "width": W, "height": H, "views": nv, "leaf_budget_mib": a.budget_mib,
                       "binning": a.binning, "loss": a.loss, "leaf_streams": a.leaf_streams,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": ("inputs larger than L2 (4.25 GB of params + Adam moments "
                              "stream every step)") if flush is None else
                             ("L2 flushed before every timed step (512 MiB fill outside the "
                              "step's CUDA events; the step's inputs fit in L2)")},
            "peak_ws_gib": peak_ws / 2 ** 30,
            "isect_per_view": isect / a.steps,
            "list_entries_per_view": entries / a.steps,
            "block_entries_per_view": sum(s.n_block_entries for s in stats) / a.steps,
            "candidates_per_view": statistics.mean(s.n_cand for s in stats),
            "leaves_per_view": statistics.mean(s.n_leaves for s in stats),
            "stage_ms_per_step": {s: round(per_step[s], 3) for s in STAGES},
            "stage_ms_source": stage_src,
            "stage_ms_per_step_overlapped": overlapped,
            "stage_launches_per_step": {s: stage_n[s] / n_steps for s in STAGES},
            "work": {"per": "mean over the views the stage times average "
                            f"({len(stage_views)} steps, views {sorted(set(stage_views))})",
                     "method_fwd_evaluations": round(cnt[2]), "method_bwd_evaluations": round(cnt[3]),
                     "fwd_pairs_evaluated": round(cnt[0]), "fwd_pairs_composited": round(cnt[1]),
                     "bwd_pairs_evaluated": round(cnt[4]), "bwd_pairs_differentiated": round(cnt[5])},
            "roofline": roof, "step_roofline": step_roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk,
        }
        print(json.dumps(out))
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_sweep(a):
    """Resolution sweep on the outdoor scene at a fixed camera pose and field
    of view (3:2 images): per width, (a) the whole-image configuration with
    a single-stage backward ("original") and (b) the bounded one (two-stage
    backward, Leaves under the budget, candidate-index projection, compact
    gradients).  Both start from the same parameters; the first step's L1
    loss is compared, then `steps` steps are timed.  One JSON line per run
    and a summary line."""
    import torch
    from gaussian_splatting_differentiable_dgs_b200 import synth
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    torch.cuda.set_device(0)
    scene, _ = synth.outdoor_scene(a.gaussians, seed=0, width=1000, height=667, n_views=1)
    jit = synth.jittered(scene, seed=1)
    budget = int(a.budget_mib * (1 << 20))
    rows = []
    clocks = ClockSampler(0)
    wall0 = time.time()
    for width in [int(w) for w in a.sweep.split(",")]:
        cam = synth.sweep_camera(width)
        jm = GaussianModel(jit.params, jit.n, jit.sh_degree)
        target_dev = Stepper(jm, budget=budget).render(cam)
        del jm
        # whole image: the view's target resident; bounded: the supervision
        # supplied one Leaf crop at a time from pinned host memory
        target_host = target_dev.cpu().pin_memory()
        losses = {}
        for mode in ("original", "bounded"):
            target = target_dev if mode == "original" else target_host
            model = GaussianModel(scene.params, scene.n, scene.sh_degree)
            stp = Stepper(model, budget=budget, mode=mode, binning=a.binning)
            if mode == "bounded":
                stp.reserve([cam])  # candidate capacity and arena sized for the view
            torch.cuda.synchronize()
            torch.cuda.reset_peak_memory_stats()
            base = torch.cuda.memory_allocated()
            st0 = stp.run_view(cam, target)
            losses[mode] = stp.last_loss()
            for _ in range(max(a.warmup - 1, 0)):
                stp.run_view(cam, target)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(a.steps):
                st = stp.run_view(cam, target)
            e1.record()
            torch.cuda.synchronize()
            stp.check()
            ms = e0.elapsed_time(e1) / a.steps
            peak = (torch.cuda.max_memory_allocated() - base) / 2 ** 30
            row = {"sweep": "resolution", "width": width, "height": cam.height, "mode": mode,
                   "target": "resident" if mode == "original" else "pinned host, per-Leaf crops",
                   "ms_per_step": round(ms, 3),
                   "working_set_gib": round(st0.peak_ws_bytes / 2 ** 30, 4),
                   "device_peak_above_model_gib": round(peak, 4),
                   "loss_first_step": losses[mode], "leaves": st.n_leaves,
                   "candidates": st.n_cand, "isect": st.n_isect_square,
                   "list_entries": st.n_isect}
            rows.append(row)
            print(json.dumps(row), flush=True)
            del stp, model
            torch.cuda.empty_cache()
        rel = abs(losses["original"] - losses["bounded"]) / max(abs(losses["original"]), 1e-30)
        rows.append({"sweep": "resolution", "width": width, "l1_rel_diff": rel})
        print(json.dumps(rows[-1]), flush=True)
        del target, target_dev, target_host
        torch.cuda.empty_cache()
    clk = clocks.stop(wall0, time.time())
    diffs = [r["l1_rel_diff"] for r in rows if "l1_rel_diff" in r]
    print(json.dumps({"sweep": "resolution", "summary": True, "max_l1_rel_diff": max(diffs),
                      "clocks": clk,
                      "workload": workload_name(a) + ", camera 0 pose, fixed field of view"}))


def run_schedules(a):
    """Schedules of one pass over the views of the outdoor scene (defaults:
    the scene at --gaussians, --width x --height, --views views):
    (1) Leaves under --budget-mib, one Adam update per view; (2) 3x3 groups,
    each with its own candidate projection, Leaves under 128 MiB, one update
    per view; (3) a fixed 8x8 grid of blocks, one Leaf and one Adam update
    per block (64 per view).  Each starts from the same parameters; the
    targets (renders of the jittered copy) are made per view outside the
    timed events.  One JSON line per schedule."""
    import torch
    from gaussian_splatting_differentiable_dgs_b200 import synth
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    torch.cuda.set_device(0)
    scene, cams = synth.outdoor_scene(a.gaussians, seed=0, width=a.width, height=a.height,
                                      n_views=a.views)
    jit = synth.jittered(scene, seed=1)
    budget = int(a.budget_mib * (1 << 20))
    plans = [("leaves", dict(budget=budget), None),
             ("groups3x3_128MiB", dict(budget=128 << 20), (3, 3)),
             ("blocks8x8", dict(budget=1 << 40), (8, 8))]
    for name, kw, split in plans:
        clocks = ClockSampler(0)
        wall0 = time.time()
        model = GaussianModel(scene.params, scene.n, scene.sh_degree)
        stp = Stepper(model, **kw)
        jm = GaussianModel(jit.params, jit.n, jit.sh_degree)
        renderer = Stepper(jm, budget=budget)
        total_ms, losses, peak, leaves, updates0 = 0.0, [], 0, 0, model.step
        for cam in cams:
            target = renderer.render(cam)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            if split is None:
                st = stp.run_view(cam, target)
            elif name.startswith("groups"):
                st = stp.run_view_grouped(cam, target, groups=split)
            else:
                st = stp.run_view_blocks(cam, target, blocks=split)
            e1.record()
            torch.cuda.synchronize()
            stp.check()
            total_ms += e0.elapsed_time(e1)
            losses.append(stp.last_loss())
            peak = max(peak, st.peak_ws_bytes)
            leaves += st.n_leaves
            del target
        clk = clocks.stop(wall0, time.time())
        print(json.dumps({"schedule": name, "views": len(cams), "ms_per_view": total_ms / len(cams),
                          "pass_s": total_ms / 1e3, "working_set_gib": peak / 2 ** 30,
                          "mean_loss": float(np.mean(losses)),
                          "adam_updates": model.step - updates0,
                          "leaves_per_view": leaves / len(cams), "clocks": clk,
                          "workload": workload_name(a)}), flush=True)
        del stp, model, renderer, jm
        torch.cuda.empty_cache()


def run_skipgs(a):
    """`skipgs` training steps cycling over the views, once with every
    backward and once behind the SkipGS gate (warm-up --skipgs-warmup
    steps, beta 0.95, rho_lo 0.5), from the same parameters; the targets
    are renders of the jittered copy.  One JSON line per run."""
    import torch
    from gaussian_splatting_differentiable_dgs_b200 import synth
    from gaussian_splatting_differentiable_dgs_b200.skipgs import BackwardGate
    from gaussian_splatting_differentiable_dgs_b200.step import GaussianModel, Stepper
    torch.cuda.set_device(0)
    scene, cams = synth.outdoor_scene(a.gaussians, seed=0, width=a.width, height=a.height,
                                      n_views=a.views)
    jit = synth.jittered(scene, seed=1)
    budget = int(a.budget_mib * (1 << 20))
    jm = GaussianModel(jit.params, jit.n, jit.sh_degree)
    targets = [Stepper(jm, budget=budget).render(c) for c in cams]
    del jm
    for gated in (False, True):
        model = GaussianModel(scene.params, scene.n, scene.sh_degree)
        stp = Stepper(model, budget=budget)
        gate = BackwardGate(warmup=a.skipgs_warmup) if gated else None
        losses = []
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k in range(a.skipgs):
            v = k % len(cams)
            stp.run_view(cams[v], targets[v], gate=gate.decide_for(v) if gated else None)
            losses.append(stp._last_loss)
        e1.record()
        torch.cuda.synchronize()
        stp.check()
        ms = e0.elapsed_time(e1) / a.skipgs
        tail = [float(x.item()) for x in losses[-len(cams):]]
        print(json.dumps({"schedule": "skipgs" if gated else "every_backward", "steps": a.skipgs,
                          "ms_per_step": ms, "backward_steps": gate.b if gated else a.skipgs,
                          "rho_min": gate.rho_min if gated else None,
                          "mean_loss_last_pass": float(np.mean(tail)),
                          "workload": workload_name(a)}), flush=True)
        del stp, model
        torch.cuda.empty_cache()


def run_reference(a, rank, world):
    """The oracle, as it stands, timed on the host cores (rank 0 only).  The
    small configurations run its whole step; the outdoor scene runs bounded
    samples of each step, scaled to the step (an estimate, marked so)."""
    if rank != 0:
        return
    from gaussian_splatting_differentiable_dgs_b200 import synth
    from oracle import oracle as O
    model_name, ncpu = cpu_model()
    scene, cams = make_workload(a, synth)
    if a.config in (1, 2):
        cam = cams[0]
        target = synth.random_image(cam.width, cam.height, 100).astype(np.float64)
        for _ in range(a.warmup if a.config == 1 else min(a.warmup, 1)):
            oracle_full_step(O, scene, cam, target)
        steps = a.steps if a.config == 1 else min(a.steps, 3)
        t0 = time.perf_counter()
        times, isect = [], 0
        for _ in range(steps):
            r = oracle_full_step(O, scene, cam, target)
            times.append(r["step_s"])
            isect += r["I_total"]
        wall = time.perf_counter() - t0
        value = isect / sum(times)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": steps, "warmup": a.warmup,
            "ms_per_step": 1e3 * sum(times) / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(a)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": O.num_threads(),
                             "cpu_model": model_name, "logical_cpus": ncpu, "kind": "oracle",
                             "sample": "the whole step, measured", "estimated": False},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "estimated": False, "wall_s": round(wall, 3)}))
        return
    jit = synth.jittered(scene, seed=1)
    cache = {}

    def target_fn(v):
        # the oracle's own render of the jittered copy, on the sampled tiles
        # only matters for the L1 sign; a seeded image stands in for it
        if v not in cache:
            cache[v] = synth.random_image(a.width, a.height, 100 + v).astype(np.float64)
        return cache[v]

    del jit
    osm = OracleSample(scene, cams, target_fn, n_tiles=a.cpu_tiles)
    for k in range(a.warmup):
        osm.step(k % len(cams))
    t0 = time.perf_counter()
    ests, isects, measured = [], [], 0.0
    for k in range(a.steps):
        r = osm.step(k % len(cams))
        ests.append(r["est_step_s"])
        isects.append(r["I_total"])
        measured += r["measured_s"]
    wall = time.perf_counter() - t0
    value = sum(isects) / sum(ests)
    # ms_per_step is the estimate of a whole oracle step from its samples; the
    # samples themselves took measured_sample_s (the run took wall_s)
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
           "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * sum(ests) / a.steps,
           "estimated": True, "measured_sample_s": round(measured, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": workload_name(a)},
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": O.num_threads(),
                            "cpu_model": model_name, "logical_cpus": ncpu,
                            "kind": "oracle", "sample": osm.describe(), "estimated": True,
                            "measured_sample_s": round(measured, 3)},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0},
           "wall_s": round(wall, 3)}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
