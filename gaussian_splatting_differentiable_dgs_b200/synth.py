"""Seeded synthetic scenes and cameras.

This module only draws inputs: Gaussian parameters in the planar layout the
library consumes, pinhole cameras, and jittered copies used to render
targets.  It holds none of the rasteriser's arithmetic and is the one module
that both the CUDA path and the CPU oracle are fed from.

Parameter layout (planar SoA, fp32, ``params[P][n_pad]``):

====================  =========================================
plane                 meaning
====================  =========================================
0, 1, 2               mean x, y, z (world)
3, 4, 5               log-scale per local axis
6, 7, 8, 9            quaternion (w, x, y, z), not normalised
10                    opacity logit (opacity = sigmoid(logit))
11 + 3*k + ch         SH coefficient k = 0 .. (D+1)^2-1, channel ch
====================  =========================================

so P = 11 + 3 (D+1)^2.  ``n_pad`` rounds n up to a multiple of 64 so every
plane starts on a 256-byte boundary; padding entries are zero and are never
read as Gaussians.

Camera convention: world->camera rotation ``R`` (row-major) and translation
``t`` (x_cam = R x_world + t), OpenCV axes (x right, y down, z forward),
principal point at the image centre, square pixels.

Scene recipes follow the workloads of "BoundedGS: memory-efficient training
for high-resolution 3D Gaussian Splatting" (section 03, Table 1 and Fig. 5:
a ~6M-Gaussian outdoor scene rendered from 1K to 16K width) at the sizes the
synthetic configurations name; none of the pages' datasets is reproduced.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Degree-0 real spherical harmonic, 1/(2 sqrt(pi)).  Used only to state the
# input distribution "degree-0 colour ~ U[0,1]" in coefficient space.
_Y00 = 0.5 / math.sqrt(math.pi)

PAD = 64


def n_params(sh_degree: int) -> int:
    return 11 + 3 * (sh_degree + 1) ** 2


def pad_n(n: int) -> int:
    return max(PAD, (n + PAD - 1) // PAD * PAD)


@dataclasses.dataclass
class Camera:
    R: np.ndarray          # (3, 3) float32, world -> camera
    t: np.ndarray          # (3,) float32
    fx: float
    fy: float
    cx: float
    cy: float
    width: int
    height: int

    def as_f32(self) -> "Camera":
        return Camera(np.asarray(self.R, np.float32).reshape(3, 3).copy(),
                      np.asarray(self.t, np.float32).reshape(3).copy(),
                      float(np.float32(self.fx)), float(np.float32(self.fy)),
                      float(np.float32(self.cx)), float(np.float32(self.cy)),
                      int(self.width), int(self.height))

    @property
    def centre(self) -> np.ndarray:
        """Camera centre in world coordinates, -R^T t (float64)."""
        R = self.R.astype(np.float64)
        return -R.T @ self.t.astype(np.float64)


@dataclasses.dataclass
class Scene:
    params: np.ndarray     # (P, n_pad) float32
    n: int
    sh_degree: int

    @property
    def n_pad(self) -> int:
        return self.params.shape[1]

    @property
    def P(self) -> int:
        return self.params.shape[0]

    def copy(self) -> "Scene":
        return Scene(self.params.copy(), self.n, self.sh_degree)


def _empty(n: int, sh_degree: int) -> np.ndarray:
    return np.zeros((n_params(sh_degree), pad_n(n)), np.float32)


def _fill(params, n, sh_degree, mean, log_scale, quat, logit, colour, rng,
          sh_rest_sigma=0.05):
    params[0:3, :n] = mean.T
    params[3:6, :n] = log_scale.T
    params[6:10, :n] = quat.T
    params[10, :n] = logit
    # degree-0 coefficient chosen so that the degree-0 colour equals `colour`
    params[11:14, :n] = ((colour - 0.5) / _Y00).T
    k_sh = (sh_degree + 1) ** 2
    if k_sh > 1:
        rest = rng.normal(0.0, sh_rest_sigma, size=(3 * (k_sh - 1), n))
        params[14:11 + 3 * k_sh, :n] = rest
    return params


def _unit_quats(rng, n):
    q = rng.normal(size=(n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    return q


def look_at(eye, target, up, f, width, height) -> Camera:
    """Pinhole camera at `eye` looking at `target`; image y points along -up."""
    eye = np.asarray(eye, np.float64)
    fwd = np.asarray(target, np.float64) - eye
    fwd /= np.linalg.norm(fwd)
    right = np.cross(fwd, np.asarray(up, np.float64))
    right /= np.linalg.norm(right)
    down = np.cross(fwd, right)
    R = np.stack([right, down, fwd])
    t = -R @ eye
    return Camera(R, t, f, f, width / 2.0, height / 2.0, width, height).as_f32()


def axis_camera(f, width, height) -> Camera:
    """Camera at the origin looking down +z (identity pose)."""
    return Camera(np.eye(3), np.zeros(3), f, f, width / 2.0, height / 2.0,
                  width, height).as_f32()


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

def tiny_oracle_scene(seed: int = 0):
    """2,000 Gaussians, degree 0, 256x256, f = 300, camera at the origin."""
    rng = np.random.default_rng(seed)
    n, D = 2000, 0
    mean = np.stack([rng.uniform(-1, 1, n), rng.uniform(-1, 1, n),
                     rng.uniform(2, 6, n)], axis=1)
    log_scale = rng.normal(-3.5, 0.5, size=(n, 3))
    quat = _unit_quats(rng, n)
    logit = rng.normal(0.0, 1.0, n)
    colour = rng.uniform(0, 1, size=(n, 3))
    params = _fill(_empty(n, D), n, D, mean, log_scale, quat, logit, colour, rng)
    return Scene(params, n, D), [axis_camera(300.0, 256, 256)]


def hd_cluster_scene(seed: int = 0):
    """100,000 Gaussians, degree 3, 64 clusters at z in [3, 15], 1920x1080."""
    rng = np.random.default_rng(seed)
    n, D, k = 100_000, 3, 64
    cz = rng.uniform(3, 15, k)
    centres = np.stack([cz * rng.uniform(-0.6, 0.6, k),
                        cz * rng.uniform(-0.34, 0.34, k), cz], axis=1)
    sig = rng.uniform(0.1, 0.5, size=(k, 3))
    member = np.repeat(np.arange(k), rng.multinomial(n, np.full(k, 1.0 / k)))
    rng.shuffle(member)
    mean = centres[member] + rng.normal(size=(n, 3)) * sig[member]
    log_scale = rng.normal(-4.0, 0.7, size=(n, 3))
    quat = _unit_quats(rng, n)
    logit = rng.normal(0.0, 1.5, n)
    colour = rng.uniform(0, 1, size=(n, 3))
    params = _fill(_empty(n, D), n, D, mean, log_scale, quat, logit, colour, rng)
    return Scene(params, n, D), [axis_camera(1500.0, 1920, 1080)]


def outdoor_scene(n: int = 6_000_000, seed: int = 0, width: int = 5000,
                  height: int = 3300, n_views: int = 8):
    """Outdoor-like scene: 70 % in 512 clusters around a central object, 20 %
    on a noisy ground plane y = -1, 10 % on a far shell at radius 30-60;
    cameras on a circle of radius 4 looking at the origin, f = 0.78125 W."""
    rng = np.random.default_rng(seed)
    D = 3
    n_cl = int(round(0.7 * n))
    n_gp = int(round(0.2 * n))
    n_sh = n - n_cl - n_gp
    # clusters: centres uniform in a ball of radius 1.5
    k = 512
    d = rng.normal(size=(k, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    centres = d * (1.5 * rng.uniform(0, 1, k) ** (1.0 / 3.0))[:, None]
    sig = rng.uniform(0.05, 0.25, size=(k, 3))
    member = np.repeat(np.arange(k), rng.multinomial(n_cl, np.full(k, 1.0 / k)))
    rng.shuffle(member)
    m_cl = centres[member] + rng.normal(size=(n_cl, 3)) * sig[member]
    # ground plane: x, z uniform in a disk of radius 25, y = -1 + N(0, 0.05)
    rad = 25.0 * np.sqrt(rng.uniform(0, 1, n_gp))
    ang = rng.uniform(0, 2 * np.pi, n_gp)
    m_gp = np.stack([rad * np.cos(ang), -1.0 + rng.normal(0, 0.05, n_gp),
                     rad * np.sin(ang)], axis=1)
    # far shell
    d = rng.normal(size=(n_sh, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    m_sh = d * rng.uniform(30, 60, n_sh)[:, None]
    mean = np.concatenate([m_cl, m_gp, m_sh])
    perm = rng.permutation(n)
    mean = mean[perm]
    log_scale = rng.normal(-4.5, 0.8, size=(n, 3))
    quat = _unit_quats(rng, n)
    logit = rng.normal(0.5, 1.5, n)
    colour = rng.uniform(0, 1, size=(n, 3))
    params = _fill(_empty(n, D), n, D, mean, log_scale, quat, logit, colour, rng)
    f = 0.78125 * width
    cams = []
    for v in range(n_views):
        th = 2 * np.pi * v / n_views
        cams.append(look_at((4 * np.cos(th), 0.0, 4 * np.sin(th)), (0, 0, 0),
                            (0, 1, 0), f, width, height))
    return Scene(params, n, D), cams


def sweep_camera(width: int):
    """Camera 0 of the outdoor scene at a given width, 3:2 aspect, fixed FOV."""
    height = int(round(2 * width / 3))
    return look_at((4.0, 0.0, 0.0), (0, 0, 0), (0, 1, 0), 0.78125 * width,
                   width, height)


def tiny_scene(n: int = 8, width: int = 48, height: int = 40, sh_degree: int = 0,
               seed: int = 0, scale_px=(1.5, 5.0), opacity=(0.2, 0.9)):
    """Small scene for finite differences: n Gaussians in front of an
    identity camera, projected sigma roughly in `scale_px` pixels."""
    rng = np.random.default_rng(seed)
    f = 60.0
    z = rng.uniform(2.0, 4.0, n)
    px = rng.uniform(0.15 * width, 0.85 * width, n)
    py = rng.uniform(0.15 * height, 0.85 * height, n)
    mean = np.stack([(px - width / 2) * z / f, (py - height / 2) * z / f, z], 1)
    sig_px = rng.uniform(scale_px[0], scale_px[1], size=(n, 3))
    log_scale = np.log(sig_px * z[:, None] / f)
    quat = _unit_quats(rng, n)
    o = rng.uniform(opacity[0], opacity[1], n)
    logit = np.log(o / (1 - o))
    colour = rng.uniform(0.05, 0.95, size=(n, 3))
    params = _fill(_empty(n, sh_degree), n, sh_degree, mean, log_scale, quat,
                   logit, colour, rng, sh_rest_sigma=0.1)
    return Scene(params, n, sh_degree), [axis_camera(f, width, height)]


def edge_needle_scene(n: int = 48, width: int = 96, height: int = 80,
                      sh_degree: int = 3, seed: int = 0, opacity=(0.02, 0.999)):
    """Needle-thin anisotropic Gaussians around the image border: one local
    axis 8-40 px long, the other two 0.2-0.6 px, random orientations; means
    within 6 px of a random border on either side of it, identity camera."""
    rng = np.random.default_rng(seed)
    f = 60.0
    z = rng.uniform(2.0, 4.0, n)
    side = rng.integers(0, 4, n)
    along = rng.uniform(0.0, 1.0, n)
    across = rng.uniform(-6.0, 6.0, n)
    px = np.where(side == 0, across, np.where(side == 1, width + across, along * width))
    py = np.where(side == 2, across, np.where(side == 3, height + across, along * height))
    mean = np.stack([(px - width / 2) * z / f, (py - height / 2) * z / f, z], 1)
    sig_px = np.stack([rng.uniform(8.0, 40.0, n), rng.uniform(0.2, 0.6, n),
                       rng.uniform(0.2, 0.6, n)], 1)
    log_scale = np.log(sig_px * z[:, None] / f)
    quat = _unit_quats(rng, n)
    o = rng.uniform(opacity[0], opacity[1], n)
    logit = np.log(o / (1 - o))
    colour = rng.uniform(0.05, 0.95, size=(n, 3))
    params = _fill(_empty(n, sh_degree), n, sh_degree, mean, log_scale, quat,
                   logit, colour, rng, sh_rest_sigma=0.1)
    return Scene(params, n, sh_degree), [axis_camera(f, width, height)]


def jittered(scene: Scene, seed: int, mean_sigma=0.02, colour_sigma=0.05) -> Scene:
    """Copy of `scene` with means + N(0, mean_sigma) and the degree-0 colour
    + N(0, colour_sigma) (higher SH bands untouched)."""
    rng = np.random.default_rng(seed)
    s = scene.copy()
    n = s.n
    s.params[0:3, :n] += rng.normal(0, mean_sigma, size=(3, n)).astype(np.float32)
    s.params[11:14, :n] += (rng.normal(0, colour_sigma, size=(3, n)) / _Y00).astype(np.float32)
    return s


def random_image(width: int, height: int, seed: int) -> np.ndarray:
    """Planar fp32 image [3][H][W] with values U[0, 1]."""
    rng = np.random.default_rng(seed)
    return rng.uniform(0, 1, size=(3, height, width)).astype(np.float32)


CONFIGS = {
    "tiny_2k_256": tiny_oracle_scene,
    "hd_100k_1080p": hd_cluster_scene,
    "outdoor_6m_5k": outdoor_scene,
}
