"""Seeded synthetic scenes for the packed 3DGS training step.

This module only draws random numbers and lays them out; it holds none of the
splatting arithmetic (no projection, no SH evaluation, no compositing), so both
the CUDA path and the CPU oracle can be fed from it.

The five workloads stand in for the scenes the pages measure on (the
``art_gallery`` scene with 5 cameras x 15M Gaussians and the ``mandeltorus``
7680x7680 scene on the "Spirula Studio VRAM" page, sections "3 key numbers" and
"4 GiB rule"), which are not available here.  Every array is float32.

Parameters are *activated*: ``scales`` = exp(log-scale), ``opacities`` =
sigmoid(logit).  Quaternions are stored (w, x, y, z) and normalised; the step
normalises them again, so any non-zero quaternion is a valid input.

Cameras are packed as ``cams[C, 20]`` = world-to-camera 4x4 view matrix
(row-major, OpenCV axes: x right, y down, z forward) followed by fx, fy, cx, cy.
"""
from __future__ import annotations

import dataclasses
import numpy as np

SQRT_PI = 1.7724538509055159  # |dc| bound that maps to rgb in [0, 1] at SH degree 0


@dataclasses.dataclass
class Scene:
    cfg: int
    C: int
    W: int
    H: int
    sh_degree: int
    N: int
    near: float
    far: float
    cams: np.ndarray        # [C, 20]
    means: np.ndarray       # [N, 3]
    quats: np.ndarray       # [N, 4]
    scales: np.ndarray      # [N, 3]
    opacities: np.ndarray   # [N]
    sh: np.ndarray          # [N, K, 3]
    upstream: str           # "uniform": v_img given; "l1": v_img = sign(img - target) * l1_scale
    v_img: np.ndarray | None      # [C, H, W, 3] when upstream == "uniform"
    target: np.ndarray | None     # [C, H, W, 3] when upstream == "l1"
    name: str = ""

    @property
    def K(self) -> int:
        return (self.sh_degree + 1) ** 2

    @property
    def l1_scale(self) -> float:
        return 1.0 / (3.0 * self.W * self.H * self.C)

    def dims(self) -> dict:
        return dict(C=self.C, W=self.W, H=self.H, sh_degree=self.sh_degree,
                    N=self.N, near=self.near, far=self.far)


def look_at(eye, target, up=(0.0, 1.0, 0.0)) -> np.ndarray:
    """World-to-camera matrix with OpenCV axes (x right, y down, z forward)."""
    eye = np.asarray(eye, np.float64)
    fwd = np.asarray(target, np.float64) - eye
    fwd /= np.linalg.norm(fwd)
    right = np.cross(fwd, np.asarray(up, np.float64))
    right /= np.linalg.norm(right)
    down = np.cross(fwd, right)
    R = np.stack([right, down, fwd])
    V = np.eye(4)
    V[:3, :3] = R
    V[:3, 3] = -R @ eye
    return V


def _cam(V, fx, fy, cx, cy) -> np.ndarray:
    return np.concatenate([np.asarray(V, np.float64).reshape(16), [fx, fy, cx, cy]]).astype(np.float32)


def _quats(rng, n):
    q = rng.standard_normal((n, 4))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    return q.astype(np.float32)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _sh(rng, n, degree, dc_low, dc_high, rest_sigma):
    K = (degree + 1) ** 2
    sh = np.empty((n, K, 3), np.float32)
    sh[:, 0, :] = rng.uniform(dc_low, dc_high, (n, 3))
    if K > 1:
        sh[:, 1:, :] = rng.standard_normal((n, K - 1, 3), dtype=np.float32) * np.float32(rest_sigma)
    return sh


def _ball(rng, n, sigma, radius):
    out = np.empty((0, 3))
    while len(out) < n:
        p = rng.normal(0.0, sigma, (2 * (n - len(out)) + 16, 3))
        p = p[np.linalg.norm(p, axis=1) <= radius]
        out = np.concatenate([out, p])
    return out[:n]


# Camera placements found once on the CPU with the oracle's visibility and
# tile counts on subsampled scenes; frozen here so every run sees the same
# scene.  Workload 3: ring of radius 8, each camera turned 47 degrees away from
# the centre (about 30% of pairs visible).  Workload 4: five cameras on a
# radius-22 ring around the room at height 1.5, turned +-41.5 degrees away from
# the centre (about 20% of pairs visible, about 2.2 tiles per row).
# Workload 5: camera 13.8 from the origin (about 5.9e8 intersections).
CFG3_YAW_DEG = 47.0
CFG4_RING = (22.0, 1.5, 41.5)
CFG5_EYE_DIR = (0.0, 4.2, 6.3)
CFG5_DIST = 13.8


def _yawed(eye, yaw_deg):
    eye = np.asarray(eye, np.float64)
    fwd = -eye / np.linalg.norm(eye)
    a = np.deg2rad(yaw_deg)
    R = np.array([[np.cos(a), 0, np.sin(a)], [0, 1, 0], [-np.sin(a), 0, np.cos(a)]])
    return look_at(eye, eye + R @ fwd)


def make_scene(cfg: int, n: int | None = None, seed: int | None = None) -> Scene:
    """Build workload ``cfg`` (1..5).  ``n`` overrides the Gaussian count (same
    distributions, fewer samples) for fast tests; ``seed`` overrides the seed
    (default cfg - 1)."""
    rng = np.random.Generator(np.random.PCG64(cfg - 1 if seed is None else seed))
    near, far = 0.01, 1e10
    if cfg == 1:
        N = 2000 if n is None else n
        means = rng.uniform(-1.0, 1.0, (N, 3))
        scales = np.exp(rng.normal(-3.5, 0.5, (N, 3)))
        quats = _quats(rng, N)
        opac = _sigmoid(rng.normal(0.0, 1.0, N))
        sh = _sh(rng, N, 0, -SQRT_PI, SQRT_PI, 0.0)  # rgb uniform in [0, 1]
        W = H = 128
        cams = np.stack([_cam(look_at((0, 0, 4), (0, 0, 0)), 120, 120, 64, 64)])
        v_img = rng.uniform(-1.0, 1.0, (1, H, W, 3)).astype(np.float32)
        return Scene(cfg, 1, W, H, 0, N, near, far, cams, means.astype(np.float32), quats,
                     scales.astype(np.float32), opac.astype(np.float32), sh, "uniform", v_img,
                     None, "tiny: 2k Gaussians, 1 camera, 128x128, SH0")
    if cfg == 2:
        N = 100_000 if n is None else n
        means = _ball(rng, N, 1.5, 4.5)
        scales = np.exp(rng.normal(-4.0, 0.6, (N, 3)))
        quats = _quats(rng, N)
        opac = _sigmoid(rng.normal(0.0, 1.5, N))
        sh = _sh(rng, N, 3, 0.0, 1.0, 0.05)
        W, H = 640, 480
        cams = np.stack([_cam(look_at((0, 0, 6), (0, 0, 0)), 500, 500, 320, 240)])
        trng = np.random.Generator(np.random.PCG64(100 + (cfg - 1 if seed is None else seed)))
        target = trng.uniform(0.0, 1.0, (1, H, W, 3)).astype(np.float32)
        return Scene(cfg, 1, W, H, 3, N, near, far, cams, means.astype(np.float32), quats,
                     scales.astype(np.float32), opac.astype(np.float32), sh, "l1", None, target,
                     "100k Gaussians, 1 camera, 640x480, SH3, L1 upstream")
    if cfg == 3:
        N = 1_000_000 if n is None else n
        n_plane = int(round(0.7 * N))
        plane = np.stack([rng.uniform(-5, 5, n_plane), -2.0 + rng.normal(0, 0.05, n_plane),
                          rng.uniform(-5, 5, n_plane)], 1)
        box = np.stack([rng.uniform(-5, 5, N - n_plane), rng.uniform(-2, 2, N - n_plane),
                        rng.uniform(-5, 5, N - n_plane)], 1)
        means = np.concatenate([plane, box])[rng.permutation(N)]
        scales = np.exp(rng.normal(-4.5, 0.7, (N, 3)))
        quats = _quats(rng, N)
        opac = _sigmoid(rng.normal(0.0, 1.5, N))
        sh = _sh(rng, N, 3, 0.0, 1.0, 0.05)
        W, H = 1280, 720
        cams = []
        for k in range(4):
            th = np.deg2rad(90.0 * k)
            cams.append(_cam(_yawed((8 * np.sin(th), 0.0, 8 * np.cos(th)), CFG3_YAW_DEG), 900, 900, 640, 360))
        trng = np.random.Generator(np.random.PCG64(100 + (cfg - 1 if seed is None else seed)))
        target = trng.uniform(0.0, 1.0, (4, H, W, 3)).astype(np.float32)
        return Scene(cfg, 4, W, H, 3, N, near, far, np.stack(cams), means.astype(np.float32), quats,
                     scales.astype(np.float32), opac.astype(np.float32), sh, "l1", None, target,
                     "1M Gaussians, 4 cameras on a ring, 1280x720, SH3")
    if cfg == 4:
        N = 15_000_000 if n is None else n
        n_shell = int(round(0.2 * N))
        n_cl = N - n_shell
        half = np.array([8.0, 3.0, 8.0])
        centres = rng.uniform(-half, half, (64, 3))
        which = rng.integers(0, 64, n_cl)
        clusters = centres[which] + rng.normal(0.0, 0.5, (n_cl, 3))
        # uniform on the six faces of the 16 x 6 x 16 room, area-weighted
        areas = np.array([6 * 16, 6 * 16, 16 * 16, 16 * 16, 16 * 6, 16 * 6], np.float64)
        face = rng.choice(6, n_shell, p=areas / areas.sum())
        shell = rng.uniform(-half, half, (n_shell, 3))
        axis = face // 2
        sign = np.where(face % 2 == 0, -1.0, 1.0)
        shell[np.arange(n_shell), axis] = sign * half[axis]
        means = np.concatenate([clusters, shell])[rng.permutation(N)]
        scales = np.exp(rng.normal(-5.0, 0.8, (N, 3)))
        quats = _quats(rng, N)
        opac = _sigmoid(rng.normal(0.0, 1.5, N))
        sh = _sh(rng, N, 3, 0.0, 1.0, 0.05)
        W, H = 1600, 1067
        D, h, yaw = CFG4_RING
        cams = []
        for k in range(5):
            th = np.deg2rad(72.0 * k + 10.0)
            cams.append(_cam(_yawed((D * np.sin(th), h, D * np.cos(th)), yaw if k % 2 else -yaw),
                             1400, 1400, 800, 533.5))
        cams = np.stack(cams)
        trng = np.random.Generator(np.random.PCG64(100 + (cfg - 1 if seed is None else seed)))
        target = trng.uniform(0.0, 1.0, (5, H, W, 3)).astype(np.float32)
        return Scene(cfg, 5, W, H, 3, N, near, far, cams, means.astype(np.float32), quats,
                     scales.astype(np.float32), opac.astype(np.float32), sh, "l1", None, target,
                     "15M Gaussians, 5 cameras in a room, 1600x1067, SH3 (75M pairs)")
    if cfg == 5:
        N = 13_000_000 if n is None else n
        R0, r0 = 2.0, 0.7
        u = rng.uniform(0, 2 * np.pi, N)
        v = rng.uniform(0, 2 * np.pi, N)
        nrm = np.stack([np.cos(u) * np.cos(v), np.sin(v), np.sin(u) * np.cos(v)], 1)
        ring = np.stack([np.cos(u), np.zeros(N), np.sin(u)], 1) * R0
        means = ring + nrm * (r0 + rng.normal(0.0, 0.02, N))[:, None]
        scales = np.exp(rng.normal(-3.8, 0.5, (N, 3)))
        quats = _quats(rng, N)
        opac = _sigmoid(rng.normal(0.0, 1.5, N))
        sh = _sh(rng, N, 3, 0.0, 1.0, 0.05)
        W = H = 7680
        eye = np.asarray(CFG5_EYE_DIR) / np.linalg.norm(CFG5_EYE_DIR) * CFG5_DIST
        cams = np.stack([_cam(look_at(eye, (0, 0, 0)), 6000, 6000, 3840, 3840)])
        trng = np.random.Generator(np.random.PCG64(100 + (cfg - 1 if seed is None else seed)))
        v_img = (trng.uniform(-1.0, 1.0, (1, H, W, 3)) / (3.0 * W * H)).astype(np.float32)
        return Scene(cfg, 1, W, H, 3, N, near, far, cams, means.astype(np.float32), quats,
                     scales.astype(np.float32), opac.astype(np.float32), sh, "uniform", v_img,
                     None, "13M Gaussians on a torus, 1 camera, 7680x7680, SH3")
    raise ValueError(f"unknown workload {cfg}")


def random_tiny(seed: int, N: int = 6, W: int = 32, H: int = 32, C: int = 1, sh_degree: int = 1,
                opacity_range=(0.1, 0.9)) -> Scene:
    """Small random scenes for brute-force and finite-difference checks."""
    rng = np.random.Generator(np.random.PCG64(1000 + seed))
    means = rng.uniform(-0.6, 0.6, (N, 3))
    scales = np.exp(rng.uniform(-2.5, -1.2, (N, 3)))
    quats = _quats(rng, N)
    opac = rng.uniform(opacity_range[0], opacity_range[1], N)
    sh = _sh(rng, N, sh_degree, 0.0, 1.0, 0.2)
    cams = []
    for c in range(C):
        th = 0.35 * c
        eye = (3.0 * np.sin(th), 0.3 * c, 3.0 * np.cos(th))
        f = 0.9 * W
        cams.append(_cam(look_at(eye, (0, 0, 0)), f, f * 1.05, 0.5 * W + 0.3, 0.5 * H - 0.2))
    v_img = rng.uniform(-1.0, 1.0, (C, H, W, 3)).astype(np.float32)
    return Scene(0, C, W, H, sh_degree, N, 0.01, 1e10, np.stack(cams), means.astype(np.float32),
                 quats, scales.astype(np.float32), opac.astype(np.float32), sh, "uniform", v_img,
                 None, f"random tiny #{seed}")
