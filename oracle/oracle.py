"""ctypes wrapper of the CPU oracle (liboracle.so).  TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this module.  It imports nothing from the CUDA package; scenes
come from the shared seeded generator, which holds no splatting arithmetic.

Every function restates one step of the packed 3DGS step in plain serial form
(see oracle.cpp for the per-step citations):
  project      packed projection + both compactions (plain flag scan and bitmask)
  intersect    tile intersections by the per-tile overlap test, range form checked
  sort         std::stable_sort by key
  tile_ranges  per-tile [start, end) by counting
  rasterize_fwd / rasterize_bwd / project_bwd  one pixel / one row at a time
  raw_gradients, adam_step                      the fused optimizer step (numpy, fp64)
  gq_quantise, gq_decode, gq_accumulate         block-quantised gradient accumulation (numpy)
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None

PAIRS_PER_BLOCK = 128
TILE = 16
ROW = 12


class Dims(ct.Structure):
    _fields_ = [("C", ct.c_int32), ("W", ct.c_int32), ("H", ct.c_int32), ("sh_degree", ct.c_int32),
                ("N", ct.c_int64), ("near_plane", ct.c_float), ("far_plane", ct.c_float)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        P = ct.c_void_p
        i64, i32 = ct.c_int64, ct.c_int
        L.orc_exp_fp32.argtypes = [ct.c_float]
        L.orc_exp_fp32.restype = ct.c_float
        L.orc_exp_fp32_vec.argtypes = [P, P, i64]
        L.orc_sh_basis_f64.argtypes = [i32, ct.c_double, ct.c_double, ct.c_double, P]
        L.orc_sh_basis_grad_f64.argtypes = [i32, ct.c_double, ct.c_double, ct.c_double, P]
        L.orc_geometry.argtypes = [P, P]
        L.orc_project.argtypes = [P, P, P, P, P, P, P, i32, P, P, P, P, P, P, P, P, P, i64, i32, i64]
        L.orc_row_boxes.argtypes = [P, P, P, P, P, P, P, P, i64, P]
        L.orc_count_tiles.argtypes = [P, P, i64, P, P]
        L.orc_intersect.argtypes = [P, P, P, P, i64, i32, P, P, i64, P, P]
        L.orc_sort.argtypes = [P, P, i64]
        L.orc_tile_ranges.argtypes = [P, i64, i64, P]
        L.orc_rasterize_fwd.argtypes = [P, P, P, P, i32, P, P, P, P, P, i32, P, P]
        L.orc_rasterize_bwd.argtypes = [P, P, P, P, P, P, i32, i64, P, i32, P, P]
        L.orc_project_bwd.argtypes = [P, P, P, P, P, P, P, P, P, i64, P, i32, P, P, P, P, P]
        L.orc_tile_counts.argtypes = [P, P, P, i64, P]
        L.orc_tile_lists.argtypes = [P, P, P, P, i64, P, i64, P, P, P, i64]
        L.orc_rasterize_tiles.argtypes = [P, P, P, P, P, P, i64, P, P, P, i32]
        L.orc_raster_bwd_rows.argtypes = [P, P, P, P, P, i64, P, P, P, i64, P, i32]
        L.orc_project_bwd_rows.argtypes = [P, P, P, P, P, P, P, P, P, i64, P, P]
        for f in ("orc_project", "orc_row_boxes", "orc_count_tiles", "orc_intersect", "orc_sort",
                  "orc_tile_ranges", "orc_rasterize_fwd", "orc_rasterize_bwd", "orc_project_bwd",
                  "orc_tile_counts", "orc_tile_lists", "orc_rasterize_tiles", "orc_raster_bwd_rows",
                  "orc_project_bwd_rows"):
            getattr(L, f).restype = ct.c_int
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ct.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def dims_of(scene) -> Dims:
    return Dims(scene.C, scene.W, scene.H, scene.sh_degree, scene.N, scene.near, scene.far)


def geometry(scene) -> dict:
    out = np.zeros(6, np.int64)
    d = dims_of(scene)
    lib().orc_geometry(ct.byref(d), _p(out))
    keys = ("tiles_x", "tiles_y", "tiles_per_cam", "n_pad", "words_per_cam", "blocks_per_cam")
    g = {k: int(v) for k, v in zip(keys, out)}
    g["n_tiles"] = g["tiles_per_cam"] * scene.C
    g["mask_words"] = g["words_per_cam"] * scene.C
    g["mask_blocks"] = g["blocks_per_cam"] * scene.C
    return g


def exp_fp32(x: float) -> float:
    return float(lib().orc_exp_fp32(ct.c_float(x)))


def exp_fp32_vec(x) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().orc_exp_fp32_vec(_p(x), _p(y), x.size)
    return y


def sh_basis(degree: int, d) -> np.ndarray:
    out = np.zeros(16)
    lib().orc_sh_basis_f64(degree, float(d[0]), float(d[1]), float(d[2]), _p(out))
    return out[: (degree + 1) ** 2]


def sh_basis_grad(degree: int, d) -> np.ndarray:
    out = np.zeros((16, 3))
    lib().orc_sh_basis_grad_f64(degree, float(d[0]), float(d[1]), float(d[2]), _p(out))
    return out[: (degree + 1) ** 2]


def _inputs(scene):
    """All oracle inputs are fp64; fp32 scene arrays convert exactly."""
    return dict(cams=_c(scene.cams, np.float64), means=_c(scene.means, np.float64),
                quats=_c(scene.quats, np.float64), scales=_c(scene.scales, np.float64),
                opac=_c(scene.opacities, np.float64), sh=_c(scene.sh, np.float64))


def project(scene, precision: int = 0, nthreads: int = 0, rows: bool = True, cap_max: int | None = None) -> dict:
    """Packed projection.  cap_max (per-image visible cap): in each camera
    with more visible pairs, keep the cap_max of highest opacity (ties to the
    lower Gaussian index)."""
    g = geometry(scene)
    d = dims_of(scene)
    x = _inputs(scene)
    mask = np.zeros(g["mask_words"], np.uint32)
    bc = np.zeros(g["mask_blocks"], np.uint32)
    bo = np.zeros(g["mask_blocks"] + 1, np.int64)
    nnz = ct.c_int64(0)
    L = lib()
    args = [ct.byref(d), _p(x["cams"]), _p(x["means"]), _p(x["quats"]), _p(x["scales"]), _p(x["opac"]),
            _p(x["sh"]), precision, _p(mask), _p(bc), _p(bo), ct.byref(nnz)]
    cap = -1 if cap_max is None else int(cap_max)
    rc = L.orc_project(*args, None, None, None, None, None, 0, nthreads, cap)
    if rc != 0:
        raise RuntimeError(f"oracle projection: compactions disagree (rc={rc})")
    out = dict(mask=mask, block_count=bc, block_off=bo, nnz=int(nnz.value))
    if not rows:
        return out
    n = out["nnz"]
    screen = np.zeros((max(n, 1), ROW), np.float64)
    aabb = np.zeros((max(n, 1), 2), np.uint32)
    row_cam = np.zeros(max(n, 1), np.int32)
    row_gauss = np.zeros(max(n, 1), np.int64)
    rgb_cl = np.zeros((max(n, 1), 3), np.uint8)
    rc = L.orc_project(*args, _p(screen), _p(aabb), _p(row_cam), _p(row_gauss), _p(rgb_cl), n, nthreads, cap)
    if rc != 0:
        raise RuntimeError(f"oracle projection failed (rc={rc})")
    out.update(screen=screen[:n], aabb=aabb[:n], row_cam=row_cam[:n], row_gauss=row_gauss[:n],
               rgb_clamped=rgb_cl[:n])
    return out


def row_boxes(scene, proj) -> np.ndarray:
    d = dims_of(scene)
    x = _inputs(scene)
    n = proj["nnz"]
    box = np.zeros((max(n, 1), 4), np.float32)
    rc = lib().orc_row_boxes(ct.byref(d), _p(x["cams"]), _p(x["means"]), _p(x["quats"]), _p(x["scales"]),
                             _p(x["opac"]), _p(_c(proj["row_cam"], np.int32)),
                             _p(_c(proj["row_gauss"], np.int64)), n, _p(box))
    if rc != 0:
        raise RuntimeError("row_boxes: row not visible")
    return box[:n]


def count_tiles(scene, aabb) -> tuple[np.ndarray, int]:
    d = dims_of(scene)
    n = len(aabb)
    per = np.zeros(max(n, 1), np.int64)
    tot = ct.c_uint64(0)
    lib().orc_count_tiles(ct.byref(d), _p(_c(aabb, np.uint32)), n, _p(per), ct.byref(tot))
    return per[:n], int(tot.value)


def intersect(scene, proj, all_pairs: bool | None = None) -> dict:
    """Intersection keys and values, rows visited in order of depth (ties by
    row index), each row's tiles row-major; `order` is that visiting order."""
    g = geometry(scene)
    d = dims_of(scene)
    n = proj["nnz"]
    _, total = count_tiles(scene, proj["aabb"])
    if all_pairs is None:
        all_pairs = n * g["tiles_per_cam"] <= 200_000_000
    keys = np.zeros(max(total, 1), np.uint64)
    vals = np.zeros(max(total, 1), np.uint32)
    order = np.zeros(max(n, 1), np.int64)
    tot = ct.c_uint64(0)
    rc = lib().orc_intersect(ct.byref(d), _p(_c(proj["screen"], np.float64)), _p(_c(proj["aabb"], np.uint32)),
                             _p(_c(proj["row_cam"], np.int32)), n, int(all_pairs), _p(keys), _p(vals), total,
                             ct.byref(tot), _p(order))
    if rc != 0:
        raise RuntimeError(f"oracle intersect: range form and overlap test disagree (rc={rc})")
    return dict(keys=keys[:total], vals=vals[:total], n_isects=int(tot.value), order=order[:n])


def sort(keys, vals) -> tuple[np.ndarray, np.ndarray]:
    k = np.array(keys, np.uint64, copy=True)
    v = np.array(vals, np.uint32, copy=True)
    lib().orc_sort(_p(k), _p(v), len(k))
    return k, v


def tile_ranges(keys, n_tiles: int) -> np.ndarray:
    off = np.zeros(n_tiles + 1, np.int64)
    k = _c(keys, np.uint64)
    if lib().orc_tile_ranges(_p(k), len(k), n_tiles, _p(off)) != 0:
        raise RuntimeError("tile id out of range")
    return off


def rasterize_fwd(scene, screen, vals_sorted, tile_off, precision: int = 0, nthreads: int = 0,
                  evals: bool = False, bg=None, depth: bool = False):
    """img, T, last (then ev, cp with evals, then the expected depth with
    depth=True).  bg: [C][3] background blended as img = C + T * bg."""
    d = dims_of(scene)
    img = np.zeros((scene.C, scene.H, scene.W, 3))
    T = np.zeros((scene.C, scene.H, scene.W))
    last = np.zeros((scene.C, scene.H, scene.W), np.int64)
    ev = np.zeros((scene.C, scene.H, scene.W), np.int64) if evals else None
    cp = np.zeros((scene.C, scene.H, scene.W), np.int64) if evals else None
    D = np.zeros((scene.C, scene.H, scene.W)) if depth else None
    bgc = None if bg is None else _c(np.asarray(bg, np.float64).reshape(scene.C, 3), np.float64)
    lib().orc_rasterize_fwd(ct.byref(d), _p(_c(screen, np.float64)), _p(_c(vals_sorted, np.uint32)),
                            _p(_c(tile_off, np.int64)), precision, _p(img), _p(T), _p(last), _p(ev), _p(cp),
                            nthreads, _p(D), _p(bgc))
    out = (img, T, last) + ((ev, cp) if evals else ()) + ((D,) if depth else ())
    return out


def rasterize_bwd(scene, screen, vals_sorted, tile_off, v_img, v_T=None, precision: int = 0,
                  nthreads: int = 0, v_depth=None, bg=None) -> np.ndarray:
    d = dims_of(scene)
    n = len(screen)
    vs = np.zeros((max(n, 1), ROW))
    vT = None if v_T is None else _c(v_T, np.float64)
    vD = None if v_depth is None else _c(v_depth, np.float64)
    bgc = None if bg is None else _c(np.asarray(bg, np.float64).reshape(scene.C, 3), np.float64)
    lib().orc_rasterize_bwd(ct.byref(d), _p(_c(screen, np.float64)), _p(_c(vals_sorted, np.uint32)),
                            _p(_c(tile_off, np.int64)), _p(_c(v_img, np.float64)), _p(vT), precision, n,
                            _p(vs), nthreads, _p(vD), _p(bgc))
    return vs[:n]


def project_bwd(scene, proj, v_screen, precision: int = 0) -> dict:
    d = dims_of(scene)
    x = _inputs(scene)
    N, K = scene.N, scene.K
    out = dict(v_means=np.zeros((N, 3)), v_quats=np.zeros((N, 4)), v_scales=np.zeros((N, 3)),
               v_opacities=np.zeros(N), v_sh=np.zeros((N, K, 3)))
    lib().orc_project_bwd(ct.byref(d), _p(x["cams"]), _p(x["means"]), _p(x["quats"]), _p(x["scales"]),
                          _p(x["opac"]), _p(x["sh"]), _p(_c(proj["row_cam"], np.int32)),
                          _p(_c(proj["row_gauss"], np.int64)), proj["nnz"], _p(_c(v_screen, np.float64)),
                          precision, _p(out["v_means"]), _p(out["v_quats"]), _p(out["v_scales"]),
                          _p(out["v_opacities"]), _p(out["v_sh"]))
    return out


def upstream(scene, img) -> np.ndarray:
    """dL/dimage of the scene: the given uniform field, or the L1 gradient
    sign(img - target) / (3 W H C) against the scene's target."""
    if scene.upstream == "uniform":
        return np.asarray(scene.v_img, np.float32)
    return (np.sign(np.asarray(img, np.float64) - scene.target) * scene.l1_scale).astype(np.float32)


def forward(scene, precision: int = 0, nthreads: int = 0, bg=None, depth: bool = False,
            cap_max: int | None = None) -> dict:
    g = geometry(scene)
    proj = project(scene, precision, nthreads, cap_max=cap_max)
    isect = intersect(scene, proj)
    ks, vs = sort(isect["keys"], isect["vals"])
    toff = tile_ranges(ks, g["n_tiles"])
    r = rasterize_fwd(scene, proj["screen"], vs, toff, precision, nthreads, bg=bg, depth=depth)
    f = dict(proj=proj, isect=isect, keys_sorted=ks, vals_sorted=vs, tile_off=toff, img=r[0], T=r[1],
             last=r[2], geo=g)
    if depth:
        f["depth"] = r[3]
    return f


def step(scene, precision: int = 0, nthreads: int = 0, v_img=None, v_T=None, v_depth=None, bg=None,
         cap_max: int | None = None) -> dict:
    """One forward+backward pass; gradients in fp64.  With v_depth the
    forward also returns the expected depth and the backward takes its
    gradient; bg blends a background colour per camera; cap_max applies the
    per-image visible cap (see project)."""
    f = forward(scene, precision, nthreads, bg=bg, depth=v_depth is not None, cap_max=cap_max)
    if v_img is None:
        v_img = upstream(scene, f["img"])
    v_screen = rasterize_bwd(scene, f["proj"]["screen"], f["vals_sorted"], f["tile_off"], v_img, v_T, precision,
                             nthreads, v_depth=v_depth, bg=bg)
    grads = project_bwd(scene, f["proj"], v_screen, precision)
    f.update(v_img=v_img, v_screen=v_screen, grads=grads)
    return f


# ---------------------------------------------------------------------------- sampled checks at full size
def tile_counts(scene, proj) -> np.ndarray:
    g = geometry(scene)
    d = dims_of(scene)
    out = np.zeros(g["n_tiles"], np.int64)
    lib().orc_tile_counts(ct.byref(d), _p(_c(proj["aabb"], np.uint32)), _p(_c(proj["row_cam"], np.int32)),
                          proj["nnz"], _p(out))
    return out


def tile_lists(scene, proj, tiles) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Sorted (key, row) lists of the given tiles: (offsets, keys, vals)."""
    d = dims_of(scene)
    sel = _c(tiles, np.int64)
    off = np.zeros(len(sel) + 1, np.int64)
    cap = 1
    while True:
        keys = np.zeros(cap, np.uint64)
        vals = np.zeros(cap, np.uint32)
        rc = lib().orc_tile_lists(ct.byref(d), _p(_c(proj["screen"], np.float64)), _p(_c(proj["aabb"], np.uint32)),
                                  _p(_c(proj["row_cam"], np.int32)), proj["nnz"], _p(sel), len(sel), _p(off),
                                  _p(keys), _p(vals), cap)
        if rc == 0:
            return off, keys[: off[-1]], vals[: off[-1]]
        cap = int(off[-1]) + 1


def rasterize_tiles(scene, proj, tiles, off, vals, starts, nthreads: int = 0):
    """Pixels of the selected tiles: img [n][256][3], T [n][256], last [n][256]
    (global sorted index; -2 outside the image)."""
    d = dims_of(scene)
    n = len(tiles)
    img = np.zeros((n, 256, 3))
    T = np.zeros((n, 256))
    last = np.zeros((n, 256), np.int64)
    lib().orc_rasterize_tiles(ct.byref(d), _p(_c(proj["screen"], np.float64)), _p(_c(vals, np.uint32)),
                              _p(_c(off, np.int64)), _p(_c(tiles, np.int64)), _p(_c(starts, np.int64)), n, _p(img),
                              _p(T), _p(last), nthreads)
    return img, T, last


def raster_bwd_rows(scene, proj, tiles, off, vals, v_img, v_T, rows, nthreads: int = 0) -> np.ndarray:
    """Screen-row gradients [len(rows)][12] of the selected rows; `tiles` must
    cover every tile those rows touch."""
    d = dims_of(scene)
    slot = np.full(proj["nnz"], -1, np.int64)
    slot[np.asarray(rows, np.int64)] = np.arange(len(rows))
    out = np.zeros((len(rows), ROW))
    vT = None if v_T is None else _c(v_T, np.float64)
    lib().orc_raster_bwd_rows(ct.byref(d), _p(_c(proj["screen"], np.float64)), _p(_c(vals, np.uint32)),
                              _p(_c(off, np.int64)), _p(_c(tiles, np.int64)), len(tiles),
                              _p(_c(v_img, np.float64)), _p(vT), _p(slot), len(rows), _p(out), nthreads)
    return out


def project_bwd_rows(scene, proj, rows, v_rows) -> np.ndarray:
    """Per-row gradient contributions [len(rows)][11 + 3K]: means(3) quats(4)
    scales(3) opacity(1) sh(3K)."""
    d = dims_of(scene)
    x = _inputs(scene)
    rows = np.asarray(rows, np.int64)
    out = np.zeros((len(rows), 11 + 3 * scene.K))
    lib().orc_project_bwd_rows(ct.byref(d), _p(x["cams"]), _p(x["means"]), _p(x["quats"]), _p(x["scales"]),
                               _p(x["opac"]), _p(x["sh"]), _p(_c(proj["row_cam"][rows], np.int32)),
                               _p(_c(proj["row_gauss"][rows], np.int64)), len(rows), _p(_c(v_rows, np.float64)),
                               _p(out))
    return out


# ---------------------------------------------------------------------------- fused optimizer step
ADAM_GROUPS = ("means", "quats", "log_scales", "logit_opacities", "sh")


def raw_gradients(grads: dict, scales, opacities) -> dict:
    """Gradients of the raw parameters from the activated ones: means and
    quaternions unchanged, log-scales through s = exp(log s) (ds/dlog s = s),
    logit-opacities through o = sigmoid(logit) (do/dlogit = o (1 - o))."""
    s = np.asarray(scales, np.float64)
    o = np.asarray(opacities, np.float64)
    return dict(means=grads["v_means"], quats=grads["v_quats"], log_scales=grads["v_scales"] * s,
                logit_opacities=grads["v_opacities"] * o * (1.0 - o), sh=grads["v_sh"])


def adam_step(params: dict, grads: dict, m: dict, v: dict, lr: dict, beta1: float, beta2: float, eps: float,
              t: int):
    """One Adam update with bias correction, element by element (fp64):
    m = b1 m + (1 - b1) g, v = b2 v + (1 - b2) g^2,
    p = p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps).
    lr maps each group to its rate; "sh" may be a pair (DC rate, rest rate)
    applied to coefficient 0 and to the others.  Returns new (params, m, v)."""
    P, M, V = {}, {}, {}
    for k in params:
        g = np.asarray(grads[k], np.float64)
        m1 = beta1 * np.asarray(m[k], np.float64) + (1.0 - beta1) * g
        v1 = beta2 * np.asarray(v[k], np.float64) + (1.0 - beta2) * g * g
        step = (m1 / (1.0 - beta1 ** t)) / (np.sqrt(v1 / (1.0 - beta2 ** t)) + eps)
        rate = lr[k]
        if k == "sh" and isinstance(rate, tuple):
            r = np.full(step.shape, rate[1])
            r[:, 0, :] = rate[0]
            rate = r
        P[k] = np.asarray(params[k], np.float64) - rate * step
        M[k], V[k] = m1, v1
    return P, M, V


# ---------------------------------------------------------------------------- block-quantised gradient accumulation
# "Spirula Studio backward pass", section 6, technique 1 (grad-quant): each
# attribute's gradient accumulator is kept as 16-bit codes in blocks of 256
# Gaussians; for every sub-batch the projection backward decodes the
# accumulator, adds the sub-batch's gradient and quantises again.  The page
# names the block size and the code width only.  Readings: one scale per
# (attribute, block) = the block's largest magnitude / 32767, codes =
# round-half-even(x / scale) (so the largest element maps to +-32767 and no
# clamp is ever needed), an all-zero block has scale 0 and codes 0; the six
# attributes are the page's gradient outputs (means, quaternions, scales,
# opacities, DC colour, higher SH coefficients).
GQ_BLOCK = 256
GQ_MAX = 32767


def gq_attributes(grads: dict) -> dict:
    """The six accumulated attributes, [N, width] each, from the gradient
    dict of project_bwd (v_sh split into its DC and higher coefficients)."""
    N = np.asarray(grads["v_means"]).shape[0]
    sh = np.asarray(grads["v_sh"], np.float64)
    return dict(means=np.asarray(grads["v_means"], np.float64).reshape(N, -1),
                quats=np.asarray(grads["v_quats"], np.float64).reshape(N, -1),
                scales=np.asarray(grads["v_scales"], np.float64).reshape(N, -1),
                opacities=np.asarray(grads["v_opacities"], np.float64).reshape(N, 1),
                sh_dc=sh[:, :1, :].reshape(N, -1), sh_rest=sh[:, 1:, :].reshape(N, -1))


def gq_quantise(x) -> tuple[np.ndarray, np.ndarray]:
    """Codes [N, w] (int16) and per-block scales [ceil(N/256)] of x [N, w]."""
    x = np.asarray(x, np.float64)
    N = x.shape[0]
    nb = (N + GQ_BLOCK - 1) // GQ_BLOCK
    codes = np.zeros(x.shape, np.int16)
    scales = np.zeros(nb, np.float64)
    for b in range(nb):
        blk = x[b * GQ_BLOCK:(b + 1) * GQ_BLOCK]
        m = float(np.abs(blk).max()) if blk.size else 0.0
        if m > 0.0:
            scales[b] = m / GQ_MAX
            codes[b * GQ_BLOCK:(b + 1) * GQ_BLOCK] = np.rint(blk / scales[b]).astype(np.int16)
    return codes, scales


def gq_decode(codes, scales) -> np.ndarray:
    """Values [N, w] of an accumulator: code times its block's scale."""
    codes = np.asarray(codes)
    N = codes.shape[0]
    per_row = np.repeat(np.asarray(scales, np.float64), GQ_BLOCK)[:N]
    return codes.astype(np.float64) * per_row.reshape((N,) + (1,) * (codes.ndim - 1))


def gq_accumulate(acc: dict | None, grads: dict) -> dict:
    """One sub-batch: decode the accumulator (None: start from zero), add the
    sub-batch's gradients, quantise again.  Returns {attribute: (codes, scales)}."""
    out = {}
    for name, g in gq_attributes(grads).items():
        x = g if acc is None else gq_decode(*acc[name]) + g
        out[name] = gq_quantise(x)
    return out
