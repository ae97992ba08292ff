"""Pins of the CPU oracle against what the pages and mathematics fix.

Nothing here calls the CUDA path.  Each test targets a mistake that could hide
in the oracle (a dropped term, a wrong sign or index, a transposed operand):

* exp:         error bound against fp64 exp on a dense sweep;
* SH basis:    the library's complex spherical harmonics (scipy) in real form,
               and finite differences of the basis for its gradient;
* projection:  closed forms (pinhole mean, isotropic 2D covariance, the
               off-axis Jacobian limit), quaternion rotation from scipy, matrix
               inverse from numpy;
* compaction:  the plain flag scan and the bitmask scan agree (checked inside the
               oracle) and the popcount bookkeeping reproduces the pages' sizes;
* AABB16:      the decoded box contains the float box exactly and the step
               sizes the page prints;
* intersect:   the all-tiles overlap test equals the range form; tile sets only
               grow by at most one tile per side;
* sort/ranges: numpy's stable lexsort and bincount;
* rasterizer:  closed form of one Gaussian, telescoping sum, the 0.99 clamp
               hand count; expected depth and background: the one-Gaussian
               closed form and, for Gaussians at one camera depth z0, the
               telescoped depth z0 * (1 - T);
* backward:    central finite differences of the fp64 instantiation, with and
               without the depth output and a background colour;
* grad-quant:  where the full code lands (every 256th Gaussian of a ramp, so
               the block size and the scale are pinned), the half-step error
               bound, exact round trips of code multiples, zero blocks, sign
               symmetry of the rounding, the two-sub-batch error bound and
               the split of the SH gradient into its DC and higher parts.
"""
import math

import numpy as np
import pytest
from scipy.spatial.transform import Rotation
from scipy.special import sph_harm_y

from conftest import golden
from gaussian_splatting_differentiable_packed_b200 import scenes
from oracle import oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def make(means, quats, scales, opac, sh, cams, W, H, sh_degree=0, v_img=None):
    N = len(means)
    C = len(cams)
    return scenes.Scene(0, C, W, H, sh_degree, N, 0.01, 1e10, np.asarray(cams, np.float32),
                        np.asarray(means, np.float32), np.asarray(quats, np.float32),
                        np.asarray(scales, np.float32), np.asarray(opac, np.float32),
                        np.asarray(sh, np.float32).reshape(N, (sh_degree + 1) ** 2, 3), "uniform",
                        v_img, None, "pin")


def ident_cam(fx, fy, cx, cy):
    return np.concatenate([np.eye(4).reshape(16), [fx, fy, cx, cy]]).astype(np.float32)


# ---------------------------------------------------------------- exp
def test_exp_error_bound_and_monotone():
    x = -np.linspace(0.0, 87.0, 2_000_001).astype(np.float32)
    y = orc.exp_fp32_vec(x).astype(np.float64)
    exact = np.exp(x.astype(np.float64))
    ulp = np.spacing(exact.astype(np.float32)).astype(np.float64)
    err = np.abs(y - exact) / ulp
    assert err.max() <= 2.0, err.max()
    assert orc.exp_fp32(0.0) == 1.0
    assert np.all(np.diff(y) <= 0.0)  # x decreasing -> non-increasing
    # early-out safety used by a rasterizer: o <= 1 and sigma > 5.6 can never reach 1/255
    assert orc.exp_fp32(-5.6) < np.float32(1.0) / np.float32(255.0)
    assert orc.exp_fp32(-88.0) == 0.0


# ---------------------------------------------------------------- SH
def real_sh_scipy(l, m, d):
    """Real SH from scipy's complex SH (Condon-Shortley phase included):
    m<0 -> sqrt2 Im Y_l^|m|, m=0 -> Y_l^0, m>0 -> sqrt2 Re Y_l^m."""
    x, y, z = d
    theta = math.acos(max(-1.0, min(1.0, z)))
    phi = math.atan2(y, x)
    if m < 0:
        return math.sqrt(2) * sph_harm_y(l, -m, theta, phi).imag
    if m == 0:
        return sph_harm_y(l, 0, theta, phi).real
    return math.sqrt(2) * sph_harm_y(l, m, theta, phi).real


def test_sh_basis_matches_library():
    rng = np.random.default_rng(7)
    for _ in range(50):
        d = rng.normal(size=3)
        d /= np.linalg.norm(d)
        got = orc.sh_basis(3, d)
        want = [real_sh_scipy(l, m, d) for l in range(4) for m in range(-l, l + 1)]
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_sh_basis_gradient_finite_difference():
    rng = np.random.default_rng(8)
    for _ in range(20):
        d = rng.normal(size=3)
        g = orc.sh_basis_grad(3, d)
        for ax in range(3):
            e = np.zeros(3)
            e[ax] = 1e-6
            fd = (orc.sh_basis(3, d + e) - orc.sh_basis(3, d - e)) / 2e-6
            np.testing.assert_allclose(g[:, ax], fd, rtol=1e-6, atol=1e-8)


# ---------------------------------------------------------------- projection
def test_pinhole_mean_and_isotropic_covariance_closed_form():
    fx, fy, cx, cy = 50.0, 60.0, 32.0, 24.0
    p = np.array([0.5, -0.25, 2.0])
    s = 0.04
    sc = make([p], [[1, 0, 0, 0]], [[s, s, s]], [0.8], [[0.0, 0.0, 0.0]], [ident_cam(fx, fy, cx, cy)], 64, 48)
    for prec in (0, 1):
        pr = orc.project(sc, precision=prec)
        assert pr["nnz"] == 1
        row = pr["screen"][0]
        u, v = p[0] / p[2], p[1] / p[2]
        np.testing.assert_allclose(row[:2], [fx * u + cx, fy * v + cy], rtol=1e-6)
        J = np.array([[fx / p[2], 0, -fx * u / p[2]], [0, fy / p[2], -fy * v / p[2]]])
        S2 = s * s * J @ J.T + 0.3 * np.eye(2)
        Q = np.linalg.inv(S2)
        np.testing.assert_allclose(row[2:5], [Q[0, 0], Q[0, 1], Q[1, 1]], rtol=2e-6)
        assert row[5] == np.float32(0.8)
        assert row[9] == np.float32(2.0)


def test_off_axis_jacobian_limit():
    # u = x/z beyond 1.3 * (W/2)/fx: the Jacobian uses the clamped value, the mean does not
    fx = fy = 40.0
    W = H = 64
    lim = 1.3 * (0.5 * W) / fx
    z = 1.0
    x = (lim + 0.5) * z
    s = 0.3
    sc = make([[x, 0.0, z]], [[1, 0, 0, 0]], [[s, s, s]], [0.9], [[0.0, 0.0, 0.0]],
              [ident_cam(fx, fy, -20.0, 32.0)], W, H)
    pr = orc.project(sc, precision=1)
    assert pr["nnz"] == 1
    row = pr["screen"][0]
    J = np.array([[fx / z, 0, -fx * lim / z], [0, fy / z, 0.0]])
    S2 = s * s * J @ J.T + 0.3 * np.eye(2)
    Q = np.linalg.inv(S2)
    np.testing.assert_allclose(row[2:5], [Q[0, 0], Q[0, 1], Q[1, 1]], rtol=1e-6)
    assert abs(row[0] - (fx * x / z - 20.0)) < 1e-4


def test_anisotropic_covariance_against_library_rotation():
    sc = scenes.random_tiny(3, N=40, W=48, H=40, C=2, sh_degree=0)
    pr = orc.project(sc, precision=1)
    assert pr["nnz"] > 10
    for r in range(pr["nnz"]):
        c, n = pr["row_cam"][r], pr["row_gauss"][r]
        V = sc.cams[c, :16].astype(np.float64).reshape(4, 4)
        fx, fy = sc.cams[c, 16:18].astype(np.float64)
        q = sc.quats[n].astype(np.float64)
        Rq = Rotation.from_quat([q[1], q[2], q[3], q[0]]).as_matrix()
        S = Rq @ np.diag(sc.scales[n].astype(np.float64) ** 2) @ Rq.T
        p = V[:3, :3] @ sc.means[n].astype(np.float64) + V[:3, 3]
        limx, limy = 1.3 * 0.5 * sc.W / fx, 1.3 * 0.5 * sc.H / fy
        ux = np.clip(p[0] / p[2], -limx, limx)
        uy = np.clip(p[1] / p[2], -limy, limy)
        J = np.array([[fx / p[2], 0, -fx * ux / p[2]], [0, fy / p[2], -fy * uy / p[2]]])
        S2 = J @ V[:3, :3] @ S @ V[:3, :3].T @ J.T + 0.3 * np.eye(2)
        Q = np.linalg.inv(S2)
        np.testing.assert_allclose(pr["screen"][r][2:5], [Q[0, 0], Q[0, 1], Q[1, 1]], rtol=1e-8)


def test_visibility_edges():
    fx = fy = 50.0
    W = H = 64
    cam = ident_cam(fx, fy, 32.0, 32.0)
    s = 0.02
    # behind the camera, in front but far off-image, and just overlapping the left edge
    sc = make([[0, 0, -2.0], [10.0, 0, 2.0], [-1.33, 0, 2.0]], [[1, 0, 0, 0]] * 3, [[s, s, s]] * 3,
              [0.5] * 3, [[0.0, 0.0, 0.0]] * 3, [cam], W, H)
    pr = orc.project(sc, precision=0)
    assert pr["nnz"] == 1 and pr["row_gauss"][0] == 2


# ---------------------------------------------------------------- compaction and sizes
def test_compaction_routes_agree_on_random_scenes():
    for seed in range(6):
        sc = scenes.random_tiny(seed, N=300 + 37 * seed, W=40, H=32, C=3, sh_degree=1)
        pr = orc.project(sc)  # raises if the plain and bitmask compactions disagree
        g = orc.geometry(sc)
        assert g["n_pad"] % 128 == 0
        assert pr["block_off"][-1] == pr["nnz"]
        assert int(np.unpackbits(pr["mask"].view(np.uint8)).sum()) == pr["nnz"]


def test_page_buffer_sizes():
    gd = golden("page_figures.txt")
    P = gd["pairs_C_times_N"]
    mib = 1024.0 * 1024.0
    assert round(P * gd["old_bridge_bytes_per_pair"] / mib, 2) == gd["old_bridge_mib"]
    per_pair = gd["mask_bytes_per_pair"] + gd["block_count_bytes_per_pair"] + gd["scan_bytes_per_pair"]
    assert per_pair == 1.0 / 8 + 2 * 4.0 / gd["pairs_per_popcount"]  # one u32 per 128 pairs, twice
    assert abs(P * per_pair / mib - gd["bitmask_bridge_mib"]) < 0.015
    # this layout: 5 cameras x 15M Gaussians padded to the 128-pair block
    sc = make(np.zeros((1, 3)), [[1, 0, 0, 0]], [[1, 1, 1]], [0.5], [[0, 0, 0]],
              [ident_cam(1, 1, 0, 0)] * 5, 1600, 1067)
    sc.N = 15_000_000
    g = orc.geometry(sc)
    mask_b = g["mask_words"] * 4
    bc_b = g["mask_blocks"] * 4
    assert abs((mask_b + 2 * bc_b) / mib - gd["bitmask_bridge_mib"]) < 0.015
    # AABB rows 16 B -> 8 B at nnz ~ 15.1M
    nnz = gd["nnz_art_gallery"]
    assert abs(16 * nnz / mib - gd["aabb_old_mib"]) < 1.0
    assert abs(8 * nnz / mib - gd["aabb_new_mib"]) < 1.0
    # 64-bit keys cross 4 GiB at 2^32 / 8 intersections
    assert abs(2**32 / gd["key_bytes"] - gd["four_gib_crossing_isects"]) < 1e6


# ---------------------------------------------------------------- AABB16
def test_aabb16_contains_float_box_and_step():
    gd = golden("page_figures.txt")
    assert round(608 / 65535, 3) == gd["aabb_step_px_608"]
    assert round(6000 / 65535, 2) == gd["aabb_step_px_6000"]
    for seed in range(4):
        sc = scenes.random_tiny(seed, N=400, W=608 if seed % 2 == 0 else 97, H=57, C=2, sh_degree=0)
        pr = orc.project(sc)
        box = orc.row_boxes(sc, pr).astype(np.float64)
        a = pr["aabb"]
        qx0, qy0 = (a[:, 0] & 0xFFFF).astype(np.int64), (a[:, 0] >> 16).astype(np.int64)
        qx1, qy1 = (a[:, 1] & 0xFFFF).astype(np.int64), (a[:, 1] >> 16).astype(np.int64)
        # exact: q*extent/65535 <= v  <=>  q*extent <= v*65535 (both exact in fp64)
        assert np.all(qx0 * sc.W <= box[:, 0] * 65535.0)
        assert np.all(qx1 * sc.W >= box[:, 1] * 65535.0)
        assert np.all(qy0 * sc.H <= box[:, 2] * 65535.0)
        assert np.all(qy1 * sc.H >= box[:, 3] * 65535.0)
        # at most one grid step wider per side
        assert np.all((qx0 + 1) * sc.W > box[:, 0] * 65535.0)
        assert np.all((qx1 - 1) * sc.W < box[:, 1] * 65535.0)


# ---------------------------------------------------------------- intersections, sort, ranges
def test_intersect_range_form_equals_overlap_test_and_only_grows():
    for seed in range(4):
        sc = scenes.random_tiny(seed, N=250, W=80, H=48, C=2, sh_degree=0)
        pr = orc.project(sc)
        it = orc.intersect(sc, pr, all_pairs=True)  # raises on any disagreement
        it2 = orc.intersect(sc, pr, all_pairs=False)
        np.testing.assert_array_equal(it["keys"], it2["keys"])
        box = orc.row_boxes(sc, pr).astype(np.float64)
        per, total = orc.count_tiles(sc, pr["aabb"])
        assert total == it["n_isects"] == per.sum()
        # float-box tile count <= decoded-box count <= float-box count widened by one tile per side
        fx = np.ceil(box[:, 1] / 16) - np.floor(box[:, 0] / 16)
        fy = np.ceil(box[:, 3] / 16) - np.floor(box[:, 2] / 16)
        assert np.all(per >= fx * fy)
        assert np.all(per <= (fx + 2) * (fy + 2))


def test_keys_layout_and_sort_against_lexsort():
    sc = scenes.random_tiny(11, N=300, W=64, H=64, C=3, sh_degree=0)
    pr = orc.project(sc)
    it = orc.intersect(sc, pr)
    g = orc.geometry(sc)
    k, v = it["keys"], it["vals"]
    tiles = (k >> np.uint64(32)).astype(np.int64)
    cams = tiles // g["tiles_per_cam"]
    np.testing.assert_array_equal(cams, pr["row_cam"][v])
    depth = (k & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    np.testing.assert_array_equal(depth, pr["screen"][v, 9].astype(np.float32))
    # written row by row in order of depth (ties by row index), each row's
    # tiles contiguous
    dbits = (k & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    assert np.all(np.diff(dbits.astype(np.int64)) >= 0)
    runs = v[np.concatenate([[True], v[1:] != v[:-1]])]
    np.testing.assert_array_equal(runs, it["order"][np.isin(it["order"], v)])
    assert len(np.unique(runs)) == len(runs)
    rd = pr["screen"][:, 9].astype(np.float32).view(np.uint32)
    np.testing.assert_array_equal(it["order"], np.lexsort((np.arange(pr["nnz"]), rd)))
    ks, vs = orc.sort(k, v)
    order = np.lexsort((np.arange(len(k)), k))
    np.testing.assert_array_equal(ks, k[order])
    np.testing.assert_array_equal(vs, v[order])
    # the sorted order is (tile, depth, row); with the rows written in depth
    # order a stable sort by the tile id alone reaches it
    by_tile = np.argsort(tiles, kind="stable")
    np.testing.assert_array_equal(k[by_tile], ks)
    np.testing.assert_array_equal(v[by_tile], vs)
    full = np.lexsort((v.astype(np.int64), dbits, tiles))
    np.testing.assert_array_equal(v[full], vs)
    off = orc.tile_ranges(ks, g["n_tiles"])
    np.testing.assert_array_equal(np.diff(off), np.bincount(tiles, minlength=g["n_tiles"]))


# ---------------------------------------------------------------- rasterizer
def render(sc, precision=0):
    return orc.forward(sc, precision)


def test_single_gaussian_closed_form():
    fx = fy = 50.0
    W = H = 64
    z, s, o = 2.0, 0.04, 0.7
    q = Rotation.from_euler("xyz", [0.3, -0.4, 0.9]).as_quat()  # (x, y, z, w)
    scl = np.array([0.05, 0.02, 0.03])
    sc = make([[0.0, 0.0, z]], [[q[3], q[0], q[1], q[2]]], [scl], [o], [[0.0, 0.0, 0.0]],
              [ident_cam(fx, fy, 32.0, 32.0)], W, H)
    f = render(sc)
    Rq = Rotation.from_quat(q).as_matrix()
    S = Rq @ np.diag(scl ** 2) @ Rq.T
    S2 = (fx / z) ** 2 * S[:2, :2] + 0.3 * np.eye(2)
    Q = np.linalg.inv(S2)
    jj, ii = np.mgrid[0:H, 0:W]
    d = np.stack([32.0 - (ii + 0.5), 32.0 - (jj + 0.5)], -1)
    sig = 0.5 * np.einsum("...i,ij,...j->...", d, Q, d)
    alpha = np.minimum(0.99, o * np.exp(-sig))
    keep = alpha >= 1.0 / 255.0
    safe = np.abs(alpha - 1.0 / 255.0) > 1e-6
    want = np.where(keep, 0.5 * alpha, 0.0)
    np.testing.assert_allclose(f["img"][0, ..., 0][safe], want[safe], atol=1e-6)
    np.testing.assert_allclose(f["T"][0][safe], np.where(keep, 1 - alpha, 1.0)[safe], atol=1e-6)
    # the Gaussian is the only entry of each tile list: last_id = that tile's start
    g = f["geo"]
    t = (jj // 16) * g["tiles_x"] + ii // 16
    np.testing.assert_array_equal(f["last"][0][keep & safe], f["tile_off"][t][keep & safe])
    assert np.all(f["last"][0][~keep & safe] == -1)


def test_weights_telescope_to_one():
    rng = np.random.default_rng(5)
    N = 60
    dc = np.full((N, 1, 3), scenes.SQRT_PI)  # rgb = C0 * sqrt(pi) + 0.5 = 1
    for prec, tol in ((0, 2e-5), (1, 1e-12)):
        sc = make(rng.uniform(-0.5, 0.5, (N, 3)) + [0, 0, 3.0], rng.normal(size=(N, 4)),
                  np.exp(rng.uniform(-3.0, -1.5, (N, 3))), rng.uniform(0.2, 0.95, N), dc,
                  [ident_cam(40, 40, 24, 20)], 48, 40)
        f = render(sc, prec)
        for ch in range(3):
            np.testing.assert_allclose(f["img"][..., ch] + f["T"], 1.0, atol=tol)
        assert np.all((f["T"] >= 0) & (f["T"] <= 1))
        # last_id lies inside the pixel's tile range
        g = f["geo"]
        jj, ii = np.mgrid[0:sc.H, 0:sc.W]
        t = (jj // 16) * g["tiles_x"] + ii // 16
        lo, hi = f["tile_off"][t], f["tile_off"][t + 1]
        L = f["last"][0]
        assert np.all((L == -1) | ((L >= lo) & (L < hi)))


def test_clamped_opacity_stops_after_one():
    # every alpha clamps at 0.99: T = 1 - 0.99f after the first, the second would
    # take T below 1e-4, so exactly one Gaussian is composited per pixel
    N = 3
    sc = make([[0, 0, 2.0], [0.1, 0, 3.0], [0, -0.1, 4.0]], [[1, 0, 0, 0]] * N, [[100.0] * 3] * N,
              [1.0] * N, [[0.0, 0.0, 0.0]] * N, [ident_cam(20, 20, 16, 16)], 32, 32)
    f = render(sc)
    one = np.float32(1.0) - np.float32(0.99)
    assert np.all(f["T"] == one)
    g = f["geo"]
    jj, ii = np.mgrid[0:32, 0:32]
    t = (jj // 16) * g["tiles_x"] + ii // 16
    np.testing.assert_array_equal(f["last"][0], f["tile_off"][t])
    np.testing.assert_allclose(f["img"][0], 0.5 * 0.99, rtol=1e-6)


def test_single_gaussian_depth_and_background():
    """One Gaussian at camera depth z: D = alpha * z and img = 0.5 alpha + (1 - alpha) bg
    where it is composited; D = 0 and img = bg elsewhere."""
    fx = fy = 50.0
    W = H = 48
    z, o = 2.5, 0.8
    bg = np.array([[0.2, 0.6, 0.9]])
    sc = make([[0.1, -0.05, z]], [[1.0, 0.0, 0.0, 0.0]], [[0.04, 0.03, 0.05]], [o], [[0.0, 0.0, 0.0]],
              [ident_cam(fx, fy, 24.0, 24.0)], W, H)
    for prec, tol in ((0, 2e-6), (1, 1e-12)):
        f = orc.forward(sc, prec, bg=bg, depth=True)
        alpha = 1.0 - f["T"][0]  # one composited entry: T = 1 - alpha
        comp = f["last"][0] >= 0
        np.testing.assert_allclose(f["depth"][0][comp], (alpha * z)[comp], rtol=tol, atol=tol)
        assert np.all(f["depth"][0][~comp] == 0.0)
        for ch in range(3):
            want = np.where(comp, 0.5 * alpha + (1.0 - alpha) * bg[0, ch], bg[0, ch])
            np.testing.assert_allclose(f["img"][0, ..., ch], want, atol=10 * tol)


def test_coplanar_depth_telescopes():
    """All Gaussians at one camera depth z0: the weights sum to 1 - T, so the
    expected depth is z0 * (1 - T) at every pixel."""
    rng = np.random.default_rng(9)
    N, z0 = 80, 3.0
    means = np.concatenate([rng.uniform(-0.6, 0.6, (N, 2)), np.full((N, 1), z0)], 1)
    for prec, tol in ((0, 3e-5), (1, 1e-12)):
        sc = make(means, rng.normal(size=(N, 4)), np.exp(rng.uniform(-3.5, -2.0, (N, 3))),
                  rng.uniform(0.2, 0.95, N), rng.uniform(0.0, 1.0, (N, 3)), [ident_cam(40, 40, 24, 20)], 48, 40)
        f = orc.forward(sc, prec, depth=True)
        np.testing.assert_allclose(f["depth"], z0 * (1.0 - f["T"]), atol=tol * z0)


def test_fp32_forward_close_to_fp64():
    sc = scenes.make_scene(1)
    a = render(sc, 0)
    b = render(sc, 1)
    assert a["proj"]["nnz"] == b["proj"]["nnz"]
    diff = np.abs(a["img"] - b["img"])
    assert np.mean(diff < 1e-4) > 0.995


# ---------------------------------------------------------------- backward vs finite differences
def loss(sc, v_img, v_T, v_D=None, bg=None):
    f = orc.forward(sc, precision=1, bg=bg, depth=v_D is not None)
    L = float(np.sum(f["img"] * v_img) + np.sum(f["T"] * v_T))
    if v_D is not None:
        L += float(np.sum(f["depth"] * v_D))
    return L


@pytest.mark.parametrize("seed,ext", [(s, False) for s in range(8)] + [(s, True) for s in (8, 9, 10, 11)])
def test_backward_central_differences(seed, ext):
    """ext: the loss also weighs the expected depth and the colour carries a
    background (the depth gradient then reaches the means through the camera
    depth, and the background through dL/dT)."""
    sc = scenes.random_tiny(seed, N=5, W=32, H=32, C=2 if seed % 2 else 1, sh_degree=seed % 4,
                            opacity_range=(0.1, 0.9))
    # fp64 parameters so the differences are not quantised to fp32
    for name in ("means", "quats", "scales", "opacities", "sh"):
        setattr(sc, name, getattr(sc, name).astype(np.float64))
    rng = np.random.default_rng(seed)
    v_img = rng.uniform(-1, 1, (sc.C, sc.H, sc.W, 3))
    v_T = rng.uniform(-1, 1, (sc.C, sc.H, sc.W))
    v_D = rng.uniform(-1, 1, (sc.C, sc.H, sc.W)) if ext else None
    bg = rng.uniform(0, 1, (sc.C, 3)) if ext else None
    r = orc.step(sc, precision=1, v_img=v_img, v_T=v_T, v_depth=v_D, bg=bg)
    gr = r["grads"]
    names = {"means": "v_means", "quats": "v_quats", "scales": "v_scales", "opacities": "v_opacities",
             "sh": "v_sh"}
    checked = skipped = 0
    for pname, gname in names.items():
        arr = getattr(sc, pname)
        flat = arr.reshape(-1)
        an = gr[gname].reshape(-1)
        for i in range(flat.size):
            x0 = flat[i]
            vals = []
            for h in (1e-6, 5e-7):
                hh = h * max(1.0, abs(x0))
                flat[i] = x0 + hh
                lp = loss(sc, v_img, v_T, v_D, bg)
                flat[i] = x0 - hh
                lm = loss(sc, v_img, v_T, v_D, bg)
                flat[i] = x0
                vals.append((lp - lm) / (2 * hh))
            # two step sizes that disagree mean a threshold (1/255, 3-sigma tile edge) was crossed
            if abs(vals[0] - vals[1]) > 1e-5 * max(1.0, abs(vals[0])):
                skipped += 1
                continue
            checked += 1
            assert abs(vals[0] - an[i]) <= 1e-4 * max(1.0, abs(an[i])), (pname, i, vals, an[i])
    assert checked > 10 * skipped


# ---------------------------------------------------------------- fused optimizer step
def test_adam_matches_library_adam():
    """The oracle's Adam against torch.optim.Adam (fp64, CPU) over three steps
    with changing gradients, per group learning rates."""
    import torch
    rng = np.random.default_rng(21)
    shapes = dict(means=(7, 3), quats=(7, 4), log_scales=(7, 3), logit_opacities=(7,), sh=(7, 4, 3))
    lr = dict(means=1e-3, quats=2e-3, log_scales=5e-3, logit_opacities=5e-2, sh=2.5e-3)
    b1, b2, eps = 0.9, 0.999, 1e-8
    p0 = {k: rng.normal(size=s) for k, s in shapes.items()}
    tp = {k: torch.tensor(p0[k], dtype=torch.float64, requires_grad=True) for k in shapes}
    opt = torch.optim.Adam([{"params": [tp[k]], "lr": lr[k]} for k in shapes], betas=(b1, b2), eps=eps)
    P = dict(p0)
    M = {k: np.zeros(s) for k, s in shapes.items()}
    V = {k: np.zeros(s) for k, s in shapes.items()}
    for t in (1, 2, 3):
        g = {k: rng.normal(size=s) * 10.0 ** rng.uniform(-4, 0) for k, s in shapes.items()}
        for k in shapes:
            tp[k].grad = torch.tensor(g[k], dtype=torch.float64)
        opt.step()
        P, M, V = orc.adam_step(P, g, M, V, lr, b1, b2, eps, t)
        for k in shapes:
            np.testing.assert_allclose(P[k], tp[k].detach().numpy(), rtol=1e-12, atol=1e-14)


def test_adam_first_step_closed_form():
    """From zero moments, step 1 moves every element by lr * g / (|g| + eps)."""
    rng = np.random.default_rng(22)
    g = {"means": rng.normal(size=(5, 3))}
    p = {"means": rng.normal(size=(5, 3))}
    z = {"means": np.zeros((5, 3))}
    P, M, V = orc.adam_step(p, g, z, z, {"means": 0.01}, 0.9, 0.999, 1e-6, 1)
    np.testing.assert_allclose(P["means"], p["means"] - 0.01 * g["means"] / (np.abs(g["means"]) + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(M["means"], 0.1 * g["means"], rtol=1e-14)
    np.testing.assert_allclose(V["means"], 0.001 * g["means"] ** 2, rtol=1e-12)


def test_raw_gradients_central_differences():
    """d L / d log s = s * dL/ds and d L / d logit = o (1 - o) dL/do, against
    central differences of the fp64 oracle in the raw parameters."""
    sc = scenes.random_tiny(13, N=5, W=32, H=32, C=1, sh_degree=1, opacity_range=(0.2, 0.8))
    for name in ("means", "quats", "scales", "opacities", "sh"):
        setattr(sc, name, getattr(sc, name).astype(np.float64))
    rng = np.random.default_rng(13)
    v_img = rng.uniform(-1, 1, (sc.C, sc.H, sc.W, 3))
    v_T = rng.uniform(-1, 1, (sc.C, sc.H, sc.W))
    r = orc.step(sc, precision=1, v_img=v_img, v_T=v_T)
    raw = orc.raw_gradients(r["grads"], sc.scales, sc.opacities)
    log_s, logit = np.log(sc.scales), np.log(sc.opacities / (1.0 - sc.opacities))
    checked = 0
    for arr, act, key in ((log_s, lambda x: np.exp(x), "log_scales"),
                          (logit, lambda x: 1.0 / (1.0 + np.exp(-x)), "logit_opacities")):
        flat = arr.reshape(-1)
        an = raw[key].reshape(-1)
        for i in range(flat.size):
            x0 = flat[i]
            vals = []
            for h in (1e-6, 5e-7):
                out = []
                for sgn in (1, -1):
                    flat[i] = x0 + sgn * h
                    if key == "log_scales":
                        sc.scales = act(log_s)
                    else:
                        sc.opacities = act(logit)
                    out.append(loss(sc, v_img, v_T))
                flat[i] = x0
                vals.append((out[0] - out[1]) / (2 * h))
            sc.scales, sc.opacities = np.exp(log_s), 1.0 / (1.0 + np.exp(-logit))
            if abs(vals[0] - vals[1]) > 1e-5 * max(1.0, abs(vals[0])):
                continue
            checked += 1
            assert abs(vals[0] - an[i]) <= 1e-4 * max(1.0, abs(an[i])), (key, i, vals, an[i])
    assert checked >= 15


# ---------------------------------------------------------------------------- block-quantised accumulation
def test_gq_full_code_at_each_blocks_largest_element():
    """A ramp x[g] = g + 1 over 700 Gaussians: each block's largest element is
    its last Gaussian, so the full code 32767 appears exactly at 255, 511 and
    699 (a wrong block size or one scale for all blocks moves it), and the
    scale is that element over 32767 (a divisor of 32768 or 65535 leaves no
    full code)."""
    x = (np.arange(700, dtype=np.float64) + 1.0).reshape(700, 1)
    codes, scales = orc.gq_quantise(x)
    assert codes.dtype == np.int16 and scales.shape == (3,)
    assert np.flatnonzero(codes[:, 0] == 32767).tolist() == [255, 511, 699]
    assert np.all(codes > 0)
    dec = orc.gq_decode(codes, scales)
    assert np.allclose(dec[[255, 511, 699], 0], [256.0, 512.0, 700.0], rtol=1e-12, atol=0)


def test_gq_half_step_error_bound_and_exact_multiples():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((1000, 4)) * np.exp(rng.uniform(-3, 3, (1000, 1)))
    codes, scales = orc.gq_quantise(x)
    err = np.abs(orc.gq_decode(codes, scales) - x)
    step = np.repeat(scales, orc.GQ_BLOCK)[:1000].reshape(1000, 1)
    assert np.all(err <= 0.5 * step * (1 + 1e-12))
    # integer multiples of one block's step come back exactly
    k = rng.integers(-32767, 32768, (256, 3)).astype(np.float64)
    k[17, 1] = 32767.0
    y = k * (3.25 / 32767.0)
    c2, s2 = orc.gq_quantise(y)
    assert np.array_equal(c2.astype(np.float64), k)
    assert np.allclose(orc.gq_decode(c2, s2), y, rtol=1e-15, atol=0)


def test_gq_zero_block_and_sign_symmetry():
    x = np.zeros((512, 2))
    x[300, 1] = -2.5e-7
    codes, scales = orc.gq_quantise(x)
    assert scales[0] == 0.0 and np.all(codes[:256] == 0)
    assert codes[300, 1] == -32767 and np.count_nonzero(codes[256:]) == 1
    rng = np.random.default_rng(8)
    y = rng.standard_normal((300, 3))
    y[5, 0] = 0.5 * (abs(y).max() / 32767.0) * 3  # an exact half step: ties go to even
    cp, sp = orc.gq_quantise(y)
    cn, sn = orc.gq_quantise(-y)
    assert np.array_equal(sp, sn) and np.array_equal(cn, -cp)


def test_gq_two_sub_batches_error_bound():
    """decode(acc2) differs from g1 + g2 by at most half a step of each
    quantisation; g2 is 50x larger than g1 so that keeping the first scale, or
    adding codes instead of values, breaks the bound."""
    rng = np.random.default_rng(9)
    N, K = 600, 16
    def grads(scale):
        return dict(v_means=rng.standard_normal((N, 3)) * scale, v_quats=rng.standard_normal((N, 4)) * scale,
                    v_scales=rng.standard_normal((N, 3)) * scale, v_opacities=rng.standard_normal(N) * scale,
                    v_sh=rng.standard_normal((N, K, 3)) * scale)
    g1, g2 = grads(1e-3), grads(5e-2)
    acc1 = orc.gq_accumulate(None, g1)
    acc2 = orc.gq_accumulate(acc1, g2)
    a1, a2 = orc.gq_attributes(g1), orc.gq_attributes(g2)
    for name in a1:
        s1 = np.repeat(acc1[name][1], orc.GQ_BLOCK)[:N].reshape(N, 1)
        s2 = np.repeat(acc2[name][1], orc.GQ_BLOCK)[:N].reshape(N, 1)
        err = np.abs(orc.gq_decode(*acc2[name]) - (a1[name] + a2[name]))
        assert np.all(err <= 0.5 * (s1 + s2) * (1 + 1e-9)), name
        c, s = orc.gq_quantise(a1[name])
        assert np.array_equal(acc1[name][0], c) and np.array_equal(acc1[name][1], s)


def test_gq_attribute_split():
    N, K = 3, 9
    sh = np.zeros((N, K, 3))
    for k in range(K):
        for c in range(3):
            sh[:, k, c] = 100 * k + c
    a = orc.gq_attributes(dict(v_means=np.zeros((N, 3)), v_quats=np.zeros((N, 4)), v_scales=np.zeros((N, 3)),
                               v_opacities=np.arange(N, dtype=float), v_sh=sh))
    assert [a[k].shape[1] for k in ("means", "quats", "scales", "opacities", "sh_dc", "sh_rest")] == [3, 4, 3, 1, 3, 24]
    assert a["sh_dc"][0].tolist() == [0, 1, 2]
    assert a["sh_rest"][0, :4].tolist() == [100, 101, 102, 200]
    assert a["opacities"][:, 0].tolist() == [0, 1, 2]
