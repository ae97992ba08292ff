"""Pins of the oracle's sampled checks against its own whole-scene step.

The full-size parity tests compare the CUDA path with five oracle helpers
that restate the step for a chosen subset of tiles or rows (tile_counts,
tile_lists, rasterize_tiles, raster_bwd_rows, project_bwd_rows), because the
whole-scene oracle is too slow at those sizes.  Here, on small scenes where
the whole-scene oracle (orc.step) runs in well under a second, each helper
must reproduce orc.step exactly:

* with every tile and every row selected: per-tile counts = the tile ranges'
  differences, the sorted slices = the sorted keys and values, img / T /
  last_id = the whole image's (pixel for pixel), the screen-row gradients and
  the per-Gaussian sums of the per-row parameter gradients = orc.step's to
  1e-12 relative (same fp64 terms, summed in another order);
* with a shuffled subset of tiles (so a slice's start in the global sorted
  list differs from its offset in the helper's list) and a subset of rows
  (only the tiles those rows cover are replayed): the same values on the
  subset.

A mistake in the remapping of last_id to the global sorted index, in the
row-to-slot map of the backward replay, in a decoded AABB half-word or in the
per-Gaussian sums fails one of these.  Nothing here calls the CUDA path.
"""
import numpy as np
import pytest

from gaussian_splatting_differentiable_packed_b200 import scenes
from oracle import oracle as orc

SCENES = [
    dict(seed=0, N=180, W=45, H=37, C=1, sh_degree=0),
    dict(seed=1, N=240, W=64, H=48, C=2, sh_degree=3),
    dict(seed=2, N=150, W=33, H=50, C=3, sh_degree=1),
    dict(seed=3, N=300, W=70, H=29, C=2, sh_degree=2),
]


def tiny(p):
    return scenes.random_tiny(p["seed"] + 600, N=p["N"], W=p["W"], H=p["H"], C=p["C"], sh_degree=p["sh_degree"])


def tiles_of_rows(sc, proj, rows):
    """Every tile the rows' AABB16s cover (the tile range of the decoded box)."""
    g = orc.geometry(sc)
    need = set()
    for r in rows:
        a = proj["aabb"][r]
        tx0 = (int(a[0] & 0xFFFF) * sc.W) // (65535 * 16)
        tx1 = min(-(-(int(a[1] & 0xFFFF) * sc.W) // (65535 * 16)), g["tiles_x"])
        ty0 = (int(a[0] >> 16) * sc.H) // (65535 * 16)
        ty1 = min(-(-(int(a[1] >> 16) * sc.H) // (65535 * 16)), g["tiles_y"])
        base = int(proj["row_cam"][r]) * g["tiles_per_cam"]
        for ty in range(ty0, ty1):
            for tx in range(tx0, tx1):
                need.add(base + ty * g["tiles_x"] + tx)
    return np.array(sorted(need), np.int64)


def pixel_grid(sc, tiles):
    """(camera, row, column) of each of the 256 pixel slots of each tile
    (row/column may lie past the image edge)."""
    g = orc.geometry(sc)
    c, tr = np.divmod(np.asarray(tiles, np.int64), g["tiles_per_cam"])
    ty, tx = np.divmod(tr, g["tiles_x"])
    q = np.arange(256)
    y = ty[:, None] * 16 + q[None, :] // 16
    x = tx[:, None] * 16 + q[None, :] % 16
    return np.broadcast_to(c[:, None], y.shape), y, x


def per_gaussian(sc, proj, rows, per_row):
    """Sum the per-row parameter gradients [rows][11 + 3K] of each Gaussian."""
    out = np.zeros((sc.N, per_row.shape[1]))
    np.add.at(out, proj["row_gauss"][rows], per_row)
    K3 = 3 * sc.K
    return dict(v_means=out[:, 0:3], v_quats=out[:, 3:7], v_scales=out[:, 7:10], v_opacities=out[:, 10],
                v_sh=out[:, 11:11 + K3].reshape(-1, sc.K, 3))


def close(a, b, rtol=1e-12):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(float(np.abs(b).max()), 1e-300)
    assert np.abs(a - b).max() <= rtol * scale, float(np.abs(a - b).max() / scale)


@pytest.fixture(scope="module", params=range(len(SCENES)))
def case(request):
    sc = tiny(SCENES[request.param])
    o = orc.step(sc, precision=0, nthreads=1)
    assert o["proj"]["nnz"] > 20 and o["isect"]["n_isects"] > 50
    return sc, o


def test_tile_counts_equal_tile_ranges(case):
    sc, o = case
    cnt = orc.tile_counts(sc, o["proj"])
    np.testing.assert_array_equal(cnt, np.diff(o["tile_off"]))


def test_tile_lists_equal_sorted_keys(case):
    sc, o = case
    tiles = np.arange(o["geo"]["n_tiles"], dtype=np.int64)
    off, keys, vals = orc.tile_lists(sc, o["proj"], tiles)
    np.testing.assert_array_equal(off, o["tile_off"])
    np.testing.assert_array_equal(keys, o["keys_sorted"])
    np.testing.assert_array_equal(vals, o["vals_sorted"])
    # a shuffled subset: each selected tile's slice is the global slice
    rng = np.random.default_rng(7)
    sub = rng.permutation(tiles)[: max(3, len(tiles) // 3)]
    off2, keys2, vals2 = orc.tile_lists(sc, o["proj"], sub)
    for i, t in enumerate(sub):
        a, b = o["tile_off"][t], o["tile_off"][t + 1]
        np.testing.assert_array_equal(keys2[off2[i]:off2[i + 1]], o["keys_sorted"][a:b])
        np.testing.assert_array_equal(vals2[off2[i]:off2[i + 1]], o["vals_sorted"][a:b])


@pytest.mark.parametrize("subset", [False, True])
def test_rasterize_tiles_equal_whole_image(case, subset):
    sc, o = case
    tiles = np.arange(o["geo"]["n_tiles"], dtype=np.int64)
    if subset:
        # shuffled, so list offsets and global starts differ for most tiles
        tiles = np.random.default_rng(11).permutation(tiles)[: max(4, len(tiles) // 2)]
    off, _, vals = orc.tile_lists(sc, o["proj"], tiles)
    img, T, last = orc.rasterize_tiles(sc, o["proj"], tiles, off, vals, o["tile_off"][tiles], nthreads=1)
    c, y, x = pixel_grid(sc, tiles)
    inside = (y < sc.H) & (x < sc.W)
    assert np.all(last[~inside] == -2) and np.all(T[~inside] == 1.0)
    ci, yi, xi = c[inside], y[inside], x[inside]
    np.testing.assert_array_equal(last[inside], o["last"][ci, yi, xi])
    np.testing.assert_array_equal(T[inside], o["T"][ci, yi, xi])
    np.testing.assert_array_equal(img[inside], o["img"][ci, yi, xi])
    assert np.any(o["last"] >= 0)
    if subset:
        assert np.any(off[:-1] != o["tile_off"][tiles])  # the remapping is exercised


def test_raster_bwd_rows_and_project_bwd_rows_all_rows(case):
    sc, o = case
    p = o["proj"]
    tiles = np.arange(o["geo"]["n_tiles"], dtype=np.int64)
    off, _, vals = orc.tile_lists(sc, p, tiles)
    rows = np.arange(p["nnz"], dtype=np.int64)
    v_rows = orc.raster_bwd_rows(sc, p, tiles, off, vals, o["v_img"], None, rows, nthreads=1)
    close(v_rows, o["v_screen"])
    per_row = orc.project_bwd_rows(sc, p, rows, v_rows)
    got = per_gaussian(sc, p, rows, per_row)
    for k, ref in o["grads"].items():
        close(got[k], ref)


def test_raster_bwd_rows_subset_of_gaussians(case):
    sc, o = case
    p = o["proj"]
    rng = np.random.default_rng(13)
    gauss = rng.choice(np.unique(p["row_gauss"]), min(8, len(np.unique(p["row_gauss"]))), replace=False)
    rows = np.nonzero(np.isin(p["row_gauss"], gauss))[0]
    # rows in a scrambled order: slot k holds rows[k]
    rows = rng.permutation(rows)
    tiles = tiles_of_rows(sc, p, rows)
    off, _, vals = orc.tile_lists(sc, p, tiles)
    v_rows = orc.raster_bwd_rows(sc, p, tiles, off, vals, o["v_img"], None, rows, nthreads=1)
    close(v_rows, o["v_screen"][rows])
    assert np.abs(v_rows[:, :9]).max() > 0
    per_row = orc.project_bwd_rows(sc, p, rows, v_rows)
    got = per_gaussian(sc, p, rows, per_row)
    for k, ref in o["grads"].items():
        close(got[k][gauss], ref[gauss])


def test_raster_bwd_rows_with_transmittance_gradient(case):
    # v_T enters each pixel's replay through T_final: the helper must pass it on
    sc, o = case
    p = o["proj"]
    rng = np.random.default_rng(17)
    v_T = rng.uniform(-1.0, 1.0, (sc.C, sc.H, sc.W))
    ref = orc.rasterize_bwd(sc, p["screen"], o["vals_sorted"], o["tile_off"], o["v_img"], v_T, nthreads=1)
    tiles = np.arange(o["geo"]["n_tiles"], dtype=np.int64)
    off, _, vals = orc.tile_lists(sc, p, tiles)
    rows = np.arange(p["nnz"], dtype=np.int64)
    v_rows = orc.raster_bwd_rows(sc, p, tiles, off, vals, o["v_img"], v_T, rows, nthreads=1)
    close(v_rows, ref)
    assert np.abs(ref - o["v_screen"]).max() > 0  # v_T changes the gradients
