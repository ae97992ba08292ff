"""Pins of the oracle's per-image visible cap (the pages' --cap-max: a cap on
the visible splats of each image that holds down nnz).

The page names the control but no selection rule; the reading is: in each
camera whose visible pairs exceed the cap, keep the cap of highest opacity,
ties going to the lower Gaussian index.  That set is fixed uniquely by three
properties, which these tests check against the uncapped projection instead
of restating the selection:

* size: each camera keeps min(cap, visible) pairs;
* subset: every kept pair is visible without the cap;
* dominance: every kept pair of a camera has a higher opacity than every
  dropped one, or the same opacity and a lower Gaussian index.

Also: a cap at or above every camera's visible count changes nothing, a cap
of 0 keeps nothing, equal opacities keep the lowest indices, and the screen
rows of kept pairs are the uncapped rows of the same pairs.
"""
import numpy as np
import pytest

from gaussian_splatting_differentiable_packed_b200 import scenes
from oracle import oracle as orc


def visible_sets(sc, p):
    """Visible Gaussian indices per camera from the mask."""
    g = orc.geometry(sc)
    bits = np.unpackbits(p["mask"].view(np.uint8), bitorder="little").reshape(sc.C, g["n_pad"])
    return [np.nonzero(bits[c, :sc.N])[0] for c in range(sc.C)]


def check_cap(sc, cap):
    full = orc.project(sc)
    capped = orc.project(sc, cap_max=cap)
    vf, vc = visible_sets(sc, full), visible_sets(sc, capped)
    o = sc.opacities.astype(np.float32)
    for c in range(sc.C):
        keep, vis = vc[c], vf[c]
        assert len(keep) == min(cap, len(vis))
        assert np.all(np.isin(keep, vis))
        drop = np.setdiff1d(vis, keep)
        if len(keep) and len(drop):
            k_min = o[keep].min()
            d_max = o[drop].max()
            assert k_min >= d_max
            # at equal opacity the kept indices come first
            tied_k = keep[o[keep] == d_max]
            tied_d = drop[o[drop] == d_max]
            if len(tied_k) and len(tied_d):
                assert tied_k.max() < tied_d.min()
    # the kept rows are the uncapped rows of the same pairs, in the same order
    key_full = full["row_cam"].astype(np.int64) * sc.N + full["row_gauss"]
    key_cap = capped["row_cam"].astype(np.int64) * sc.N + capped["row_gauss"]
    assert np.all(np.diff(key_cap) > 0)
    pos = np.searchsorted(key_full, key_cap)
    np.testing.assert_array_equal(key_full[pos], key_cap)
    np.testing.assert_array_equal(capped["screen"], full["screen"][pos])
    np.testing.assert_array_equal(capped["aabb"], full["aabb"][pos])
    assert capped["nnz"] == sum(min(cap, len(v)) for v in vf)
    return full, capped


@pytest.mark.parametrize("seed,cap", [(0, 40), (1, 1), (2, 123), (3, 250)])
def test_cap_properties_random(seed, cap):
    sc = scenes.random_tiny(800 + seed, N=300 + 40 * seed, W=48, H=40, C=1 + seed % 3, sh_degree=seed % 4)
    full, _ = check_cap(sc, cap)
    assert max(len(v) for v in visible_sets(sc, full)) > cap  # the cap binds


def test_cap_on_a_partly_visible_scene():
    # workload 3's distributions with few Gaussians: cameras see different subsets
    sc = scenes.make_scene(3, n=20_000)
    full, capped = check_cap(sc, 1500)
    assert capped["nnz"] < full["nnz"]


def test_cap_at_or_above_visible_changes_nothing():
    sc = scenes.random_tiny(810, N=400, W=40, H=32, C=2, sh_degree=1)
    full = orc.project(sc)
    most = max(len(v) for v in visible_sets(sc, full))
    for cap in (most, most + 1, 10**9):
        capped = orc.project(sc, cap_max=cap)
        np.testing.assert_array_equal(capped["mask"], full["mask"])
        np.testing.assert_array_equal(capped["block_off"], full["block_off"])
        np.testing.assert_array_equal(capped["screen"], full["screen"])


def test_cap_zero_keeps_nothing():
    sc = scenes.random_tiny(811, N=200, W=40, H=32, C=2, sh_degree=0)
    p = orc.project(sc, cap_max=0)
    assert p["nnz"] == 0 and not p["mask"].any()


def test_equal_opacities_keep_lowest_indices():
    sc = scenes.random_tiny(812, N=300, W=48, H=40, C=1, sh_degree=0)
    sc.opacities = np.full(sc.N, 0.5, np.float32)
    vis = visible_sets(sc, orc.project(sc))[0]
    keep = visible_sets(sc, orc.project(sc, cap_max=17))[0]
    np.testing.assert_array_equal(keep, vis[:17])


def test_capped_step_runs_end_to_end():
    # the later stages see only the kept rows: intersections and gradients of
    # dropped pairs vanish
    sc = scenes.random_tiny(813, N=350, W=48, H=40, C=2, sh_degree=2)
    o = orc.step(sc, cap_max=60)
    p = o["proj"]
    assert p["nnz"] == 120
    kept = np.zeros(sc.N, bool)
    kept[p["row_gauss"]] = True
    assert np.all(o["grads"]["v_opacities"][~kept] == 0)
    assert np.abs(o["grads"]["v_opacities"][kept]).max() > 0
