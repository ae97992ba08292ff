"""Parity at the full workload sizes, in the launch configuration bench.py
times (PackedStep over the whole scene), on outputs the oracle can compute:

* the whole visibility mask, block counts and offsets, nnz, every screen row
  and AABB16 (the oracle's projection runs over all C*N pairs);
* n_isects and the full tile_off array (exact per-tile counts);
* the sorted (key, value) slices of at least 200 sampled tiles: the heaviest
  ones, tiles around the median entry count, tiles on the four image edges
  of every camera (partial tiles where the image size is not a multiple of
  16) and random non-empty ones;
* image, transmittance and last_id of every pixel of those tiles;
* the screen-row gradients and the Gaussian gradients of at least 200
  sampled Gaussians (those seen by the most cameras, those with a row at an
  image edge, random ones; every pixel of every tile they touch is replayed
  by the oracle).

The upstream gradient is a seeded uniform field (the L1 gradient would need
the oracle's whole image).  Workload 5 has n_isects > 2^29 (keys > 4 GiB).
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss
from oracle import oracle as orc
from test_gpu_parity import grad_close, u32

pytestmark = pytest.mark.gpu

THREADS = 16


def gaussian_grads(scene, proj, rows, per_row):
    """Sum per-row contributions [rows][11+3K] per Gaussian."""
    K3 = 3 * scene.K
    out = {}
    for r, v in zip(rows, per_row):
        n = int(proj["row_gauss"][r])
        out[n] = out.get(n, 0) + v
    ns = sorted(out)
    arr = np.stack([out[n] for n in ns])
    return ns, dict(v_means=arr[:, 0:3], v_quats=arr[:, 3:7], v_scales=arr[:, 7:10], v_opacities=arr[:, 10],
                    v_sh=arr[:, 11:11 + K3].reshape(-1, scene.K, 3))


def tile_pixels(g, tiles):
    """(camera, row, column) of the 256 pixel slots of each tile."""
    c, tr = np.divmod(np.asarray(tiles, np.int64), g["tiles_per_cam"])
    ty, tx = np.divmod(tr, g["tiles_x"])
    q = np.arange(256)
    y = ty[:, None] * 16 + q[None, :] // 16
    x = tx[:, None] * 16 + q[None, :] % 16
    return np.broadcast_to(c[:, None], y.shape), y, x


def sample_tiles(sc, g, cnt, rng, n=216):
    """Heaviest, median-count, edge and random non-empty tiles (at least n
    in all when that many are non-empty)."""
    nonempty = np.nonzero(cnt)[0]
    order = nonempty[np.argsort(cnt[nonempty], kind="stable")]
    heavy = order[-24:]
    mid = len(order) // 2
    median = order[max(0, mid - 12):mid + 12]
    tr = nonempty % g["tiles_per_cam"]
    ty, tx = np.divmod(tr, g["tiles_x"])
    edge_all = nonempty[(tx == 0) | (ty == 0) | (tx == g["tiles_x"] - 1) | (ty == g["tiles_y"] - 1)]
    edge = rng.choice(edge_all, min(48, len(edge_all)), replace=False)
    picked = np.unique(np.concatenate([heavy, median, edge]))
    rest = np.setdiff1d(nonempty, picked)
    rand = rng.choice(rest, min(max(0, n - len(picked)), len(rest)), replace=False)
    return np.unique(np.concatenate([picked, rand])).astype(np.int64)


def sample_gaussians(sc, p, rng, n=200):
    """Gaussians visible in the most cameras, with a row touching an image
    edge, and random ones (at least n in all)."""
    rg = p["row_gauss"]
    uniq, seen = np.unique(rg, return_counts=True)
    most = uniq[np.argsort(-seen, kind="stable")[:40]]
    a = p["aabb"]
    at_edge = (((a[:, 0] & 0xFFFF) == 0) | ((a[:, 0] >> 16) == 0) | ((a[:, 1] & 0xFFFF) == 65535)
               | ((a[:, 1] >> 16) == 65535))
    edge_g = np.unique(rg[at_edge])
    edge = rng.choice(edge_g, min(40, len(edge_g)), replace=False) if len(edge_g) else np.zeros(0, np.int64)
    picked = np.unique(np.concatenate([most, edge]))
    rest = np.setdiff1d(uniq, picked)
    rand = rng.choice(rest, max(0, n - len(picked)), replace=False)
    return np.unique(np.concatenate([picked, rand])).astype(np.int64)


@pytest.mark.parametrize("cfg", [4, 5])
def test_full_size_sampled(cfg):
    sc = scenes.make_scene(cfg)
    rng = np.random.default_rng(500 + cfg)
    v_img = (rng.uniform(-1.0, 1.0, (sc.C, sc.H, sc.W, 3)) / (3.0 * sc.W * sc.H * sc.C)).astype(np.float32)
    d = ss.scene_dims(sc)
    step = ss.PackedStep(d, "cuda")
    step.forward(*ss.scene_tensors(sc))
    step.backward(torch.from_numpy(v_img).cuda())
    torch.cuda.synchronize()

    # --- projection: everything
    p = orc.project(sc, nthreads=THREADS)
    g = orc.geometry(sc)
    np.testing.assert_array_equal(u32(step.mask[: g["mask_words"]]), p["mask"])
    np.testing.assert_array_equal(u32(step.block_count[: g["mask_blocks"]]), p["block_count"])
    np.testing.assert_array_equal(step.block_off.cpu().numpy(), p["block_off"])
    n = p["nnz"]
    assert step.nnz == n
    gs = step.screen[:n].cpu().numpy()
    np.testing.assert_array_equal(gs[:, :10].view(np.uint32), p["screen"][:, :10].astype(np.float32).view(np.uint32))
    np.testing.assert_array_equal(u32(step.aabb16[:n]), p["aabb"])
    del gs

    # --- intersections and tile ranges: exact counts everywhere
    _, total = orc.count_tiles(sc, p["aabb"])
    assert step.n_isects == total
    cnt = orc.tile_counts(sc, p)
    toff = np.concatenate([[0], np.cumsum(cnt)])
    np.testing.assert_array_equal(step.tile_off.cpu().numpy(), toff)
    if cfg == 5:
        assert total * 8 > 2**32  # the key buffer crosses 4 GiB

    # --- sampled tiles: sorted slices and every pixel
    tiles = sample_tiles(sc, g, cnt, rng)
    assert len(tiles) >= 200
    off, keys, vals = orc.tile_lists(sc, p, tiles)
    gk = step.keys
    gv = step.vals
    for i, t in enumerate(tiles):
        a, b = toff[t], toff[t + 1]
        np.testing.assert_array_equal(gk[a:b].cpu().numpy().view(np.uint64), keys[off[i]:off[i + 1]])
        np.testing.assert_array_equal(u32(gv[a:b]), vals[off[i]:off[i + 1]])
    img, T, last = orc.rasterize_tiles(sc, p, tiles, off, vals, toff[tiles], nthreads=THREADS)
    c, y, x = tile_pixels(g, tiles)
    inside = last != -2
    assert np.array_equal(inside, (y < sc.H) & (x < sc.W))
    ci, yi, xi = (torch.from_numpy(np.ascontiguousarray(a[inside])).cuda() for a in (c, y, x))
    np.testing.assert_array_equal(step.last[ci, yi, xi].cpu().numpy(), last[inside])
    assert np.abs(step.T[ci, yi, xi].cpu().numpy() - T[inside]).max() <= 1e-5
    assert np.abs(step.img[ci, yi, xi].cpu().numpy() - img[inside]).max() <= 1e-5

    # --- sampled Gaussians: screen-row and parameter gradients
    gauss = sample_gaussians(sc, p, rng)
    assert len(gauss) >= 200
    rows = np.nonzero(np.isin(p["row_gauss"], gauss))[0]
    need = set()
    for r in rows:
        a = p["aabb"][r]
        tx0 = (int(a[0] & 0xFFFF) * sc.W) // (65535 * 16)
        tx1 = min(-(-(int(a[1] & 0xFFFF) * sc.W) // (65535 * 16)), g["tiles_x"])
        ty0 = (int(a[0] >> 16) * sc.H) // (65535 * 16)
        ty1 = min(-(-(int(a[1] >> 16) * sc.H) // (65535 * 16)), g["tiles_y"])
        base = int(p["row_cam"][r]) * g["tiles_per_cam"]
        for ty in range(ty0, ty1):
            for tx in range(tx0, tx1):
                need.add(base + ty * g["tiles_x"] + tx)
    need = np.array(sorted(need), np.int64)
    off2, _, vals2 = orc.tile_lists(sc, p, need)
    v_rows = orc.raster_bwd_rows(sc, p, need, off2, vals2, v_img, None, rows, nthreads=THREADS)
    gvs = step.v_screen[torch.from_numpy(rows).cuda()].cpu().numpy()
    grad_close("v_screen rows", gvs[:, :9], v_rows[:, :9])
    per_row = orc.project_bwd_rows(sc, p, rows, v_rows)
    ns, ref = gaussian_grads(sc, p, rows, per_row)
    idx = torch.tensor(ns).cuda()
    for k, r in ref.items():
        grad_close(k, getattr(step, k)[idx].cpu().numpy(), r)
