"""Parity at the full workload sizes, in the launch configuration bench.py
times (PackedStep over the whole scene), on outputs the oracle can compute:

* the whole visibility mask, block counts and offsets, nnz, every screen row
  and AABB16 (the oracle's projection runs over all C*N pairs);
* n_isects and the full tile_off array (exact per-tile counts);
* the sorted (key, value) slices of sampled tiles, including the longest one;
* image, transmittance and last_id of every pixel of those tiles;
* the screen-row gradients and the Gaussian gradients of sampled Gaussians
  (every pixel of every tile they touch is replayed by the oracle).

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
    nonempty = np.nonzero(cnt)[0]
    tiles = np.unique(np.concatenate([[int(np.argmax(cnt))], rng.choice(nonempty, 23, replace=False)]))
    off, keys, vals = orc.tile_lists(sc, p, tiles)
    gk = step.keys
    gv = step.vals
    for i, t in enumerate(tiles):
        a, b = toff[t], toff[t + 1]
        np.testing.assert_array_equal(gk[a:b].cpu().numpy().view(np.uint64), keys[off[i]:off[i + 1]])
        np.testing.assert_array_equal(u32(gv[a:b]), vals[off[i]:off[i + 1]])
    img, T, last = orc.rasterize_tiles(sc, p, tiles, off, vals, toff[tiles], nthreads=THREADS)
    gimg = step.img.cpu().numpy()
    gT = step.T.cpu().numpy()
    glast = step.last.cpu().numpy()
    for i, t in enumerate(tiles):
        c, tr = divmod(int(t), g["tiles_per_cam"])
        ty, tx = divmod(tr, g["tiles_x"])
        for q in range(256):
            y, x = ty * 16 + q // 16, tx * 16 + q % 16
            if last[i, q] == -2:
                continue
            assert glast[c, y, x] == last[i, q], (t, q)
            assert abs(gT[c, y, x] - T[i, q]) <= 1e-5
            assert np.abs(gimg[c, y, x] - img[i, q]).max() <= 1e-5

    # --- sampled Gaussians: screen-row and parameter gradients
    gauss = rng.choice(np.unique(p["row_gauss"]), 10, replace=False)
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
