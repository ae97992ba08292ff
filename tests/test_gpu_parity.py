"""Parity of the CUDA path (libss.so through the C ABI) with the CPU oracle.

Integer outputs must be bit-exact: visibility mask, block counts and offsets,
nnz, screen rows (the forward is specified in canonical fp32 order, so the
rows are bit-identical too), AABB16, n_isects, per-row offsets, keys and
values before and after the sort, tile ranges, last_id.  Images and final
transmittance within 1e-5 absolute.  Gradients within 1e-3 relative +
1e-5 absolute of the oracle's fp64 gradients (atomic order varies), plus a
scale-aware bound (error / max|reference| <= 1e-4) so that small-valued
gradient fields are not passed by the absolute term alone.
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

ORACLE_THREADS = 16


def u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def run_gpu(scene, v_img=None, v_T=None, **kw):
    d = ss.scene_dims(scene)
    step = ss.PackedStep(d, "cuda", **kw)
    t = ss.scene_tensors(scene)
    step.forward(*t)
    if v_img is not None:
        vi = torch.from_numpy(np.ascontiguousarray(v_img, np.float32)).cuda()
        vt = None if v_T is None else torch.from_numpy(np.ascontiguousarray(v_T, np.float32)).cuda()
        step.backward(vi, vt)
    torch.cuda.synchronize()
    return step


def grad_close(name, gpu, ref, rtol=1e-3, atol=1e-5, scale_tol=1e-4):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, name
    if ref.size == 0:
        return
    err = np.abs(gpu - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not bad.any(), (name, int(bad.sum()), float(err[bad].max()), np.argwhere(bad)[:5].tolist())
    scale = max(float(np.abs(ref).max()), 1e-30)
    assert float(err.max()) / scale <= scale_tol, (name, float(err.max()) / scale)


def check_forward(scene, o, step):
    g = o["geo"]
    p = o["proj"]
    np.testing.assert_array_equal(u32(step.mask[: g["mask_words"]]), p["mask"])
    np.testing.assert_array_equal(u32(step.block_count[: g["mask_blocks"]]), p["block_count"])
    np.testing.assert_array_equal(step.block_off.cpu().numpy(), p["block_off"])
    assert step.nnz == p["nnz"]
    n = p["nnz"]
    if n:
        gs = step.screen[:n].cpu().numpy()
        np.testing.assert_array_equal(gs[:, :10].view(np.uint32), p["screen"][:, :10].astype(np.float32).view(np.uint32))
        assert np.all(gs[:, 10:] == 0)
        np.testing.assert_array_equal(u32(step.aabb16[:n]), p["aabb"])
    I = o["isect"]["n_isects"]
    assert step.n_isects == I
    per, _ = orc.count_tiles(scene, p["aabb"])
    # rows are written in depth order: the offsets follow that order
    order = o["isect"]["order"]
    np.testing.assert_array_equal(step.isect_off[: n + 1].cpu().numpy(), np.concatenate([[0], np.cumsum(per[order])]))
    if I:
        np.testing.assert_array_equal(step.keys[:I].cpu().numpy().view(np.uint64), o["keys_sorted"])
        np.testing.assert_array_equal(u32(step.vals[:I]), o["vals_sorted"])
    np.testing.assert_array_equal(step.tile_off.cpu().numpy(), o["tile_off"])
    img = step.img.cpu().numpy().astype(np.float64)
    T = step.T.cpu().numpy().astype(np.float64)
    assert np.abs(img - o["img"]).max() <= 1e-5
    assert np.abs(T - o["T"]).max() <= 1e-5
    np.testing.assert_array_equal(step.last.cpu().numpy(), o["last"])


def check_unsorted(scene, o, step):
    """Keys/values as written by the intersection pass (before the sort)."""
    p = o["proj"]
    it = orc.intersect(scene, p)
    # the sort ping-pongs; re-run the intersect call alone to read its output
    I = it["n_isects"]
    keys = torch.empty(max(I, 1), dtype=torch.int64, device="cuda")
    vals = torch.empty(max(I, 1), dtype=torch.int32, device="cuda")
    hist = torch.full((4 * 256,), -1, dtype=torch.int32, device="cuda")
    n = ss.ss_intersect_tiles(step.d, step.row_depth, step.aabb16, step.block_off, step.nnz, step.isect_off, keys, vals,
                              I, step.temp_isect, key_hist=hist)
    torch.cuda.synchronize()
    assert n == I
    if I:
        np.testing.assert_array_equal(keys[:I].cpu().numpy().view(np.uint64), it["keys"])
        np.testing.assert_array_equal(u32(vals[:I]), it["vals"])
    # the digit counts of the keys' tile-id bytes it wrote for the sort (the
    # bytes past the tile ids' width stay zero)
    tiles = it["keys"] >> np.uint64(32)
    nb = max(1, (int(np.ceil(np.log2(max(ss.size(step.d, ss.SIZE_N_TILES), 1)))) + 7) // 8) if I else 0
    want = np.zeros((4, 256), np.int64)
    for b in range(nb):
        want[b] = np.bincount(((tiles >> np.uint64(8 * b)) & np.uint64(255)).astype(np.int64), minlength=256)
    np.testing.assert_array_equal(hist.cpu().numpy().reshape(4, 256), want)


def check_backward(scene, o, step):
    n = o["proj"]["nnz"]
    vs = step.v_screen[:n].cpu().numpy()
    ref = o["v_screen"]
    grad_close("v_screen", vs[:, :9], ref[:, :9])
    assert np.all(vs[:, 9:] == 0)
    for k, ref in o["grads"].items():
        grad_close(k, getattr(step, k).cpu().numpy(), ref)


def full_parity(scene, with_unsorted=True):
    o = orc.step(scene, precision=0, nthreads=ORACLE_THREADS)
    step = run_gpu(scene, o["v_img"])
    check_forward(scene, o, step)
    if with_unsorted:
        check_unsorted(scene, o, step)
    check_backward(scene, o, step)
    return o, step


@pytest.mark.parametrize("seed", range(6))
def test_random_tiny_scenes(seed):
    sc = scenes.random_tiny(seed, N=300 + 61 * seed, W=37 + 16 * seed, H=29 + 5 * seed, C=1 + seed % 3,
                            sh_degree=seed % 4)
    full_parity(sc)


def test_config1_tiny():
    o, step = full_parity(scenes.make_scene(1))
    assert o["proj"]["nnz"] > 1000 and o["isect"]["n_isects"] > 1000


def test_config2_100k():
    o, step = full_parity(scenes.make_scene(2))
    assert o["proj"]["nnz"] > 50_000


def test_config3_reduced():
    # the 1M x 4 workload's distributions and cameras with 1/10 of the Gaussians
    full_parity(scenes.make_scene(3, n=100_000), with_unsorted=False)


def test_config3_full_size():
    # the 1M-Gaussian, 4-camera 1280x720 workload, every output compared whole
    o, step = full_parity(scenes.make_scene(3), with_unsorted=False)
    assert o["proj"]["nnz"] > 1_000_000


def test_many_cameras_ragged():
    # 33 cameras (two camera chunks per CTA), N not a multiple of 128, partial tiles
    full_parity(scenes.random_tiny(40, N=517, W=45, H=23, C=33, sh_degree=2))


def test_non_rigid_viewmat_and_edge_gaussians():
    # view matrices whose 3x3 part is scaled and sheared (rows of unequal norm,
    # row 0 not orthogonal to row 2) and Gaussians spread across and past the
    # image edges: the visibility decisions near the edges and with a
    # non-orthonormal camera rotation must stay bit-exact
    sc = scenes.random_tiny(42, N=900, W=53, H=41, C=3, sh_degree=1)
    rng = np.random.default_rng(42)
    sc.means = rng.uniform(-2.2, 2.2, (sc.N, 3)).astype(np.float32)
    cams = sc.cams.copy()
    for c in range(sc.C):
        R = cams[c, :12].reshape(3, 4)[:, :3].astype(np.float64)
        R2 = R.copy()
        R2[0] = 1.25 * R[0] + 0.1 * R[2]
        R2[1] = 0.8 * R[1] - 0.07 * R[2]
        R2[2] = 1.1 * R[2]
        m = cams[c, :12].reshape(3, 4).copy()
        m[:, :3] = R2
        cams[c, :12] = m.reshape(-1)
    sc.cams = cams.astype(np.float32)
    o = orc.step(sc, precision=0, nthreads=ORACLE_THREADS)
    assert 0 < o["proj"]["nnz"] < sc.C * sc.N
    step = run_gpu(sc, o["v_img"])
    check_forward(sc, o, step)
    check_unsorted(sc, o, step)
    vs = step.v_screen[: o["proj"]["nnz"]].cpu().numpy()
    grad_close("v_screen", vs[:, :9], o["v_screen"][:, :9])
    # Parameter gradients: a few Gaussians here sum camera terms that cancel
    # (v_means[520, 2] = 0.34 from terms of size ~3), where the float oracle
    # itself is 2e-4 of the largest gradient away from the fp64 oracle; so
    # the bound is relative to each gradient's scale.
    for k, ref in o["grads"].items():
        gpu = np.asarray(getattr(step, k).cpu().numpy(), np.float64)
        err = np.abs(gpu - np.asarray(ref, np.float64))
        assert err.max() <= 1e-3 * max(float(np.abs(ref).max()), 1e-30), (k, float(err.max()))


def test_opacity_above_one():
    # opacities in (0.5, 1.6): entries with o > 1 take no skip threshold and no
    # culling (every pixel evaluates them), the alpha clamp at 0.99 is hit
    full_parity(scenes.random_tiny(41, N=600, W=48, H=40, C=2, sh_degree=1, opacity_range=(0.5, 1.6)))


def test_empty_scene():
    sc = scenes.random_tiny(1, N=0, W=40, H=24)
    o = orc.step(sc)
    step = run_gpu(sc, o["v_img"])
    assert step.nnz == 0 and step.n_isects == 0
    assert np.all(step.img.cpu().numpy() == 0) and np.all(step.T.cpu().numpy() == 1)
    assert np.all(step.last.cpu().numpy() == -1)


def test_all_invisible():
    sc = scenes.random_tiny(2, N=200, W=40, H=24)
    sc.means = sc.means + np.float32(100.0)  # everything far off to the side / behind
    o = orc.step(sc)
    assert o["proj"]["nnz"] == 0
    step = run_gpu(sc, o["v_img"])
    check_forward(sc, o, step)
    for k in ("v_means", "v_quats", "v_scales", "v_opacities", "v_sh"):
        assert np.all(getattr(step, k).cpu().numpy() == 0)


def test_capacity_errors_report_exact_counts():
    sc = scenes.make_scene(1)
    o = orc.forward(sc)
    d = ss.scene_dims(sc)
    t = ss.scene_tensors(sc)
    step = ss.PackedStep(d, "cuda", cap_rows=10, cap_isects=10)
    with pytest.raises(ss.SSError) as e:
        ss.ss_project_packed(d, *t, step.mask, step.block_count, step.block_off, step.screen, step.aabb16,
                             step.row_depth, step.cap_rows, step.temp_project)
    assert e.value.status == ss.SS_ERR_CAPACITY and e.value.count == o["proj"]["nnz"]
    # count-only mode
    assert ss.ss_project_packed(d, *t, step.mask, step.block_count, step.block_off, None, None, None, 0,
                                step.temp_project) == o["proj"]["nnz"]
    step._rows(o["proj"]["nnz"])
    nnz = ss.ss_project_packed(d, *t, step.mask, step.block_count, step.block_off, step.screen, step.aabb16,
                               step.row_depth, step.cap_rows, step.temp_project)
    with pytest.raises(ss.SSError) as e:
        ss.ss_intersect_tiles(d, step.row_depth, step.aabb16, step.block_off, nnz, step.isect_off, step.keys_a,
                              step.vals_a, 10, step.temp_isect)
    assert e.value.status == ss.SS_ERR_CAPACITY and e.value.count == o["isect"]["n_isects"]


def test_counts_past_2_pow_32_are_exact():
    # 4400 large Gaussians over a 16384^2 image: every row covers all 1M tiles,
    # so n_isects = 4400 * 2^20 > 2^32.  The count must not wrap and the call
    # must refuse to write (32-bit values); no key buffer is allocated.
    W = H = 16384
    N = 4400
    rng = np.random.default_rng(3)
    cam = np.concatenate([np.eye(4).reshape(16), [8000.0, 8000.0, W / 2, H / 2]]).astype(np.float32)
    sc = scenes.Scene(0, 1, W, H, 0, N, 0.01, 1e10, cam[None], rng.uniform(-0.01, 0.01, (N, 3)).astype(np.float32)
                      + np.float32([0, 0, 2.0]), np.tile(np.float32([1, 0, 0, 0]), (N, 1)),
                      np.full((N, 3), 5.0, np.float32), np.full(N, 0.5, np.float32),
                      np.zeros((N, 1, 3), np.float32), "uniform", None, None, "huge")
    p = orc.project(sc)
    per, total = orc.count_tiles(sc, p["aabb"])
    assert total > 2**32
    d = ss.scene_dims(sc)
    t = ss.scene_tensors(sc)
    step = ss.PackedStep(d, "cuda", cap_rows=N, cap_isects=1)
    nnz = ss.ss_project_packed(d, *t, step.mask, step.block_count, step.block_off, step.screen, step.aabb16,
                               step.row_depth, step.cap_rows, step.temp_project)
    assert nnz == p["nnz"] == N
    with pytest.raises(ss.SSError) as e:
        ss.ss_intersect_tiles(d, step.row_depth, step.aabb16, step.block_off, nnz, step.isect_off, None, None,
                              2**62, step.temp_isect)
    assert e.value.status == ss.SS_ERR_OVERFLOW
    assert e.value.count == total


def test_rasterizer_work_counts_match_oracle():
    # the counting forward reports the per-pixel work the definition implies
    sc = scenes.make_scene(2, n=30_000)
    o = orc.forward(sc, nthreads=ORACLE_THREADS)
    _, _, _, ev, cp = orc.rasterize_fwd(sc, o["proj"]["screen"], o["vals_sorted"], o["tile_off"], evals=True,
                                        nthreads=ORACLE_THREADS)
    step = run_gpu(sc)
    w = ss.raster_work(step.d, step)
    assert w["evals"] == int(ev.sum())
    assert w["comps"] == int(cp.sum())
    g = o["geo"]
    jj, ii = np.mgrid[0:sc.H, 0:sc.W]
    t = (jj // 16) * g["tiles_x"] + ii // 16
    last = o["last"][0]
    replay = np.where(last >= 0, last - o["tile_off"][t] + 1, 0)
    assert w["bwd_evals"] == int(replay.sum())
    np.testing.assert_array_equal(step.last.cpu().numpy(), o["last"])


# ---------------------------------------------------------------- depth output and background
def depth_bg_parity(scene, seed):
    """Forward with a background per camera and the expected depth, backward
    with v_T and v_depth: images, depth, T and last_id against the oracle,
    every screen-row gradient including the depth column, and the Gaussian
    gradients (the depth gradient reaches the means through the camera z)."""
    rng = np.random.default_rng(700 + seed)
    shp = (scene.C, scene.H, scene.W)
    bg = rng.uniform(0.0, 1.0, (scene.C, 3)).astype(np.float32)
    v_img = (rng.uniform(-1, 1, shp + (3,)) / (3.0 * scene.W * scene.H)).astype(np.float32)
    v_T = (rng.uniform(-1, 1, shp) / (scene.W * scene.H)).astype(np.float32)
    v_D = (rng.uniform(-1, 1, shp) / (scene.W * scene.H)).astype(np.float32)
    o = orc.step(scene, precision=0, nthreads=ORACLE_THREADS, v_img=v_img, v_T=v_T, v_depth=v_D, bg=bg)
    step = ss.PackedStep(ss.scene_dims(scene), "cuda")
    step.forward(*ss.scene_tensors(scene), bg=torch.from_numpy(bg).cuda(), depth=True)
    step.backward(torch.from_numpy(v_img).cuda(), torch.from_numpy(v_T).cuda(), v_depth=torch.from_numpy(v_D).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(step.last.cpu().numpy(), o["last"])
    assert np.abs(step.T.cpu().numpy() - o["T"]).max() <= 1e-5
    assert np.abs(step.img.cpu().numpy() - o["img"]).max() <= 1e-5
    D = step.depth.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(D - o["depth"]) <= 1e-5 * np.maximum(1.0, np.abs(o["depth"])))
    n = o["proj"]["nnz"]
    vs = step.v_screen[:n].cpu().numpy()
    grad_close("v_screen", vs[:, :10], o["v_screen"][:, :10])
    assert np.abs(o["v_screen"][:, 9]).max() > 0  # the depth column is exercised
    for k, ref in o["grads"].items():
        grad_close(k, getattr(step, k).cpu().numpy(), ref)


@pytest.mark.parametrize("seed", range(4))
def test_depth_and_background_random_tiny(seed):
    sc = scenes.random_tiny(50 + seed, N=400 + 37 * seed, W=41 + 8 * seed, H=33 + 3 * seed, C=1 + seed % 2,
                            sh_degree=(seed + 1) % 4)
    depth_bg_parity(sc, seed)


def test_depth_and_background_config2():
    depth_bg_parity(scenes.make_scene(2), 9)
