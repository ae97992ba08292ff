"""The per-image visible cap of ss_project_packed (the pages' --cap-max)
against the oracle's sort-and-truncate reading: the capped mask, block counts
and offsets, nnz, rows and AABB16s bit-exact, and the whole step after it
(intersections, sorted keys, image, last_id, gradients) as in the uncapped
parity tests."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss
from oracle import oracle as orc
from test_gpu_parity import check_backward, check_forward

pytestmark = pytest.mark.gpu


def capped_parity(sc, cap):
    o = orc.step(sc, precision=0, nthreads=16, cap_max=cap)
    step = ss.PackedStep(ss.scene_dims(sc), "cuda", cap_visible=cap)
    step.forward(*ss.scene_tensors(sc))
    step.backward(torch.from_numpy(np.ascontiguousarray(o["v_img"], np.float32)).cuda())
    torch.cuda.synchronize()
    check_forward(sc, o, step)
    check_backward(sc, o, step)
    return o, step


@pytest.mark.parametrize("seed,cap", [(0, 40), (1, 1), (2, 123), (3, 250)])
def test_cap_random_tiny(seed, cap):
    sc = scenes.random_tiny(800 + seed, N=300 + 40 * seed, W=48, H=40, C=1 + seed % 3, sh_degree=seed % 4)
    o, _ = capped_parity(sc, cap)
    assert o["proj"]["nnz"] < orc.project(sc, rows=False)["nnz"]


def test_cap_partly_visible_cameras():
    # cameras see different numbers of pairs: some capped, some not
    sc = scenes.make_scene(3, n=20_000)
    full = orc.project(sc, rows=False)
    cam_counts = np.diff(full["block_off"][:: orc.geometry(sc)["blocks_per_cam"]])
    cap = int(np.median(cam_counts))
    o, _ = capped_parity(sc, cap)
    assert o["proj"]["nnz"] < full["nnz"]


def test_cap_ties_zero_and_no_op():
    sc = scenes.random_tiny(812, N=300, W=48, H=40, C=2, sh_degree=0)
    sc.opacities = np.full(sc.N, 0.5, np.float32)  # every opacity equal: lowest indices stay
    capped_parity(sc, 17)
    o, step = capped_parity(sc, 0)
    assert step.nnz == 0
    big = orc.project(sc, rows=False)["nnz"]
    o, step = capped_parity(sc, big)
    assert step.nnz == big


def test_cap_count_only_mode():
    sc = scenes.random_tiny(814, N=500, W=48, H=40, C=3, sh_degree=1)
    d = ss.scene_dims(sc)
    step = ss.PackedStep(d, "cuda")
    t = ss.scene_tensors(sc)
    n = ss.ss_project_packed(d, *t, step.mask, step.block_count, step.block_off, None, None, None, 0,
                             step.temp_project, cap_visible=77)
    assert n == orc.project(sc, rows=False, cap_max=77)["nnz"] == 3 * 77
