"""ss_tile_order and the rasterizers' tile order.

The order only schedules the rasterizers' CTAs: it must be a permutation of
the tiles with heavier tiles first (four bins per power of two of the entry
count, so a later tile never holds 5/4 or more of the entries of an earlier
one; empty tiles last), the forward's outputs must be bit-identical with and
without it, and the backward's row gradients equal up to the order of the
float additions.
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss

pytestmark = pytest.mark.gpu


def _forward(sc):
    d = ss.scene_dims(sc)
    step = ss.PackedStep(d)
    t = ss.scene_tensors(sc)
    step.forward(*t)
    torch.cuda.synchronize()
    return d, step, t


@pytest.mark.parametrize("cfg", [2, 3])
def test_order_is_heaviest_first_permutation(cfg):
    sc = scenes.make_scene(cfg, n=100_000 if cfg == 3 else None)
    d, step, _ = _forward(sc)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    order = step.tile_order[:n_tiles].cpu().numpy().view(np.uint32).astype(np.int64)
    np.testing.assert_array_equal(np.sort(order), np.arange(n_tiles))
    toff = step.tile_off.cpu().numpy()
    cnt = (toff[1:] - toff[:-1])[order].astype(np.float64)
    nz = cnt > 0
    # empty tiles form the tail
    k = int(nz.sum())
    assert nz[:k].all() and not nz[k:].any()
    # within 5/4 of every earlier tile's count
    run_min = np.minimum.accumulate(cnt[:k])
    assert np.all(cnt[1:k] < 1.25 * run_min[:-1])
    assert 1.25 * cnt[0] > cnt.max()  # the first tile is in the heaviest bin


def test_ordered_rasterizers_match_index_order():
    sc = scenes.make_scene(2)
    d, step, t = _forward(sc)
    img0, T0, last0 = step.img.clone(), step.T.clone(), step.last.clone()
    img = torch.empty_like(img0)
    T = torch.empty_like(T0)
    last = torch.empty_like(last0)
    ss.ss_rasterize_fwd(d, step.screen, step.vals, step.tile_off, img, T, last)  # tile index order
    torch.cuda.synchronize()
    assert torch.equal(img, img0) and torch.equal(T, T0) and torch.equal(last, last0)
    g = torch.Generator(device="cpu").manual_seed(5)
    v_img = (torch.rand(img0.shape, generator=g) * 2 - 1).cuda()
    vs_ordered = torch.empty_like(step.v_screen)
    vs_index = torch.empty_like(step.v_screen)
    ss.ss_rasterize_bwd(d, step.screen, step.vals, step.tile_off, step.T, step.last, v_img, None, vs_ordered,
                        step.nnz, tile_order=step.tile_order)
    ss.ss_rasterize_bwd(d, step.screen, step.vals, step.tile_off, step.T, step.last, v_img, None, vs_index,
                        step.nnz)
    torch.cuda.synchronize()
    a = vs_ordered[: step.nnz].double().cpu().numpy()
    b = vs_index[: step.nnz].double().cpu().numpy()
    err = np.abs(a - b)
    assert np.all(err <= 1e-5 + 1e-4 * np.abs(b)), float(err.max())


def test_empty_tile_list():
    sc = scenes.random_tiny(3, N=0, W=40, H=24)
    d, step, _ = _forward(sc)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    order = step.tile_order[:n_tiles].cpu().numpy().view(np.uint32)
    np.testing.assert_array_equal(np.sort(order), np.arange(n_tiles))
