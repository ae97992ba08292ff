"""The allocation-free sort entry point (ss_sort_isects_noalloc).

It exists for callers that cannot call cudaMalloc themselves (code running
inside another runtime's allocator callbacks, where a nested cudaMalloc would
re-enter that allocator, or hosts that hand out only fixed device buffers):
its scratch is a static device array inside libss.so, so the caller passes
only the key/value buffers and tile_off.

Checked here through the C ABI: two calls in a row give exactly the results of
the allocating ss_sort_isects (integer outputs, so the tolerance is equality),
and a key count beyond the static limit is refused before any device work.
The file sorts last so that a failure here never hides another test.
"""
import ctypes as ct

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 24 << 20


def max_keys(d):
    """Largest key count whose sort scratch fits the 24 MiB static array."""
    lo, hi = 1, 1 << 31
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if ss.workspace_bytes(d, ss.WS_SORT, mid) <= SCRATCH_BYTES else (lo, mid)
    return lo


def unsorted_keys(cfg):
    sc = scenes.make_scene(cfg)
    d = ss.scene_dims(sc)
    step = ss.PackedStep(d, "cuda")
    step.forward(*ss.scene_tensors(sc))
    n = step.n_isects
    # the intersection pass alone: keys/values in row-major order
    keys = torch.empty(n, dtype=torch.int64, device="cuda")
    vals = torch.empty(n, dtype=torch.int32, device="cuda")
    ss.ss_intersect_tiles(d, step.row_depth, step.aabb16, step.block_off, step.nnz, step.isect_off, keys, vals, n,
                          step.temp_isect)
    torch.cuda.synchronize()
    return d, keys, vals, n


def sort_with(d, keys, vals, n, noalloc):
    ka, va = keys.clone(), vals.clone()
    kb, vb = torch.empty_like(ka), torch.empty_like(va)
    tile_off = torch.empty(ss.size(d, ss.SIZE_N_TILES) + 1, dtype=torch.int64, device="cuda")
    if noalloc:
        in_b = ss.ss_sort_isects_noalloc(d, ka, va, kb, vb, n, tile_off)
    else:
        temp = torch.empty(ss.workspace_bytes(d, ss.WS_SORT, n), dtype=torch.uint8, device="cuda")
        in_b = ss.ss_sort_isects(d, ka, va, kb, vb, n, temp, tile_off)
    torch.cuda.synchronize()
    k, v = (kb, vb) if in_b else (ka, va)
    return k.cpu().numpy(), v.cpu().numpy(), tile_off.cpu().numpy()


@pytest.mark.parametrize("cfg", [2, 3])
def test_noalloc_sort_matches_allocating_sort_twice(cfg):
    d, keys, vals, n = unsorted_keys(cfg)
    assert n > 0
    ref = sort_with(d, keys, vals, n, noalloc=False)
    for _ in range(2):  # the static scratch keeps the previous call's contents
        got = sort_with(d, keys, vals, n, noalloc=True)
        for a, b in zip(got, ref):
            np.testing.assert_array_equal(a, b)


def test_noalloc_sort_rejects_more_than_its_limit():
    d = ss.make_dims(1, 64, 64, 0, 10)
    limit = max_keys(d)
    assert limit == 50_311_168  # the limit the header states
    in_b = ct.c_int(0)
    fake = ct.c_void_p(256)  # never dereferenced: the size check comes first
    st = ss.lib().ss_sort_isects_noalloc(ct.byref(d), fake, fake, fake, fake, limit + 1, fake, ct.byref(in_b),
                                         None)
    assert st == ss.SS_ERR_INVALID_ARG
    assert f"at most {limit} keys".encode() in ss.lib().ss_last_error()
