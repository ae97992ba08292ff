"""Direct parity of ss_sort_isects with the oracle's stable sort on seeded
synthetic (tile << 32 | depth) keys with skewed tile populations (uniform
tiles, a few tiles holding thousands of keys as the heavy tiles of the large
workloads do), and a tile count needing 17 tile-id bits.  The sort skips
the digit bytes that are equal in every key, so the pass count (and the
buffer pair that ends up holding the result) follows from the keys.
Depths repeat (ties must keep input order) and values are not ordered by
position, so only a stable sort by key matches.  Keys, values and tile
offsets must be bit-exact.
"""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import ss
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


def make_keys(rng, n_tiles, n, hot=()):
    """n keys over uniform tiles plus `hot` = [(tile, count), ...] extra keys;
    depths drawn from a small pool half of the time so that many tie."""
    tiles = [rng.integers(0, n_tiles, n)]
    for t, c in hot:
        tiles.append(np.full(c, t))
    tiles = np.concatenate(tiles).astype(np.uint64)
    rng.shuffle(tiles)
    m = len(tiles)
    pool = rng.uniform(0.2, 50.0, 40).astype(np.float32)
    depth = np.where(rng.random(m) < 0.5, rng.choice(pool, m), rng.uniform(0.2, 50.0, m).astype(np.float32))
    bits = depth.astype(np.float32).view(np.uint32).astype(np.uint64)
    keys = (tiles << np.uint64(32)) | bits
    vals = rng.permutation(m).astype(np.uint32) * np.uint32(7) + np.uint32(3)
    return keys, vals


def digit_hist(keys):
    """Counts of each value of byte b of the keys' tile ids, [4][256] int32."""
    tiles = (np.asarray(keys, np.uint64) >> np.uint64(32)).astype(np.uint64)
    h = np.zeros((4, 256), np.int64)
    for b in range(4):
        h[b] = np.bincount(((tiles >> np.uint64(8 * b)) & np.uint64(255)).astype(np.int64), minlength=256)
    return h.astype(np.int32).reshape(-1)


def run_sort(d, keys, vals, presorted_depth=False, with_hist=False):
    n = len(keys)
    ka = torch.from_numpy(keys.view(np.int64).copy()).cuda()
    va = torch.from_numpy(vals.view(np.int32).copy()).cuda()
    kb = torch.empty_like(ka)
    vb = torch.empty_like(va)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    tile_off = torch.empty(n_tiles + 1, dtype=torch.int64, device="cuda")
    temp = torch.empty(ss.workspace_bytes(d, ss.WS_SORT, n), dtype=torch.uint8, device="cuda")
    hist = torch.from_numpy(digit_hist(keys)).cuda() if with_hist else None
    in_b = ss.ss_sort_isects(d, ka, va, kb, vb, n, temp, tile_off, presorted_depth=presorted_depth, key_hist=hist)
    torch.cuda.synchronize()
    k, v = (kb, vb) if in_b else (ka, va)
    return in_b, k.cpu().numpy().view(np.uint64), v.cpu().numpy().view(np.uint32), tile_off.cpu().numpy()


@pytest.mark.parametrize("case", ["small", "large", "lsd", "three_tile_bytes"])
def test_sort_paths(case):
    rng = np.random.default_rng({"small": 11, "large": 12, "lsd": 13, "three_tile_bytes": 14}[case])
    if case == "three_tile_bytes":
        d = ss.make_dims(5, 2048, 2048, 0, 1, 0.01, 1e10)  # 81920 tiles: 17 tile-id bits
    else:
        d = ss.make_dims(1, 1024, 1024, 0, 1, 0.01, 1e10)  # 4096 tiles
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    hot = {"small": [], "large": [(17, 9000), (4000, 2100)], "lsd": [(5, 20000), (6, 3000)],
           "three_tile_bytes": [(81919, 2500)]}[case]
    keys, vals = make_keys(rng, n_tiles, 300_000, hot)
    in_b, gk, gv, toff = run_sort(d, keys, vals)
    assert in_b == bool(ss.sort_passes_for(torch.from_numpy(keys.view(np.int64)), d, presorted_depth=False) & 1)
    ok, ov = orc.sort(keys, vals)
    np.testing.assert_array_equal(gk, ok)
    np.testing.assert_array_equal(gv, ov)
    np.testing.assert_array_equal(toff, orc.tile_ranges(ok, n_tiles))


def test_sort_single_bucket_and_tiny():
    """Every key in one tile (one 1500-key bucket), and a 3-key input."""
    d = ss.make_dims(1, 64, 64, 0, 1, 0.01, 1e10)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    rng = np.random.default_rng(15)
    for keys, vals in [make_keys(rng, 1, 1500), make_keys(rng, n_tiles, 3)]:
        in_b, gk, gv, toff = run_sort(d, keys, vals)
        ok, ov = orc.sort(keys, vals)
        np.testing.assert_array_equal(gk, ok)
        np.testing.assert_array_equal(gv, ov)
        np.testing.assert_array_equal(toff, orc.tile_ranges(ok, n_tiles))


def test_sort_skipped_digit_plans():
    """Digit bytes equal in every key are skipped: every key equal (no pass,
    the result stays in the first pair), keys differing in one low bit (one
    pass), depths sharing their top byte (one pass fewer), and full 32-bit
    low words with the top bit set (every pass)."""
    d = ss.make_dims(1, 1024, 1024, 0, 1, 0.01, 1e10)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    rng = np.random.default_rng(16)
    same = np.full(5000, (np.uint64(77) << np.uint64(32)) | np.uint64(0x40a00000), np.uint64)
    one_bit = same ^ rng.integers(0, 2, 5000).astype(np.uint64)
    top = (rng.integers(0, n_tiles, 100_000).astype(np.uint64) << np.uint64(32)) | \
        (np.uint64(0x41000000) + rng.integers(0, 1 << 23, 100_000).astype(np.uint64))
    full = (rng.integers(0, n_tiles, 200_000).astype(np.uint64) << np.uint64(32)) | \
        rng.integers(0, 2**32, 200_000, dtype=np.uint64)
    for keys, passes in ((same, 0), (one_bit, 1), (top, 5), (full, 6)):
        vals = rng.permutation(len(keys)).astype(np.uint32)
        p = ss.sort_passes_for(torch.from_numpy(keys.view(np.int64)), d, presorted_depth=False)
        assert p == passes
        in_b, gk, gv, toff = run_sort(d, keys, vals)
        assert in_b == bool(p & 1)
        ok, ov = orc.sort(keys, vals)
        np.testing.assert_array_equal(gk, ok)
        np.testing.assert_array_equal(gv, ov)
        np.testing.assert_array_equal(toff, orc.tile_ranges(ok, n_tiles))


@pytest.mark.parametrize("case", ["tiles4096", "tiles81920"])
def test_sort_presorted_depth(case):
    """Keys that arrive in depth order (ties in the order to keep), as the
    intersection writes them: sorting the tile-id bytes alone gives the full
    stable key order."""
    rng = np.random.default_rng(17)
    d = ss.make_dims(1, 1024, 1024, 0, 1, 0.01, 1e10) if case == "tiles4096" else \
        ss.make_dims(5, 2048, 2048, 0, 1, 0.01, 1e10)
    n_tiles = ss.size(d, ss.SIZE_N_TILES)
    keys, vals = make_keys(rng, n_tiles, 300_000, [(n_tiles - 1, 3000), (3, 9000)])
    order = np.argsort((keys & np.uint64(0xFFFFFFFF)).astype(np.uint32), kind="stable")
    keys, vals = keys[order], vals[order]
    ok, ov = orc.sort(keys, vals)
    # with the sort's own histogram read, and with the digit counts given as
    # the intersection writes them
    for with_hist in (False, True):
        in_b, gk, gv, toff = run_sort(d, keys, vals, presorted_depth=True, with_hist=with_hist)
        assert in_b == bool(ss.sort_passes_for(torch.from_numpy(keys.view(np.int64)), d, presorted_depth=True) & 1)
        np.testing.assert_array_equal(gk, ok)
        np.testing.assert_array_equal(gv, ov)
        np.testing.assert_array_equal(toff, orc.tile_ranges(ok, n_tiles))
