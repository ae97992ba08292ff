"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
exports every function include/ss.h declares, derives the documented sizes,
and rejects bad arguments before touching the device."""
import ctypes as ct
import os
import re

import pytest

from conftest import ROOT
from gaussian_splatting_differentiable_packed_b200 import build as ssbuild
from gaussian_splatting_differentiable_packed_b200 import ss


@pytest.fixture(scope="module")
def L():
    ssbuild.build()
    return ss.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "ss.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ss_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_function(L):
    names = header_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(ss.EXPORTS)


def test_sizes_match_layout(L):
    d = ss.make_dims(5, 1600, 1067, 3, 15_000_000)
    n_pad = (15_000_000 + 127) // 128 * 128
    assert ss.size(d, ss.SIZE_N_PAD) == n_pad
    assert ss.size(d, ss.SIZE_MASK_WORDS) == 5 * n_pad // 32
    assert ss.size(d, ss.SIZE_MASK_BLOCKS) == 5 * n_pad // 128
    assert ss.size(d, ss.SIZE_TILES_X) == 100 and ss.size(d, ss.SIZE_TILES_Y) == 67
    assert ss.size(d, ss.SIZE_N_TILES) == 5 * 100 * 67
    for which, count in ((ss.WS_PROJECT, 0), (ss.WS_INTERSECT, 15_000_000), (ss.WS_SORT, 30_000_000),
                         (ss.WS_TILE_ORDER, 0)):
        assert ss.workspace_bytes(d, which, count) > 0


def test_tile_order_rejects_bad_arguments_on_host(L):
    """ss_tile_order checks its pointers and scratch size before any device
    work (the fake pointers are never dereferenced)."""
    d = ss.make_dims(1, 64, 64, 0, 10)
    fake = ct.c_void_p(256)
    need = ss.workspace_bytes(d, ss.WS_TILE_ORDER, 0)
    assert L.ss_tile_order(ct.byref(d), None, fake, fake, need, None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_tile_order(ct.byref(d), fake, None, fake, need, None) == ss.SS_ERR_INVALID_ARG
    assert L.ss_tile_order(ct.byref(d), fake, fake, fake, need - 1, None) == ss.SS_ERR_INVALID_ARG
    assert b"temp" in L.ss_last_error()
    bad = ss.make_dims(1, 0, 64, 0, 10)
    assert L.ss_tile_order(ct.byref(bad), fake, fake, fake, need, None) == ss.SS_ERR_INVALID_ARG


def test_oracle_and_library_agree_on_geometry(L):
    from gaussian_splatting_differentiable_packed_b200 import scenes
    from oracle import oracle as orc
    for cfg, n in ((1, None), (2, 1000), (3, 777), (4, 5000), (5, 300)):
        sc = scenes.make_scene(cfg, n=n)
        g = orc.geometry(sc)
        d = ss.scene_dims(sc)
        assert ss.size(d, ss.SIZE_MASK_WORDS) == g["mask_words"]
        assert ss.size(d, ss.SIZE_MASK_BLOCKS) == g["mask_blocks"]
        assert ss.size(d, ss.SIZE_N_TILES) == g["n_tiles"]


@pytest.mark.parametrize("bad", [dict(C=0), dict(W=0), dict(sh_degree=4), dict(N=-1), dict(near=0.0),
                                 dict(far=0.001)])
def test_invalid_dims_rejected_on_host(L, bad):
    kw = dict(C=1, W=64, H=64, sh_degree=0, N=10, near=0.01, far=100.0)
    kw.update(bad)
    d = ss.make_dims(kw["C"], kw["W"], kw["H"], kw["sh_degree"], kw["N"], kw["near"], kw["far"])
    assert L.ss_size(ct.byref(d), 0) == -1
    assert L.ss_workspace_bytes(ct.byref(d), 0, 0) == 0
    nnz = ct.c_int64(0)
    st = L.ss_project_packed(ct.byref(d), *([None] * 12), 0, -1, None, 0, ct.byref(nnz), None)
    assert st == ss.SS_ERR_INVALID_ARG
    assert b"dims" in L.ss_last_error()


def test_sort_overflow_rejected_before_device_work(L):
    d = ss.make_dims(1, 64, 64, 0, 10)
    in_b = ct.c_int(0)
    st = L.ss_sort_isects(ct.byref(d), None, None, None, None, 2**31, 0, None, None, 0, ct.c_void_p(16),
                          ct.byref(in_b), None)
    assert st == ss.SS_ERR_OVERFLOW
    assert L.ss_status_string(st) == b"count overflows 32-bit indices"


def test_grad_quant_rejects_bad_arguments_on_host(L):
    """ss_project_bwd_gq checks its accumulator before any device work (the
    fake pointers are never dereferenced)."""
    d = ss.make_dims(1, 64, 64, 3, 1000)
    f = ct.c_void_p(256)
    args = [ct.byref(d)] + [f] * 9
    assert L.ss_project_bwd_gq(*args, None, 1, None) == ss.SS_ERR_INVALID_ARG
    acc = ss.ss_gq_accum(256, 256, 256, 256, 256, None, 256)  # degree 3 needs the higher-SH codes
    assert L.ss_project_bwd_gq(*args, ct.byref(acc), 1, None) == ss.SS_ERR_INVALID_ARG
    assert b"accumulator" in L.ss_last_error()
    acc = ss.ss_gq_accum(256, 256, 256, 256, 256 + 2, 256, 256)  # DC codes off a 16-byte boundary
    assert L.ss_project_bwd_gq(*args, ct.byref(acc), 1, None) == ss.SS_ERR_INVALID_ARG
    assert b"16-byte" in L.ss_last_error()


def test_null_and_short_temp_rejected(L):
    d = ss.make_dims(1, 64, 64, 0, 10)
    nnz = ct.c_int64(0)
    fake = ct.c_void_p(256)  # never dereferenced: the temp size check fails first
    st = L.ss_project_packed(ct.byref(d), fake, fake, fake, fake, fake, fake, fake, fake, fake, None, None, None, 0,
                             -1, fake, 1, ct.byref(nnz), None)
    assert st == ss.SS_ERR_INVALID_ARG
    n = ct.c_uint64(0)
    st = L.ss_intersect_tiles(ct.byref(d), fake, fake, fake, 5, fake, fake, fake, None, 100, fake, 1, ct.byref(n),
                              None)
    assert st == ss.SS_ERR_INVALID_ARG


def test_noalloc_sort_limit_on_host(L):
    """The allocation-free sort's key limit is the largest count whose sort
    scratch fits its 24 MiB static array: the workspace query agrees at the
    boundary, and one key more is refused with the limit in the message."""
    d = ss.make_dims(1, 64, 64, 0, 10)
    limit = 50_311_168
    assert ss.workspace_bytes(d, ss.WS_SORT, limit) <= 24 << 20
    assert ss.workspace_bytes(d, ss.WS_SORT, limit + 1) > 24 << 20
    in_b = ct.c_int(0)
    fake = ct.c_void_p(256)  # never dereferenced: the size check comes first
    st = L.ss_sort_isects_noalloc(ct.byref(d), fake, fake, fake, fake, limit + 1, fake, ct.byref(in_b), None)
    assert st == ss.SS_ERR_INVALID_ARG
    assert f"at most {limit} keys".encode() in L.ss_last_error()
