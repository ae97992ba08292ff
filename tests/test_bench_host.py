"""Host-side logic of bench.py and the binding that the bench line rests on
(no GPU needed): the traffic record's guards, the per-step launch count, the
oracle sample bound and the stage model's bytes."""
import json
import os

import pytest

import bench
from gaussian_splatting_differentiable_packed_b200 import ss


def test_traffic_record_guards(tmp_path, monkeypatch):
    rec = json.load(open(bench.TRAFFIC_FILE))
    stage = "rasterize_bwd"
    wl = rec["_workload"]
    # a record whose digest matches the sources as they are now is reported
    good = dict(rec)
    good[stage] = dict(rec[stage], sha256=bench.source_digest(rec[stage]["sources"]))
    p = tmp_path / "traffic.json"
    p.write_text(json.dumps(good))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.recorded_traffic(stage, wl["config"], wl["n"]) == float(rec[stage]["dram_bytes_per_launch"])
    # another workload: no traffic
    assert bench.recorded_traffic(stage, 3, None) is None
    assert bench.recorded_traffic(stage, wl["config"], 3_000_001) is None
    # sources that differ from the capture's: no traffic
    bad = dict(rec)
    bad[stage] = dict(rec[stage], sha256="0" * 64)
    p.write_text(json.dumps(bad))
    assert bench.recorded_traffic(stage, wl["config"], wl["n"]) is None
    # a capture of a smaller case scales by the units the kernel processes
    small = dict(rec)
    small[stage] = dict(rec[stage], sha256=bench.source_digest(rec[stage]["sources"]),
                        workload={"config": wl["config"], "n": 3_000_000}, units={"name": "n_isects", "value": 1000})
    p.write_text(json.dumps(small))
    got = bench.recorded_traffic(stage, wl["config"], None, dict(n_isects=3000))
    assert got == 3 * float(rec[stage]["dram_bytes_per_launch"])
    assert bench.recorded_traffic(stage, wl["config"], None, dict(nnz=3000)) is None
    assert bench.recorded_traffic(stage, 3, None, dict(n_isects=3000)) is None
    # a missing stage or file: no traffic
    assert bench.recorded_traffic("no_such_stage", wl["config"], wl["n"]) is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic(stage, wl["config"], wl["n"]) is None


def test_launches_per_step():
    """projection 5, intersection 3 plus one per depth-sort pass, the sort's
    bases (its digit counts come with the keys), one kernel per digit pass
    that runs and tile ranges, the tile order 3, rasterizers 2, projection
    backward 1."""
    d = ss.make_dims(5, 1600, 1067, 3, 15_000_000)
    assert ss.launches_per_step(d, 15_000_000, 33_000_000, 2, 3) == 5 + (3 + 3) + (2 + 2) + 3 + 2 + 1
    assert ss.launches_per_step(d, 15_000_000, 0, 0, 3) == 5 + (3 + 3) + 0 + 3 + 2 + 1
    assert ss.launches_per_step(d, 0, 0, 0, 0) == 5 + 0 + 0 + 3 + 2 + 1
    assert ss.launches_per_step(ss.make_dims(1, 64, 64, 0, 0), 0, 0, 0, 0) == 3 + 2


def test_sort_passes_skip_constant_bytes():
    """A byte equal in every key takes no pass: 16 tile-id bits and depths
    whose top byte is fixed take 5 of the 6 byte passes; keys that differ in
    one low bit take one; equal keys none."""
    import torch
    d = ss.make_dims(5, 1600, 1067, 3, 15_000_000)
    tiles = torch.arange(0, 33_500, dtype=torch.int64)
    depth = torch.full_like(tiles, 0x41000000) + (tiles * 1237) % (1 << 23)
    assert ss.sort_passes_for((tiles << 32) | depth, d, presorted_depth=False) == 5
    assert ss.sort_passes_for(torch.tensor([7, 6], dtype=torch.int64), d, presorted_depth=False) == 1
    assert ss.sort_passes_for(torch.tensor([5, 5], dtype=torch.int64), d, presorted_depth=False) == 0
    # keys in depth order: the tile-id bytes only
    assert ss.sort_passes_for((tiles << 32) | depth, d) == 2
    assert ss.depth_sort_passes(torch.tensor([1.5, 2.5, 3.0])) == 2


def test_oracle_sample_never_exceeds_the_workload():
    assert bench.oracle_sample(1, 300_000).N == 2_000
    assert bench.oracle_sample(2, 300_000).N == 100_000
    assert bench.oracle_sample(3, 300_000).N == 300_000


def test_stage_model_counts_every_stage():
    d = ss.make_dims(5, 1600, 1067, 3, 15_000_000)
    work = dict(evals=1.6e9, exps=1.1e8, comps=9e7, bwd_evals=1.6e9, bwd_exps=1.1e8)
    m = bench.stage_model(d, 16, 15_000_000, 33_000_000, 6, 33_500, work)
    for name in ("project_packed", "intersect_tiles", "sort_isects", "rasterize_fwd", "rasterize_bwd", "project_bwd",
                 "project_bwd_adam", "project_bwd_gq"):
        assert m[name]["bytes"] > 0, name
    # the projection backward reads and writes 236 B per Gaussian at SH 3,
    # plus the screen rows and the mask
    assert m["project_bwd"]["bytes"] > 2 * 236 * 15_000_000
    # the 16-bit accumulators are read and written (118 B each way per
    # Gaussian) where the plain call writes 236 B of fp32 gradients: about
    # the same traffic, half the memory; the fused Adam moves far more
    gq, plain = m["project_bwd_gq"]["bytes"], m["project_bwd"]["bytes"]
    assert abs(gq - plain) < 0.02 * plain
    assert plain < m["project_bwd_adam"]["bytes"]
