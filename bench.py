"""Benchmark of the packed 3DGS forward+backward step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

A step is one pass of the whole path over the workload: ss_project_packed,
ss_intersect_tiles, ss_sort_isects, ss_tile_order, ss_rasterize_fwd, ss_rasterize_bwd,
ss_project_bwd.  The upstream dL/dimage is an input of the step (the L1
gradient against the workload's seeded target, computed once from the forward
image before timing; the step's work does not depend on its values).

Default workload: configuration 4 (15M Gaussians x 5 cameras at 1600x1067,
SH degree 3; 75M pairs, ~15M visible, ~33M tile intersections), the shape of
the pages' art_gallery measurement.  Inputs (3.5 GB of parameters) are larger
than L2, so no flush is needed between steps.

Multi-GPU: the step does not shard on one GPU's problem; N ranks run N
independent replicas (weak scaling), timed on the device, max over ranks.

--impl reference times the CPU oracle (as it stands) on a bounded sample of
the same workload on the host cores; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd step ms at 1 B200; isects/s; per-stage % of HBM/FP32 roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), sm_max_mhz=float(p.get("sm_max_mhz", 1965.0)), src="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, sm_max_mhz=1965.0, src="fallback")


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def source_digest(paths) -> str:
    """sha256 over the kernel's source files (the capture is void once they change)."""
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(stage: str, config: int, n, units=None):
    """DRAM bytes per launch of the stage's kernel from a recorded ncu capture,
    or None when there is none, it was taken on another workload, or the
    kernel's sources changed since.  A capture of a smaller case of the same
    workload (fewer Gaussians) is scaled to this launch by the units the
    kernel processes (record["units"]: the unit's name and its count in the
    capture; `units` maps names to this run's counts), when the record says
    that its traffic grows in proportion to them."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        rec = t[stage]
        wl = rec.get("workload", t["_workload"])
        if source_digest(rec["sources"]) != rec["sha256"]:
            return None
        if wl == {"config": config, "n": n}:
            return float(rec["dram_bytes_per_launch"])
        if wl.get("config") != config or "units" not in rec or not units:
            return None
        name, captured = rec["units"]["name"], float(rec["units"]["value"])
        if name not in units or captured <= 0:
            return None
        return float(rec["dram_bytes_per_launch"]) * float(units[name]) / captured
    except Exception:
        return None


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return dict(sm_mhz=float(np.median(sm)) if sm else None, sm_max_mhz=mx, reasons=sorted(reasons),
                    samples=len(sm))


# ---------------------------------------------------------------------------- roofline model
def stage_model(d, K, nnz, n_isects, passes, n_tiles, work, n_seen=None, depth_passes=4):
    """Algorithmic bytes (HBM) and FP32 instruction counts per call.

    bytes: every input the stage needs read once and every output written
    once, at the stage's own layout (the SH coefficients only of the n_seen
    Gaussians some camera sees: the colour of the others is never
    evaluated); instr: FP32-pipe instructions of the canonical per-item
    sequences (counted from the source), for the ALU-bound stages.
    """
    if n_seen is None:
        n_seen = d.N
    C, N, W, H = d.C, d.N, d.W, d.H
    P = C * N
    X = C * W * H
    row = 48
    par = 40  # means 12 + quats 16 + scales 12
    shb = 12 * K
    m = {}
    m["project_packed"] = dict(bytes=par * N + P / 8 + P / 32 + P / 16 + (par + 4) * N + shb * n_seen
                               + (row + 8 + 4) * nnz, instr=P * 140.0 + nnz * 160.0)
    # depth keys of the rows, the count and the depth digits (depth 4 B and
    # AABB 8 B read, key 8 B written), their keys-only sort (16 B per byte
    # pass), the write (key 8 B, AABB 8 B, offsets 8 B; 12 B per key)
    m["intersect_tiles"] = dict(bytes=nnz * (20 + 16 * depth_passes + 24) + 12 * n_isects, instr=0.0)
    # 12 B read + 12 B written per key per digit pass that runs (the tile-id
    # bytes: the keys arrive in depth order, with their digit counts from the
    # intersection), tile offsets
    m["sort_isects"] = dict(bytes=n_isects * (24 * passes) + 8 * (n_tiles + 1), instr=0.0)
    # per-pixel FP32 instructions of the canonical sequences: 11 per evaluated
    # entry (offsets, sigma, tests), 16 per exp (range reduction, degree-7
    # polynomial, scaling, alpha), 7 per composite; backward: 11 per replayed
    # entry, 17 per exp, 30 per contributing entry (T recovery, nine gradients)
    # second model, the measurement plan's FLOP counts: forward E * (12 + 1
    # exp) + C * 10 over the evaluated entries E and composited entries C; the
    # backward about three times that on the replayed entries (against 2
    # FLOPs per FMA lane per clock)
    m["rasterize_fwd"] = dict(bytes=n_isects * (4 + row) + X * 20 + 8 * (n_tiles + 1),
                              instr=work["evals"] * 11.0 + work["exps"] * 16.0 + work["comps"] * 7.0,
                              flops=work["evals"] * 13.0 + work["comps"] * 10.0)
    m["rasterize_bwd"] = dict(bytes=n_isects * (4 + row) + X * 24 + nnz * row * 2,
                              instr=work["bwd_evals"] * 11.0 + work["bwd_exps"] * 17.0 + work["comps"] * 30.0,
                              flops=3.0 * (work["bwd_evals"] * 13.0 + work["comps"] * 10.0))
    m["project_bwd"] = dict(bytes=par * N + shb * n_seen + row * nnz + P / 8 + P / 16 + (par + 4 + shb) * N,
                            instr=nnz * 700.0)
    # fused with Adam: parameters, activated copies and both moments read and
    # written once, no gradient arrays
    pa = par + 4 + shb
    m["project_bwd_adam"] = dict(bytes=(pa + 16) * N + 2 * pa * N + row * nnz + P / 8 + P / 16
                                 + (pa + 16) * N + 2 * pa * N, instr=nnz * 700.0)
    # with block-quantised accumulators: parameters and SH read once, the
    # 16-bit codes read and written (2 bytes per gradient element), scales
    q = 2 * (11 + 3 * K)
    m["project_bwd_gq"] = dict(bytes=(par + 4 + shb) * N + row * nnz + P / 8 + P / 16 + 2 * q * N + 2 * 6 * 4 * N / 256,
                               instr=nnz * 700.0)
    return m


def fp32_peak_instr_per_s(sm_mhz: float) -> float:
    # 148 SMs x 128 FP32 lanes, one instruction per lane per clock
    return 148 * 128 * sm_mhz * 1e6


def fp32_peak_flops(sm_mhz: float) -> float:
    # the same lanes counted as 2 FLOPs per FMA
    return 2.0 * fp32_peak_instr_per_s(sm_mhz)


# ---------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, device) -> float:
    """Largest x over all ranks (a replicated step's time is its slowest
    rank's); x itself when no process group is running."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput of `world` replicas each processing
    units_per_rank in a step whose slowest rank took ms."""
    return world * units_per_rank / (ms / 1e3)


# ---------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from gaussian_splatting_differentiable_packed_b200 import scenes, ss

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    dev = torch.device("cuda", local)

    sc = scenes.make_scene(args.config, n=args.n)
    d = ss.scene_dims(sc)
    inputs = ss.scene_tensors(sc, dev)
    step = ss.PackedStep(d, dev)
    # optional depth output + background blend (forward) and depth gradient
    # (backward), seeded inputs
    fkw, bkw, bg_t, v_D = {}, {}, None, None
    if args.depth_bg:
        g_ext = torch.Generator(device="cpu").manual_seed(1234)
        bg_t = torch.rand((d.C, 3), generator=g_ext).to(dev)
        v_D = ((torch.rand((d.C, d.H, d.W), generator=g_ext) * 2 - 1) / (d.W * d.H)).to(dev)
        fkw, bkw = dict(bg=bg_t, depth=True), dict(v_depth=v_D)
    step.forward(*inputs, **fkw)
    torch.cuda.synchronize()
    # capacities with headroom, then the upstream gradient from this forward
    step._rows(int(step.nnz * 1.05) + 1)
    step._isects(int(step.n_isects * 1.05) + 1)
    img = step.forward(*inputs, **fkw)
    if sc.upstream == "l1":
        target = torch.from_numpy(sc.target).to(dev)
        v_img = (torch.sign(img - target) * sc.l1_scale).contiguous()
        del target
    else:
        v_img = torch.from_numpy(sc.v_img).to(dev)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()

    # optional fused projection backward + Adam: raw parameters, activated
    # copies and moments on the device, updated in place every step
    trainer = None
    if args.adam:
        cams, means, quats, scales, opac, sh = inputs
        trainer = ss.AdamTrainer(step, cams, means, quats, torch.log(scales).contiguous(),
                                 torch.log(opac / (1.0 - opac)).contiguous(), sh, eps=1e-8)
        inputs = (cams, means, quats, trainer.scales, trainer.opacities, sh)

    # optional block-quantised gradient accumulation: every step after the
    # first decodes, adds and re-quantises (the sub-batch update)
    gq = ss.GradQuantAccum(d.N, (d.sh_degree + 1) ** 2, dev) if args.grad_quant else None
    gq_first = [True]

    last_stage = "project_bwd_adam" if args.adam else ("project_bwd_gq" if gq is not None else "project_bwd")
    names = ["project_packed", "intersect_tiles", "sort_isects", "rasterize_fwd", "rasterize_bwd", last_stage]

    def backward_rest():
        if gq is not None:
            ss.ss_project_bwd_gq(d, *inputs, step.mask, step.block_off, step.v_screen, gq, first=gq_first[0])
            gq_first[0] = False
        elif trainer is None:
            ss.ss_project_bwd(d, *inputs, step.mask, step.block_off, step.v_screen, step.v_means, step.v_quats,
                              step.v_scales, step.v_opacities, step.v_sh)
        else:
            trainer.hp.step += 1
            ss.ss_project_bwd_adam(d, trainer.cams, trainer.means, trainer.quats, trainer.log_scales,
                                   trainer.scales, trainer.logit_opacities, trainer.opacities, trainer.sh, step.mask,
                                   step.block_off, step.v_screen, trainer.state, trainer.hp)

    def whole_step():
        step.forward(*inputs, **fkw)
        if trainer is None and gq is None:
            step.backward(v_img, **bkw)
        else:
            ss.ss_rasterize_bwd(d, step.screen, step.vals, step.tile_off, step.T, step.last, v_img, None,
                                step.v_screen, step.nnz, tile_order=step.tile_order)
            backward_rest()

    def run_step(ev=None):
        if ev is not None:
            ev[0].record(st)
        step.forward(*inputs, stream=None, **fkw) if ev is None else _timed_forward(ev)
        if ev is None:
            step.backward(v_img, **bkw)
        else:
            ss.ss_rasterize_bwd(d, step.screen, step.vals, step.tile_off, step.T, step.last, v_img, None,
                                step.v_screen, step.nnz, v_depth=v_D, bg=bg_t, tile_order=step.tile_order)
            ev[5].record(st)
            backward_rest()
            ev[6].record(st)

    def _timed_forward(ev):
        cams, means, quats, scales, opac, sh = inputs
        nnz = ss.ss_project_packed(d, cams, means, quats, scales, opac, sh, step.mask, step.block_count,
                                   step.block_off, step.screen, step.aabb16, step.row_depth, step.cap_rows,
                                   step.temp_project)
        ev[1].record(st)
        n = ss.ss_intersect_tiles(d, step.row_depth, step.aabb16, step.block_off, nnz, step.isect_off, step.keys_a,
                                  step.vals_a, step.cap_isects, step.temp_isect, key_hist=step.key_hist)
        ev[2].record(st)
        in_b = ss.ss_sort_isects(d, step.keys_a, step.vals_a, step.keys_b, step.vals_b, n, step.temp_sort,
                                 step.tile_off, presorted_depth=True, key_hist=step.key_hist)
        step.vals = step.vals_b if in_b else step.vals_a
        ev[3].record(st)
        # the rasterizers' tile order is part of the forward rasterizer's stage
        ss.ss_tile_order(d, step.tile_off, step.tile_order, step.temp_order)
        ss.ss_rasterize_fwd(d, step.screen, step.vals, step.tile_off, step.img, step.T, step.last,
                            step.depth if args.depth_bg else None, bg_t, tile_order=step.tile_order)
        ev[4].record(st)
        step.nnz, step.n_isects = nnz, n

    for _ in range(args.warmup):
        whole_step()
    torch.cuda.synchronize()

    # ---- headline: K whole steps, device-timed, max over ranks
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for _ in range(args.steps):
        whole_step()
    t1.record(st)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)

    # ---- per-stage times (separate pass, events between the calls)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for k in range(args.steps):
        run_step(evs[k])
    torch.cuda.synchronize()
    stage_ms = {nm: float(np.mean([evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)]))
                for i, nm in enumerate(names)}

    # ---- work counts for the ALU roofline (outside every timed region)
    work = ss.raster_work(d, step) if hasattr(ss, "raster_work") else dict(
        evals=0.0, exps=0.0, comps=0.0, bwd_evals=0.0, bwd_exps=0.0)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and not args.adam and not args.grad_quant:  # those keep their state on the device
        host_in = [t.cpu().pin_memory() for t in inputs]
        host_vimg = v_img.cpu().pin_memory()
        host_out = {k: torch.empty(tuple(getattr(step, k).shape), dtype=torch.float32).pin_memory()
                    for k in ("v_means", "v_quats", "v_scales", "v_opacities", "v_sh")}
        dev_in = [torch.empty_like(t) for t in inputs]
        dev_vimg = torch.empty_like(v_img)
        h2d = sum(t.numel() * 4 for t in host_in) + host_vimg.numel() * 4
        d2h = sum(t.numel() * 4 for t in host_out.values())

        # the public host-memory API: next step's inputs up and last step's
        # gradients down on their own streams while the current step runs
        pipe = ss.HostPipeline(step, inputs, v_img)
        ke = max(2, min(args.steps, 6))
        plan = [(host_in, host_vimg, host_out)] * ke
        if fkw or bkw:
            pipe = None  # the extension run keeps the plain host loop below
        if pipe is not None:
            pipe.run(plan[:2])
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a0 = torch.cuda.Event(enable_timing=True)
            a0.record(st)
            a1 = pipe.run(plan, start=a0)
            torch.cuda.synchronize()
            e_ms = a0.elapsed_time(a1) / ke
        else:
            def e2e_step():
                for a, b in zip(dev_in, host_in):
                    a.copy_(b, non_blocking=True)
                dev_vimg.copy_(host_vimg, non_blocking=True)
                step.forward(*dev_in, **fkw)
                g = step.backward(dev_vimg, **bkw)
                for k, h in host_out.items():
                    h.copy_(g[k], non_blocking=True)

            e2e_step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(st)
            for _ in range(ke):
                e2e_step()
            a1.record(st)
            torch.cuda.synchronize()
            e_ms = a0.elapsed_time(a1) / ke
        e_ms = max_over_ranks(e_ms, dev)
        e2e = dict(value=job_throughput(step.n_isects, world, e_ms), unit="isects/s", ms_per_step=e_ms,
                   h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h))

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    peaks = load_peaks()
    passes = ss.sort_passes_for(step.keys[: step.n_isects], d)
    n_seen = ss.seen_gaussians(d, step.mask)
    depth_passes = ss.depth_sort_passes(step.row_depth[: step.nnz])
    model = stage_model(d, (d.sh_degree + 1) ** 2, step.nnz, step.n_isects, passes, ss.size(d, ss.SIZE_N_TILES),
                        work, n_seen, depth_passes)
    sm_mhz = clocks["sm_mhz"] or peaks["sm_max_mhz"]
    stages = {}
    for nm in names:
        t = stage_ms[nm] / 1e3
        b = model[nm]["bytes"]
        ins = model[nm]["instr"]
        hbm = b / t / 1e9
        alu = ins / t
        f_hbm = hbm / peaks["hbm_gbs"]
        f_alu = alu / fp32_peak_instr_per_s(sm_mhz) if ins else 0.0
        stages[nm] = dict(ms=round(stage_ms[nm], 4), hbm_gbs=round(hbm, 1), hbm_frac=round(f_hbm, 4),
                          alu_frac=round(f_alu, 4), bound="alu" if f_alu > f_hbm else "hbm")
        if "flops" in model[nm]:
            stages[nm]["flop_frac"] = round(model[nm]["flops"] / t / fp32_peak_flops(sm_mhz), 4)
    # whole-step fraction: sum over stages of the roofline time (the slower of
    # bytes at the HBM peak and FP32 instructions at the FP32 peak) over the
    # sum of measured stage times
    t_roof = sum(max(model[nm]["bytes"] / (peaks["hbm_gbs"] * 1e9),
                     model[nm]["instr"] / fp32_peak_instr_per_s(sm_mhz)) for nm in names)
    step_frac = t_roof / (sum(stage_ms.values()) / 1e3)
    # the same with the rasterizers priced by the FLOP model
    t_roof_fl = sum(max(model[nm]["bytes"] / (peaks["hbm_gbs"] * 1e9),
                        model[nm].get("flops", model[nm]["instr"] * 2.0) / fp32_peak_flops(sm_mhz)) for nm in names)
    step_frac_fl = t_roof_fl / (sum(stage_ms.values()) / 1e3)
    dom = max(names, key=lambda k: stage_ms[k])
    units = dict(N=d.N, nnz=step.nnz, n_isects=step.n_isects, pixels=d.C * d.W * d.H)
    sd = stages[dom]
    if sd["bound"] == "hbm":
        roof = dict(bound="hbm", achieved=sd["hbm_gbs"], peak=peaks["hbm_gbs"], unit="GB/s", frac=sd["hbm_frac"],
                    traffic=recorded_traffic(dom, args.config, args.n, units), kernel=dom, peak_source=peaks["src"])
    else:
        ach = model[dom]["instr"] / (stage_ms[dom] / 1e3) / 1e12
        pk = fp32_peak_instr_per_s(sm_mhz) / 1e12
        roof = dict(bound="alu", achieved=round(ach, 3), peak=round(pk, 3), unit="T FP32 instr/s",
                    frac=round(ach / pk, 4), traffic=recorded_traffic(dom, args.config, args.n, units), kernel=dom,
                    peak_source=f"148 SMs x 128 FP32 lanes x {sm_mhz:.0f} MHz (median SM clock under load)",
                    model="FP32 instructions of the canonical per-pixel sequences")
        if "flops" in model[dom]:
            fa = model[dom]["flops"] / (stage_ms[dom] / 1e3) / 1e12
            fp = fp32_peak_flops(sm_mhz) / 1e12
            roof["flop_model"] = dict(achieved=round(fa, 3), peak=round(fp, 3), unit="TFLOP/s", frac=round(fa / fp, 4),
                                      model="E * (12 + 1 exp) + C * 10 per pass, x3 for the backward")
    launches = ss.launches_per_step(d, step.nnz, step.n_isects, passes, depth_passes) * args.steps
    out_work = dict(work)
    out = dict(metric=METRIC, value=job_throughput(step.n_isects, world, ms), unit="isects/s", n_gpus=world,
               steps=args.steps, warmup=args.warmup, ms_per_step=round(ms, 4), higher_is_better=True,
               scaling="weak", vs_baseline=None, dtype="f32", data="synthetic",
               config=dict(workload=sc.name if args.n is None else f"{sc.name}, N overridden to {d.N}",
                           C=d.C, N=d.N, W=d.W, H=d.H,
                           sh_degree=d.sh_degree, pairs=d.C * d.N, nnz=step.nnz, n_isects=step.n_isects,
                           sort_passes=passes, depth_sort_passes=depth_passes, gaussians_seen=n_seen, l2="inputs larger than L2 (3.5 GB parameters), no flush",
                           parallelism=f"replicas x{world}", depth_and_background=bool(args.depth_bg),
                           fused_adam=bool(args.adam), grad_quant=bool(args.grad_quant)),
               pairs_per_s=world * d.C * d.N / (ms / 1e3),
               pixel_gaussian_evals_per_s=world * work["evals"] / (stage_ms["rasterize_fwd"] / 1e3),
               step_roofline_frac=round(step_frac, 4), step_roofline_frac_flop_model=round(step_frac_fl, 4),
               raster_work=out_work, stages=stages, roofline=roof,
               clocks=clocks,
               e2e=e2e, gpu_launches=launches)
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.config, args.cpu_sample)
    print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- CPU oracle
# Gaussian count of each workload (the sample never exceeds the workload)
WORKLOAD_N = {1: 2_000, 2: 100_000, 3: 1_000_000, 4: 15_000_000, 5: 13_000_000}


def oracle_sample(config: int, n: int):
    from gaussian_splatting_differentiable_packed_b200 import scenes
    full = WORKLOAD_N.get(config)
    return scenes.make_scene(config, n=None if full is not None and n >= full else n)


def cpu_baseline(config: int, n_sample: int, repeats: int = 1):
    from oracle import oracle as orc
    cores = os.cpu_count() or 1
    sc = oracle_sample(config, n_sample)
    t = time.perf_counter()
    isects = 0
    for _ in range(repeats):
        r = orc.step(sc, precision=0, nthreads=cores)
        isects += r["isect"]["n_isects"]
    dt = time.perf_counter() - t
    return dict(value=isects / dt, unit="isects/s", cores=cores, kind="oracle",
                sample=f"the workload's distributions and cameras ({sc.name}) with N={sc.N} Gaussians "
                       f"({r['isect']['n_isects']} intersections, full image size), {repeats} step(s) "
                       f"in {dt:.1f} s")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from oracle import oracle as orc
    cores = os.cpu_count() or 1
    sc = oracle_sample(args.config, args.cpu_sample)
    for _ in range(min(args.warmup, 1)):
        orc.step(sc, precision=0, nthreads=cores)
    t = time.perf_counter()
    isects = 0
    for _ in range(args.steps):
        r = orc.step(sc, precision=0, nthreads=cores)
        isects += r["isect"]["n_isects"]
    dt = time.perf_counter() - t
    v = isects / dt
    out = dict(impl="reference", metric=METRIC, value=v, unit="isects/s", n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=1e3 * dt / args.steps, higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="f32", data="synthetic",
               config=dict(workload=f"{sc.name}: bounded sample with N={sc.N} Gaussians"),
               cpu_baseline=dict(value=v, unit="isects/s", cores=cores, kind="oracle",
                                 sample=f"{sc.name} with N={sc.N} Gaussians per step"),
               e2e=dict(value=v, unit="isects/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--n", type=int, default=None, help="override the Gaussian count (profiling captures)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample", type=int, default=300_000)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--adam", action="store_true",
                    help="train: the projection backward fused with an Adam step updates the parameters in place")
    ap.add_argument("--grad-quant", action="store_true",
                    help="accumulate the projection backward's gradients into block-quantised 16-bit accumulators")
    ap.add_argument("--depth-bg", action="store_true",
                    help="also render the expected depth over a background colour and back-propagate a depth gradient")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
