"""HostPipeline: steps over pinned host inputs with overlapped transfers give
the same gradients as PackedStep on device inputs, step by step, when the
inputs change between steps (so a buffer reused too early would show)."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss

pytestmark = pytest.mark.gpu


def test_pipeline_matches_direct_steps():
    scs = [scenes.make_scene(2, seed=s) for s in (0, 1, 2, 3)]
    d = ss.scene_dims(scs[0])
    rng = np.random.default_rng(3)
    v_imgs = [(rng.uniform(-1, 1, (d.C, d.H, d.W, 3)) / (3.0 * d.W * d.H)).astype(np.float32) for _ in scs]
    # reference: one PackedStep per input set, device inputs
    ref = []
    for sc, vi in zip(scs, v_imgs):
        st = ss.PackedStep(d, "cuda")
        st.forward(*ss.scene_tensors(sc))
        g = st.backward(torch.from_numpy(vi).cuda())
        ref.append({k: v.cpu().numpy().copy() for k, v in g.items()})
    # pipeline over pinned host buffers
    step = ss.PackedStep(d, "cuda")
    ex = ss.scene_tensors(scs[0])
    step.forward(*ex)
    pipe = ss.HostPipeline(step, ex, torch.from_numpy(v_imgs[0]).cuda())
    plan = []
    for sc, vi in zip(scs, v_imgs):
        hin = [t.cpu().pin_memory() for t in ss.scene_tensors(sc)]
        hv = torch.from_numpy(vi).pin_memory()
        hout = {k: torch.empty(tuple(getattr(step, k).shape), dtype=torch.float32).pin_memory()
                for k in ss.HostPipeline.GRADS}
        plan.append((hin, hv, hout))
    fin = pipe.run(plan)
    fin.synchronize()
    torch.cuda.synchronize()
    # the rasterizer's float atomics may add in another order: compare with a
    # relative bound plus a small fraction of the field's largest value
    for r, (_, _, hout) in zip(ref, plan):
        for k in ss.HostPipeline.GRADS:
            got, want = hout[k].numpy().astype(np.float64), r[k].astype(np.float64)
            tol = 1e-4 * np.abs(want) + 1e-5 * np.abs(want).max()
            assert np.all(np.abs(got - want) <= tol), k
