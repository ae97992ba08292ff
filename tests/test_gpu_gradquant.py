"""ss_project_bwd_gq: the projection backward accumulating into block-quantised
16-bit gradient accumulators, over two sub-batches of cameras.

* After the first sub-batch the decoded accumulator is the plain projection
  backward's gradient (same inputs, same arithmetic) within half a
  quantisation step; after the second it is the first accumulator plus the
  second sub-batch's gradient within half a step of the new scale.
* Against the oracle (fp64 gradients of each sub-batch, the same two-step
  accumulation): the decoded accumulators within the gradient tolerance of
  each sub-batch plus the quantisation steps of both sides, and the block
  scales within that tolerance over 32767.
Cases: three quantisation blocks with an even number of 128-Gaussian CTAs,
an odd CTA count (the cluster's extra CTA) and SH degree 0 (no higher SH
coefficients).
"""
import dataclasses

import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

ATTR_OF_GRAD = dict(means="v_means", quats="v_quats", scales="v_scales", opacities="v_opacities")


def sub_scene(sc, cams):
    return dataclasses.replace(sc, C=len(cams), cams=np.ascontiguousarray(sc.cams[cams]),
                               v_img=np.ascontiguousarray(sc.v_img[cams]))


def gpu_plain(step, K):
    N = step.v_means.shape[0]
    sh = step.v_sh.double().cpu().numpy().reshape(N, K, 3)
    out = {a: getattr(step, g).double().cpu().numpy().reshape(N, -1) for a, g in ATTR_OF_GRAD.items()}
    out["sh_dc"] = sh[:, :1, :].reshape(N, -1)
    out["sh_rest"] = sh[:, 1:, :].reshape(N, -1)
    return out


def steps_of(acc):
    return {a: np.repeat(acc.block_scale[i].double().cpu().numpy(), ss.GQ_BLOCK)[: acc.N].reshape(acc.N, 1)
            for i, a in enumerate(ss.GQ_ATTRS)}


@pytest.mark.parametrize("N,deg", [(700, 3), (300, 2), (130, 0)])
def test_two_sub_batches(N, deg):
    sc = scenes.random_tiny(60 + N, N=N, W=48, H=40, C=4, sh_degree=deg)
    acc = ss.GradQuantAccum(N, sc.K)
    plain, refs, dec_prev = [], [], None
    for k, cams in enumerate(([0, 1], [2, 3])):
        sub = sub_scene(sc, cams)
        o = orc.step(sub)
        refs.append(o["grads"])
        d = ss.scene_dims(sub)
        step = ss.PackedStep(d)
        t = ss.scene_tensors(sub)
        step.forward(*t)
        step.backward(torch.from_numpy(np.ascontiguousarray(o["v_img"], np.float32)).cuda())
        ss.ss_project_bwd_gq(d, *t, step.mask, step.block_off, step.v_screen, acc, first=(k == 0))
        torch.cuda.synchronize()
        g = gpu_plain(step, sc.K)
        dec = acc.decoded()
        st = steps_of(acc)
        for a in ss.GQ_ATTRS:
            x = g[a] if dec_prev is None else dec_prev[a] + g[a]
            # half a step, plus the rounding of the fp32 division x / scale
            bound = 0.51 * st[a] + 1e-7 * np.abs(x)
            assert np.all(np.abs(dec[a] - x) <= bound), (k, a, float(np.abs(dec[a] - x).max()))
            assert np.all(np.abs(acc.codes[a][:, : acc.widths[a]].cpu().numpy().astype(np.int32)) <= 32767)
        plain.append(g)
        dec_prev = dec
    # oracle: the same accumulation from its fp64 gradients
    acc_o = orc.gq_accumulate(orc.gq_accumulate(None, refs[0]), refs[1])
    r0, r1 = orc.gq_attributes(refs[0]), orc.gq_attributes(refs[1])
    st = steps_of(acc)
    dec = acc.decoded()
    for i, a in enumerate(ss.GQ_ATTRS):
        if acc.widths[a] == 0:
            continue
        ref_dec = orc.gq_decode(*acc_o[a])
        ref_step = np.repeat(acc_o[a][1], ss.GQ_BLOCK)[:N].reshape(N, 1)
        gtol = 1e-3 * (np.abs(r0[a]) + np.abs(r1[a])) + 2e-5
        # each side carries half a step of both quantisations (the first
        # scale is within the tolerance of the last one's order)
        tol = gtol + 1.5 * (st[a] + ref_step)
        err = np.abs(dec[a] - ref_dec)
        assert np.all(err <= tol), (a, float((err - tol).max()))
        s_gpu = acc.block_scale[i].double().cpu().numpy()[: len(acc_o[a][1])]
        nb = len(acc_o[a][1])
        for b in range(nb):
            blk = slice(b * ss.GQ_BLOCK, (b + 1) * ss.GQ_BLOCK)
            assert abs(s_gpu[b] - acc_o[a][1][b]) <= (gtol[blk].max() + 0.5 * (st[a][blk].max() + ref_step[blk].max())) / 32767 + 1e-12, (a, b)
