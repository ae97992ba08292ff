"""ss_project_bwd_adam (projection backward fused with an Adam step) against
the oracle: the oracle's gradients taken to the raw parameters and one Adam
step in fp64, from a random optimizer state at step t = 3.  The moments give
back the gradient ((m' - b1 m) / (1 - b1) = g), which is held to the gradient
tolerance plus the floor that this recovery itself sets: m' is stored in
fp32, so its rounding (up to about one ulp of b1 m for the product and one
of m' for the sum) comes back divided by 1 - b1; the parameter updates and
the refreshed activated copies are compared with the oracle's."""
import numpy as np
import pytest
import torch

from gaussian_splatting_differentiable_packed_b200 import scenes, ss
from oracle import oracle as orc
from test_gpu_parity import grad_close

pytestmark = pytest.mark.gpu

LR = dict(means=1.6e-4, quats=1e-3, log_scales=5e-3, logit_opacities=5e-2, sh=(2.5e-3, 1.25e-4))
B1, B2, EPS, T = 0.9, 0.999, 1e-8, 3


def run(sc, seed):
    rng = np.random.default_rng(seed)
    d = ss.scene_dims(sc)
    v_img = (rng.uniform(-1, 1, (sc.C, sc.H, sc.W, 3)) / (3.0 * sc.W * sc.H)).astype(np.float32)
    o = orc.step(sc, precision=0, nthreads=16, v_img=v_img)
    raw_g = orc.raw_gradients(o["grads"], sc.scales, sc.opacities)
    params = dict(means=sc.means.astype(np.float64), quats=sc.quats.astype(np.float64),
                  log_scales=np.log(sc.scales.astype(np.float64)),
                  logit_opacities=np.log(sc.opacities / (1.0 - sc.opacities)).astype(np.float64),
                  sh=sc.sh.astype(np.float64))
    m0 = {k: (rng.normal(size=v.shape) * 1e-4).astype(np.float32) for k, v in params.items()}
    v0 = {k: rng.uniform(1e-8, 1e-6, v.shape).astype(np.float32) for k, v in params.items()}
    P, M, V = orc.adam_step(params, raw_g, m0, v0, LR, B1, B2, EPS, T)

    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    cams, means, quats, scales, opac, sh = ss.scene_tensors(sc)
    log_s = f(params["log_scales"])
    logit = f(params["logit_opacities"])
    step = ss.PackedStep(d, "cuda")
    step.forward(cams, means, quats, scales, opac, sh)
    ss.ss_rasterize_bwd(d, step.screen, step.vals, step.tile_off, step.T, step.last, f(v_img), None, step.v_screen,
                        step.nnz)
    names = dict(means="means", quats="quats", scales="log_scales", opacities="logit_opacities", sh="sh")
    state = {}
    for short, key in names.items():
        state["m_" + short] = f(m0[key])
        state["v_" + short] = f(v0[key])
    hp = ss.ss_adam(LR["means"], LR["quats"], LR["log_scales"], LR["logit_opacities"], LR["sh"][0], LR["sh"][1],
                    B1, B2, EPS, T)
    ss.ss_project_bwd_adam(d, cams, means, quats, log_s, scales, logit, opac, sh, step.mask, step.block_off,
                           step.v_screen, state, hp)
    torch.cuda.synchronize()
    got = dict(means=means, quats=quats, log_scales=log_s, logit_opacities=logit, sh=sh)
    for short, key in names.items():
        gm = state["m_" + short].cpu().numpy().astype(np.float64)
        gv = state["v_" + short].cpu().numpy().astype(np.float64)
        # the gradient the kernel used, from its moments; the scale-aware bound
        # gets the recovery's own floor: two ulps of the largest moment over 1 - b1
        floor = 2.0 * float(np.spacing(np.float32(max(np.abs(m0[key]).max(), np.abs(gm).max())))) / (1.0 - B1)
        scale = max(float(np.abs(raw_g[key]).max()), 1e-30)
        grad_close("g " + key, (gm - B1 * m0[key]) / (1.0 - B1), raw_g[key], scale_tol=1e-4 + floor / scale)
        g2 = (gv - B2 * v0[key].astype(np.float64)) / (1.0 - B2)
        # v' is stored in fp32: recovering g^2 from it loses about 1.2e-4 * v0
        assert np.all(np.abs(g2 - raw_g[key] ** 2) <= 3e-3 * raw_g[key] ** 2 + 1e-6 * np.abs(raw_g[key] ** 2).max()
                      + 2e-3 * np.abs(v0[key])), key
        dp = got[key].cpu().numpy().astype(np.float64) - params[key]
        dref = P[key] - params[key]
        tol = 3e-3 * np.abs(dref) + 1e-3 * np.abs(dref).max() + 1e-6 * np.abs(params[key])
        assert np.all(np.abs(dp - dref) <= tol), (key, float(np.abs(dp - dref).max()))
    np.testing.assert_allclose(scales.cpu().numpy(), np.exp(log_s.cpu().numpy().astype(np.float64)), rtol=2e-6)
    lo = logit.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(opac.cpu().numpy(), 1.0 / (1.0 + np.exp(-lo)), rtol=2e-6)
    assert np.abs(raw_g["means"]).max() > 0


@pytest.mark.parametrize("seed", range(3))
def test_fused_adam_random_tiny(seed):
    run(scenes.random_tiny(60 + seed, N=350 + 50 * seed, W=40, H=36, C=1 + seed % 2, sh_degree=seed + 1,
                           opacity_range=(0.1, 0.9)), seed)


def test_fused_adam_config2():
    run(scenes.make_scene(2), 7)
