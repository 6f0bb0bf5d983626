"""GPU parity of the sampler entry points (dit_sampler_step, dit_sample) against the
sampler oracle (deterministic DDPM step and rectified-flow Euler step around the
denoiser; "Sora / DiT" training objective, "GOKU" §2.3)."""
import numpy as np
import pytest
import torch

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding
from diffusion_transformer_denoiser_dit_b200.binding import DiT, DitError
from oracle import dit_oracle as O
from oracle import sampler as SM

pytestmark = pytest.mark.gpu


def small_image_bf16():        # DiT-B/4 layout, T = 64, learned-Sigma head (C_out = 2C)
    return S.DIT_B4_BF16.with_(hidden=256, heads=4, mlp_hidden=1024, depth=2, batch=3, index=-1)


def small_video_bf16():        # velocity head (C_out = C), QK-RMSNorm + 3D RoPE, T = 48
    return S.VIDEO_RF.with_(hidden=288, heads=4, mlp_hidden=1152, depth=2, in_channels=4, frames=3, height=8, width=8,
                            batch=2, index=-1)


def small_video_f32():
    return S.VIDEO_RF.with_(dtype=S.DTYPE_F32, hidden=144, heads=2, mlp_hidden=576, depth=2, in_channels=4, frames=3,
                            height=8, width=6, batch=2, index=-1)


def rel_l2(got, want):
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


@pytest.mark.parametrize("kind,a,b", [(SM.DDIM, 0.3, 0.5), (SM.DDIM, 0.9, 0.2), (SM.DDIM, 0.6, 1.0),
                                      (SM.EULER, 0.0, 0.25), (SM.EULER, 0.8, 0.3)])
@pytest.mark.parametrize("offset", [0, 1], ids=["vector", "scalar"])
def test_sampler_step_matches_oracle(kind, a, b, offset):
    cfg = small_image_bf16()
    m = DiT(cfg, S.make_weights(cfg))
    rng = np.random.default_rng(11)
    B = cfg.batch
    x = rng.standard_normal(cfg.x_shape()).astype(np.float32)
    out = rng.standard_normal(cfg.out_shape()).astype(np.float32)
    want = SM.step(kind, x, out, a, b)
    # offset = 1 puts every buffer one float past a 16-byte boundary: the scalar path
    bx = torch.zeros(x.size + 4, device="cuda")
    bo = torch.zeros(out.size + 4, device="cuda")
    bn = torch.zeros(x.size + 4, device="cuda")
    dx = bx[offset:offset + x.size].view(x.shape)
    do = bo[offset:offset + out.size].view(out.shape)
    dn = bn[offset:offset + x.size].view(x.shape)
    dx.copy_(torch.from_numpy(x))
    do.copy_(torch.from_numpy(out))
    m.sampler_step(kind, dx, do, a, b, x_next=dn)
    got = dn.cpu().numpy()
    # fp32 arithmetic with coefficients rounded to fp32: a few ulps of |c0 x| + |c1 eps|
    assert np.abs(got - want).max() <= 4e-6 * (1.0 + np.abs(want).max())
    m.sampler_step(kind, dx, do, a, b, x_next=dx)          # in place
    assert np.array_equal(dx.cpu().numpy(), got)
    assert m.sync_status() == 0
    m.close()


@pytest.mark.parametrize("name,kind,model_t,levels,tol", [
    ("img_bf16", SM.DDIM, [700.0, 500.0, 300.0], [0.3, 0.5, 0.7, 0.9], 2e-2),
    ("video_bf16", SM.EULER, [0.1, 0.4, 0.7], [0.1, 0.4, 0.7, 1.0], 2e-2),
    ("video_f32", SM.EULER, [0.05, 0.5], [0.05, 0.5, 1.0], 1e-4),
])
def test_sample_loop_matches_oracle(name, kind, model_t, levels, tol):
    """Whole loop (forward + update per step) against the oracle loop around the oracle
    forward.  Each update is x' = c0 x + c1 pred with |c1| < 1 on these schedules, so the
    denoiser's per-step error enters the result scaled down: the forward's bar (rel-L2 2e-2
    for bf16, 1e-4 for fp32) is the bar for the final latent too."""
    cfg = {"img_bf16": small_image_bf16, "video_bf16": small_video_bf16, "video_f32": small_video_f32}[name]()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    Wd = S.weight_dict(cfg, W)
    s = cfg.cfg_scale

    def model(xv, tv):
        return O.forward(cfg, Wd, xv, np.full(cfg.batch, tv), inp["y"], cfg_scale=s)

    want = SM.sample(kind, model, inp["x"], model_t, levels)
    x = torch.from_numpy(np.ascontiguousarray(inp["x"])).cuda()
    y = torch.from_numpy(np.ascontiguousarray(inp["y"])).cuda()
    m.sample(kind, x, y, s, model_t, levels)
    got = x.cpu().numpy()
    assert m.sync_status() == 0
    assert rel_l2(got, want) <= tol, rel_l2(got, want)
    m.close()


def test_sample_graph_replay_matches_direct_loop():
    cfg = small_image_bf16()
    m = DiT(cfg, S.make_weights(cfg))
    inp = S.make_inputs(cfg)
    x0 = torch.from_numpy(np.ascontiguousarray(inp["x"])).cuda()
    y = torch.from_numpy(np.ascontiguousarray(inp["y"])).cuda()
    sched = ([900.0, 600.0, 300.0, 100.0], [0.05, 0.3, 0.6, 0.85, 0.97])
    x = x0.clone()
    m.sample(SM.DDIM, x, y, 1.5, *sched)
    want = x.cpu().numpy()
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    for _ in range(4):                       # direct, captured, replayed, replayed
        x.copy_(x0)
        m.sample(SM.DDIM, x, y, 1.5, *sched)
        assert np.array_equal(x.cpu().numpy(), want)
    # the model timesteps are uploaded every call: a new schedule of the same length replays
    x.copy_(x0)
    m.set_option(binding.DIT_OPT_USE_GRAPH, 0)
    m.sample(SM.DDIM, x, y, 1.5, [800.0, 500.0, 250.0, 50.0], sched[1])
    want2 = x.cpu().numpy()
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    x.copy_(x0)
    m.sample(SM.DDIM, x, y, 1.5, [800.0, 500.0, 250.0, 50.0], sched[1])
    assert np.array_equal(x.cpu().numpy(), want2)
    assert m.sync_status() == 0
    m.close()


def test_sampler_host_errors_launch_nothing():
    cfg = small_image_bf16()
    m = DiT(cfg, S.make_weights(cfg))
    x = torch.zeros(cfg.x_shape(), device="cuda")
    out = torch.zeros(cfg.out_shape(), device="cuda")
    y = torch.zeros(cfg.batch, dtype=torch.int32, device="cuda")
    for kind, a, b in [(7, 0.5, 0.6), (SM.DDIM, 0.0, 0.5), (SM.DDIM, 0.5, 1.5), (SM.EULER, float("nan"), 0.5)]:
        with pytest.raises(DitError) as e:
            m.sampler_step(kind, x, out, a, b, x_next=x)
        assert e.value.code == binding.DIT_ERR_INVALID_ARG
    with pytest.raises(DitError):
        m.sample(SM.DDIM, x, y, 1.5, [500.0], [0.5, 1.2])
    with pytest.raises(ValueError):
        m.sample(SM.DDIM, x, y, 1.5, [500.0, 100.0], [0.5, 0.9])
    assert float(x.abs().max()) == 0.0
    assert m.sync_status() == 0
    m.close()
