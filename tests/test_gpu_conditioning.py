"""The four conditioning designs of "확산 트랜스포머" (itwiki.kr), section "조건 주입 방식":
in-context tokens, cross-attention, adaLN and adaLN-Zero, on the GPU through the C ABI against
the oracle (GPU only).  Same tolerances as the adaLN-Zero parity tests.
"""
import numpy as np
import pytest
import torch

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding
from diffusion_transformer_denoiser_dit_b200.binding import DiT
from oracle import dit_oracle as O
from test_gpu_parity import assert_parity, dev, small_image_bf16_dh64, small_image_bf16_dh72, small_video_bf16, \
    small_video_f32

pytestmark = pytest.mark.gpu

KINDS = {"in_context": S.BLOCK_IN_CONTEXT, "cross_attn": S.BLOCK_CROSS_ATTN, "adaln": S.BLOCK_ADALN}
CONFIGS = {
    "img_bf16_dh72": small_image_bf16_dh72,      # T = 225 (+2 in context), guided
    "img_bf16_dh64": small_image_bf16_dh64,      # T = 64, unguided
    "video_bf16": small_video_bf16,              # QK-RMSNorm + 3D RoPE, text vector
    "s8_f32": lambda: S.DIT_S8_F32.with_(depth=3),
    "video_f32": small_video_f32,
}


@pytest.mark.parametrize("cname", list(CONFIGS))
@pytest.mark.parametrize("kname", list(KINDS))
def test_conditioning_design_parity(kname, cname):
    cfg = CONFIGS[cname]().with_(block_kind=KINDS[kname])
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert_parity(cfg, got, want, f"{kname} {cname}")
    m.close()


@pytest.mark.parametrize("kname", ["in_context", "cross_attn"])
@pytest.mark.parametrize("cname", ["img_bf16_dh72", "video_bf16", "video_f32"])
def test_conditioning_design_residual_per_block(kname, cname):
    """The residual stream after every block (in context: T + 2 tokens per row, the two
    condition tokens first) against the oracle."""
    cfg = CONFIGS[cname]().with_(block_kind=KINDS[kname])
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    for k in range(cfg.depth + 1):
        got = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, k).cpu().numpy()
        want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=k)
        assert got.shape == want.shape == (got.shape[0], cfg.seq_tokens, cfg.hidden)
        assert_parity(cfg, got, want, f"{kname} {cname} after block {k}")
    m.close()


@pytest.mark.parametrize("kname", list(KINDS))
def test_conditioning_design_graph_replay_and_launch_count(kname):
    """Graph replay is bit-identical to direct launches, and the library's launch count is
    the number of graph nodes."""
    cfg = small_image_bf16_dh72().with_(block_kind=KINDS[kname])
    m = DiT(cfg, S.make_weights(cfg))
    d = dev(S.make_inputs(cfg))
    want = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    m.profile(True)
    m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale)
    m.profile(False)
    recs = sum(v[1] for v in m.profile_read().values())
    n = m.launch_count(cfg.batch, cfg.cfg_scale)
    assert recs <= n <= recs + 2   # the condition record covers its three kernels
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    out = torch.empty(cfg.out_shape(), device="cuda")
    for _ in range(3):
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out)
    assert np.array_equal(out.cpu().numpy(), want)
    m.close()


@pytest.mark.parametrize("kname", ["in_context", "cross_attn"])
def test_conditioning_design_full_size_sample(kname):
    """DiT-XL/2 with guidance at 256px (32 rows; in context 258 tokens per row, a ragged third
    key tile): the last sample against the oracle, every sample against a one-sample forward."""
    cfg = S.DIT_XL2_CFG256.with_(block_kind=KINDS[kname])
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    for b in (0, cfg.batch // 2):
        one = m.forward(d["x"][b:b + 1].contiguous(), d["t"][b:b + 1].contiguous(), d["y"][b:b + 1].contiguous(),
                        cfg.cfg_scale).cpu().numpy()
        rel = np.linalg.norm(one[0] - got[b]) / np.linalg.norm(got[b])
        assert rel < 1e-5, (b, rel)
    m.close()
    b = cfg.batch - 1
    want = O.forward(cfg, S.weight_dict(cfg, W), inp["x"][b:b + 1], inp["t"][b:b + 1], inp["y"][b:b + 1])
    assert_parity(cfg, got[b:b + 1], want, f"{kname} XL/2 sample {b}")
