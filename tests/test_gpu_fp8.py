"""The FP8 (E4M3) linears on the tensor cores (tcgen05 kind::f8f6f4), GPU only: the
feed-forward (ffn_fp8) and the self-attention's in- and out-projection (attn_fp8).

The GEMM building block is checked against its definition on E4M3 operands (exact up to
float32 accumulation).  The forward with ffn_fp8 and / or attn_fp8 = 1 is checked against the
oracle's E4M3 linears (oracle.forward(..., ffn_fp8=..., attn_fp8=...)) with an FP8 tolerance,
derived here:
both sides quantise with the same rule, but from inputs that differ by the bf16 path's own
error (about 4e-3 relative, from the bf16 operands of every other matmul).  An E4M3 step is
2^-3 relative (2^-4 to the rounding boundary), so about 4e-3 / 2^-4 ~ 6% of the quantised
codes fall on the other side of a boundary and move by one step; each such move perturbs a
matmul output by ~sqrt(0.06) x 2^-3 / sqrt(3) ~ 2% relative, compounded over the blocks'
quantised matmuls (two, or four with both switches).  Hence rel-L2 <= 5e-2 and max|gpu - oracle| / std(oracle) <= 0.2,
about twice the observed worst case, against 2e-2 / 5e-2 for bf16.  The oracle's E4M3
linears themselves are pinned in tests/test_oracle_fp8_pins.py.
"""

FP8_REL = 5e-2
FP8_MAXN = 0.2


def assert_fp8_parity(got, want, what):
    assert got.shape == want.shape and np.all(np.isfinite(got)), what
    rel, maxn = metrics(got, want)
    assert rel <= FP8_REL and maxn <= FP8_MAXN, (what, rel, maxn)
    return rel, maxn
import numpy as np
import pytest
import torch

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding
from diffusion_transformer_denoiser_dit_b200.binding import DiT
from oracle import dit_oracle as O
from test_gpu_parity import dev, metrics, small_image_bf16_dh64, small_image_bf16_dh72, small_video_bf16

pytestmark = pytest.mark.gpu


def quantise(a):
    """Per-row E4M3 quantisation with torch: bytes and scales (amax / 448)."""
    s = a.abs().amax(dim=1).clamp_min(1e-30) / 448.0
    q = (a / s[:, None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), s.float()


@pytest.mark.parametrize("M,N,K,bn", [
    (128, 128, 128, 128), (300, 256, 1152, 256), (77, 64, 160, 64), (513, 1152, 4608, 128),
    (8192, 4608, 1152, 256), (1000, 192, 2304, 64),
])
def test_e4m3_linear_matches_definition(M, N, K, bn):
    g = torch.Generator(device="cuda").manual_seed(M + 3 * N + K)
    x = torch.randn(M, K, device="cuda", generator=g) * 2.0
    w = torch.randn(N, K, device="cuda", generator=g) * 0.05
    b = torch.randn(N, device="cuda", generator=g)
    x8, sx = quantise(x)
    w8, sw = quantise(w)
    y = binding.linear_e4m3(x8, w8, sx, sw, b, block_n=bn)
    torch.cuda.synchronize()
    xd = x8.view(torch.float8_e4m3fn).double().cpu().numpy() * sx.double().cpu().numpy()[:, None]
    wd = w8.view(torch.float8_e4m3fn).double().cpu().numpy() * sw.double().cpu().numpy()[:, None]
    ref = xd @ wd.T + b.double().cpu().numpy()
    err = np.abs(y.cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


FP8_CONFIGS = {
    "img_dh72": small_image_bf16_dh72,     # T = 225, guided
    "img_dh64": small_image_bf16_dh64,
    "video": small_video_bf16,             # QK-RMSNorm + 3D RoPE
}


@pytest.mark.parametrize("cname", list(FP8_CONFIGS))
@pytest.mark.parametrize("gates", ["random", "strong"])
def test_fp8_feed_forward_parity(cname, gates):
    cfg = FP8_CONFIGS[cname]().with_(ffn_fp8=1)
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], ffn_fp8=True)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert_fp8_parity(got, want, f"fp8 {cname} {gates}")
    m.close()


def test_fp8_residual_per_block_and_conditioning_designs():
    cfg = small_image_bf16_dh72().with_(ffn_fp8=1)
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    for k in range(cfg.depth + 1):
        got = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, k).cpu().numpy()
        want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=k, ffn_fp8=True)
        assert_fp8_parity(got, want, f"fp8 after block {k}")
    m.close()
    for kind in (S.BLOCK_IN_CONTEXT, S.BLOCK_CROSS_ATTN):
        c2 = cfg.with_(block_kind=kind)
        W2 = S.make_weights(c2)
        want = O.forward(c2, W2, inp["x"], inp["t"], inp["y"], ffn_fp8=True)
        m = DiT(c2, W2)
        got = m.forward(d["x"], d["t"], d["y"], c2.cfg_scale).cpu().numpy()
        assert m.sync_status() == binding.DIT_OK
        assert_fp8_parity(got, want, f"fp8 block kind {kind}")
        m.close()


def test_fp8_full_size_sample():
    """DiT-XL/2 with guidance at 256px with the FP8 feed-forward: the last sample against the
    FP8 oracle; the distance to the exact forward stays within a few percent."""
    cfg = S.DIT_XL2_CFG256.with_(ffn_fp8=1)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    m.close()
    b = cfg.batch - 1
    Wd = S.weight_dict(cfg, W)
    sl = slice(b, b + 1)
    want = O.forward(cfg, Wd, inp["x"][sl], inp["t"][sl], inp["y"][sl], ffn_fp8=True)
    assert_fp8_parity(got[sl], want, "fp8 XL/2 256px")
    exact = O.forward(cfg, Wd, inp["x"][sl], inp["t"][sl], inp["y"][sl])
    assert metrics(got[sl], exact)[0] < 5e-2


@pytest.mark.parametrize("cname", list(FP8_CONFIGS))
@pytest.mark.parametrize("gates", ["random", "strong"])
def test_fp8_attention_projection_parity(cname, gates):
    """attn_fp8: E4M3 in-projection (swapped scatter for images, whole-head epilogue with
    QK-RMSNorm and RoPE for video), bf16 attention, per-token E4M3 of the heads' output and
    the E4M3 out-projection into the float32 stream."""
    cfg = FP8_CONFIGS[cname]().with_(attn_fp8=1)
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], attn_fp8=True)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert_fp8_parity(got, want, f"attn fp8 {cname} {gates}")
    m.close()


@pytest.mark.parametrize("cname", ["img_dh72", "video"])
def test_fp8_all_four_linears_parity(cname):
    cfg = FP8_CONFIGS[cname]().with_(attn_fp8=1, ffn_fp8=1)
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], attn_fp8=True, ffn_fp8=True)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert_fp8_parity(got, want, f"all fp8 {cname}")
    m.close()


def test_fp8_attention_per_block_and_conditioning_designs():
    cfg = small_image_bf16_dh72().with_(attn_fp8=1)
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    for k in range(cfg.depth + 1):
        got = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, k).cpu().numpy()
        want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=k, attn_fp8=True)
        assert_fp8_parity(got, want, f"attn fp8 after block {k}")
    m.close()
    for kind in (S.BLOCK_IN_CONTEXT, S.BLOCK_CROSS_ATTN, S.BLOCK_ADALN):
        c2 = cfg.with_(block_kind=kind)
        W2 = S.make_weights(c2)
        want = O.forward(c2, W2, inp["x"], inp["t"], inp["y"], attn_fp8=True)
        m = DiT(c2, W2)
        got = m.forward(d["x"], d["t"], d["y"], c2.cfg_scale).cpu().numpy()
        assert m.sync_status() == binding.DIT_OK
        assert_fp8_parity(got, want, f"attn fp8 block kind {kind}")
        m.close()


def test_fp8_all_linears_full_size_sample():
    """DiT-XL/2 with guidance at 256px with all four block linears in E4M3: the last sample
    against the FP8 oracle; the distance to the exact forward stays within a few percent."""
    cfg = S.DIT_XL2_CFG256.with_(ffn_fp8=1, attn_fp8=1)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    m.close()
    b = cfg.batch - 1
    Wd = S.weight_dict(cfg, W)
    sl = slice(b, b + 1)
    want = O.forward(cfg, Wd, inp["x"][sl], inp["t"][sl], inp["y"][sl], ffn_fp8=True, attn_fp8=True)
    assert_fp8_parity(got[sl], want, "all fp8 XL/2 256px")
    exact = O.forward(cfg, Wd, inp["x"][sl], inp["t"][sl], inp["y"][sl])
    assert metrics(got[sl], exact)[0] < 6e-2
