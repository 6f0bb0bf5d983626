"""CUDA path vs the CPU oracle, through the C ABI (GPU only).

Tolerances (from the workload definition): float32 path relative L2 <= 1e-4;
bf16 path relative L2 <= 2e-2 and max|gpu - oracle| / std(oracle) <= 5e-2.
"""
import numpy as np
import pytest
import torch

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding
from diffusion_transformer_denoiser_dit_b200.binding import DiT
from oracle import dit_oracle as O

pytestmark = pytest.mark.gpu

F32_REL = 1e-4
BF16_REL = 2e-2
BF16_MAXN = 5e-2


def metrics(got, want):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    maxn = np.abs(got - want).max() / want.std()
    return rel, maxn


def assert_parity(cfg, got, want, what=""):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    rel, maxn = metrics(got, want)
    if cfg.dtype == S.DTYPE_F32:
        assert rel <= F32_REL, (what, rel, maxn)
    else:
        assert rel <= BF16_REL and maxn <= BF16_MAXN, (what, rel, maxn)
    return rel, maxn


def dev(inp):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}


# ----------------------------------------------------------------------------- configs
def small_video_f32():
    return S.VIDEO_RF.with_(dtype=S.DTYPE_F32, hidden=144, heads=2, mlp_hidden=576, depth=2, in_channels=4, frames=3,
                            height=8, width=6, batch=2, index=-1)


def small_image_bf16_dh72():   # T = 225 (ragged), 6 rows with guidance, M = 1350
    return S.DIT_XL2_CFG256.with_(hidden=288, heads=4, mlp_hidden=1152, depth=2, height=30, width=30, batch=3,
                                  index=-1)


def small_image_bf16_dh64():   # T = 64, M = 320, no guidance
    return S.DIT_B4_BF16.with_(hidden=256, heads=4, mlp_hidden=1024, depth=2, batch=5, index=-1)


def small_video_bf16():        # T = 48, QK-RMSNorm + 3D RoPE
    return S.VIDEO_RF.with_(hidden=288, heads=4, mlp_hidden=1152, depth=2, in_channels=4, frames=3, height=8, width=8,
                            batch=2, index=-1)


def small_image_bf16_dh64_ragged():   # dh 64, T = 225 (two key tiles, ragged), 6 guided rows
    return S.DIT_XL2_CFG256.with_(hidden=256, heads=4, mlp_hidden=1024, depth=2, height=30, width=30, batch=3,
                                  index=-1)


SMALL = {
    "s8_f32": lambda: S.DIT_S8_F32,
    "video_f32": small_video_f32,
    "img_bf16_dh72": small_image_bf16_dh72,
    "img_bf16_dh64": small_image_bf16_dh64,
    "img_bf16_dh64_ragged": small_image_bf16_dh64_ragged,
    "video_bf16": small_video_bf16,
    "b4_bf16_full": lambda: S.DIT_B4_BF16,
}


# ----------------------------------------------------------------------------- GEMM building block
@pytest.mark.parametrize("M,N,K,bn", [
    (128, 128, 64, 128), (300, 144, 1152, 144), (77, 50, 72, 64), (1000, 192, 200, 192),
    (513, 256, 4608, 256), (64, 16, 1152, 16), (200, 32, 1152, 32), (8192, 3456, 1152, 144),
])
def test_tcgen05_linear_matches_definition(M, N, K, bn):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N)
    x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    b = torch.randn(N, device="cuda", generator=g)
    y = binding.linear_bf16(x, w, b, block_n=bn)
    torch.cuda.synchronize()
    ref = x.double().cpu().numpy() @ w.double().cpu().numpy().T + b.double().cpu().numpy()
    err = np.abs(y.cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


@pytest.mark.parametrize("M,N,K,bn", [
    (256, 128, 64, 128), (300, 144, 1152, 144), (77, 64, 72, 64), (1000, 192, 200, 192),
    (513, 256, 4608, 256), (8192, 3456, 1152, 144), (8192, 1152, 4608, 128), (8192, 4608, 1152, 256),
])
def test_tcgen05_pair_linear_matches_definition(M, N, K, bn):
    g = torch.Generator(device="cuda").manual_seed(M * 11 + N)
    x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    b = torch.randn(N, device="cuda", generator=g)
    y = binding.linear_bf16(x, w, b, block_n=bn, pair=True)
    torch.cuda.synchronize()
    ref = x.double().cpu().numpy() @ w.double().cpu().numpy().T + b.double().cpu().numpy()
    err = np.abs(y.cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


# ----------------------------------------------------------------------------- end to end
@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("gates", ["random", "strong"])
def test_forward_parity(name, gates):
    cfg = SMALL[name]()
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale)
    assert m.sync_status() == binding.DIT_OK
    assert_parity(cfg, got.cpu().numpy(), want, name)
    m.close()


@pytest.mark.parametrize("name", ["s8_f32", "img_bf16_dh72", "img_bf16_dh64_ragged", "video_bf16", "video_f32"])
def test_residual_stream_parity_per_block(name):
    cfg = SMALL[name]()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    for k in range(cfg.depth + 1):
        got = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, k).cpu().numpy()
        want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=k)
        assert_parity(cfg, got, want, f"{name} after block {k}")
    m.close()


def test_condition_vector_parity():
    cfg = small_image_bf16_dh72()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    c = m.debug_condition(d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    yy = np.concatenate([inp["y"], np.full(cfg.batch, cfg.num_classes)])
    tt = np.concatenate([inp["t"], inp["t"]])
    want = O.condition(cfg, S.weight_dict(cfg, W), tt, yy)
    assert np.abs(c - want).max() / np.abs(want).max() < 1e-5
    m.close()


def test_zero_adaln_blocks_are_identity_on_gpu():
    cfg = small_image_bf16_dh72()
    W = S.set_adaln(cfg, S.make_weights(cfg), zero=True)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    h0 = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, 0).cpu()
    hN = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, cfg.depth).cpu()
    assert torch.equal(h0, hN)
    m.close()


def test_guidance_special_cases_on_gpu():
    cfg = small_image_bf16_dh72()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    null = torch.full_like(d["y"], cfg.num_classes)
    cond = m.forward(d["x"], d["t"], d["y"], 1.0).cpu().numpy()
    uncond = m.forward(d["x"], d["t"], null, 1.0).cpu().numpy()
    s0 = m.forward(d["x"], d["t"], d["y"], 0.0).cpu().numpy()
    s15 = m.forward(d["x"], d["t"], d["y"], 1.5).cpu().numpy()
    assert metrics(s0, uncond)[0] < 1e-5
    assert metrics(s15, uncond + 1.5 * (cond - uncond))[0] < 1e-4
    m.set_option(binding.DIT_OPT_FORCE_GUIDANCE, 1)
    s1 = m.forward(d["x"], d["t"], d["y"], 1.0).cpu().numpy()
    assert metrics(s1, cond)[0] < 1e-5
    m.close()


def test_host_entry_point_matches_device_entry_point():
    cfg = small_image_bf16_dh64()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    a = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    b = m.forward_host(inp["x"], inp["t"], inp["y"], cfg.cfg_scale)
    assert np.array_equal(a, b)
    m.close()


@pytest.mark.parametrize("name", ["img_bf16_dh72", "video_f32"])
def test_graph_replay_matches_direct_launches(name):
    """DIT_OPT_USE_GRAPH: first call direct, second captured, third replayed; a new
    output buffer starts over.  Same kernels on the same inputs: bit-identical results."""
    cfg = SMALL[name]()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    want = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    out = torch.empty(cfg.out_shape(), device="cuda")
    for _ in range(4):
        out.fill_(float("nan"))
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out)
        assert np.array_equal(out.cpu().numpy(), want)
    out2 = torch.empty(cfg.out_shape(), device="cuda")
    for _ in range(3):
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out2)
        assert np.array_equal(out2.cpu().numpy(), want)
    # new inputs in the same buffers are picked up by the replayed graph
    d["x"].mul_(0.5).add_(0.25)
    m.set_option(binding.DIT_OPT_USE_GRAPH, 0)
    want2 = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out2)
    assert np.array_equal(out2.cpu().numpy(), want2)
    assert m.sync_status() == 0
    m.close()


def test_batch_smaller_than_max_and_rows_independent():
    cfg = small_image_bf16_dh72()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W, max_batch=cfg.batch)
    d = dev(inp)
    full = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    one = m.forward(d["x"][1:2].contiguous(), d["t"][1:2].contiguous(), d["y"][1:2].contiguous(),
                    cfg.cfg_scale).cpu().numpy()
    assert metrics(one[0], full[1])[0] < 1e-5
    m.close()


def test_bad_label_is_reported_and_clamped():
    cfg = small_image_bf16_dh64()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    inp["y"][0] = 5000
    m = DiT(cfg, W)
    d = dev(inp)
    out = m.forward(d["x"], d["t"], d["y"], 1.0)
    assert m.sync_status() == binding.DIT_ERR_BAD_LABEL
    assert torch.isfinite(out).all()
    assert m.sync_status() == binding.DIT_OK   # cleared by the read


def test_bounded_wait_times_out_and_context_survives():
    cfg = small_image_bf16_dh64()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    m.wait_probe(2000)   # 2 ms on a flag nothing sets
    assert m.sync_status() == binding.DIT_ERR_DEVICE_TIMEOUT
    d = dev(inp)
    out = m.forward(d["x"], d["t"], d["y"], 1.0)
    assert m.sync_status() == binding.DIT_OK
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    assert_parity(cfg, out.cpu().numpy(), want, "after timeout")
    m.close()


def test_host_side_errors_launch_nothing():
    cfg = small_image_bf16_dh64()
    m = DiT(cfg, S.make_weights(cfg))
    d = dev(S.make_inputs(cfg, batch=cfg.batch + 1))
    with pytest.raises(binding.DitError) as e:
        m.forward(d["x"], d["t"], d["y"], 1.0)
    assert e.value.code == binding.DIT_ERR_INVALID_ARG
    m.close()


def tie_keys_to_queries(cfg, W, f):
    """Copy of W whose key projections equal the query projections scaled by f (and the
    query projections scaled by f): every logit q_i . q_j then peaks on its own token, far
    above the first key tile's best, so the attention's running maximum must move."""
    W = [w.copy() for w in W]
    names = [n for n, _, _ in S.weight_specs(cfg)]
    d = cfg.hidden
    for i in range(cfg.depth):
        w, b = W[names.index(f"blocks.{i}.qkv.w")], W[names.index(f"blocks.{i}.qkv.b")]
        w[:d] *= f
        b[:d] *= f
        w[d:2 * d] = w[:d]
        b[d:2 * d] = b[:d]
    return W


def test_attention_rescale_path_in_the_forward():
    """A model whose logits span far more than 2^8 across key tiles (T = 576, five key
    tiles): the forward's attention takes its rescale path (read back through the handle's
    counter) and still matches the oracle, per block and at the output."""
    cfg = small_image_bf16_dh72().with_(height=48, width=48, batch=2)
    W = tie_keys_to_queries(cfg, S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0), 8.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    assert m.attention_rescales() == 0
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    events = m.attention_rescales()
    assert events > 0
    assert_parity(cfg, got, O.forward(cfg, W, inp["x"], inp["t"], inp["y"]), "rescale forward")
    h1 = m.debug_residual(d["x"], d["t"], d["y"], cfg.cfg_scale, 1).cpu().numpy()
    assert_parity(cfg, h1, O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=1), "after block 1")
    # the standard weights never take that path
    m.close()
    m = DiT(cfg, S.make_weights(cfg))
    m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale)
    assert m.attention_rescales() == 0
    m.close()


# ----------------------------------------------------------------------------- full-size workloads
# The benchmark's launch configuration (standard weights/inputs, full batch) on the GPU;
# the oracle recomputes one sampled sample (rows of a batch are independent, so sample
# b of the batched GPU output must equal the oracle run on sample b alone).
FULL = [S.DIT_XL2_CFG256, S.DIT_XL2_CFG512, S.VIDEO_RF]
FULL_IDS = ["xl2_cfg256", "xl2_cfg512", "video_rf"]


@pytest.mark.parametrize("cfg", FULL, ids=FULL_IDS)
@pytest.mark.parametrize("gates", ["random", "strong"])
def test_full_size_sampled_parity(cfg, gates):
    """Standard weights: the last sample (its guided partner is the batch's last row).
    Gate biases 1.0, so every block moves the residual stream strongly: the first and the
    last sample.  Every other sample is checked against a single-sample GPU forward."""
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert got.shape == cfg.out_shape() and np.all(np.isfinite(got))
    # rows are independent: each sample of the batched forward equals the same sample alone
    for b in range(cfg.batch):
        one = m.forward(d["x"][b:b + 1].contiguous(), d["t"][b:b + 1].contiguous(), d["y"][b:b + 1].contiguous(),
                        cfg.cfg_scale).cpu().numpy()
        assert metrics(one[0], got[b])[0] < 1e-5, b
    m.close()
    Wd = S.weight_dict(cfg, W)
    for b in ([cfg.batch - 1] if gates == "random" else [0, cfg.batch - 1]):
        want = O.forward(cfg, Wd, inp["x"][b:b + 1], inp["t"][b:b + 1], inp["y"][b:b + 1])
        assert_parity(cfg, got[b:b + 1], want, f"{cfg.name} sample {b} {gates} gates")


# ----------------------------------------------------------------------------- edge shapes
EDGE = {
    # no blocks at all: the forward is the final layer of the embedding
    "depth0_bf16": lambda: small_image_bf16_dh72().with_(depth=0),
    "depth0_f32": lambda: small_video_f32().with_(depth=0),
    # one token per row: softmax over a single key is 1, attention returns V
    "one_token_bf16": lambda: small_image_bf16_dh64().with_(height=4, width=4),
    "one_token_guided_dh72": lambda: small_image_bf16_dh72().with_(height=2, width=2),
    # the widest supported models for each head dim (hidden <= 1536)
    "widest_dh64": lambda: small_image_bf16_dh64().with_(hidden=1536, heads=24, mlp_hidden=6144, depth=1, batch=2),
    "widest_dh72": lambda: small_image_bf16_dh72().with_(hidden=1440, heads=20, mlp_hidden=5760, depth=1, height=16,
                                                         width=16, batch=2),
    # a single sample
    "batch1_video": lambda: small_video_bf16().with_(batch=1),
    # dh 64 over eight key tiles (T = 1024), guided
    "dh64_T1024": lambda: small_image_bf16_dh64_ragged().with_(height=64, width=64, depth=1, batch=1),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_edge_shape_parity(name):
    cfg = EDGE[name]()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    m = DiT(cfg, W)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale)
    assert m.sync_status() == binding.DIT_OK
    assert_parity(cfg, got.cpu().numpy(), want, name)
    m.close()


def test_empty_batch_is_rejected_without_launch():
    cfg = small_image_bf16_dh64()
    m = DiT(cfg, S.make_weights(cfg))
    d = dev(S.make_inputs(cfg, batch=1))
    out = torch.full((8,), 7.0, device="cuda")
    rc = m.lib.dit_forward(m.h, d["x"].data_ptr(), d["t"].data_ptr(), d["y"].data_ptr(), 0, 1.0, out.data_ptr(), None)
    assert rc == binding.DIT_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    assert m.sync_status() == binding.DIT_OK
    m.close()


def test_guidance_on_the_first_channels_only():
    """DIT_OPT_CFG_CHANNELS = 3 against the oracle's cfg_channels = 3; the option is part of
    the graph cache key, so replay picks up a change."""
    cfg = small_image_bf16_dh72()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    want = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], cfg_channels=3)
    m = DiT(cfg, W)
    d = dev(inp)
    m.set_option(binding.DIT_OPT_CFG_CHANNELS, 3)
    direct = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert_parity(cfg, direct, want, "cfg_channels=3")
    m.set_option(binding.DIT_OPT_CFG_CHANNELS, 0)
    full = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert np.array_equal(full[:, :3], direct[:, :3]) and not np.array_equal(full[:, 3:], direct[:, 3:])
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    out = torch.empty(cfg.out_shape(), device="cuda")
    for _ in range(3):
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out)
    assert np.array_equal(out.cpu().numpy(), full)
    m.set_option(binding.DIT_OPT_CFG_CHANNELS, 3)
    for _ in range(3):
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out)
        assert np.array_equal(out.cpu().numpy(), direct)
    with pytest.raises(binding.DitError):
        m.set_option(binding.DIT_OPT_CFG_CHANNELS, -1)
    assert m.sync_status() == binding.DIT_OK
    m.close()


def test_split_k_residual_gemms_match_unsplit():
    """DIT_OPT_SPLIT_K: the out-projection's K slices each add their share into the residual
    stream; any split gives the unsplit result up to float32 summation order, and parity.
    A reordered float32 sum can flip the bf16 rounding of a later activation (2^-9 relative),
    so two splits agree to about 1e-3, not to float32 precision."""
    cfg = small_image_bf16_dh72()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    d = dev(inp)
    outs = {}
    for sk in (1, 2, 3, 8):
        m.set_option(binding.DIT_OPT_SPLIT_K, sk)
        outs[sk] = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    for sk in (2, 3, 8):
        assert metrics(outs[sk], outs[1])[0] < 5e-3, sk
    assert_parity(cfg, outs[2], O.forward(cfg, W, inp["x"], inp["t"], inp["y"]), "split-K 2")
    with pytest.raises(binding.DitError):
        m.set_option(binding.DIT_OPT_SPLIT_K, 0)
    m.close()


@pytest.mark.parametrize("name", ["img_bf16_dh72", "b4_bf16_full", "video_bf16", "img_bf16_dh64_ragged"])
def test_pair_gemm_forward_parity(name):
    """DIT_OPT_PAIR_GEMM: the block GEMMs on SM pairs (cta_group::2, 256-row tiles, ragged
    token counts included) match the oracle, and graph replay of that forward is bit-identical."""
    cfg = SMALL[name]()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    m = DiT(cfg, W)
    m.set_option(binding.DIT_OPT_PAIR_GEMM, 1)
    d = dev(inp)
    got = m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale).cpu().numpy()
    assert m.sync_status() == binding.DIT_OK
    assert_parity(cfg, got, O.forward(cfg, W, inp["x"], inp["t"], inp["y"]), f"pair {name}")
    m.set_option(binding.DIT_OPT_USE_GRAPH, 1)
    out = torch.empty(cfg.out_shape(), device="cuda")
    for _ in range(3):
        m.forward(d["x"], d["t"], d["y"], cfg.cfg_scale, out=out)
    assert np.array_equal(out.cpu().numpy(), got)
    m.close()
