"""Pins of the CPU oracle to things other than itself (CPU only).

Each test fixes a part of the oracle against a value printed on the pages
(tests/golden/*.txt), a closed form, an invariant, a special case that reduces to
a stock library routine, or brute force on a tiny input.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import dit_synth as S
from oracle import dit_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(fname):
    with open(os.path.join(GOLDEN, fname)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def small_image(**kw):
    base = S.DIT_S8_F32.with_(depth=2, hidden=96, heads=4, mlp_hidden=384, num_classes=10,
                              height=16, width=16, patch_h=4, patch_w=4, batch=2, index=-1)
    return base.with_(**kw)


def small_video(**kw):
    base = S.VIDEO_RF.with_(depth=2, hidden=72, heads=2, mlp_hidden=288, in_channels=3, frames=3,
                            height=8, width=6, patch_t=1, patch_h=2, patch_w=2, batch=2, index=-1)
    return base.with_(**kw)


# ----------------------------------------------------------------------------- shapes / FLOPs
def test_token_count_and_decoder_width():
    for side, ch, p, tokens, width in (map(int, r) for r in _rows("shapes.txt")):
        cfg = S.DIT_XL2_CFG256.with_(height=side, width=side, in_channels=ch, patch_h=p, patch_w=p)
        assert cfg.tokens == tokens
        assert cfg.out_dim == width
        x = np.zeros((1, ch, 1, side, side))
        assert O.patchify(x, 1, p, p).shape == (1, tokens, ch * p * p)


@pytest.mark.parametrize("row", _rows("gflops_table.txt"))
def test_mac_counter_reproduces_printed_gflops(row):
    size, depth, hidden, heads, patch, side, printed = row
    cfg = S.DIT_XL2_CFG256.with_(depth=int(depth), hidden=int(hidden), heads=int(heads),
                                 mlp_hidden=4 * int(hidden), patch_h=int(patch), patch_w=int(patch),
                                 height=int(side), width=int(side))
    g = O.count_forward_macs(cfg) / 1e9
    assert abs(g - float(printed)) <= 0.1, (size, g, printed)


@pytest.mark.parametrize("row", _rows("gflops_conditioning.txt"))
def test_mac_counter_reproduces_conditioning_table(row):
    """The four conditioning designs' printed DiT-XL/2 Gflops: in-context adds two tokens to
    every row, cross-attention adds a query and an output projection per token and block, and
    neither keeps the per-block modulation MLP (with it, 119.58 and 137.83 would be off)."""
    name, kind, printed = row
    cfg = S.DIT_XL2_CFG256.with_(block_kind=int(kind))
    g = O.count_forward_macs(cfg) / 1e9
    assert abs(g - float(printed)) <= 0.1, (name, g, printed)


def test_mac_counter_range_ends():
    rng = dict((r[0], float(r[1])) for r in _rows("gflops_range.txt"))
    low = O.count_forward_macs(S.DIT_S8_F32) / 1e9
    high = O.count_forward_macs(S.DIT_XL2_CFG256) / 1e9
    assert math.floor(low * 10) / 10 == rng["low"]
    assert abs(high - rng["high"]) < 0.05


def test_mac_counter_dry_equals_real():
    cfg = small_image()
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg, batch=1)
    O.reset_mac_counter()
    O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    real = O.mac_count()
    assert real == O.count_forward_macs(cfg)
    assert real > 0


# ----------------------------------------------------------------------------- elementwise
def test_layernorm_moments_and_library():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7, 96)) * 3 + 1.5
    y = O.layernorm(x)
    assert np.allclose(y.mean(-1), 0, atol=1e-12)
    assert np.allclose(y.var(-1), 1, atol=1e-5)  # eps 1e-6 shrinks var by ~eps/var
    ref = F.layer_norm(torch.from_numpy(x), (96,), eps=1e-6).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # constant row -> zeros (eps keeps it finite)
    assert np.all(O.layernorm(np.full((1, 8), 3.0)) == 0)


def test_rmsnorm_unit_rms_and_library():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 72)) * 5
    g = rng.standard_normal(72)
    assert np.allclose(np.sqrt((O.rmsnorm(x, np.ones(72)) ** 2).mean(-1)), 1, atol=1e-6)
    ref = F.rms_norm(torch.from_numpy(x), (72,), torch.from_numpy(g), eps=1e-6).numpy()
    assert np.allclose(O.rmsnorm(x, g), ref, rtol=1e-12, atol=1e-12)


def test_gelu_silu_library_and_special_values():
    x = np.linspace(-8, 8, 1001)
    assert np.allclose(O.gelu_tanh(x), F.gelu(torch.from_numpy(x), approximate="tanh").numpy(),
                       rtol=1e-13, atol=1e-13)
    assert np.allclose(O.silu(x), F.silu(torch.from_numpy(x)).numpy(), rtol=1e-13, atol=1e-13)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu_tanh(np.array([20.0]))[0] - 20.0) < 1e-12
    assert abs(O.gelu_tanh(np.array([-20.0]))[0]) < 1e-12


def test_modulate_identity_at_zero():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 3, 8))
    z = np.zeros((2, 8))
    assert np.array_equal(O.modulate(x, z, z), x)
    sh = rng.standard_normal((2, 8))
    out = O.modulate(x, sh, z)
    assert np.allclose(out - x, np.broadcast_to(sh[:, None], x.shape))


# ----------------------------------------------------------------------------- attention
def test_attention_two_token_closed_form():
    # q0 = (1,0) sees logits (1/sqrt2, 0): weight on key 0 is sigmoid(1/sqrt2);
    # q1 = 0 sees equal logits: the mean of the values.
    q = np.array([[1.0, 0.0], [0.0, 0.0]])
    k = np.array([[1.0, 0.0], [0.0, 1.0]])
    v = np.array([[1.0, 2.0], [3.0, 4.0]])
    w0 = 1.0 / (1.0 + math.exp(-1.0 / math.sqrt(2.0)))
    want = np.array([w0 * v[0] + (1 - w0) * v[1], (v[0] + v[1]) / 2])
    assert np.allclose(O.attention(q, k, v), want, rtol=1e-14, atol=1e-14)


def test_attention_zero_query_is_mean_and_library():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((9, 6)) for _ in range(3))
    assert np.allclose(O.attention(np.zeros_like(q), k, v), np.broadcast_to(v.mean(0), v.shape))
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a)[None] for a in (q, k, v)))[0].numpy()
    assert np.allclose(O.attention(q, k, v), ref, rtol=1e-12, atol=1e-12)


def test_attention_brute_force_tiny():
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((3, 4)) for _ in range(3))
    out = np.zeros((3, 4))
    for i in range(3):
        e = [math.exp(sum(q[i, a] * k[j, a] for a in range(4)) / 2.0) for j in range(3)]
        z = sum(e)
        for a in range(4):
            out[i, a] = sum(e[j] / z * v[j, a] for j in range(3))
    assert np.allclose(O.attention(q, k, v), out, rtol=1e-13, atol=1e-13)


def test_attention_permutation():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((7, 5)) for _ in range(3))
    p = rng.permutation(7)
    base = O.attention(q, k, v)
    assert np.allclose(O.attention(q, k[p], v[p]), base)   # keys/values: invariant
    assert np.allclose(O.attention(q[p], k, v), base[p])   # queries: equivariant


# ----------------------------------------------------------------------------- embeddings
def test_timestep_embedding_invariants():
    e = O.timestep_embedding(np.array([0.0, 1.0, 999.0]), 256)
    assert e.shape == (3, 256)
    assert np.all(e[0, :128] == 1) and np.all(e[0, 128:] == 0)      # t = 0
    assert np.allclose(e[:, :128] ** 2 + e[:, 128:] ** 2, 1)         # cos^2 + sin^2
    assert np.allclose((e ** 2).sum(1), 128)                         # |e|^2 = dim/2
    assert abs(e[1, 0] - math.cos(1.0)) < 1e-15 and abs(e[1, 128] - math.sin(1.0)) < 1e-15  # f_0 = 1
    assert abs(math.acos(e[1, 127]) - 10000 ** (-127 / 128)) < 1e-12  # slowest frequency
    e2 = O.timestep_embedding(np.array([0.5]), 256, t_scale=1000.0)
    assert np.allclose(e2, O.timestep_embedding(np.array([500.0]), 256))


def test_sincos_2d_invariants():
    d, gh, gw = 96, 3, 5
    pe = O.pos_embed_sincos_2d(gh, gw, d)
    assert pe.shape == (gh * gw, d)
    q = d // 4
    first = pe[0]
    assert np.all(first[:q] == 0) and np.all(first[q:2 * q] == 1)
    assert np.all(first[2 * q:3 * q] == 0) and np.all(first[3 * q:] == 1)
    assert np.allclose((pe ** 2).sum(1), d / 2)
    tok = lambda r, c: r * gw + c
    assert np.array_equal(pe[tok(2, 1), :d // 2], pe[tok(2, 4), :d // 2])   # same row
    assert np.array_equal(pe[tok(0, 3), d // 2:], pe[tok(2, 3), d // 2:])   # same column
    assert abs(pe[tok(0, 1), d // 2] - math.sin(1.0)) < 1e-15               # w_0 = 1


def test_token_coords_follow_the_patchify_token_order():
    """Each token's (frame, row, col) on the patch grid, fixed by the tokenisation itself: a
    latent whose channels hold each element's own frame, row and column index is patchified
    (patchify is pinned to a Conv3d with kernel = stride = patch below), and token tau's patch
    must start at (frame, row, col) = patch extent x token_coords(tau)."""
    for (pt, ph, pw), (F_, H, W) in (((1, 2, 2), (3, 8, 6)), ((2, 1, 3), (4, 5, 9)), ((1, 4, 4), (1, 16, 8))):
        f, i, j = np.meshgrid(np.arange(F_), np.arange(H), np.arange(W), indexing="ij")
        x = np.stack([f, i, j]).astype(np.float64)[None]          # [1, 3, F, H, W]
        v = O.patchify(x, pt, ph, pw)[0]                           # [T, 3 * pt * ph * pw]
        n = pt * ph * pw
        start = np.stack([v[:, 0], v[:, n], v[:, 2 * n]], axis=1)  # first element of each channel
        grid = (F_ // pt, H // ph, W // pw)
        assert np.array_equal(O.token_coords(grid) * np.array([pt, ph, pw]), start)
    # a frame/row swap is caught whenever the two extents differ
    swapped = O.token_coords((2, 3, 4))[:, [1, 0, 2]]
    assert not np.array_equal(swapped, O.token_coords((2, 3, 4)))


def test_rope_invariants():
    rng = np.random.default_rng(6)
    # explicit (frame, row, col) triples, independent of token_coords
    coords = np.array([[f, r, c] for f in range(2) for r in range(3) for c in range(4)])
    q = rng.standard_normal((24, 72))
    k = rng.standard_normal((24, 72))
    rq = O.rope_3d(q, coords)
    assert np.allclose(np.linalg.norm(rq, axis=1), np.linalg.norm(q, axis=1))
    assert np.array_equal(O.rope_3d(q, np.zeros_like(coords)), q)
    shifted = coords + np.array([3, -2, 5])
    assert np.allclose(O.rope_3d(q, coords) @ O.rope_3d(k, coords).T,
                       O.rope_3d(q, shifted) @ O.rope_3d(k, shifted).T)
    # the first pair of each slice (theta_0 = 1) turns by exactly that axis' coordinate:
    # token 23 is (frame 1, row 2, col 3)
    for a, want in enumerate((1, 2, 3)):
        ang = math.atan2(rq[23, 24 * a + 1], rq[23, 24 * a]) - math.atan2(q[23, 24 * a + 1], q[23, 24 * a])
        assert abs(math.remainder(ang - want, 2 * math.pi)) < 1e-12


def test_patchify_is_conv_and_unpatchify_is_rearrange():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 3, 4, 8, 6))
    w = rng.standard_normal((5, 3 * 2 * 2 * 3))
    tok = O.patchify(x, 2, 2, 3) @ w.T
    ref = F.conv3d(torch.from_numpy(x), torch.from_numpy(w).view(5, 3, 2, 2, 3), stride=(2, 2, 3))
    assert np.allclose(tok, ref.flatten(2).transpose(1, 2).numpy(), rtol=1e-12, atol=1e-12)
    grid = (2, 4, 2)
    z = rng.standard_normal((2, 16, 2 * 2 * 3 * 3))
    img = O.unpatchify(z, 3, grid, 2, 2, 3)
    import einops
    ref = einops.rearrange(z, "n (f h w) (a p q c) -> n c (f a) (h p) (w q)", f=2, h=4, w=2, a=2, p=2, q=3, c=3)
    assert np.array_equal(img, ref)


def test_unpatchify_inverts_channel_last_patchify():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, 4, 1, 8, 8))
    v = O.patchify(x, 1, 2, 2).reshape(2, 16, 4, 1, 2, 2).transpose(0, 1, 3, 4, 5, 2).reshape(2, 16, 16)
    assert np.array_equal(O.unpatchify(v, 4, (1, 4, 4), 1, 2, 2), x)


def test_one_hot_embedding_picks_input_element():
    cfg = small_image(depth=0)
    W = S.weight_dict(cfg, S.make_weights(cfg))
    x = np.random.default_rng(9).standard_normal(cfg.x_shape(1))
    W = dict(W)
    w = np.zeros_like(W["pe.w"])
    c, ih, iw = 2, 1, 3
    w[0, c * 16 + ih * 4 + iw] = 1.0
    W["pe.w"] = w
    W["pe.b"] = np.zeros_like(W["pe.b"])
    h = O.linear(O.patchify(x[:, :, None], 1, 4, 4), W["pe.w"], W["pe.b"])
    for i in range(4):
        for j in range(4):
            assert h[0, i * 4 + j, 0] == x[0, c, 4 * i + ih, 4 * j + iw]


# ----------------------------------------------------------------------------- blocks / forward
def test_zero_adaln_block_is_identity_bit_exact():
    cfg = small_image()
    W = S.weight_dict(cfg, S.set_adaln(cfg, S.make_weights(cfg), zero=True))
    rng = np.random.default_rng(10)
    x = rng.standard_normal((3, cfg.tokens, cfg.hidden))
    sc = O.silu(rng.standard_normal((3, cfg.hidden)))
    assert np.array_equal(O.dit_block(x, sc, W, "blocks.0.", cfg.heads), x)


def test_zero_adaln_forward_skips_blocks():
    cfg = small_image()
    W = S.weight_dict(cfg, S.set_adaln(cfg, S.make_weights(cfg), zero=True))
    inp = S.make_inputs(cfg)
    out = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    h = O.embed(cfg, W, inp["x"][:, :, None])
    sc = O.silu(O.condition(cfg, W, inp["t"], inp["y"]))
    z = O.final_layer(h, sc, W)
    want = O.unpatchify(z, cfg.out_channels, cfg.grid, 1, 4, 4)[:, :, 0]
    assert np.array_equal(out, want)
    assert np.array_equal(O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=2), h)


def test_block_is_token_permutation_equivariant():
    cfg = small_image()
    W = S.weight_dict(cfg, S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0))
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, cfg.tokens, cfg.hidden))
    sc = O.silu(rng.standard_normal((2, cfg.hidden)))
    p = rng.permutation(cfg.tokens)
    a = O.dit_block(x, sc, W, "blocks.0.", cfg.heads)[:, p]
    b = O.dit_block(x[:, p], sc, W, "blocks.0.", cfg.heads)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_batch_rows_independent():
    cfg = small_image(batch=3)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    full = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    for i in range(3):
        one = O.forward(cfg, W, inp["x"][i:i + 1], inp["t"][i:i + 1], inp["y"][i:i + 1])
        assert np.allclose(one[0], full[i], rtol=1e-12, atol=1e-12)


def test_guidance_special_cases():
    cfg = small_image(cfg_scale=1.5)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    x, t, y = inp["x"], inp["t"], inp["y"]
    cond = O.forward(cfg, W, x, t, y, cfg_scale=1.0)
    uncond = O.forward(cfg, W, x, t, np.full_like(y, cfg.num_classes), cfg_scale=1.0)
    s1 = O.forward(cfg, W, x, t, y, cfg_scale=1.0, force_guidance=True)
    s0 = O.forward(cfg, W, x, t, y, cfg_scale=0.0)
    s15 = O.forward(cfg, W, x, t, y)
    s3 = O.forward(cfg, W, x, t, y, cfg_scale=3.0)
    assert np.allclose(s1, cond, rtol=1e-12, atol=1e-12)
    assert np.allclose(s0, uncond, rtol=1e-12, atol=1e-12)
    assert np.array_equal(O.cfg_combine(cond, uncond, 0.0), uncond)
    assert np.allclose(s15, uncond + 1.5 * (cond - uncond), rtol=1e-12, atol=1e-12)
    assert np.allclose(s3 - s15, (3.0 - 1.5) * (cond - uncond), rtol=1e-10, atol=1e-10)


def test_guidance_on_the_first_channels_only():
    """[DiT-wiki] "ImageNet 클래스 조건 생성": the official code guides only the first three
    output channels.  Those channels equal full guidance; the rest equal the unguided
    conditional prediction (computed here by a separate, unduplicated forward)."""
    cfg = small_image(cfg_scale=1.5)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    x, t, y = inp["x"], inp["t"], inp["y"]
    full = O.forward(cfg, W, x, t, y)
    part = O.forward(cfg, W, x, t, y, cfg_channels=3)
    cond = O.forward(cfg, W, x, t, y, cfg_scale=1.0)
    assert cfg.out_channels > 3
    assert np.array_equal(part[:, :3], full[:, :3])
    assert np.allclose(part[:, 3:], cond[:, 3:], rtol=1e-12, atol=1e-12)
    assert not np.allclose(part[:, 3:], full[:, 3:], rtol=1e-6, atol=1e-6)     # the guidance mattered there
    assert np.array_equal(O.forward(cfg, W, x, t, y, cfg_channels=cfg.out_channels), full)
    assert np.array_equal(O.forward(cfg, W, x, t, y, cfg_channels=0), full)
    # planted slip: the unguided channels taken from the unconditional rows
    uncond = O.forward(cfg, W, x, t, np.full_like(y, cfg.num_classes), cfg_scale=1.0)
    assert not np.allclose(uncond[:, 3:], cond[:, 3:], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("kind", ["image", "image_guided", "video"])
def test_forward_matches_torch_layers(kind):
    from torch_reference import reference_forward
    if kind == "video":
        cfg = small_video()
    else:
        cfg = small_image(cfg_scale=1.5 if kind == "image_guided" else 1.0)
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    inp = S.make_inputs(cfg)
    got = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    want = reference_forward(cfg, S.weight_dict(cfg, W), inp["x"], inp["t"], inp["y"])
    assert got.shape == want.shape == cfg.out_shape()
    assert np.allclose(got, want, rtol=1e-9, atol=1e-10), np.abs(got - want).max()


@pytest.mark.parametrize("kind,video", [(1, False), (2, False), (3, False), (1, True), (2, True)],
                         ids=["in_context", "cross_attn", "adaln", "in_context_video", "cross_attn_video"])
def test_conditioning_designs_match_torch_layers(kind, video):
    """The in-context, cross-attention and adaLN designs against stock torch layers
    (LayerNorm with affine, nn.MultiheadAttention for the cross-attention)."""
    from torch_reference import reference_forward
    cfg = (small_video() if video else small_image(cfg_scale=1.5)).with_(block_kind=kind)
    W = S.make_weights(cfg)
    inp = S.make_inputs(cfg)
    got = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    want = reference_forward(cfg, S.weight_dict(cfg, W), inp["x"], inp["t"], inp["y"])
    assert got.shape == want.shape == cfg.out_shape()
    assert np.allclose(got, want, rtol=1e-9, atol=1e-10), np.abs(got - want).max()


def test_cross_attention_closed_forms():
    """Two equal keys weigh both values 1/2; queries identical across tokens give identical
    outputs; a zero output projection makes the sublayer vanish."""
    rng = np.random.default_rng(21)
    d, heads = 8, 2
    u = rng.standard_normal((1, 5, d))
    ctx = rng.standard_normal((1, 2, d))
    wq, bq = rng.standard_normal((d, d)), rng.standard_normal(d)
    wkv, bkv = rng.standard_normal((2 * d, d)), rng.standard_normal(2 * d)
    wo, bo = np.eye(d), np.zeros(d)
    same = np.repeat(ctx[:, :1], 2, axis=1)
    k0v = O.linear(same, wkv, bkv)[0, 0, d:]
    out = O.cross_attention(u, same, wq, bq, wkv, bkv, wo, bo, heads)
    assert np.allclose(out[0], np.broadcast_to(k0v, (5, d)), rtol=1e-12, atol=1e-12)
    v = O.linear(ctx, wkv, bkv)[0, :, d:]
    out = O.cross_attention(u, ctx, wq, bq, wkv, bkv, wo, bo, heads)
    for hd in range(heads):   # each head's output is a convex mix of the two values
        sl = slice(hd * 4, hd * 4 + 4)
        lam = (out[0, :, sl] - v[1, sl]) / (v[0, sl] - v[1, sl])
        assert np.allclose(lam, lam[:, :1], rtol=1e-9, atol=1e-9) and np.all((lam > 0) & (lam < 1))
    assert np.array_equal(O.cross_attention(u, ctx, wq, bq, wkv, bkv, 0 * wo, bo, heads), np.zeros((1, 5, d)))


def test_in_context_tokens_are_dropped_and_blocks_see_them():
    """In-context: the residual stream carries T + 2 tokens, the first two being e_t and e_y
    before any block; the output has the patch tokens only, and the condition reaches it."""
    cfg = small_image(cfg_scale=1.0, block_kind=1)
    W = S.weight_dict(cfg, S.make_weights(cfg))
    inp = S.make_inputs(cfg)
    h0 = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], stop_after_block=0)
    et, ey = O.condition_parts(cfg, W, inp["t"], inp["y"])
    assert h0.shape == (cfg.batch, cfg.tokens + 2, cfg.hidden)
    assert np.array_equal(h0[:, 0], et) and np.array_equal(h0[:, 1], ey)
    out = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    other = O.forward(cfg, W, inp["x"], inp["t"], (inp["y"] + 1) % cfg.num_classes)
    assert out.shape == cfg.out_shape() and not np.allclose(out, other)


@pytest.mark.parametrize("plant", ["kv_swapped", "ln_gain_dropped", "ctx_from_c", "adaln_gate_kept"])
def test_conditioning_cross_check_catches_planted_mistakes(plant, monkeypatch):
    """Slips in the other conditioning designs (keys and values swapped in the cross-attention,
    the learned LN gain dropped, the summed c used as both condition tokens, a gate applied in
    the gateless adaLN block) make the torch-layer cross-check fail."""
    from torch_reference import reference_forward
    kind = {"kv_swapped": 2, "ln_gain_dropped": 1, "ctx_from_c": 2, "adaln_gate_kept": 3}[plant]
    cfg = small_image(cfg_scale=1.5, block_kind=kind)
    Wd = S.weight_dict(cfg, S.make_weights(cfg))
    inp = S.make_inputs(cfg)
    want = reference_forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    if plant == "kv_swapped":
        orig = O.cross_attention
        d = cfg.hidden
        monkeypatch.setattr(O, "cross_attention", lambda u, ctx, wq, bq, wkv, bkv, wo, bo, h: orig(
            u, ctx, wq, bq, np.concatenate([wkv[d:], wkv[:d]]), np.concatenate([bkv[d:], bkv[:d]]), wo, bo, h))
    elif plant == "ln_gain_dropped":
        orig = O.layernorm_affine
        monkeypatch.setattr(O, "layernorm_affine", lambda x, g, b, eps=1e-6: orig(x, np.ones_like(g), b, eps))
    elif plant == "ctx_from_c":
        orig = O.condition_parts
        monkeypatch.setattr(O, "condition_parts", lambda c_, W_, t_, y_: (lambda a: (a[0] + a[1], a[0] + a[1]))(
            orig(c_, W_, t_, y_)))
    else:
        orig = O.adaln_block

        def gated(x, sc, W_, prefix, heads, coords=None):
            g = O.silu(sc) * 0.5 + 0.25    # any gate other than 1
            return x + g[:, None, :] * (orig(x, sc, W_, prefix, heads, coords) - x)
        monkeypatch.setattr(O, "adaln_block", gated)
    got = O.forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel > 1e-7, rel


_PLANTS = {
    "erf_gelu": ("gelu_tanh", lambda x: 0.5 * np.asarray(x) * (1 + np.vectorize(math.erf)(np.asarray(x) / math.sqrt(2)))),
    "chunk_order": ("adaln_chunks", None),
    "no_gate": ("dit_block", None),
    "ln_eps": ("layernorm", lambda x, eps=1e-6: O.__dict__["_orig_layernorm"](x, eps=1e-2)),
    "attn_scale": ("attention", None),
}


def test_oracle_catches_a_frame_row_swap_in_token_coords(monkeypatch):
    """The torch-layer cross-check derives each token's RoPE coordinates from the Conv3d
    output layout, not from the oracle, so swapping frame and row in token_coords shows."""
    from torch_reference import reference_forward
    cfg = small_video()
    assert cfg.grid[0] != cfg.grid[1]
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    Wd = S.weight_dict(cfg, W)
    inp = S.make_inputs(cfg)
    want = reference_forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    orig = O.token_coords
    monkeypatch.setattr(O, "token_coords", lambda grid: orig(grid)[:, [1, 0, 2]])
    got = O.forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel > 1e-7, rel


@pytest.mark.parametrize("plant", sorted(_PLANTS))
def test_oracle_catches_planted_mistakes(plant, monkeypatch):
    """A plausible slip planted in the oracle (wrong GELU, swapped modulation
    chunks, a dropped gate, a wrong LN eps, a wrong attention scale) makes the
    torch-layer cross-check fail by far more than its tolerance."""
    from torch_reference import reference_forward
    cfg = small_image()
    W = S.set_adaln(cfg, S.make_weights(cfg), gate_bias=1.0)
    Wd = S.weight_dict(cfg, W)
    inp = S.make_inputs(cfg)
    want = reference_forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    name, fn = _PLANTS[plant]
    orig = getattr(O, name)
    monkeypatch.setitem(O.__dict__, "_orig_layernorm", O.layernorm)
    if plant == "chunk_order":
        fn = lambda sc, w, b, n: orig(sc, w, b, n)[::-1]
    elif plant == "no_gate":
        def fn(x, sc, W_, prefix, heads, coords=None):
            W2 = dict(W_)
            W2[prefix + "ada.b"] = W_[prefix + "ada.b"].copy()
            W2[prefix + "ada.b"][2 * cfg.hidden:3 * cfg.hidden] = 0.0
            W2[prefix + "ada.w"] = W_[prefix + "ada.w"].copy()
            W2[prefix + "ada.w"][2 * cfg.hidden:3 * cfg.hidden] = 0.0
            return orig(x, sc, W2, prefix, heads, coords)
    elif plant == "attn_scale":
        fn = lambda q, k, v: orig(q * math.sqrt(q.shape[1]) ** 0.5, k, v)
    monkeypatch.setattr(O, name, fn)
    got = O.forward(cfg, Wd, inp["x"], inp["t"], inp["y"])
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel > 1e-7, rel  # the cross-check above holds the oracle to ~1e-9
