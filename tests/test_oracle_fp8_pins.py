"""Pins of the oracle's FP8 (E4M3) linears: the feed-forward and the attention projections (CPU only).

The quantiser is checked against torch's float8_e4m3fn cast (a library routine) on every
representable value, every midpoint between neighbours (ties to even) and random values; the
quantised matmul against its closed forms (exact on the E4M3 grid, error within the format's
half-step bound); the hidden activation's scale against the bound it claims.
"""
import numpy as np
import pytest
import torch

import dit_synth as S
from oracle import dit_oracle as O


def e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    v = np.unique(codes[np.isfinite(codes)].astype(np.float64))
    return v


def test_grid_is_the_e4m3_value_set():
    v = e4m3_values()
    assert v.max() == 448.0 and v.min() == -448.0 and len(v) == 253   # 2 x 126 nonzero + one zero
    assert np.array_equal(O.round_e4m3(v), v)                         # representable -> itself


def test_midpoints_round_to_even_like_the_library():
    v = e4m3_values()
    pos = v[v >= 0]
    mid = (pos[:-1] + pos[1:]) / 2
    want = torch.from_numpy(mid.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(O.round_e4m3(mid), want)
    assert np.array_equal(O.round_e4m3(-mid), -want)


def test_random_values_match_the_library_and_saturate():
    rng = np.random.default_rng(31)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x[np.abs(x) < 464].astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(O.round_e4m3(x.astype(np.float64)), want)
    assert np.array_equal(O.round_e4m3(np.array([470.0, -1e6])), np.array([448.0, -448.0]))


def test_quantised_linear_closed_forms():
    rng = np.random.default_rng(32)
    v = e4m3_values()
    x = rng.choice(v[np.abs(v) <= 16], size=(5, 24))
    x[:, 0] = 448.0                                   # per-row amax 448 -> scale 1, exact
    w = rng.choice(v[np.abs(v) <= 16], size=(7, 24))
    w[:, 0] = 448.0
    b = rng.standard_normal(7)
    assert np.allclose(O.linear_e4m3(x, w, b), O.linear(x, w, b), rtol=1e-15, atol=1e-12)
    # general inputs: each operand within half a step of itself (2^-4 relative for normals,
    # 2^-10 of the scale below 2^-6 of it)
    xr, wr = rng.standard_normal((6, 40)), rng.standard_normal((9, 40))
    xs, ws = O.amax_scale(xr), O.amax_scale(wr)
    xq, wq = O.quantize_rows(xr, xs), O.quantize_rows(wr, ws)
    assert np.all(np.abs(xq - xr) <= np.maximum(np.abs(xr) * 2.0 ** -4, xs[:, None] * 2.0 ** -10) + 1e-15)
    assert np.all(np.abs(wq - wr) <= np.maximum(np.abs(wr) * 2.0 ** -4, ws[:, None] * 2.0 ** -10) + 1e-15)
    y = O.linear_e4m3(xr, wr, np.zeros(9))
    assert np.allclose(y, xq @ wq.T, rtol=1e-13, atol=1e-13)


def test_hidden_scale_bounds_the_hidden_activation():
    """The per-token bound ||u|| max_n ||W1_n|| + max|b1| is never below max |GELU(z)|."""
    cfg = S.DIT_XL2_CFG256.with_(hidden=96, heads=2, mlp_hidden=384, depth=1, index=-1)
    W = S.weight_dict(cfg, S.make_weights(cfg))
    rng = np.random.default_rng(33)
    u = rng.standard_normal((3, 50, 96)) * 3.0
    z = O.linear_e4m3(u, W["blocks.0.fc1.w"], W["blocks.0.fc1.b"])
    bound = np.linalg.norm(u, axis=-1) * np.linalg.norm(W["blocks.0.fc1.w"], axis=1).max() + \
        np.abs(W["blocks.0.fc1.b"]).max()
    assert np.all(np.abs(O.gelu_tanh(z)).max(axis=-1) <= bound)


@pytest.mark.parametrize("gates", ["random", "strong"])
def test_fp8_forward_stays_near_the_exact_forward(gates):
    """The E4M3 feed-forward perturbs the forward by a few percent at most on these workloads
    (3 mantissa bits: ~2^-4 / sqrt(3) relative rounding per operand)."""
    cfg = S.DIT_XL2_CFG256.with_(hidden=288, heads=4, mlp_hidden=1152, depth=2, height=16, width=16, batch=2,
                                 index=-1)
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    a = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    b = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], ffn_fp8=True)
    rel = np.linalg.norm(a - b) / np.linalg.norm(a)
    assert 0 < rel < 5e-2, rel
    assert np.array_equal(O.forward(cfg, W, inp["x"], inp["t"], inp["y"]), a)   # the switch is scoped


def _torch_linear_e4m3(x, w, b):
    """linear_e4m3 written with torch's float8_e4m3fn cast (per-row amax / 448 scales)."""
    def q(a):
        s = a.abs().amax(dim=-1, keepdim=True) / 448.0
        s = torch.where(s > 0, s, torch.ones_like(s))
        return (a / s).to(torch.float8_e4m3fn).to(torch.float64) * s
    return q(x) @ q(w).T + b


def test_attn_fp8_self_attention_matches_a_torch_float8_composition():
    """Both projections of the E4M3 self-attention, written independently with torch's float8
    cast and torch's softmax: in-projection on the LN output's rows, out-projection on the
    concatenated heads' rows (a slip such as leaving the out-projection exact fails here)."""
    rng = np.random.default_rng(34)
    r, t, d, heads = 2, 20, 48, 3
    u = rng.standard_normal((r, t, d)) * 2.0
    wqkv, bqkv = rng.standard_normal((3 * d, d)) * 0.2, rng.standard_normal(3 * d) * 0.1
    wo, bo = rng.standard_normal((d, d)) * 0.2, rng.standard_normal(d) * 0.1
    O._STATE["attn_fp8"] = True
    try:
        got = O.self_attention(u, wqkv, bqkv, wo, bo, heads)
    finally:
        O._STATE["attn_fp8"] = False
    U = torch.from_numpy(u)
    qkv = _torch_linear_e4m3(U.reshape(r * t, d), torch.from_numpy(wqkv), torch.from_numpy(bqkv)).reshape(r, t, 3 * d)
    dh = d // heads
    q = qkv[..., :d].reshape(r, t, heads, dh).transpose(1, 2)
    k = qkv[..., d:2 * d].reshape(r, t, heads, dh).transpose(1, 2)
    v = qkv[..., 2 * d:].reshape(r, t, heads, dh).transpose(1, 2)
    o = torch.softmax(q @ k.transpose(-1, -2) / dh ** 0.5, dim=-1) @ v
    o = o.transpose(1, 2).reshape(r * t, d)
    want = _torch_linear_e4m3(o, torch.from_numpy(wo), torch.from_numpy(bo)).reshape(r, t, d).numpy()
    assert np.allclose(got, want, rtol=1e-10, atol=1e-10)
    exact = O.self_attention(u, wqkv, bqkv, wo, bo, heads)
    assert not np.allclose(got, exact, rtol=1e-4, atol=1e-4)     # the switch does something


@pytest.mark.parametrize("gates", ["random", "strong"])
def test_attn_fp8_forward_stays_near_the_exact_forward(gates):
    """E4M3 attention projections (and with them the E4M3 feed-forward) perturb the forward
    by a few percent at most; the switches are scoped to the call."""
    cfg = S.DIT_XL2_CFG256.with_(hidden=288, heads=4, mlp_hidden=1152, depth=2, height=16, width=16, batch=2,
                                 index=-1)
    W = S.make_weights(cfg)
    if gates == "strong":
        W = S.set_adaln(cfg, W, gate_bias=1.0)
    inp = S.make_inputs(cfg)
    a = O.forward(cfg, W, inp["x"], inp["t"], inp["y"])
    b = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], attn_fp8=True)
    c = O.forward(cfg, W, inp["x"], inp["t"], inp["y"], attn_fp8=True, ffn_fp8=True)
    for z in (b, c):
        rel = np.linalg.norm(a - z) / np.linalg.norm(a)
        assert 0 < rel < 5e-2, rel
    assert not np.array_equal(b, c)
    assert np.array_equal(O.forward(cfg, W, inp["x"], inp["t"], inp["y"]), a)
