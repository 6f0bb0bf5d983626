"""CPU oracle for the DiT denoiser forward pass — TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 numpy restatement of what the method computes.  Only the
tests, the package's smoke check and the benchmark's CPU-baseline leg may import
it; the product path (the CUDA library) never does, and the two share no code.

Sources (web pages on the Diffusion Transformer; cited by title and section):
  [DiT-wiki]  "확산 트랜스포머" (Diffusion Transformer), itwiki.kr — sections
              "잠재 공간과 패치화" (latent space and patchify), "조건 주입 방식"
              (conditioning), "adaLN-Zero", "모델 크기" (model size table),
              "ImageNet 클래스 조건 생성" (class-conditional results), "구현"
              (implementation: the DiT block listing and the patchify remark).
  [Sora-DiT]  "Sora / DiT", cv-learn.com — section "방법 및 아키텍처" (method and
              architecture): patchify, adaLN-Zero, linear decoder to p×p×2C,
              classifier-free guidance formula.
  [Sora-obs]  "Sora: 확산 기반 비디오 생성 모델", obsidian-dorae222 — section
              "시공간 패치 토큰화" (spacetime patch tokenisation).
  [Goku]      "GOKU : Flow Based Video Generative Foundation Models", blog.outta.ai —
              §2.2 (full attention, 3D RoPE, Q-K normalisation), §2.3 (rectified
              flow: the network predicts a velocity).

Readings taken where the pages are silent:
  * timestep sinusoid: 256 dims, half = 128, f_i = 10000^(-i/128), layout
    [cos | sin], argument t * t_scale (t_scale = 1 for integer steps, 1000 for
    t in [0, 1));
  * 2D sin-cos positions: first d/2 dims encode the patch row, last d/2 the
    column; each half is [sin(pos w_k) | cos(pos w_k)], w_k = 10000^(-k/(d/4));
  * LayerNorm without affine, eps 1e-6, population variance;
  * attention: heads are contiguous dh-slices of d, in-projection rows ordered
    [q | k | v], scale 1/sqrt(dh), no mask;
  * final layer: an adaLN (shift, scale) modulation of a no-affine LayerNorm,
    then a linear decoder; decoder vector index (i_t, i_h, i_w, c), c fastest;
  * patch vector index (c, i_t, i_h, i_w), i.e. the flattened Conv weight;
  * QK-RMSNorm per head over dh, eps 1e-6, learnable gain; 3D RoPE splits dh
    into three equal slices (t, h, w), rotates adjacent pairs (2k, 2k+1) by
    pos * 10000^(-2k/(dh/3)), applied after the QK norm;
  * classifier-free guidance on every output channel; internal row order
    [conditional; unconditional].

Parity of the whole forward against a trained checkpoint is unpinned (no
checkpoints exist offline); every step below is pinned by the tests in
tests/test_oracle_*.py.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

F64 = np.float64

# multiply-add counter: the pages' "Gflops" column counts one per multiply-add
# (see count_forward_macs); linear() and attention() add to it.
_STATE = {"macs": 0, "dry": False}


def reset_mac_counter(dry: bool = False) -> None:
    _STATE["macs"] = 0
    _STATE["dry"] = dry


def mac_count() -> int:
    return _STATE["macs"]


# --------------------------------------------------------------------------- #
# elementwise pieces
# --------------------------------------------------------------------------- #
def silu(x):
    """SiLU(x) = x * sigmoid(x): the activation in front of the adaLN MLP
    ([DiT-wiki] "구현": the modulation branch is SiLU then Linear(d, 6d))."""
    x = np.asarray(x, dtype=F64)
    return x / (1.0 + np.exp(-x))


def gelu_tanh(x):
    """tanh-approximated GELU used inside the FFN ([DiT-wiki] "구현": GELU with the
    tanh approximation):  0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=F64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def layernorm(x, eps: float = 1e-6):
    """LayerNorm over the last axis with no learnable affine ([DiT-wiki]
    "adaLN-Zero": LN has no learnable affine parameters; "구현": eps = 1e-6).
    Population (biased) variance, the plain definition of layer normalisation."""
    x = np.asarray(x, dtype=F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def rmsnorm(x, gain, eps: float = 1e-6):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * gain
    ([Goku] §2.2 Q-K normalisation; [DiT-wiki] "MMDiT": RMSNorm on Q and K)."""
    x = np.asarray(x, dtype=F64)
    return x / np.sqrt((x ** 2).mean(axis=-1, keepdims=True) + eps) * np.asarray(gain, dtype=F64)


def layernorm_affine(x, gain, bias, eps: float = 1e-6):
    """LayerNorm with its learned per-feature scale and shift, the normalisation of the
    in-context and cross-attention designs ([DiT-wiki] "조건 주입 방식": adaLN replaces
    exactly these learned constants with values regressed from t + c)."""
    return layernorm(x, eps) * np.asarray(gain, dtype=F64) + np.asarray(bias, dtype=F64)


def modulate(x, shift, scale):
    """x * (1 + scale) + shift, shift/scale broadcast over the token axis
    ([DiT-wiki] "adaLN-Zero": LN(x)(1 + gamma) + beta)."""
    return x * (1.0 + scale[:, None, :]) + shift[:, None, :]


# --------------------------------------------------------------------------- #
# contractions (the only places multiply-adds are counted)
# --------------------------------------------------------------------------- #
def linear(x, w, b):
    """y = x W^T + b with W stored [out, in] (a library matmul serves as the step)."""
    x = np.asarray(x, dtype=F64)
    w = np.asarray(w)
    rows = int(np.prod(x.shape[:-1]))
    _STATE["macs"] += rows * w.shape[0] * w.shape[1]
    if _STATE["dry"]:
        return np.zeros(x.shape[:-1] + (w.shape[0],), dtype=F64)
    return x @ w.astype(F64).T + np.asarray(b, dtype=F64)


def attention(q, k, v):
    """Scaled dot-product softmax attention for one head, no mask:
    softmax(q k^T / sqrt(dh)) v over all T keys ([DiT-wiki] "adaLN-Zero": Attn is
    multi-head self-attention over every token; [Goku] §2.2: full attention).
    q, k, v: [T, dh].  The softmax subtracts the row maximum before exp."""
    t, dh = q.shape
    _STATE["macs"] += 2 * t * k.shape[0] * dh
    if _STATE["dry"]:
        return np.zeros((t, v.shape[1]), dtype=F64)
    s = (q @ k.T) / math.sqrt(dh)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


# --------------------------------------------------------------------------- #
# embeddings and positions
# --------------------------------------------------------------------------- #
def timestep_embedding(t, dim: int = 256, t_scale: float = 1.0):
    """Sinusoidal timestep features [cos(t' f_i) | sin(t' f_i)], f_i = 10000^(-i/half),
    t' = t * t_scale (reading of the 256-dim sinusoidal embedding; see header)."""
    half = dim // 2
    freqs = np.exp(-math.log(10000.0) * np.arange(half, dtype=F64) / half)
    arg = np.asarray(t, dtype=F64)[:, None] * t_scale * freqs[None, :]
    return np.concatenate([np.cos(arg), np.sin(arg)], axis=1)


def pos_embed_sincos_2d(gh: int, gw: int, d: int):
    """ViT-style fixed 2D sin-cos table [gh*gw, d] ([Sora-DiT] patchify bullet;
    [DiT-wiki] "잠재 공간과 패치화": 2D sine-cosine position embedding added to every
    token).  Row-major token order; first half encodes the row, second the column."""
    assert d % 4 == 0
    q = d // 4
    omega = 1.0 / (10000.0 ** (np.arange(q, dtype=F64) / q))

    def one_axis(pos):
        a = np.asarray(pos, dtype=F64)[:, None] * omega[None, :]
        return np.concatenate([np.sin(a), np.cos(a)], axis=1)

    rows = np.repeat(np.arange(gh), gw)
    cols = np.tile(np.arange(gw), gh)
    return np.concatenate([one_axis(rows), one_axis(cols)], axis=1)


def rope_3d(x, coords):
    """Rotary position embedding over three axes ([Goku] §2.2, 3D RoPE).
    x: [T, dh]; coords: [T, 3] integer (frame, row, col) of each token.
    dh is split into three equal slices; slice a rotates its adjacent pairs
    (2k, 2k+1) by angle coords[:, a] * 10000^(-2k/(dh/3))."""
    t, dh = x.shape
    assert dh % 6 == 0
    sl = dh // 3
    out = np.array(x, dtype=F64, copy=True)
    k = np.arange(sl // 2, dtype=F64)
    theta = 10000.0 ** (-2.0 * k / sl)
    for a in range(3):
        ang = np.asarray(coords[:, a], dtype=F64)[:, None] * theta[None, :]
        c, s = np.cos(ang), np.sin(ang)
        x0 = x[:, a * sl + 0:(a + 1) * sl:2].astype(F64)
        x1 = x[:, a * sl + 1:(a + 1) * sl:2].astype(F64)
        out[:, a * sl + 0:(a + 1) * sl:2] = x0 * c - x1 * s
        out[:, a * sl + 1:(a + 1) * sl:2] = x0 * s + x1 * c
    return out


def token_coords(grid):
    """(frame, row, col) of every token in raster order over the patch grid."""
    gf, gh, gw = grid
    f, r, c = np.meshgrid(np.arange(gf), np.arange(gh), np.arange(gw), indexing="ij")
    return np.stack([f.ravel(), r.ravel(), c.ravel()], axis=1)


# --------------------------------------------------------------------------- #
# patchify / unpatchify ([DiT-wiki] "잠재 공간과 패치화"; [Sora-obs] spacetime patches)
# --------------------------------------------------------------------------- #
def patchify(x, pt: int, ph: int, pw: int):
    """Cut latents [N, C, F, H, W] into non-overlapping pt×ph×pw patches.
    Returns [N, T, C*pt*ph*pw]; token order (f, i, j) raster, patch vector order
    (c, it, ih, iw) — the flattening of a Conv weight with kernel = stride = patch."""
    n, c, f, h, w = x.shape
    gf, gh, gw = f // pt, h // ph, w // pw
    v = np.asarray(x, dtype=F64).reshape(n, c, gf, pt, gh, ph, gw, pw)
    v = v.transpose(0, 2, 4, 6, 1, 3, 5, 7)  # n, gf, gh, gw, c, pt, ph, pw
    return v.reshape(n, gf * gh * gw, c * pt * ph * pw)


def unpatchify(z, c_out: int, grid, pt: int, ph: int, pw: int):
    """Inverse arrangement of the decoder output ([Sora-DiT]: each token is decoded to
    p×p×2C; [DiT-wiki]: the decoded tokens are put back in the spatial layout).
    z: [N, T, pt*ph*pw*c_out] with vector index (it, ih, iw, c), c fastest.
    Returns [N, c_out, F, H, W]."""
    n = z.shape[0]
    gf, gh, gw = grid
    v = np.asarray(z, dtype=F64).reshape(n, gf, gh, gw, pt, ph, pw, c_out)
    v = v.transpose(0, 7, 1, 4, 2, 5, 3, 6)  # n, c, gf, pt, gh, ph, gw, pw
    return v.reshape(n, c_out, gf * pt, gh * ph, gw * pw)


# --------------------------------------------------------------------------- #
# condition and guidance
# --------------------------------------------------------------------------- #
def condition_parts(cfg, W: Dict[str, np.ndarray], t, y):
    """The two condition embeddings: e_t = MLP(sinusoid(t)) (a two-layer SiLU MLP on the
    timestep features) and e_y = the class embedding (a row of the label table), or for the
    text-conditioned video model the pooled text vector itself."""
    e = timestep_embedding(t, cfg.freq_dim, cfg.t_scale)
    hid = silu(linear(e, W["t.w1"], W["t.b1"]))
    et = linear(hid, W["t.w2"], W["t.b2"])
    if cfg.cond_kind == 0:
        ey = np.asarray(W["y.table"], dtype=F64)[np.asarray(y, dtype=np.int64)]
    else:
        ey = np.asarray(y, dtype=F64)
    return et, ey


def condition(cfg, W: Dict[str, np.ndarray], t, y):
    """c = e_t + e_y: the timestep embedding summed with the class embedding ([DiT-wiki]
    "adaLN-Zero": c is the sum of the time and class embeddings; "조건 주입 방식": gamma,
    beta regressed from t + c)."""
    et, ey = condition_parts(cfg, W, t, y)
    return et + ey


def cfg_combine(eps_cond, eps_uncond, s: float, channels: Optional[int] = None):
    """Classifier-free guidance: eps(∅) + s (eps(c) - eps(∅)) ([Sora-DiT] guidance bullet).
    With `channels` = n, only output channels c < n are guided, the variant [DiT-wiki]
    "ImageNet 클래스 조건 생성" attributes to the official code (n = 3); the other channels
    keep the conditional prediction (reading: the page does not say what they hold)."""
    g = eps_uncond + s * (eps_cond - eps_uncond)
    if channels is None or channels <= 0 or channels >= eps_cond.shape[1]:
        return g
    out = np.array(eps_cond, dtype=F64, copy=True)
    out[:, :channels] = g[:, :channels]
    return out


# --------------------------------------------------------------------------- #
# one DiT block ([DiT-wiki] "adaLN-Zero" block equations)
# --------------------------------------------------------------------------- #
def self_attention(u, wqkv, bqkv, wo, bo, heads: int, qn=None, kn=None, coords=None):
    """Multi-head self-attention on u [R, T, d]: in-projection to [q | k | v],
    per-head attention, heads concatenated, out-projection.  Optional per-head
    QK-RMSNorm (gains qn, kn) and 3D RoPE (coords) for the video model."""
    r, t, d = u.shape
    dh = d // heads
    fp8 = _STATE.get("attn_fp8")
    qkv = linear_e4m3(u, wqkv, bqkv) if fp8 else linear(u, wqkv, bqkv)
    q, k, v = qkv[..., :d], qkv[..., d:2 * d], qkv[..., 2 * d:]
    o = np.zeros((r, t, d), dtype=F64)
    for i in range(r):
        for hd in range(heads):
            sl = slice(hd * dh, (hd + 1) * dh)
            qh, kh, vh = q[i, :, sl], k[i, :, sl], v[i, :, sl]
            if qn is not None:
                qh, kh = rmsnorm(qh, qn), rmsnorm(kh, kn)
            if coords is not None:
                qh, kh = rope_3d(qh, coords), rope_3d(kh, coords)
            o[i, :, sl] = attention(qh, kh, vh)
    return linear_e4m3(o, wo, bo) if fp8 else linear(o, wo, bo)


def ffn(u, w1, b1, w2, b2):
    """Linear(d, 4d) -> tanh-GELU -> Linear(4d, d) ([DiT-wiki] "구현")."""
    if _STATE.get("ffn_fp8"):
        return ffn_e4m3(u, w1, b1, w2, b2)
    return linear(gelu_tanh(linear(u, w1, b1)), w2, b2)


# --------------------------------------------------------------------------- #
# FP8 (E4M3) linears: a reading, not the pages' ([DiT-wiki] "U-Net과 비교" names mixed
# precision among the techniques that carry over from language models; the pages fix no
# format, so this is the quantised computation the FP8 path is held to).  With attn_fp8 the
# self-attention's in-projection and out-projection are linear_e4m3 (per-token amax scales of
# the LN output and of the concatenated heads); with ffn_fp8 the feed-forward is ffn_e4m3.
# --------------------------------------------------------------------------- #
E4M3_MAX = 448.0


def round_e4m3(x):
    """Nearest FP8 E4M3 value (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits:
    normal magnitudes 2^-6 .. 448 in binades of 8 steps, subnormal steps of 2^-9 below 2^-6),
    ties to the even mantissa, magnitudes past 448 saturated to 448."""
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))   # binade of each magnitude
    e = np.maximum(e, -6.0)                            # one step size below 2^-6
    step = np.exp2(e - 3.0)                            # 8 steps per binade
    q = np.minimum(np.round(a / step) * step, E4M3_MAX)   # np.round: ties to even
    return np.sign(x) * q


def quantize_rows(a, scale):
    """s * Q(a / s) row by row: the value an E4M3 operand with per-row scale s stands for."""
    s = np.asarray(scale, dtype=F64)[..., None]
    return round_e4m3(np.asarray(a, dtype=F64) / s) * s


def amax_scale(a):
    """Per-row scale amax(|a|) / 448 (1 for an all-zero row), so that a row's largest
    magnitude maps onto the largest E4M3 value."""
    m = np.abs(np.asarray(a, dtype=F64)).max(axis=-1)
    return np.where(m > 0, m / E4M3_MAX, 1.0)


def linear_e4m3(x, w, b, x_scale=None):
    """y = x W^T + b with both operands in E4M3: x with a per-row (token) scale (amax unless
    given), W with a per-output-channel scale; products accumulated exactly."""
    x = np.asarray(x, dtype=F64)
    sx = amax_scale(x) if x_scale is None else np.asarray(x_scale, dtype=F64)
    wq = quantize_rows(w, amax_scale(w))
    return linear(quantize_rows(x, sx), wq, b)


def ffn_e4m3(u, w1, b1, w2, b2):
    """The feed-forward with both matmuls in E4M3.  The hidden activation g = GELU(z) gets a
    per-token scale from a bound known before z is formed: |g| <= |z| <= ||u||_2 max_n ||W1_n||_2
    + max |b1| (Cauchy-Schwarz), so g's scale is that bound / 448."""
    u = np.asarray(u, dtype=F64)
    z = linear_e4m3(u, w1, b1)
    g = gelu_tanh(z)
    w1 = np.asarray(w1, dtype=F64)
    bound = np.linalg.norm(u, axis=-1) * np.linalg.norm(w1, axis=1).max() + np.abs(np.asarray(b1, F64)).max()
    return linear_e4m3(g, w2, b2, x_scale=np.where(bound > 0, bound / E4M3_MAX, 1.0))


def adaln_chunks(sc, w, b, n: int):
    """Regress n modulation vectors from SiLU(c): (shift1, scale1, gate1, shift2,
    scale2, gate2) for a block, (shift, scale) for the final layer ([DiT-wiki]
    "adaLN-Zero": (beta1, gamma1, alpha1, beta2, gamma2, alpha2) = MLP(c))."""
    m = linear(sc, w, b)
    d = m.shape[-1] // n
    return [m[:, i * d:(i + 1) * d] for i in range(n)]


def dit_block(x, sc, W: Dict[str, np.ndarray], prefix: str, heads: int, coords=None):
    """x <- x + a1 ⊙ Attn(LN(x)(1+g1)+b1);  x <- x + a2 ⊙ FFN(LN(x)(1+g2)+b2)."""
    sh1, sc1, g1, sh2, sc2, g2 = adaln_chunks(sc, W[prefix + "ada.w"], W[prefix + "ada.b"], 6)
    qn = W.get(prefix + "q_norm.g")
    kn = W.get(prefix + "k_norm.g")
    u = modulate(layernorm(x), sh1, sc1)
    a = self_attention(u, W[prefix + "qkv.w"], W[prefix + "qkv.b"], W[prefix + "proj.w"],
                       W[prefix + "proj.b"], heads, qn, kn, coords)
    x = x + g1[:, None, :] * a
    u = modulate(layernorm(x), sh2, sc2)
    f = ffn(u, W[prefix + "fc1.w"], W[prefix + "fc1.b"], W[prefix + "fc2.w"], W[prefix + "fc2.b"])
    return x + g2[:, None, :] * f


def cross_attention(u, ctx, wq, bq, wkv, bkv, wo, bo, heads: int):
    """Multi-head cross-attention of the tokens u [R, T, d] onto the condition sequence
    ctx [R, S, d] ([DiT-wiki] "조건 주입 방식": t and c embeddings kept as a separate
    sequence, a cross-attention layer added to every block; [Sora-DiT]: a multi-head
    cross-attention layer after the self-attention layer): queries from u, keys and values
    from ctx, per-head softmax attention, heads concatenated, output projection."""
    r, t, d = u.shape
    dh = d // heads
    q = linear(u, wq, bq)
    kv = linear(ctx, wkv, bkv)
    k, v = kv[..., :d], kv[..., d:]
    o = np.zeros((r, t, d), dtype=F64)
    for i in range(r):
        for hd in range(heads):
            sl = slice(hd * dh, (hd + 1) * dh)
            o[i, :, sl] = attention(q[i, :, sl], k[i, :, sl], v[i, :, sl])
    return linear(o, wo, bo)


def plain_block(x, W: Dict[str, np.ndarray], prefix: str, heads: int, coords=None, ctx=None):
    """The block of the in-context and cross-attention designs: a pre-norm transformer block
    with learned LayerNorm affines and no modulation or gate.
        x <- x + Attn(LN1(x));  [x <- x + CrossAttn(LNx(x), ctx)];  x <- x + FFN(LN2(x))."""
    qn = W.get(prefix + "q_norm.g")
    kn = W.get(prefix + "k_norm.g")
    u = layernorm_affine(x, W[prefix + "ln1.g"], W[prefix + "ln1.b"])
    x = x + self_attention(u, W[prefix + "qkv.w"], W[prefix + "qkv.b"], W[prefix + "proj.w"],
                           W[prefix + "proj.b"], heads, qn, kn, coords)
    if ctx is not None:
        u = layernorm_affine(x, W[prefix + "xln.g"], W[prefix + "xln.b"])
        x = x + cross_attention(u, ctx, W[prefix + "xq.w"], W[prefix + "xq.b"], W[prefix + "xkv.w"],
                                W[prefix + "xkv.b"], W[prefix + "xo.w"], W[prefix + "xo.b"], heads)
    u = layernorm_affine(x, W[prefix + "ln2.g"], W[prefix + "ln2.b"])
    return x + ffn(u, W[prefix + "fc1.w"], W[prefix + "fc1.b"], W[prefix + "fc2.w"], W[prefix + "fc2.b"])


def adaln_block(x, sc, W: Dict[str, np.ndarray], prefix: str, heads: int, coords=None):
    """The adaLN design ([DiT-wiki] "조건 주입 방식": LN's scale and shift regressed from the
    t + c embedding instead of learned constants; no residual gate):
        (b1, g1, b2, g2) = Linear(SiLU(c));  x <- x + Attn(LN(x)(1+g1)+b1);  x <- x + FFN(LN(x)(1+g2)+b2)."""
    sh1, sc1, sh2, sc2 = adaln_chunks(sc, W[prefix + "ada.w"], W[prefix + "ada.b"], 4)
    qn = W.get(prefix + "q_norm.g")
    kn = W.get(prefix + "k_norm.g")
    u = modulate(layernorm(x), sh1, sc1)
    x = x + self_attention(u, W[prefix + "qkv.w"], W[prefix + "qkv.b"], W[prefix + "proj.w"],
                           W[prefix + "proj.b"], heads, qn, kn, coords)
    u = modulate(layernorm(x), sh2, sc2)
    return x + ffn(u, W[prefix + "fc1.w"], W[prefix + "fc1.b"], W[prefix + "fc2.w"], W[prefix + "fc2.b"])


def final_layer(x, sc, W):
    """Final modulated LN and linear decoder to pt*ph*pw*C_out per token."""
    shift, scale = adaln_chunks(sc, W["final.ada.w"], W["final.ada.b"], 2)
    return linear(modulate(layernorm(x), shift, scale), W["dec.w"], W["dec.b"])


# --------------------------------------------------------------------------- #
# the whole forward
# --------------------------------------------------------------------------- #
def _as_ncfhw(cfg, x):
    x = np.asarray(x)
    return x if x.ndim == 5 else x[:, :, None]


def embed(cfg, W, x5):
    """Patchify + linear embed (+ 2D sin-cos positions for images)."""
    h = linear(patchify(x5, cfg.patch_t, cfg.patch_h, cfg.patch_w), W["pe.w"], W["pe.b"])
    if cfg.pos_kind == 0:
        gf, gh, gw = cfg.grid
        assert gf == 1
        h = h + pos_embed_sincos_2d(gh, gw, cfg.hidden)[None]
    return h


def forward(cfg, weights: Sequence[np.ndarray] | Dict[str, np.ndarray], x, t, y,
            cfg_scale: Optional[float] = None, force_guidance: bool = False,
            stop_after_block: Optional[int] = None, cfg_channels: Optional[int] = None,
            ffn_fp8: bool = False, attn_fp8: bool = False):
    """ffn_fp8: every block's feed-forward in E4M3 (ffn_e4m3) instead of exact arithmetic.
    attn_fp8: every self-attention's in- and out-projection in E4M3 (linear_e4m3)."""
    prev = (_STATE.get("ffn_fp8", False), _STATE.get("attn_fp8", False))
    _STATE["ffn_fp8"] = bool(ffn_fp8)
    _STATE["attn_fp8"] = bool(attn_fp8)
    try:
        return _forward(cfg, weights, x, t, y, cfg_scale, force_guidance, stop_after_block, cfg_channels)
    finally:
        _STATE["ffn_fp8"], _STATE["attn_fp8"] = prev


def _forward(cfg, weights, x, t, y, cfg_scale, force_guidance, stop_after_block, cfg_channels):
    """Denoiser output for a batch.

    Returns the guided prediction [B, C_out, (F,) H, W] (float64), or, when
    ``stop_after_block`` is k, the residual stream [rows, T, d] after k blocks
    (k = 0: right after the embedding), rows ordered [cond; uncond] if guided.
    Guidance runs when the model is class-conditional and s != 1 (or when
    forced): rows [x; x] with labels [y; null] are evaluated and combined, on every output
    channel or, with ``cfg_channels`` = n > 0, on channels c < n only.
    """
    from_list = not isinstance(weights, dict)
    if from_list:
        from dit_synth import weight_specs  # names only
        W = {n: w for (n, _, _), w in zip(weight_specs(cfg), weights)}
    else:
        W = weights
    s = cfg.cfg_scale if cfg_scale is None else cfg_scale
    x5 = _as_ncfhw(cfg, x)
    b = x5.shape[0]
    guided = cfg.cond_kind == 0 and (force_guidance or s != 1.0)
    t = np.asarray(t)
    if guided:
        x5 = np.concatenate([x5, x5], axis=0)
        t = np.concatenate([t, t], axis=0)
        y = np.concatenate([np.asarray(y), np.full(b, cfg.num_classes, dtype=np.int64)], axis=0)
    kind = getattr(cfg, "block_kind", 0)
    h = embed(cfg, W, x5)
    et, ey = condition_parts(cfg, W, t, y)
    sc = silu(et + ey)
    coords = token_coords(cfg.grid) if cfg.pos_kind == 1 else None
    ctx = None
    if kind == 1:
        # in-context: the two condition embeddings become two extra tokens in front of the
        # patch tokens ([DiT-wiki] "조건 주입 방식": appended like ViT's cls token); they carry
        # no position (3D RoPE, when used, gives them coordinate 0, an identity rotation)
        h = np.concatenate([et[:, None, :], ey[:, None, :], h], axis=1)
        if coords is not None:
            coords = np.concatenate([np.zeros((2, 3), dtype=coords.dtype), coords], axis=0)
    elif kind == 2:
        ctx = np.stack([et, ey], axis=1)   # the separate length-two condition sequence
    if stop_after_block == 0:
        return h
    for i in range(cfg.depth):
        p = f"blocks.{i}."
        if kind == 0:
            h = dit_block(h, sc, W, p, cfg.heads, coords)
        elif kind == 3:
            h = adaln_block(h, sc, W, p, cfg.heads, coords)
        else:
            h = plain_block(h, W, p, cfg.heads, coords, ctx)
        if stop_after_block is not None and i + 1 == stop_after_block:
            return h
    if kind in (1, 2):
        # the condition tokens leave the sequence after the last block; final LN (learned
        # affine) and the linear decoder ([DiT-wiki] "잠재 공간과 패치화": final layer norm,
        # then the linear decoder)
        h = h[:, 2:] if kind == 1 else h
        z = linear(layernorm_affine(h, W["final.ln.g"], W["final.ln.b"]), W["dec.w"], W["dec.b"])
    else:
        z = final_layer(h, sc, W)
    img = unpatchify(z, cfg.out_channels, cfg.grid, cfg.patch_t, cfg.patch_h, cfg.patch_w)
    if guided:
        img = cfg_combine(img[:b], img[b:], s, cfg_channels)
    if img.shape[2] == 1 and np.asarray(x).ndim == 4:
        img = img[:, :, 0]
    return img


def count_forward_macs(cfg, batch: int = 1) -> int:
    """Multiply-adds of one forward (the pages' "Gflops" unit: [DiT-wiki] "모델 크기"
    and "조건 주입 방식" tables count one per multiply-add), obtained by running the
    forward's control flow with the contractions only counted, not computed."""
    from dit_synth import weight_specs  # shapes only
    W = {n: np.zeros(shape, dtype=np.float32) for n, shape, _ in weight_specs(cfg)}
    x = np.zeros(cfg.x_shape(batch), dtype=np.float32)
    t = np.zeros(batch, dtype=np.float32)
    y = np.zeros(batch, dtype=np.int64) if cfg.cond_kind == 0 else np.zeros((batch, cfg.hidden), np.float32)
    reset_mac_counter(dry=True)
    try:
        forward(cfg, W, x, t, y, cfg_scale=1.0)
        return mac_count()
    finally:
        reset_mac_counter(dry=False)
