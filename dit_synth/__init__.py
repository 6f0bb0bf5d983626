"""Seeded synthetic workloads for the DiT denoiser forward pass.

This module names model shapes, lays out the weight list in the library's fixed
order, and draws random numbers.  It holds none of the forward pass's arithmetic,
so both the CUDA path and the CPU oracle can consume what it produces without
sharing any computation.

Workload recipe (stands in for class-conditional ImageNet latents and for
text-to-video latents, neither of which is available offline):
  * latents x ~ N(0, 1) float32, NCHW (images) or NCFHW (video);
  * image timesteps: integers uniform in [0, 1000) stored as float32;
    video timesteps: t ~ U(0, 1) float32;
  * class labels uniform in [0, 1000) (int32); the null label is num_classes;
  * pooled-text condition vector ~ N(0, 1) float32 [B, hidden] (video);
  * every parameter tensor ~ N(0, 0.02) float32, biases included, except the
    QK-RMSNorm gains, which are 1.0;
  * weights seed = 1000 + config index, inputs seed = 2000 + config index.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, List, Tuple

import numpy as np

DTYPE_F32, DTYPE_BF16 = 0, 1
POS_SINCOS2D, POS_ROPE3D = 0, 1
COND_CLASS, COND_VECTOR = 0, 1
# how the condition enters the blocks (the four designs of the DiT paper's comparison)
BLOCK_ADALN_ZERO, BLOCK_IN_CONTEXT, BLOCK_CROSS_ATTN, BLOCK_ADALN = 0, 1, 2, 3


@dataclass(frozen=True)
class DiTConfig:
    """One model + workload.  Field meanings match ``dit_config`` in include/dit.h."""

    name: str
    dtype: int
    in_channels: int
    frames: int
    height: int
    width: int
    patch_t: int
    patch_h: int
    patch_w: int
    hidden: int
    depth: int
    heads: int
    mlp_hidden: int
    learn_sigma: int
    pos_kind: int
    qk_norm: int
    cond_kind: int
    num_classes: int
    freq_dim: int
    t_scale: float
    batch: int
    cfg_scale: float
    index: int = -1  # position in the standard workload list (seeds); -1 = ad hoc
    block_kind: int = BLOCK_ADALN_ZERO
    ffn_fp8: int = 0   # 1: the feed-forward matmuls on FP8 E4M3 operands
    attn_fp8: int = 0  # 1: the self-attention's in- and out-projection on FP8 E4M3 operands

    # ---- derived shapes (no arithmetic of the method) ----
    @property
    def grid(self) -> Tuple[int, int, int]:
        return (self.frames // self.patch_t, self.height // self.patch_h, self.width // self.patch_w)

    @property
    def tokens(self) -> int:
        g = self.grid
        return g[0] * g[1] * g[2]

    @property
    def cond_tokens(self) -> int:
        """Condition tokens ahead of the patch tokens in each row (in-context design: 2)."""
        return 2 if self.block_kind == BLOCK_IN_CONTEXT else 0

    @property
    def seq_tokens(self) -> int:
        """Tokens per row inside the blocks."""
        return self.tokens + self.cond_tokens

    @property
    def mod_per_block(self) -> int:
        """Modulation vectors regressed per block: 6 (adaLN-Zero), 4 (adaLN), 0 (others)."""
        return {BLOCK_ADALN_ZERO: 6, BLOCK_ADALN: 4}.get(self.block_kind, 0)

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads

    @property
    def out_channels(self) -> int:
        return 2 * self.in_channels if self.learn_sigma else self.in_channels

    @property
    def patch_dim(self) -> int:
        return self.in_channels * self.patch_t * self.patch_h * self.patch_w

    @property
    def out_dim(self) -> int:
        return self.patch_t * self.patch_h * self.patch_w * self.out_channels

    @property
    def is_video(self) -> bool:
        return self.frames > 1 or self.patch_t > 1 or self.pos_kind == POS_ROPE3D

    @property
    def guided(self) -> bool:
        return self.cond_kind == COND_CLASS and self.cfg_scale != 1.0

    @property
    def rows(self) -> int:
        return 2 * self.batch if self.guided else self.batch

    def x_shape(self, batch: int | None = None) -> Tuple[int, ...]:
        b = self.batch if batch is None else batch
        if self.is_video:
            return (b, self.in_channels, self.frames, self.height, self.width)
        return (b, self.in_channels, self.height, self.width)

    def out_shape(self, batch: int | None = None) -> Tuple[int, ...]:
        b = self.batch if batch is None else batch
        if self.is_video:
            return (b, self.out_channels, self.frames, self.height, self.width)
        return (b, self.out_channels, self.height, self.width)

    def with_(self, **kw) -> "DiTConfig":
        return replace(self, **kw)


def _image(name, dtype, size, patch, hidden, depth, heads, batch, cfg_scale, index, height=None):
    return DiTConfig(name=name, dtype=dtype, in_channels=4, frames=1, height=height or size, width=size,
                     patch_t=1, patch_h=patch, patch_w=patch, hidden=hidden, depth=depth, heads=heads,
                     mlp_hidden=4 * hidden, learn_sigma=1, pos_kind=POS_SINCOS2D, qk_norm=0,
                     cond_kind=COND_CLASS, num_classes=1000, freq_dim=256, t_scale=1.0,
                     batch=batch, cfg_scale=cfg_scale, index=index)


# The five standard workloads, in order.
DIT_S8_F32 = _image("DiT-S/8 fp32", DTYPE_F32, 32, 8, 384, 12, 6, 2, 1.0, 0)
DIT_B4_BF16 = _image("DiT-B/4 bf16", DTYPE_BF16, 32, 4, 768, 12, 12, 8, 1.0, 1)
DIT_XL2_CFG256 = _image("DiT-XL/2 CFG 256px bf16", DTYPE_BF16, 32, 2, 1152, 28, 16, 16, 1.5, 2)
DIT_XL2_CFG512 = _image("DiT-XL/2 CFG 512px bf16", DTYPE_BF16, 64, 2, 1152, 28, 16, 8, 1.5, 3)
VIDEO_RF = DiTConfig(name="video RF DiT bf16", dtype=DTYPE_BF16, in_channels=16, frames=16, height=32,
                     width=32, patch_t=1, patch_h=2, patch_w=2, hidden=1152, depth=28, heads=16,
                     mlp_hidden=4608, learn_sigma=0, pos_kind=POS_ROPE3D, qk_norm=1,
                     cond_kind=COND_VECTOR, num_classes=0, freq_dim=256, t_scale=1000.0,
                     batch=2, cfg_scale=1.0, index=4)

STANDARD = [DIT_S8_F32, DIT_B4_BF16, DIT_XL2_CFG256, DIT_XL2_CFG512, VIDEO_RF]


def weights_seed(cfg: DiTConfig) -> int:
    return 1000 + (cfg.index if cfg.index >= 0 else 50)


def inputs_seed(cfg: DiTConfig) -> int:
    return 2000 + (cfg.index if cfg.index >= 0 else 50)


def weight_specs(cfg: DiTConfig) -> List[Tuple[str, Tuple[int, ...], str]]:
    """(name, shape, init) for every weight, in the library's fixed order.

    Linear weights are row-major [out, in].  ``init`` is "normal" (N(0, std)), "one"
    (filled with 1.0, used for the QK-RMSNorm gains) or "gain" (1 + N(0, 0.1), the learned
    LayerNorm gains of the in-context and cross-attention designs).
    """
    d, f, m = cfg.hidden, cfg.freq_dim, cfg.mlp_hidden
    dh = cfg.head_dim
    kind = cfg.block_kind
    s: List[Tuple[str, Tuple[int, ...], str]] = [
        ("pe.w", (d, cfg.patch_dim), "normal"), ("pe.b", (d,), "normal"),
        ("t.w1", (d, f), "normal"), ("t.b1", (d,), "normal"),
        ("t.w2", (d, d), "normal"), ("t.b2", (d,), "normal"),
    ]
    if cfg.cond_kind == COND_CLASS:
        s.append(("y.table", (cfg.num_classes + 1, d), "normal"))
    modulated = kind in (BLOCK_ADALN_ZERO, BLOCK_ADALN)
    for i in range(cfg.depth):
        p = f"blocks.{i}."
        if modulated:
            nm = cfg.mod_per_block
            s += [(p + "ada.w", (nm * d, d), "normal"), (p + "ada.b", (nm * d,), "normal")]
        else:
            s += [(p + "ln1.g", (d,), "gain"), (p + "ln1.b", (d,), "normal")]
        s += [(p + "qkv.w", (3 * d, d), "normal"), (p + "qkv.b", (3 * d,), "normal")]
        if cfg.qk_norm:
            s += [(p + "q_norm.g", (dh,), "one"), (p + "k_norm.g", (dh,), "one")]
        s += [(p + "proj.w", (d, d), "normal"), (p + "proj.b", (d,), "normal")]
        if kind == BLOCK_CROSS_ATTN:
            s += [(p + "xln.g", (d,), "gain"), (p + "xln.b", (d,), "normal"),
                  (p + "xq.w", (d, d), "normal"), (p + "xq.b", (d,), "normal"),
                  (p + "xkv.w", (2 * d, d), "normal"), (p + "xkv.b", (2 * d,), "normal"),
                  (p + "xo.w", (d, d), "normal"), (p + "xo.b", (d,), "normal")]
        if not modulated:
            s += [(p + "ln2.g", (d,), "gain"), (p + "ln2.b", (d,), "normal")]
        s += [(p + "fc1.w", (m, d), "normal"), (p + "fc1.b", (m,), "normal"),
              (p + "fc2.w", (d, m), "normal"), (p + "fc2.b", (d,), "normal")]
    if modulated:
        s += [("final.ada.w", (2 * d, d), "normal"), ("final.ada.b", (2 * d,), "normal")]
    else:
        s += [("final.ln.g", (d,), "gain"), ("final.ln.b", (d,), "normal")]
    s += [("dec.w", (cfg.out_dim, d), "normal"), ("dec.b", (cfg.out_dim,), "normal")]
    return s


def make_weights(cfg: DiTConfig, seed: int | None = None, std: float = 0.02) -> List[np.ndarray]:
    """Draw every weight tensor in ``weight_specs`` order from one PCG64 stream."""
    rng = np.random.default_rng(weights_seed(cfg) if seed is None else seed)
    out = []
    for _, shape, init in weight_specs(cfg):
        if init == "one":
            a = np.ones(shape, dtype=np.float32)
        elif init == "gain":
            a = np.float32(1.0) + np.float32(0.1) * rng.standard_normal(shape, dtype=np.float32)
        else:
            a = rng.standard_normal(shape, dtype=np.float32)
            a *= np.float32(std)
        out.append(np.ascontiguousarray(a))
    return out


def weight_dict(cfg: DiTConfig, weights: List[np.ndarray]) -> Dict[str, np.ndarray]:
    return {name: w for (name, _, _), w in zip(weight_specs(cfg), weights)}


def set_adaln(cfg: DiTConfig, weights: List[np.ndarray], *, zero: bool = False,
              gate_bias: float | None = None) -> List[np.ndarray]:
    """Copy of ``weights`` with the per-block modulation layers edited.

    zero=True zeroes every block's ada.w and ada.b (the adaLN-Zero initial state);
    gate_bias=v sets the two gate slices [2d,3d) and [5d,6d) of every ada.b to v,
    so that the blocks change the residual stream strongly.
    """
    d = cfg.hidden
    out = [w.copy() for w in weights]
    names = [n for n, _, _ in weight_specs(cfg)]
    if cfg.block_kind != BLOCK_ADALN_ZERO:
        if cfg.block_kind == BLOCK_ADALN and zero:
            for i in range(cfg.depth):
                out[names.index(f"blocks.{i}.ada.w")][...] = 0.0
                out[names.index(f"blocks.{i}.ada.b")][...] = 0.0
        return out   # gates exist only in the adaLN-Zero design
    for i in range(cfg.depth):
        wi = names.index(f"blocks.{i}.ada.w")
        bi = names.index(f"blocks.{i}.ada.b")
        if zero:
            out[wi][...] = 0.0
            out[bi][...] = 0.0
        if gate_bias is not None:
            out[bi][2 * d:3 * d] = gate_bias
            out[bi][5 * d:6 * d] = gate_bias
    return out


def make_inputs(cfg: DiTConfig, seed: int | None = None, batch: int | None = None) -> Dict[str, np.ndarray]:
    """x, t, y for one forward call (y is int32 labels or a float32 text vector)."""
    rng = np.random.default_rng(inputs_seed(cfg) if seed is None else seed)
    b = cfg.batch if batch is None else batch
    x = rng.standard_normal(cfg.x_shape(b), dtype=np.float32)
    if cfg.t_scale == 1.0:
        t = rng.integers(0, 1000, size=b).astype(np.float32)
    else:
        t = rng.random(b, dtype=np.float32)
    if cfg.cond_kind == COND_CLASS:
        y = rng.integers(0, cfg.num_classes, size=b).astype(np.int32)
    else:
        y = rng.standard_normal((b, cfg.hidden), dtype=np.float32)
    return {"x": np.ascontiguousarray(x), "t": t, "y": np.ascontiguousarray(y)}

