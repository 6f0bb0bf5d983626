"""An independent float64 CPU restatement of the DiT forward built from torch.nn layers.

Test-only.  It pins the oracle's wiring against stock library layers: the patch
embedding is a Conv with kernel = stride = patch (the pages' remark that patchify
is one such convolution), attention is ``nn.MultiheadAttention`` (in-projection
[q|k|v] with bias, out-projection with bias) or ``scaled_dot_product_attention``,
LayerNorm is ``nn.LayerNorm(elementwise_affine=False, eps=1e-6)``, the FFN uses
``nn.GELU(approximate="tanh")``, unpatchify is an einops rearrangement of the
literal p x p x C_out token vector.  The fixed tables (timestep sinusoid, 2D
sin-cos positions, RoPE rotation) are taken from the oracle because each is
pinned on its own by invariants in test_oracle_pins.py; the tokens' RoPE
coordinates are derived here from the patch layout, not taken from the oracle.
"""
from __future__ import annotations

import einops
import numpy as np
import torch
import torch.nn as nn
import torch.nn.functional as F

from oracle import dit_oracle as O

T64 = torch.float64


def _t(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


class RefBlock(nn.Module):
    """kind 0: adaLN-Zero (six modulation vectors incl. gates); 3: adaLN (four, no gates);
    1: in-context and 2: cross-attention (learned LayerNorm affines, no modulation)."""

    def __init__(self, d, heads, mlp, qk_norm, kind=0):
        super().__init__()
        self.heads = heads
        self.qk_norm = qk_norm
        self.kind = kind
        affine = kind in (1, 2)
        self.norm1 = nn.LayerNorm(d, elementwise_affine=affine, eps=1e-6)
        self.norm2 = nn.LayerNorm(d, elementwise_affine=affine, eps=1e-6)
        self.attn = nn.MultiheadAttention(d, heads, batch_first=True)
        self.mlp = nn.Sequential(nn.Linear(d, mlp), nn.GELU(approximate="tanh"), nn.Linear(mlp, d))
        if kind in (0, 3):
            self.ada = nn.Sequential(nn.SiLU(), nn.Linear(d, (6 if kind == 0 else 4) * d))
        if kind == 2:
            self.normx = nn.LayerNorm(d, eps=1e-6)
            self.xattn = nn.MultiheadAttention(d, heads, batch_first=True)
        self.qg = None
        self.kg = None

    def load(self, W, p):
        with torch.no_grad():
            if self.kind in (0, 3):
                self.ada[1].weight.copy_(_t(W[p + "ada.w"]))
                self.ada[1].bias.copy_(_t(W[p + "ada.b"]))
            else:
                self.norm1.weight.copy_(_t(W[p + "ln1.g"]))
                self.norm1.bias.copy_(_t(W[p + "ln1.b"]))
                self.norm2.weight.copy_(_t(W[p + "ln2.g"]))
                self.norm2.bias.copy_(_t(W[p + "ln2.b"]))
            if self.kind == 2:
                self.normx.weight.copy_(_t(W[p + "xln.g"]))
                self.normx.bias.copy_(_t(W[p + "xln.b"]))
                self.xattn.in_proj_weight.copy_(torch.cat([_t(W[p + "xq.w"]), _t(W[p + "xkv.w"])]))
                self.xattn.in_proj_bias.copy_(torch.cat([_t(W[p + "xq.b"]), _t(W[p + "xkv.b"])]))
                self.xattn.out_proj.weight.copy_(_t(W[p + "xo.w"]))
                self.xattn.out_proj.bias.copy_(_t(W[p + "xo.b"]))
            self.attn.in_proj_weight.copy_(_t(W[p + "qkv.w"]))
            self.attn.in_proj_bias.copy_(_t(W[p + "qkv.b"]))
            self.attn.out_proj.weight.copy_(_t(W[p + "proj.w"]))
            self.attn.out_proj.bias.copy_(_t(W[p + "proj.b"]))
            self.mlp[0].weight.copy_(_t(W[p + "fc1.w"]))
            self.mlp[0].bias.copy_(_t(W[p + "fc1.b"]))
            self.mlp[2].weight.copy_(_t(W[p + "fc2.w"]))
            self.mlp[2].bias.copy_(_t(W[p + "fc2.b"]))
        if self.qk_norm:
            self.qg = _t(W[p + "q_norm.g"])
            self.kg = _t(W[p + "k_norm.g"])

    def _attend(self, h, coords):
        if not self.qk_norm and coords is None:
            return self.attn(h, h, h, need_weights=False)[0]
        # video path: explicit projections so QK-RMSNorm and RoPE can sit between them
        r, t, d = h.shape
        dh = d // self.heads
        qkv = F.linear(h, self.attn.in_proj_weight, self.attn.in_proj_bias)
        q, k, v = qkv.split(d, dim=-1)
        q = q.view(r, t, self.heads, dh).transpose(1, 2)
        k = k.view(r, t, self.heads, dh).transpose(1, 2)
        v = v.view(r, t, self.heads, dh).transpose(1, 2)
        if self.qk_norm:
            q = F.rms_norm(q, (dh,), self.qg, eps=1e-6)
            k = F.rms_norm(k, (dh,), self.kg, eps=1e-6)
        if coords is not None:
            q = torch.stack([torch.stack([_t(O.rope_3d(q[i, j].numpy(), coords)) for j in range(self.heads)])
                             for i in range(r)])
            k = torch.stack([torch.stack([_t(O.rope_3d(k[i, j].numpy(), coords)) for j in range(self.heads)])
                             for i in range(r)])
        o = F.scaled_dot_product_attention(q, k, v)
        o = o.transpose(1, 2).reshape(r, t, d)
        return self.attn.out_proj(o)

    def forward(self, x, c, coords=None, ctx=None):
        if self.kind == 0:
            sh1, sc1, g1, sh2, sc2, g2 = self.ada(c).chunk(6, dim=1)
            h = self.norm1(x) * (1 + sc1[:, None]) + sh1[:, None]
            x = x + g1[:, None] * self._attend(h, coords)
            h = self.norm2(x) * (1 + sc2[:, None]) + sh2[:, None]
            return x + g2[:, None] * self.mlp(h)
        if self.kind == 3:
            sh1, sc1, sh2, sc2 = self.ada(c).chunk(4, dim=1)
            x = x + self._attend(self.norm1(x) * (1 + sc1[:, None]) + sh1[:, None], coords)
            return x + self.mlp(self.norm2(x) * (1 + sc2[:, None]) + sh2[:, None])
        x = x + self._attend(self.norm1(x), coords)
        if self.kind == 2:
            x = x + self.xattn(self.normx(x), ctx, ctx, need_weights=False)[0]
        return x + self.mlp(self.norm2(x))


def conv_token_coords(cfg, extent):
    """(frame, row, col) of every token, read off the tokenisation itself: three planes holding
    each latent element's own frame, row and column index go through the same stride-p
    pooling and flatten(2) as the patch tokens, so token tau gets the coordinate of the patch it
    came from (divided by the patch extent)."""
    F_, H, W = (int(e) for e in extent)
    axes = torch.meshgrid(torch.arange(F_, dtype=T64), torch.arange(H, dtype=T64), torch.arange(W, dtype=T64),
                          indexing="ij")
    k = (cfg.patch_t, cfg.patch_h, cfg.patch_w)
    pooled = F.avg_pool3d(torch.stack(axes)[None], k, stride=k).flatten(2)[0]   # [3, T] patch centres
    low = pooled - (torch.tensor(k, dtype=T64)[:, None] - 1) / 2                 # patch start
    return (low / torch.tensor(k, dtype=T64)[:, None]).round().to(torch.int64).T.numpy()


def reference_forward(cfg, weights_by_name, x, t, y, cfg_scale=None, force_guidance=False):
    W = weights_by_name
    d = cfg.hidden
    s = cfg.cfg_scale if cfg_scale is None else cfg_scale
    x = _t(x)
    video = x.ndim == 5
    b = x.shape[0]
    guided = cfg.cond_kind == 0 and (force_guidance or s != 1.0)
    t = np.asarray(t)
    if guided:
        x = torch.cat([x, x])
        t = np.concatenate([t, t])
        y = np.concatenate([np.asarray(y), np.full(b, cfg.num_classes)])
    with torch.no_grad():
        if video:
            conv = nn.Conv3d(cfg.in_channels, d, (cfg.patch_t, cfg.patch_h, cfg.patch_w),
                             stride=(cfg.patch_t, cfg.patch_h, cfg.patch_w)).to(T64)
            conv.weight.copy_(_t(W["pe.w"]).view(d, cfg.in_channels, cfg.patch_t, cfg.patch_h, cfg.patch_w))
        else:
            conv = nn.Conv2d(cfg.in_channels, d, cfg.patch_h, stride=cfg.patch_h).to(T64)
            conv.weight.copy_(_t(W["pe.w"]).view(d, cfg.in_channels, cfg.patch_h, cfg.patch_w))
        conv.bias.copy_(_t(W["pe.b"]))
        h = conv(x).flatten(2).transpose(1, 2)
        if cfg.pos_kind == 0:
            gf, gh, gw = cfg.grid
            h = h + _t(O.pos_embed_sincos_2d(gh, gw, d))[None]

        tmlp = nn.Sequential(nn.Linear(cfg.freq_dim, d), nn.SiLU(), nn.Linear(d, d)).to(T64)
        tmlp[0].weight.copy_(_t(W["t.w1"])); tmlp[0].bias.copy_(_t(W["t.b1"]))
        tmlp[2].weight.copy_(_t(W["t.w2"])); tmlp[2].bias.copy_(_t(W["t.b2"]))
        et = tmlp(_t(O.timestep_embedding(t, cfg.freq_dim, cfg.t_scale)))
        if cfg.cond_kind == 0:
            emb = nn.Embedding(cfg.num_classes + 1, d).to(T64)
            emb.weight.copy_(_t(W["y.table"]))
            ey = emb(torch.as_tensor(np.asarray(y, dtype=np.int64)))
        else:
            ey = _t(y)
        c = et + ey
        kind = cfg.block_kind

        coords = conv_token_coords(cfg, x.shape[2:]) if cfg.pos_kind == 1 else None
        ctx = None
        if kind == 1:    # two condition tokens in front, without position
            h = torch.cat([et[:, None], ey[:, None], h], dim=1)
            if coords is not None:
                coords = np.concatenate([np.zeros((2, 3), dtype=coords.dtype), coords])
        elif kind == 2:  # a separate two-token condition sequence
            ctx = torch.stack([et, ey], dim=1)
        for i in range(cfg.depth):
            blk = RefBlock(d, cfg.heads, cfg.mlp_hidden, cfg.qk_norm, kind).to(T64)
            blk.load(W, f"blocks.{i}.")
            h = blk(h, c, coords, ctx)

        dec = nn.Linear(d, cfg.out_dim).to(T64)
        dec.weight.copy_(_t(W["dec.w"])); dec.bias.copy_(_t(W["dec.b"]))
        if kind in (1, 2):
            norm = nn.LayerNorm(d, eps=1e-6).to(T64)
            norm.weight.copy_(_t(W["final.ln.g"])); norm.bias.copy_(_t(W["final.ln.b"]))
            z = dec(norm(h[:, 2:] if kind == 1 else h))
        else:
            fada = nn.Sequential(nn.SiLU(), nn.Linear(d, 2 * d)).to(T64)
            fada[1].weight.copy_(_t(W["final.ada.w"])); fada[1].bias.copy_(_t(W["final.ada.b"]))
            shift, scale = fada(c).chunk(2, dim=1)
            norm = nn.LayerNorm(d, elementwise_affine=False, eps=1e-6)
            z = dec(norm(h) * (1 + scale[:, None]) + shift[:, None])
        gf, gh, gw = cfg.grid
        img = einops.rearrange(z, "n (f h w) (a p q c) -> n c (f a) (h p) (w q)", f=gf, h=gh, w=gw,
                               a=cfg.patch_t, p=cfg.patch_h, q=cfg.patch_w, c=cfg.out_channels)
        if guided:
            img = img[b:] + s * (img[:b] - img[b:])
        if not video:
            img = img[:, :, 0]
        return img.numpy()
