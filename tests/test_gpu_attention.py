"""The bf16 tensor-core attention kernel on its own, through dit_op_attention_bf16 (GPU only).

Reference: the oracle's softmax attention (float64) on the same bf16-rounded q, k, v, so the
only differences are the kernel's float32 accumulation and its bf16 P and O.  Shapes cover
both head dims with one and many key tiles and a ragged last tile, and inputs crafted so
that the online softmax must move its reference maximum ("확산 트랜스포머", section
"adaLN-Zero": Attn is full multi-head self-attention; section "U-Net과 비교": its cost is
quadratic in the token count).
"""
import numpy as np
import pytest
import torch

from diffusion_transformer_denoiser_dit_b200 import binding
from oracle import dit_oracle as O

pytestmark = pytest.mark.gpu

REL = 1e-2     # bf16 P and bf16 output: ~2^-9 relative per element
MAXN = 3e-2


def padded(x, T, dh):
    """[R*H, T, dh] float -> bf16 [R*H, Tpad, DP] with zero padding (the kernel's q / k layout)."""
    RH = x.shape[0]
    Tpad, DP = (T + 127) // 128 * 128, (dh + 15) // 16 * 16
    out = torch.zeros((RH, Tpad, DP), dtype=torch.bfloat16, device="cuda")
    out[:, :T, :dh] = x.to(torch.bfloat16)
    return out


def run(q, k, v, R, H, T, dh):
    """q, k, v: float32 CUDA [R*H, T, dh].  Returns (kernel output [R, T, H*dh] float64,
    float64 reference on the bf16-rounded inputs, rescale count)."""
    qp, kp, vp = padded(q, T, dh), padded(k, T, dh), padded(v, T, dh)
    vt = vp.transpose(1, 2).contiguous()                     # [R*H, DP, Tpad]
    o = torch.full((R * T, H * dh), float("nan"), dtype=torch.bfloat16, device="cuda")
    counters = torch.zeros(2, dtype=torch.int32, device="cuda")
    binding.attention_bf16(qp, kp, vt, o, R, H, T, dh, counters)
    torch.cuda.synchronize()
    assert int(counters[0].item()) == 0
    got = o.double().cpu().numpy().reshape(R, T, H, dh)
    qd, kd, vd = (a[:, :T, :dh].double().cpu().numpy() for a in (qp, kp, vp))
    want = np.zeros_like(got)
    for rh in range(R * H):
        r, h = divmod(rh, H)
        want[r, :, h] = O.attention(qd[rh], kd[rh], vd[rh])
    return got.reshape(R, T, H * dh), want.reshape(R, T, H * dh), int(counters[1].item())


def check(got, want):
    assert np.all(np.isfinite(got))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    maxn = np.abs(got - want).max() / want.std()
    assert rel <= REL and maxn <= MAXN, (rel, maxn)


@pytest.mark.parametrize("R,H,T,dh", [
    (2, 2, 256, 72),     # two key tiles, one query-tile pair
    (1, 3, 225, 64),     # dh 64, ragged second key tile
    (1, 2, 1024, 64),    # dh 64, eight key tiles, several items per CTA
    (2, 1, 1000, 72),    # dh 72, ragged eighth tile, odd query-tile count
    (1, 1, 4096, 72),    # the video workload's row length
    (3, 1, 129, 64),     # one key past a tile boundary
    (2, 2, 1, 72),       # one token: the output is v
])
def test_attention_matches_definition(R, H, T, dh):
    g = torch.Generator(device="cuda").manual_seed(R * 1000 + T + dh)
    q, k, v = (torch.randn((R * H, T, dh), device="cuda", generator=g) for _ in range(3))
    got, want, events = run(q, k, v, R, H, T, dh)
    check(got, want)
    assert events == 0   # logits of std ~1.4 (log2 units): the row maximum never jumps by 2^8


@pytest.mark.parametrize("dh", [64, 72])
def test_lazy_rescale_path(dh):
    """Keys whose scale grows tile by tile, so each row's maximum climbs by more than 2^8
    several times: the kernel must rescale its running output (and counts that it did)."""
    R, H, T = 1, 2, 1024
    g = torch.Generator(device="cuda").manual_seed(7 + dh)
    q = torch.randn((R * H, T, dh), device="cuda", generator=g)
    k = torch.randn((R * H, T, dh), device="cuda", generator=g)
    v = torch.randn((R * H, T, dh), device="cuda", generator=g)
    tile = torch.arange(T, device="cuda") // 128
    k *= (0.5 + 1.0 * tile.float())[None, :, None]
    got, want, events = run(q, k, v, R, H, T, dh)
    check(got, want)
    assert events >= R * H * (T // 32)   # every warp of query rows rescaled at least once
