"""dit_condition_static — the entry point for callers that cannot allocate device
memory (its scratch is a fixed array inside the library) — must give the same
condition vector as the handle-based path, call after call."""
import numpy as np
import pytest
import torch

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding
from diffusion_transformer_denoiser_dit_b200.binding import DiT

pytestmark = pytest.mark.gpu


def _static_condition(lib, cfg, Wd, t, y, guided, status):
    dev = {k: torch.from_numpy(np.ascontiguousarray(Wd[k])).cuda() for k in ("t.w1", "t.b1", "t.w2", "t.b2", "y.table")}
    B = t.shape[0]
    rows = 2 * B if guided else B
    c = torch.full((rows, cfg.hidden), float("nan"), device="cuda")
    rc = lib.dit_condition_static(t.data_ptr(), y.data_ptr(), B, int(guided), dev["t.w1"].data_ptr(),
                                  dev["t.b1"].data_ptr(), dev["t.w2"].data_ptr(), dev["t.b2"].data_ptr(),
                                  dev["y.table"].data_ptr(), cfg.cond_kind, cfg.num_classes, cfg.freq_dim,
                                  cfg.hidden, cfg.t_scale, c.data_ptr(), status.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return rc, c


def test_static_scratch_condition_matches_handle_path_twice():
    cfg = S.DIT_XL2_CFG256.with_(depth=1, batch=6, index=-1)
    W = S.make_weights(cfg)
    Wd = S.weight_dict(cfg, W)
    model = DiT(cfg, W)
    lib = binding.load()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    for call in range(2):   # the second call must not see the first call's leftovers
        inp = S.make_inputs(cfg, seed=777 + call, batch=cfg.batch - call)
        t = torch.from_numpy(inp["t"]).cuda()
        y = torch.from_numpy(inp["y"]).cuda()
        want = model.debug_condition(t, y, cfg.cfg_scale)
        torch.cuda.synchronize()
        rc, got = _static_condition(lib, cfg, Wd, t, y, True, status)
        assert rc == binding.DIT_OK
        assert torch.isfinite(got).all()
        assert torch.allclose(got, want, rtol=1e-6, atol=1e-6), (got - want).abs().max().item()
    assert int(status[0].item()) == 0
    model.close()


def test_static_scratch_refuses_sizes_beyond_its_limit():
    cfg = S.DIT_XL2_CFG256.with_(depth=1, batch=65, index=-1)   # 130 guided rows > 128
    Wd = S.weight_dict(cfg, S.make_weights(cfg))
    inp = S.make_inputs(cfg)
    t = torch.from_numpy(inp["t"]).cuda()
    y = torch.from_numpy(inp["y"]).cuda()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    rc, got = _static_condition(binding.load(), cfg, Wd, t, y, True, status)
    assert rc == binding.DIT_ERR_INVALID_ARG
    assert torch.isnan(got).all()   # nothing was launched
