"""The C-ABI library loads and exports every symbol include/dit.h declares; host-side
argument checks reject bad configurations before any CUDA call (CPU only)."""
import ctypes
import os
import re

import numpy as np
import pytest

import dit_synth as S
from diffusion_transformer_denoiser_dit_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "dit.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dit_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    lib = binding.load()
    declared = header_functions()
    assert len(declared) >= 10
    assert sorted(binding.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_weight_count_matches_generator():
    lib = binding.load()
    for cfg in S.STANDARD:
        for kind in (S.BLOCK_ADALN_ZERO, S.BLOCK_IN_CONTEXT, S.BLOCK_CROSS_ATTN, S.BLOCK_ADALN):
            c = binding.make_config(cfg.with_(block_kind=kind))
            assert lib.dit_weight_count(ctypes.byref(c)) == len(S.weight_specs(cfg.with_(block_kind=kind)))


def _create(cfg, weights=None, n=None):
    lib = binding.load()
    c = binding.make_config(cfg)
    if weights is None:
        weights = [np.zeros(1, np.float32)] * len(S.weight_specs(cfg))
    ptrs = (ctypes.c_void_p * len(weights))(*[w.ctypes.data for w in weights])
    h = ctypes.c_void_p()
    return lib.dit_create(ctypes.byref(c), ptrs, len(weights) if n is None else n, ctypes.byref(h)), h


@pytest.mark.parametrize("change,code", [
    (dict(hidden=0), binding.DIT_ERR_INVALID_ARG),
    (dict(heads=5), binding.DIT_ERR_INVALID_ARG),           # 384 % 5 != 0
    (dict(height=30), binding.DIT_ERR_INVALID_ARG),         # patch 8 does not divide 30
    (dict(dtype=7), binding.DIT_ERR_INVALID_ARG),
    (dict(batch=0), binding.DIT_ERR_INVALID_ARG),
    (dict(freq_dim=255), binding.DIT_ERR_INVALID_ARG),
    (dict(block_kind=4), binding.DIT_ERR_INVALID_ARG),
    (dict(ffn_fp8=2), binding.DIT_ERR_INVALID_ARG),
    (dict(ffn_fp8=1), binding.DIT_ERR_UNSUPPORTED),          # FP8 feed-forward needs the bf16 path
    (dict(attn_fp8=3), binding.DIT_ERR_INVALID_ARG),
    (dict(attn_fp8=1), binding.DIT_ERR_UNSUPPORTED),         # FP8 attention projections need the bf16 path
    (dict(heads=12), binding.DIT_ERR_UNSUPPORTED),           # head dim 32
    (dict(hidden=2048, heads=32, mlp_hidden=8192), binding.DIT_ERR_UNSUPPORTED),  # hidden > 1536
])
def test_bad_configs_rejected_on_host(change, code):
    cfg = S.DIT_S8_F32.with_(**change)
    rc, h = _create(cfg)
    assert rc == code
    assert not h.value


def test_wrong_weight_count_rejected():
    rc, _ = _create(S.DIT_S8_F32, n=3)
    assert rc == binding.DIT_ERR_INVALID_ARG


def test_no_device_reported_without_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, _ = _create(S.DIT_S8_F32.with_(depth=1))
    assert rc == binding.DIT_ERR_NO_DEVICE


def test_status_strings():
    lib = binding.load()
    for code in range(8):
        assert lib.dit_status_string(code).decode().startswith("DIT_")
