"""ctypes binding of libdit_b200.so (include/dit.h).

Argument marshalling only: every step of the forward runs in the library's CUDA
kernels.  torch provides device memory and streams.  If the library is missing or
cannot be loaded, every call raises; there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_uint16, c_void_p
from typing import Optional, Sequence

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdit_b200.so")

DIT_OK, DIT_ERR_INVALID_ARG, DIT_ERR_UNSUPPORTED, DIT_ERR_OOM, DIT_ERR_CUDA = 0, 1, 2, 3, 4
DIT_ERR_DEVICE_TIMEOUT, DIT_ERR_BAD_LABEL, DIT_ERR_NO_DEVICE = 5, 6, 7
DIT_OPT_FORCE_GUIDANCE, DIT_OPT_USE_GRAPH, DIT_OPT_OVERLAP_LAUNCH, DIT_OPT_CFG_CHANNELS = 1, 2, 3, 4
DIT_OPT_REPEAT_KIND, DIT_OPT_SPLIT_K, DIT_OPT_PAIR_GEMM = 5, 6, 7
DIT_SAMPLER_DDIM, DIT_SAMPLER_EULER = 0, 1

# every exported symbol declared in include/dit.h
EXPORTS = [
    "dit_create", "dit_weight_count", "dit_forward", "dit_forward_host", "dit_sync_status", "dit_last_error",
    "dit_status_string", "dit_destroy", "dit_set_option", "dit_debug_residual", "dit_debug_condition",
    "dit_debug_wait_probe", "dit_op_linear_bf16", "dit_forward_launch_count", "dit_profile_enable",
    "dit_profile_read", "dit_condition_static", "dit_op_linear_bf16_pair", "dit_sampler_step", "dit_sample",
    "dit_op_attention_bf16", "dit_debug_attention_rescales", "dit_op_linear_e4m3",
]

KERNEL_KINDS = ["cond", "adaln", "patch", "ln", "qkv", "attn", "proj", "fc1", "fc2", "decode", "sampler"]


class DitConfig(ctypes.Structure):
    _fields_ = [("dtype", c_int), ("in_channels", c_int), ("frames", c_int), ("height", c_int), ("width", c_int),
                ("patch_t", c_int), ("patch_h", c_int), ("patch_w", c_int), ("hidden", c_int), ("depth", c_int),
                ("heads", c_int), ("mlp_hidden", c_int), ("learn_sigma", c_int), ("pos_kind", c_int),
                ("qk_norm", c_int), ("cond_kind", c_int), ("num_classes", c_int), ("freq_dim", c_int),
                ("max_batch", c_int), ("t_scale", c_float), ("block_kind", c_int), ("ffn_fp8", c_int),
                ("attn_fp8", c_int)]


class DitError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


_LIB = None


def load() -> ctypes.CDLL:
    """Load the library (raises if it was not built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m diffusion_transformer_denoiser_dit_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "dit_create": (c_int, [POINTER(DitConfig), POINTER(c_void_p), c_int, POINTER(c_void_p)]),
        "dit_weight_count": (c_int, [POINTER(DitConfig)]),
        "dit_forward": (c_int, [P, P, P, P, c_int, c_float, P, P]),
        "dit_forward_host": (c_int, [P, P, P, P, c_int, c_float, P, P]),
        "dit_sampler_step": (c_int, [P, c_int, P, P, c_int, c_float, c_float, P, P]),
        "dit_sample": (c_int, [P, c_int, P, P, c_int, c_float, c_int, POINTER(c_float), POINTER(c_float), P]),
        "dit_sync_status": (c_int, [P]),
        "dit_last_error": (ctypes.c_char_p, [P]),
        "dit_status_string": (ctypes.c_char_p, [c_int]),
        "dit_destroy": (None, [P]),
        "dit_set_option": (c_int, [P, c_int, c_int]),
        "dit_debug_residual": (c_int, [P, P, P, P, c_int, c_float, c_int, P, P]),
        "dit_debug_condition": (c_int, [P, P, P, c_int, c_float, P, P]),
        "dit_debug_wait_probe": (c_int, [P, c_int, P]),
        "dit_op_linear_bf16": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, P]),
        "dit_op_linear_bf16_pair": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, P]),
        "dit_forward_launch_count": (c_int, [P, c_int, c_float]),
        "dit_profile_enable": (c_int, [P, c_int]),
        "dit_profile_read": (c_int, [P, POINTER(c_float), POINTER(c_int)]),
        "dit_condition_static": (c_int, [P, P, c_int, c_int, P, P, P, P, P, c_int, c_int, c_int, c_int, c_float,
                                         P, P, P]),
        "dit_op_attention_bf16": (c_int, [P, P, P, P, c_int, c_int, c_int, c_int, P, P]),
        "dit_debug_attention_rescales": (c_int, [P, POINTER(ctypes.c_longlong)]),
        "dit_op_linear_e4m3": (c_int, [P, P, P, P, P, P, c_int, c_int, c_int, c_int, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def make_config(cfg, max_batch: Optional[int] = None) -> DitConfig:
    """dit_config from any object with the same field names (e.g. dit_synth.DiTConfig)."""
    mb = max_batch if max_batch is not None else cfg.batch
    return DitConfig(cfg.dtype, cfg.in_channels, cfg.frames, cfg.height, cfg.width, cfg.patch_t, cfg.patch_h,
                     cfg.patch_w, cfg.hidden, cfg.depth, cfg.heads, cfg.mlp_hidden, cfg.learn_sigma, cfg.pos_kind,
                     cfg.qk_norm, cfg.cond_kind, cfg.num_classes, cfg.freq_dim, mb, float(cfg.t_scale),
                     int(getattr(cfg, "block_kind", 0)), int(getattr(cfg, "ffn_fp8", 0)),
                     int(getattr(cfg, "attn_fp8", 0)))


def status_string(code: int) -> str:
    return load().dit_status_string(code).decode()


def _ptr(t) -> int:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class DiT:
    """A created model: device weights + workspace owned by the library."""

    def __init__(self, cfg, weights: Sequence[np.ndarray], max_batch: Optional[int] = None):
        self.lib = load()
        self.cfg = cfg
        self._c = make_config(cfg, max_batch)
        arrs = [np.ascontiguousarray(w, dtype=np.float32) for w in weights]
        ptrs = (c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
        h = c_void_p()
        rc = self.lib.dit_create(ctypes.byref(self._c), ptrs, len(arrs), ctypes.byref(h))
        if rc != DIT_OK:
            raise DitError(rc, f"dit_create failed: {status_string(rc)}")
        self.h = h

    # ---- helpers
    def _check(self, rc: int, what: str):
        if rc != DIT_OK:
            msg = self.lib.dit_last_error(self.h).decode() if self.h else ""
            raise DitError(rc, f"{what}: {status_string(rc)} {msg}")

    def rows(self, B: int, cfg_scale: float) -> int:
        return 2 * B if (self.cfg.cond_kind == 0 and cfg_scale != 1.0) else B

    def out_shape(self, B: int):
        return self.cfg.out_shape(B)

    # ---- calls
    def forward(self, x, t, y, cfg_scale: float, out=None, stream=None):
        import torch
        B = x.shape[0]
        if out is None:
            out = torch.empty(self.out_shape(B), dtype=torch.float32, device=x.device)
        rc = self.lib.dit_forward(self.h, _ptr(x), _ptr(t), _ptr(y), B, float(cfg_scale), _ptr(out), _stream(stream))
        self._check(rc, "dit_forward")
        return out

    def forward_host(self, x: np.ndarray, t: np.ndarray, y: np.ndarray, cfg_scale: float, out: np.ndarray = None,
                     stream=None):
        B = x.shape[0]
        if out is None:
            out = np.empty(self.out_shape(B), dtype=np.float32)
        rc = self.lib.dit_forward_host(self.h, x.ctypes.data, t.ctypes.data, y.ctypes.data, B, float(cfg_scale),
                                       out.ctypes.data, _stream(stream))
        self._check(rc, "dit_forward_host")
        return out

    def forward_host_ptr(self, x_ptr: int, t_ptr: int, y_ptr: int, B: int, cfg_scale: float, out_ptr: int,
                         stream=None):
        rc = self.lib.dit_forward_host(self.h, x_ptr, t_ptr, y_ptr, B, float(cfg_scale), out_ptr, _stream(stream))
        self._check(rc, "dit_forward_host")

    def debug_residual(self, x, t, y, cfg_scale: float, after_block: int, stream=None):
        import torch
        B = x.shape[0]
        R = self.rows(B, cfg_scale) if not getattr(self, "_force", False) else 2 * B
        h = torch.empty((R, getattr(self.cfg, "seq_tokens", self.cfg.tokens), self.cfg.hidden), dtype=torch.float32,
                        device=x.device)
        rc = self.lib.dit_debug_residual(self.h, _ptr(x), _ptr(t), _ptr(y), B, float(cfg_scale), after_block, _ptr(h),
                                         _stream(stream))
        self._check(rc, "dit_debug_residual")
        return h

    def debug_condition(self, t, y, cfg_scale: float, stream=None):
        import torch
        B = t.shape[0]
        R = self.rows(B, cfg_scale) if not getattr(self, "_force", False) else 2 * B
        c = torch.empty((R, self.cfg.hidden), dtype=torch.float32, device=t.device)
        rc = self.lib.dit_debug_condition(self.h, _ptr(t), _ptr(y), B, float(cfg_scale), _ptr(c), _stream(stream))
        self._check(rc, "dit_debug_condition")
        return c

    def sampler_step(self, kind: int, x, model_out, a: float, b: float, x_next=None, stream=None):
        """One sampler update (DIT_SAMPLER_DDIM: a, b = abar now / next; DIT_SAMPLER_EULER:
        a, b = t now / next) of the device latent x given dit_forward's output; in place when
        x_next is x."""
        import torch
        if x_next is None:
            x_next = torch.empty_like(x)
        rc = self.lib.dit_sampler_step(self.h, int(kind), _ptr(x), _ptr(model_out), x.shape[0], float(a), float(b),
                                       _ptr(x_next), _stream(stream))
        self._check(rc, "dit_sampler_step")
        return x_next

    def sample(self, kind: int, x, y, cfg_scale: float, model_t, levels, stream=None):
        """len(model_t) steps of forward + update, in place on the device latent x."""
        mt = np.ascontiguousarray(model_t, dtype=np.float32)
        lv = np.ascontiguousarray(levels, dtype=np.float32)
        if lv.size != mt.size + 1:
            raise ValueError("levels needs one more entry than model_t")
        fp = POINTER(c_float)
        rc = self.lib.dit_sample(self.h, int(kind), _ptr(x), _ptr(y), x.shape[0], float(cfg_scale), int(mt.size),
                                 mt.ctypes.data_as(fp), lv.ctypes.data_as(fp), _stream(stream))
        self._check(rc, "dit_sample")
        return x

    def set_option(self, option: int, value: int):
        self._check(self.lib.dit_set_option(self.h, option, value), "dit_set_option")
        if option == DIT_OPT_FORCE_GUIDANCE:
            self._force = bool(value)

    def sync_status(self) -> int:
        return self.lib.dit_sync_status(self.h)

    def wait_probe(self, timeout_us: int, stream=None):
        self._check(self.lib.dit_debug_wait_probe(self.h, timeout_us, _stream(stream)), "dit_debug_wait_probe")

    def attention_rescales(self) -> int:
        """Attention reference-maximum moves (per warp of 32 query rows) since the last read."""
        n = ctypes.c_longlong(0)
        self._check(self.lib.dit_debug_attention_rescales(self.h, ctypes.byref(n)), "dit_debug_attention_rescales")
        return int(n.value)

    def launch_count(self, B: int, cfg_scale: float) -> int:
        return self.lib.dit_forward_launch_count(self.h, B, float(cfg_scale))

    def profile(self, enable: bool, kind: Optional[str] = None):
        """Per-launch event timing on (every kind, or only `kind`, one of KERNEL_KINDS) or off."""
        mode = 0 if not enable else (1 if kind is None else 2 + KERNEL_KINDS.index(kind))
        self._check(self.lib.dit_profile_enable(self.h, mode), "dit_profile_enable")

    def profile_read(self):
        """{kind: (total_ms, launches)} of the launches recorded since the last read."""
        n = len(KERNEL_KINDS)
        ms = (c_float * n)()
        cnt = (c_int * n)()
        self._check(self.lib.dit_profile_read(self.h, ms, cnt), "dit_profile_read")
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}

    def close(self):
        if getattr(self, "h", None):
            self.lib.dit_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def linear_bf16(x, w, b, block_n: int = 128, stream=None, pair: bool = False):
    """y = x W^T + b on the tensor-core GEMM (x, w: torch bf16 CUDA tensors);
    pair=True runs the SM-pair (cta_group::2) kernel."""
    import torch
    lib = load()
    M, K = x.shape
    N = w.shape[0]
    y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    fn = lib.dit_op_linear_bf16_pair if pair else lib.dit_op_linear_bf16
    rc = fn(_ptr(x), _ptr(w), _ptr(b), _ptr(y), M, N, K, block_n, _stream(stream))
    if rc != DIT_OK:
        raise DitError(rc, f"dit_op_linear_bf16: {status_string(rc)}")
    return y


def attention_bf16(q, k, v, o, R: int, H: int, T: int, dh: int, counters=None, stream=None):
    """The bf16 tensor-core attention kernel on the forward's workspace layouts (see
    dit_op_attention_bf16 in include/dit.h): q, k [R*H, Tpad, DP], v [R*H, DP, Tpad] and
    o [R*T, H*dh], torch bf16 CUDA tensors; counters an int32 CUDA tensor of 2 or None."""
    lib = load()
    rc = lib.dit_op_attention_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(o), R, H, T, dh, _ptr(counters), _stream(stream))
    if rc != DIT_OK:
        raise DitError(rc, f"dit_op_attention_bf16: {status_string(rc)}")
    return o


def linear_e4m3(x8, w8, sx, sw, b, block_n: int = 128, stream=None):
    """y = sx[m] sw[n] (x8 w8^T)[m, n] + b[n] on the FP8 tensor-core GEMM (x8, w8: uint8 CUDA
    tensors of E4M3 bytes; sx, sw, b: float32 CUDA tensors, b may be None)."""
    import torch
    lib = load()
    M, K = x8.shape
    N = w8.shape[0]
    y = torch.empty((M, N), dtype=torch.float32, device=x8.device)
    rc = lib.dit_op_linear_e4m3(_ptr(x8), _ptr(w8), _ptr(sx), _ptr(sw), _ptr(b), _ptr(y), M, N, K, block_n,
                                _stream(stream))
    if rc != DIT_OK:
        raise DitError(rc, f"dit_op_linear_e4m3: {status_string(rc)}")
    return y
