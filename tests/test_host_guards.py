"""Host-side guards that need no GPU: the product path has no CPU fallback (it fails loudly
without the built library and never reaches the oracle), and the newer entry points reject
a null handle before touching the device."""
import ast
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "diffusion_transformer_denoiser_dit_b200")


def test_package_never_imports_the_oracle():
    for name in os.listdir(PKG):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, name)).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                mods = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                mods = [node.module or ""]
            else:
                continue
            assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), (name, mods)


def test_missing_library_fails_loudly():
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from diffusion_transformer_denoiser_dit_b200 import binding\n"
        "binding.LIB_PATH = '/nonexistent/libdit_b200.so'\n"
        "try:\n"
        "    binding.load()\n"
        "except RuntimeError as e:\n"
        "    print('raised:', e)\n"
        "    sys.exit(0)\n"
        "sys.exit(3)\n" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "missing" in r.stdout


@pytest.fixture(scope="module")
def lib():
    from diffusion_transformer_denoiser_dit_b200 import binding
    if not os.path.exists(binding.LIB_PATH):
        pytest.skip("library not built")
    return binding.load()


def test_null_handle_is_rejected_by_every_new_entry_point(lib):
    from ctypes import POINTER, c_float

    from diffusion_transformer_denoiser_dit_b200 import binding
    bad = binding.DIT_ERR_INVALID_ARG
    assert lib.dit_sampler_step(None, 0, None, None, 1, 0.5, 0.6, None, None) == bad
    assert lib.dit_sample(None, 0, None, None, 1, 1.0, 1, POINTER(c_float)(), POINTER(c_float)(), None) == bad
    assert lib.dit_set_option(None, binding.DIT_OPT_CFG_CHANNELS, 3) == bad
    assert lib.dit_set_option(None, binding.DIT_OPT_USE_GRAPH, 1) == bad
