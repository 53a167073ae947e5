"""The C-ABI library loads and exports every entry point that include/*.h
declares (no compute calls: runs without a GPU)."""

import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "discrete_diffusion_moe_b200", "libdg.so")


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dg_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "dg_build", os.path.join(ROOT, "discrete_diffusion_moe_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("dg_encode_context", "dg_denoise_step", "dg_decode_block", "dg_context_create",
              "dg_weights_bytes", "dg_workspace_bytes", "dg_kv_bytes", "dg_model_init_random",
              "dg_canvas_init", "dg_check_device_error", "dg_last_error", "dg_context_destroy"):
        assert n in names, n


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_exports_are_c_symbols():
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in _declared():
        assert n in exported, f"{n} is not an unmangled export"


def test_size_queries_and_argument_errors_without_gpu(lib):
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(30, 2816, 16, 8, 176, 128, 8, 704, 262144, self_cond=True)
    nbytes = dg.dg_weights_bytes(cfg)
    # 30 layers of attention (2816 x 8448) and 128 experts (3 x 704 x 2816), router, the
    # embedding (plus its transposed copy), LM head and self-conditioning matrix, all bf16
    layer = 2816 * (2816 + 2 * 1408) + 2816 * 2816 + 128 * 2816 + 128 * 3 * 704 * 2816 + 2 * 2816
    glob_ = 3 * 262144 * 2816 + 2816 * 2816 + 2816
    assert abs(nbytes - 2 * (30 * layer + glob_)) < 1e6
    assert dg.dg_kv_bytes(cfg, 1, 1280) == 30 * 8 * 1280 * 176 * 2
    bad = dg.model_config(1, 100, 1, 1, 32, 4, 2, 64, 4096)  # d_model not a multiple of 64
    assert dg.dg_weights_bytes(bad) == 0
    assert "d_model" in dg.last_error()
    with pytest.raises(dg.DgError) as e:
        dg.dg_context_create(cfg, None, None, 0, 1)
    assert e.value.status == dg.DG_ERR_INVALID_ARG


def test_workspace_too_small_is_refused_before_any_device_work(lib):
    # the size check comes before the context touches the workspace, so fake
    # (aligned, never dereferenced) addresses suffice and no GPU is needed
    import discrete_diffusion_moe_b200 as dg
    cfg = dg.model_config(2, 256, 8, 8, 32, 16, 2, 512, 4096)
    need = dg.dg_workspace_bytes(cfg, 2)
    assert need > 0
    with pytest.raises(dg.DgError) as e:
        dg.dg_context_create(cfg, 1 << 20, 2 << 20, need - 256, 2)
    assert e.value.status == dg.DG_ERR_WORKSPACE
    assert "workspace too small" in dg.last_error()
    # a misaligned workspace is an argument error
    with pytest.raises(dg.DgError) as e:
        dg.dg_context_create(cfg, 1 << 20, (2 << 20) + 8, need, 2)
    assert e.value.status == dg.DG_ERR_INVALID_ARG
    # so is a batch outside [1, 64]
    with pytest.raises(dg.DgError) as e:
        dg.dg_context_create(cfg, 1 << 20, 2 << 20, need, 65)
    assert e.value.status == dg.DG_ERR_INVALID_ARG


def test_binding_structs_match_the_header():
    """The Python binding's ctypes mirrors of the ABI structs have the sizes
    the C build gives them (a field added on one side only shifts every later
    one)."""
    import discrete_diffusion_moe_b200 as dg
    for name in ("dg_model_config", "dg_sampler_config", "dg_kv", "dg_canvas", "dg_step_args",
                 "dg_step_out", "dg_block_stats", "dg_profile"):
        c_size = dg.lib.dg_test_struct_size(name.encode())
        assert c_size > 0, name
        assert ctypes.sizeof(getattr(dg, name)) == c_size, (name, ctypes.sizeof(getattr(dg, name)), c_size)
    assert dg.lib.dg_test_struct_size(b"no_such_struct") == 0
