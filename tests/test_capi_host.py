"""Host-side checks of the C-ABI library that need no GPU: it loads, it exports
every entry point include/mla.h declares, and the argument validation that
runs before any CUDA call rejects bad input with the documented codes."""
import ctypes
import os
import re
import subprocess

import pytest

import mla_latent_kv_19_b200 as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    return sorted(set(re.findall(r"^MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_path():
    names = _declared()
    for n in ("mla_create", "mla_destroy", "mla_cache_append", "mla_absorb_q", "mla_decode",
              "mla_decode_partial", "mla_decode_combine", "mla_out_proj"):
        assert n in names


def test_every_declared_symbol_is_exported():
    out = subprocess.run(["nm", "-D", "--defined-only", m.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (mla_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    # and the binding wraps each one
    assert sorted(m.EXPORTED_SYMBOLS) == _declared()
    for n in _declared():
        assert hasattr(m.lib, n)


def test_status_strings():
    assert m.mla_status_string(0) == "MLA_OK"
    assert m.mla_status_string(-6) == "MLA_ERR_BAD_INDEX"
    assert m.mla_status_string(-7) == "MLA_ERR_TIMEOUT"
    assert m.mla_status_string(-9) == "MLA_ERR_RANGE"
    assert m.mla_status_string(12345) == "MLA_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(num_heads=128, d_c=512, d_r=64, d_nope=128, d_v=128, d_model=5120, block_size=64,
                act_dtype=m.MLA_BF16, cache_dtype=m.MLA_BF16, softmax_scale=192 ** -0.5,
                rope_base=10000.0, max_position=4096)
    base.update(kw)
    return m.MlaConfig(*[base[f] for f, _ in m.MlaConfig._fields_])


def _create(cfg):
    h = ctypes.c_void_p()
    return m.lib.mla_create(ctypes.byref(cfg), ctypes.byref(h)), h


@pytest.mark.parametrize("bad", [
    dict(num_heads=0), dict(d_c=-512), dict(d_r=63), dict(softmax_scale=0.0),
    dict(softmax_scale=float("nan")), dict(rope_base=0.5), dict(max_position=0), dict(block_size=0),
])
def test_create_rejects_invalid_config(bad):
    st, h = _create(_cfg(**bad))
    assert st == -1 and not h.value


@pytest.mark.parametrize("bad", [
    dict(act_dtype=m.MLA_FP32, cache_dtype=m.MLA_BF16),
    dict(act_dtype=m.MLA_FP32, cache_dtype=m.MLA_FP8_E4M3),
    dict(d_c=1024), dict(d_c=520),
])
def test_create_rejects_unsupported(bad):
    st, h = _create(_cfg(**bad))
    assert st == -2 and not h.value


def test_null_arguments():
    assert m.lib.mla_create(None, None) == -1
    assert m.lib.mla_destroy(None) == 0
    assert m.lib.mla_cache_row_bytes(None) == 0
    assert m.lib.mla_decode_workspace_bytes(None, 4, 2, 100) == 0
    assert m.lib.mla_decode_auto_splits(None, 4, 100) == 1
    null = ctypes.c_void_p()
    assert m.lib.mla_cache_append(null, None, None, None, None, 1, None, 1, 1, None, None, 1, None) == -1
    assert m.lib.mla_absorb_q(null, None, None, None, None, 1, None, None) == -1
    assert m.lib.mla_decode(null, None, None, None, 1, None, 1, None, 1, 64, 0, None, 0, None, None, None) == -1
    assert m.lib.mla_out_proj(null, None, None, None, 1, None, 0, None, None, None) == -1
    assert m.lib.mla_last_device_error(null, None) == -1
    assert m.lib.mla_set_wait_limit(null, 5) == -1
    assert m.lib.mla_set_launch_overlap(null, 1) == -1
    assert m.lib.mla_set_w_o_layout(null, 1) == -1
    assert m.lib.mla_pack_w_o(null, None, None, None) == -1
    assert m.lib.mla_combine_out_proj(null, 1, 64, 1, None, 0, None, None, None, 0, None, None, None, None,
                                      None) == -1


def test_create_without_device_reports_cuda_error():
    """A valid configuration reaches the device query; with no GPU present that
    fails with MLA_ERR_CUDA and no handle is returned."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st, h = _create(_cfg())
    assert st == -8 and not h.value


def test_binding_counts_pages_from_the_cache_size():
    """The page count handed to the library (its bounds check on page-table
    entries) comes from the cache's size, whatever the tensor's shape."""
    import types

    import torch
    h = types.SimpleNamespace(cfg=types.SimpleNamespace(block_size=64, d_c=512, d_r=64))
    assert m._num_blocks(h, torch.empty(10 * 64, 576, dtype=torch.bfloat16)) == 10
    assert m._num_blocks(h, torch.empty(7, 64, 576, dtype=torch.uint8)) == 7
    with pytest.raises(ValueError):
        m._num_blocks(h, torch.empty(100, 576))


def test_binding_checks_the_scale_array_length():
    """An fp8 cache's scales need one fp32 per cache row: a shorter array would
    let the kernels read past it, so the binding refuses it before any call."""
    import types

    import torch
    h = types.SimpleNamespace(cfg=types.SimpleNamespace(block_size=64, d_c=512, d_r=64))
    cache = torch.empty(3 * 64, 576, dtype=torch.uint8)
    assert m._scale_ptr(h, cache, None) is None
    assert m._scale_ptr(h, cache, torch.empty(3 * 64, dtype=torch.float32)) is not None
    with pytest.raises(ValueError):
        m._scale_ptr(h, cache, torch.empty(3 * 64 - 1, dtype=torch.float32))
    with pytest.raises(ValueError):
        m._scale_ptr(h, cache, torch.empty(3 * 64, dtype=torch.float64))
