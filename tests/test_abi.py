"""CPU checks of the C ABI: the library builds and loads, exports every symbol
include/pae.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

import flow_matching_action_pi0_b200 as fm
from flow_matching_action_pi0_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "pae.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(pae_[a-z_0-9]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    return fm.lib()


def test_every_declared_symbol_is_exported(lib):
    decl = declared_symbols()
    assert "pae_denoise" in decl and "pae_create" in decl
    for name in decl:
        assert hasattr(lib, name), f"{name} not exported"
    assert sorted(fm.EXPORTS) == decl


def test_library_links_no_cuda_shared_objects():
    # The static runtime is linked in; the driver is loaded at first use, so the
    # library loads where no GPU exists.
    fbuild.build()
    import subprocess
    out = subprocess.run(["ldd", fbuild.LIB], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libcuda.so" not in out


def _cfg(**kw):
    base = dict(layers=2, width=256, n_q_heads=4, n_kv_heads=1, head_dim=64, mlp_dim=1024, action_dim=8,
                chunk=16, max_batch=1, max_prefix=64, dtype="bf16")
    base.update(kw)
    return fm.make_config(**base)


def _create_status(cfg, weights=None):
    out = ctypes.c_void_p()
    w = fm.pae_weights() if weights is None else weights
    st = fm.lib().pae_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(out))
    return st, out.value, fm.lib().pae_last_error(None).decode()


def test_create_rejects_bad_configs(lib):
    st, ctx, msg = _create_status(_cfg(width=0))
    assert st == fm.PAE_ERR_ARG and ctx is None and "positive" in msg
    st, ctx, msg = _create_status(_cfg(n_q_heads=6, n_kv_heads=4))
    assert st == fm.PAE_ERR_UNSUPPORTED and "multiple" in msg
    st, ctx, msg = _create_status(_cfg(width=160))
    assert st == fm.PAE_ERR_UNSUPPORTED
    st, ctx, msg = _create_status(_cfg(dtype=7))
    assert st == fm.PAE_ERR_ARG
    st, ctx, msg = _create_status(_cfg(chunk=300))
    assert st == fm.PAE_ERR_UNSUPPORTED
    # a valid config with missing weights
    st, ctx, msg = _create_status(_cfg())
    assert st == fm.PAE_ERR_ARG and "NULL" in msg


def test_null_arguments(lib):
    assert lib.pae_create(None, None, None) == fm.PAE_ERR_ARG
    assert lib.pae_denoise(None, None, None, 1, None) == fm.PAE_ERR_ARG
    assert lib.pae_set_prefix(None, 0, None, None, 0, None) == fm.PAE_ERR_ARG
    assert lib.pae_precompute_tables(None, None, 1, None) == fm.PAE_ERR_ARG
    lib.pae_destroy(None)
    assert lib.pae_last_error(None) is not None
