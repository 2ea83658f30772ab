"""The allocation-free table build (pae_precompute_tables_static) against the
context's own table build (pae_precompute_tables).

Callers that may not allocate device memory while they run (a real-time
control process after its set-up, a framework that owns all device memory, a
stream being captured into a CUDA graph) use the static entry point with
buffers they own.  It must give the same tables as the context path, call
after call, although every call reuses one fixed scratch array.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import flow_matching_action_pi0_b200 as fm
import workloads as wl
from tests.helpers import TOL_FP32_MAX_ABS, build_expert
from workloads import device as wd

pytestmark = pytest.mark.gpu


def _weights_struct(dev_w):
    w = fm.pae_weights()
    for name in ("w_t1", "b_t1", "w_t2", "b_t2", "w_mod", "b_mod", "w_modf", "b_modf"):
        setattr(w, name, dev_w[name].data_ptr())
    return w


@pytest.mark.parametrize("cfg", [wl.TINY_FP32, wl.TINY_FP32.replace(name="tiny_bf16_t", dtype=wl.BF16),
                                 wl.PI05_BF16_BS1], ids=["fp32", "bf16", "pi05_bf16"])
def test_static_tables_match_context_tables(cfg):
    W = wl.make_weights(cfg)
    ex, _ = build_expert(cfg, W=W)
    try:
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        ex.sync()
        want_tab = np.frombuffer(ex.debug_copy("tables").tobytes(), dtype=np.float32)
        want_dt = np.frombuffer(ex.debug_copy("dt").tobytes(), dtype=np.float32)
    finally:
        ex.close()
    K = cfg.steps
    rows = (6 * cfg.layers + 2) * cfg.width
    dev_w = wd.upload_weights(cfg, W)
    w = _weights_struct(dev_w)
    code = fm.DTYPE_CODES[cfg.dtype]
    for call in range(2):   # two calls in a row share the scratch array
        tables = torch.full((K, rows), float("nan"), dtype=torch.float32, device="cuda")
        dt = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
        fm.pae_precompute_tables_static(cfg.layers, cfg.width, code, w, list(grid), tables.data_ptr(),
                                        dt.data_ptr())
        torch.cuda.synchronize()
        got_tab = tables.cpu().numpy().reshape(-1)
        got_dt = dt.cpu().numpy()
        assert np.all(np.isfinite(got_tab)), f"call {call}: unwritten table entries"
        assert np.max(np.abs(got_tab - want_tab[:got_tab.size])) <= TOL_FP32_MAX_ABS, f"call {call}: tables differ"
        assert np.max(np.abs(got_dt - want_dt[:K])) <= TOL_FP32_MAX_ABS, f"call {call}: dt differs"
        ref_tab, _ = _oracle_table_rows(cfg, W, grid)
        assert np.max(np.abs(got_tab.reshape(K, rows) - ref_tab)) <= TOL_FP32_MAX_ABS, f"call {call}: vs oracle"


def _oracle_table_rows(cfg, W, grid):
    """The oracle's per-step tables in the library's layout: per layer l and
    norm j the rows (scale, shift, gate), then the final (scale, shift)."""
    import oracle
    p = oracle.params_from_weights(cfg, W)
    out = []
    for tab in oracle.modulation_tables(grid, p):
        parts = []
        for l in range(cfg.layers):
            for j in range(2):
                parts += [tab.scale[l, j], tab.shift[l, j], tab.gate[l, j]]
        parts += [tab.scale_f, tab.shift_f]
        out.append(np.concatenate(parts))
    return np.stack(out), np.array([t.dt for t in oracle.modulation_tables(grid, p)])


# Sizes at the edges of the fixed scratch array and of the 16-step passes of its
# batched GEMV: K = 17 (a second, one-step pass), K = 64 at width 2048 (the whole
# array), and the int4 mode (its modulation weights are bf16 as in bf16 mode).
EDGE_CASES = [
    wl.TINY_FP32.replace(name="k17_fp32", steps=17),
    wl.TINY_FP32.replace(name="k64_w2048_bf16", dtype=wl.BF16, layers=1, width=2048, mlp_dim=128, steps=64),
    wl.TINY_FP32.replace(name="k64_w2048_fp32", layers=1, width=2048, mlp_dim=128, steps=64),
    wl.TINY_FP32.replace(name="tiny_w4a16_t", dtype=wl.W4A16, steps=10),
]


@pytest.mark.parametrize("cfg", EDGE_CASES, ids=[c.name for c in EDGE_CASES])
def test_static_tables_edge_sizes_match_oracle(cfg):
    W = wl.make_weights(cfg)
    grid = wl.uniform_grid(cfg.steps)
    want_tab, want_dt = _oracle_table_rows(cfg, W, grid)
    K = cfg.steps
    rows = (6 * cfg.layers + 2) * cfg.width
    dev_w = wd.upload_weights(cfg, W)
    w = _weights_struct(dev_w)
    code = fm.DTYPE_CODES[cfg.dtype]
    for call in range(2):
        tables = torch.full((K, rows), float("nan"), dtype=torch.float32, device="cuda")
        dt = torch.full((K,), float("nan"), dtype=torch.float32, device="cuda")
        fm.pae_precompute_tables_static(cfg.layers, cfg.width, code, w, list(grid), tables.data_ptr(),
                                        dt.data_ptr())
        torch.cuda.synchronize()
        got = tables.cpu().numpy()
        assert np.all(np.isfinite(got)), f"call {call}: unwritten table entries"
        err = float(np.max(np.abs(got - want_tab)))
        assert err <= TOL_FP32_MAX_ABS, f"{cfg.name} call {call}: tables differ from the oracle by {err:.3e}"
        assert np.max(np.abs(dt.cpu().numpy() - want_dt)) <= 1e-6, f"{cfg.name} call {call}: dt differs"


def test_static_tables_reject_sizes_beyond_the_scratch():
    cfg = wl.TINY_FP32
    dev_w = wd.upload_weights(cfg, wl.make_weights(cfg))
    w = _weights_struct(dev_w)
    out = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(fm.PaeError) as e:
        fm.pae_precompute_tables_static(cfg.layers, cfg.width, fm.PAE_FP32, w, list(wl.uniform_grid(65)),
                                        out.data_ptr(), out.data_ptr())
    assert e.value.status == fm.PAE_ERR_ARG and "64" in str(e.value)
    with pytest.raises(fm.PaeError) as e:
        fm.pae_precompute_tables_static(cfg.layers, 4096, fm.PAE_FP32, w, list(wl.uniform_grid(2)),
                                        out.data_ptr(), out.data_ptr())
    assert e.value.status == fm.PAE_ERR_ARG and "2048" in str(e.value)
