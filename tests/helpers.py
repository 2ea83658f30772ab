"""Shared test helpers: build a pae context from a workload config and compare
results with the oracle under the stated tolerances."""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np

import workloads as wl

# Tolerances on final actions after K steps (fp32: max-abs; bf16/W4A16:
# max-abs and relative RMS), as the benchmark spec fixes them.
TOL_FP32_MAX_ABS = 1e-4
TOL_BF16_MAX_ABS = 2e-2
TOL_BF16_REL_RMS = 1e-2


def max_abs(a, b) -> float:
    """Largest absolute difference (0 for empty arrays, e.g. a zero-length prefix)."""
    d = np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))
    return float(d.max()) if d.size else 0.0


def assert_bf16_slot_close(got, ref, what: str) -> None:
    """K/V slot contents stored in bf16: the bf16-mode absolute bound 2e-2
    (the task's figure for final actions) plus the storage rounding a value of
    magnitude m carries, up to m * 2^-8, taken as m / 128 per element (the
    final actions are checked separately at the task's own tolerances)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if got.size == 0:
        return
    excess = np.abs(got - ref) - (2e-2 + np.abs(ref) / 128.0)
    assert excess.max() <= 0.0, f"{what}: max excess over the bf16 bound {excess.max():.3e}"


def rel_rms(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def assert_parity(gpu, ref, dtype: str, what: str = ""):
    ma = max_abs(gpu, ref)
    rr = rel_rms(gpu, ref)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    if dtype == wl.FP32:
        assert ma <= TOL_FP32_MAX_ABS, f"{what}: max-abs {ma:.3e} > {TOL_FP32_MAX_ABS} (rel-rms {rr:.3e})"
    else:
        assert ma <= TOL_BF16_MAX_ABS and rr <= TOL_BF16_REL_RMS, \
            f"{what}: max-abs {ma:.3e} (tol {TOL_BF16_MAX_ABS}), rel-rms {rr:.3e} (tol {TOL_BF16_REL_RMS})"
    return ma, rr


def build_expert(cfg: wl.ExpertConfig, W=None, max_batch: Optional[int] = None,
                 max_prefix: Optional[int] = None):
    import flow_matching_action_pi0_b200 as fm
    from workloads import device as wd
    if W is None:
        W = wl.make_weights(cfg)
    dev_w = wd.upload_weights(cfg, W)
    ex = fm.ActionExpert(fm.make_config(**wd.abi_config(cfg, max_batch, max_prefix)), dev_w)
    del dev_w
    return ex, W


def set_prefixes(ex, cfg, ks, vs, rows: Optional[Sequence[int]] = None):
    from workloads import device as wd
    kd, vd = wd.upload_prefix(cfg, ks, vs)
    rows = range(len(ks)) if rows is None else rows
    for i, b in enumerate(rows):
        ex.set_prefix(b, kd[i], vd[i], int(ks[i][0].shape[0]))
    return kd, vd


def run_gpu(ex, noise: np.ndarray) -> np.ndarray:
    import torch
    x = torch.from_numpy(noise).cuda()
    out = ex.denoise(x)
    ex.sync()
    return out.cpu().numpy()


def oracle_rows(cfg, W, ks, vs, noise, grid, rows: Optional[List[int]] = None):
    import oracle
    p = oracle.params_from_weights(cfg, W)
    return oracle.denoise(noise.astype(np.float64), grid, p, ks, vs, rows=rows)
