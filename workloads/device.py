"""Copy generated inputs into CUDA tensors laid out as the C ABI expects.

Data movement only (float32 -> bf16 of values that are already bf16, int4
records as packed bytes plus bf16 scales); no arithmetic of the method.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np
import torch

from . import BF16, FP32, LAYER_MATS, W4A16, ExpertConfig

SCALE_KEYS = {"w_qkv": "s_qkv", "w_o": "s_o", "w_gate": "s_gate", "w_up": "s_up", "w_down": "s_down"}


def act_dtype(cfg: ExpertConfig):
    return torch.float32 if cfg.dtype == FP32 else torch.bfloat16


def to_dev(a: np.ndarray, dtype, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device).to(dtype).contiguous()


def upload_weights(cfg: ExpertConfig, W: Dict[str, object], device="cuda") -> Dict[str, object]:
    dt = act_dtype(cfg)
    out: Dict[str, object] = {}
    for k in ("w_in", "b_in", "w_out", "b_out", "w_t1", "b_t1", "w_t2", "b_t2",
              "w_mod", "b_mod", "w_modf", "b_modf"):
        out[k] = to_dev(W[k], dt, device)
    for name in LAYER_MATS:
        if cfg.dtype == W4A16:
            out[name] = [torch.from_numpy(m.packed).to(device) for m in W[name]]
            out[SCALE_KEYS[name]] = [to_dev(m.scales, torch.bfloat16, device) for m in W[name]]
        else:
            out[name] = [to_dev(m, dt, device) for m in W[name]]
    if "w_prefix_kv" in W:  # prefix production weights (activation dtype)
        out["w_prefix_kv"] = [to_dev(m, dt, device) for m in W["w_prefix_kv"]]
    return out


def upload_prefix(cfg: ExpertConfig, ks: List[List[np.ndarray]], vs: List[List[np.ndarray]], device="cuda"):
    dt = act_dtype(cfg)
    return ([[to_dev(a, dt, device) for a in row] for row in ks],
            [[to_dev(a, dt, device) for a in row] for row in vs])


def abi_config(cfg: ExpertConfig, max_batch=None, max_prefix=None) -> Dict[str, object]:
    """Keyword arguments for flow_matching_action_pi0_b200.make_config."""
    return dict(layers=cfg.layers, width=cfg.width, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads,
                head_dim=cfg.head_dim, mlp_dim=cfg.mlp_dim, action_dim=cfg.action_dim, chunk=cfg.chunk,
                max_batch=cfg.batch if max_batch is None else max_batch,
                max_prefix=cfg.prefix if max_prefix is None else max_prefix,
                dtype=cfg.dtype, group_size=cfg.group_size, rms_eps=cfg.rms_eps, rope_base=cfg.rope_base,
                prefix_width=cfg.prefix_width)


__all__ = ["upload_weights", "upload_prefix", "abi_config", "act_dtype", "to_dev", "BF16", "FP32", "W4A16"]
