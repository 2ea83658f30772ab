"""Seeded synthetic inputs for the action-expert denoise loop.

This module only draws numbers: configuration shapes, weights, prefix K/V,
noise and timestep grids.  It holds none of the expert's arithmetic, so the
CPU oracle and the CUDA path can both take their inputs from here without
sharing any computation.

Workload shapes follow the pi0.5 setting the PhyAI report measures ("PhyAI:
Real-Time Physical AI at the Edge", Sec. 5.3 PI0.5 paragraph and Figure 5:
BF16, three cameras, a 50-action chunk, ten Euler steps).  The prefix length
968 is 3 camera views x 256 image tokens + 200 text tokens.  No dataset item
is used: weights, prefix K/V and noise are Gaussian draws that stand in for a
trained checkpoint and for real observations.

Random recipe (NumPy PCG64):
  * weights and biases ~ N(0, 0.02), seed 0 + config index;
  * prefix K/V ~ N(0, 1), seed 1 + config index (ragged lengths from the
    same stream, uniform on [512, 1024]);
  * noise ~ N(0, 1), seed 2 + config index;
  * W4A16 group scales ~ U(0.005, 0.02), drawn from the weight stream.
In bf16 and W4A16 modes every stored value is rounded to bf16 here, so both
sides see exactly the same numbers.  W4A16 codes come from the offline
round-to-nearest quantiser the report describes (Sec. 5.4, "During
training"): q = clamp(rint(w / s), -8, 7).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

FP32, BF16, W4A16 = "fp32", "bf16", "w4a16"
DTYPE_CODE = {FP32: 0, BF16: 1, W4A16: 2}


@dataclasses.dataclass(frozen=True)
class ExpertConfig:
    name: str
    layers: int
    width: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    mlp_dim: int
    action_dim: int
    chunk: int
    prefix: int            # prefix tokens per request (max for ragged)
    steps: int
    batch: int
    dtype: str
    group_size: int = 128  # W4A16 quantisation group along K
    rms_eps: float = 1e-6
    ragged: bool = False   # per-request prefix lengths drawn on [512, 1024]
    index: int = 0         # config index, added to every seed
    rope_base: float = 0.0  # rotary embedding base (0: off)
    prefix_width: int = 0   # width of the prefix model's hidden states (0: no prefix production)

    @property
    def qkv_dim(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def attn_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    def replace(self, **kw) -> "ExpertConfig":
        return dataclasses.replace(self, **kw)


TINY_FP32 = ExpertConfig("tiny_fp32", layers=2, width=256, n_q_heads=4, n_kv_heads=1,
                         head_dim=64, mlp_dim=1024, action_dim=8, chunk=16, prefix=64,
                         steps=4, batch=1, dtype=FP32, index=0)
PI05_BF16_BS1 = ExpertConfig("pi05_bf16_bs1", layers=18, width=1024, n_q_heads=8,
                             n_kv_heads=1, head_dim=256, mlp_dim=4096, action_dim=32,
                             chunk=50, prefix=968, steps=10, batch=1, dtype=BF16, index=1)
PI05_BF16_BS32 = PI05_BF16_BS1.replace(name="pi05_bf16_bs32", batch=32, index=2)
PI05_W4A16_BS1 = PI05_BF16_BS1.replace(name="pi05_w4a16_bs1", dtype=W4A16, index=3)
RAGGED_BF16_BS16 = PI05_BF16_BS1.replace(name="ragged_bf16_bs16", batch=16, prefix=1024,
                                         ragged=True, index=4)

CONFIGS: Dict[str, ExpertConfig] = {c.name: c for c in (
    TINY_FP32, PI05_BF16_BS1, PI05_BF16_BS32, PI05_W4A16_BS1, RAGGED_BF16_BS16)}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bf16 (ties to even); returns float32."""
    a32 = np.array(a, dtype=np.float32, copy=True, order="C")
    u = a32.view(np.uint32)          # finite inputs: the add cannot wrap
    lsb = (u >> 16) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return a32


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of bf16-representable float32 values (uint16)."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    return (a32.view(np.uint32) >> 16).astype(np.uint16)


def _normal(g: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    w = (g.standard_normal(size=shape, dtype=np.float32) * np.float32(std))
    return round_bf16(w) if dtype in (BF16, W4A16) else w


# Names of the per-layer projection matrices, in the order the C ABI takes them.
LAYER_MATS = ("w_qkv", "w_o", "w_gate", "w_up", "w_down")


def layer_shapes(cfg: ExpertConfig) -> Dict[str, tuple]:
    D, F = cfg.width, cfg.mlp_dim
    return {"w_qkv": (cfg.qkv_dim, D), "w_o": (D, cfg.attn_dim),
            "w_gate": (F, D), "w_up": (F, D), "w_down": (D, F)}


@dataclasses.dataclass
class Quantized:
    """Int4 weights: codes in [-8, 7] (int8 [N][K]), packed nibbles
    (uint8 [N][K/2], low nibble = even k) and bf16-valued scales
    (float32 [N][K/group])."""
    codes: np.ndarray
    packed: np.ndarray
    scales: np.ndarray


def quantize_rtn(w: np.ndarray, scales: np.ndarray, group: int) -> Quantized:
    """Offline round-to-nearest int4 quantiser (input preparation only)."""
    N, K = w.shape
    s_full = np.repeat(scales.astype(np.float64), group, axis=1)
    codes = np.clip(np.rint(w.astype(np.float64) / s_full), -8, 7).astype(np.int8)
    nib = (codes.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return Quantized(codes=codes, packed=packed, scales=scales.astype(np.float32))


def make_weights(cfg: ExpertConfig, seed: Optional[int] = None) -> Dict[str, object]:
    """All expert parameters, drawn N(0, 0.02).

    Returns a dict of float32 arrays (bf16-representable in bf16/W4A16 mode):
      w_in [D][A], b_in [D], w_out [A][D], b_out [A],
      w_t1 [D][D], b_t1 [D], w_t2 [D][D], b_t2 [D],
      w_mod [L*2][3D][D], b_mod [L*2][3D]  (index 2l = attention norm,
      2l+1 = MLP norm; chunks ordered scale, shift, gate),
      w_modf [2D][D], b_modf [2D]           (final norm: scale, shift),
      and per layer lists w_qkv, w_o, w_gate, w_up, w_down ([out][in]).
    In W4A16 mode the per-layer matrices are replaced by Quantized records
    under the same keys (their dequantised values are codes * scales).
    """
    g = rng(cfg.index if seed is None else seed)
    D, A, L = cfg.width, cfg.action_dim, cfg.layers
    dt = cfg.dtype
    std = 0.02
    W: Dict[str, object] = {}
    W["w_in"] = _normal(g, (D, A), std, dt)
    W["b_in"] = _normal(g, (D,), std, dt)
    W["w_out"] = _normal(g, (A, D), std, dt)
    W["b_out"] = _normal(g, (A,), std, dt)
    W["w_t1"] = _normal(g, (D, D), std, dt)
    W["b_t1"] = _normal(g, (D,), std, dt)
    W["w_t2"] = _normal(g, (D, D), std, dt)
    W["b_t2"] = _normal(g, (D,), std, dt)
    W["w_mod"] = _normal(g, (2 * L, 3 * D, D), std, dt)
    W["b_mod"] = _normal(g, (2 * L, 3 * D), std, dt)
    W["w_modf"] = _normal(g, (2 * D, D), std, dt)
    W["b_modf"] = _normal(g, (2 * D,), std, dt)
    shapes = layer_shapes(cfg)
    for name in LAYER_MATS:
        W[name] = []
    for _l in range(L):
        for name in LAYER_MATS:
            shp = shapes[name]
            if dt == W4A16:
                w = g.standard_normal(size=shp, dtype=np.float32) * np.float32(std)
                s = round_bf16(g.uniform(0.005, 0.02, size=(shp[0], shp[1] // cfg.group_size))
                               .astype(np.float32))
                W[name].append(quantize_rtn(w, s, cfg.group_size))
            else:
                W[name].append(_normal(g, shp, std, dt))
    return W


def make_prefix_model(cfg: ExpertConfig, prefix_len: Optional[int] = None,
                      seed: Optional[int] = None) -> Dict[str, object]:
    """A stand-in for the vision-language model that produces the prefix: per
    layer a QKV projection [(Hq + 2 Hkv) d][Dp], an output projection
    [Dp][Hq d] and a GeGLU MLP (F x Dp), all ~N(0, 0.05), and the prefix's
    input hidden states z [P][Dp] ~N(0, 1) (Dp = cfg.prefix_width; seed
    3 + config index).  Values are bf16-rounded in bf16 and W4A16 modes.
    "w_prefix_kv" holds each layer's key and value rows of its QKV projection,
    the weights the prefix production step projects with."""
    Dp = cfg.prefix_width
    if Dp <= 0:
        raise ValueError("make_prefix_model needs cfg.prefix_width > 0")
    g = rng((3 + cfg.index) if seed is None else seed)
    dt = BF16 if cfg.dtype in (BF16, W4A16) else FP32
    P = cfg.prefix if prefix_len is None else prefix_len
    L, F, std = cfg.layers, cfg.mlp_dim, 0.05
    M: Dict[str, object] = {"w_qkv": [], "w_o": [], "w_gate": [], "w_up": [], "w_down": []}
    for _l in range(L):
        M["w_qkv"].append(_normal(g, (cfg.qkv_dim, Dp), std, dt))
        M["w_o"].append(_normal(g, (Dp, cfg.attn_dim), std, dt))
        M["w_gate"].append(_normal(g, (F, Dp), std, dt))
        M["w_up"].append(_normal(g, (F, Dp), std, dt))
        M["w_down"].append(_normal(g, (Dp, F), std, dt))
    M["z"] = _normal(g, (P, Dp), 1.0, dt)
    qd = cfg.attn_dim
    M["w_prefix_kv"] = [np.ascontiguousarray(w[qd:]) for w in M["w_qkv"]]
    return M


def dequantized(W: Dict[str, object], name: str, layer: int) -> np.ndarray:
    """Float64 value of a per-layer matrix as the kernels see it."""
    m = W[name][layer]
    if isinstance(m, Quantized):
        grp = m.codes.shape[1] // m.scales.shape[1]
        return m.codes.astype(np.float64) * np.repeat(m.scales.astype(np.float64), grp, axis=1)
    return np.asarray(m, dtype=np.float64)


def prefix_lengths(cfg: ExpertConfig, seed: Optional[int] = None) -> List[int]:
    if not cfg.ragged:
        return [cfg.prefix] * cfg.batch
    g = rng((1 + cfg.index) if seed is None else seed)
    return [int(v) for v in g.integers(512, 1024, size=cfg.batch, endpoint=True)]


def make_prefix(cfg: ExpertConfig, lengths: Optional[List[int]] = None,
                seed: Optional[int] = None, std: float = 1.0):
    """Per-request cached prefix K/V: lists (over rows) of lists (over layers)
    of float32 arrays [len][Hkv][head_dim], ~N(0, std)."""
    g = rng((1 + cfg.index) if seed is None else seed)
    if lengths is None:
        lengths = prefix_lengths(cfg)
        if cfg.ragged:
            g.integers(512, 1024, size=cfg.batch, endpoint=True)  # keep streams aligned
    ks, vs = [], []
    for n in lengths:
        kr, vr = [], []
        for _l in range(cfg.layers):
            kr.append(_normal(g, (n, cfg.n_kv_heads, cfg.head_dim), std, cfg.dtype))
            vr.append(_normal(g, (n, cfg.n_kv_heads, cfg.head_dim), std, cfg.dtype))
        ks.append(kr)
        vs.append(vr)
    return ks, vs


def make_noise(cfg: ExpertConfig, batch: Optional[int] = None,
               seed: Optional[int] = None) -> np.ndarray:
    g = rng((2 + cfg.index) if seed is None else seed)
    B = cfg.batch if batch is None else batch
    return g.standard_normal(size=(B, cfg.chunk, cfg.action_dim), dtype=np.float32)


def uniform_grid(steps: int, t0: float = 1.0, t1: float = 0.0) -> np.ndarray:
    """t_k = t0 + (t1 - t0) k / K, k = 0..K (float64)."""
    return np.array([t0 + (t1 - t0) * k / steps for k in range(steps + 1)], dtype=np.float64)
