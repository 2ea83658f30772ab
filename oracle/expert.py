"""Float64 oracle of the action-expert flow-matching denoise loop.

TEST INFRASTRUCTURE ONLY.  Nothing in the product library imports or runs this
file; it shares no code with the CUDA path.  Only tests, the smoke check and
the benchmark's CPU-baseline leg call it.

What it computes, and where each step comes from:

* The loop structure is the pi0.5 path of the PhyAI report ("PhyAI: Real-Time
  Physical AI at the Edge", Sec. 5.1 "Follow one pi0.5 request through cache
  reuse and graph replay", and Sec. 5.5 "Reuse only valid conditions"): the
  vision-language prefix is computed once, its per-layer K/V is cached, the
  timestep/modulation tables are precomputed, and ten Euler steps advance the
  action tokens while the prefix stays fixed.
* The layer is the action expert as the benchmark spec defines it: a small
  transformer over the action chunk with timestep-conditioned adaptive
  RMSNorm, GQA attention over [cached prefix | action tokens] and a GeGLU MLP,
  an input projection from actions and an output projection to a velocity.
* The pages do not print the expert's equations.  The readings taken where
  they are silent are listed in the design notes and repeated beside each
  function below; both sides implement them independently.

Notation: L layers, D width, Hq/Hkv heads, d head_dim, F MLP width, A action
dim, H chunk, P_b prefix length of request b, K Euler steps, t_0 = 1 > ... >
t_K = 0 (noise at t = 1, data at t = 0), dt_k = t_{k+1} - t_k.

Parity status: every function here is pinned by the tests in
``tests/test_oracle_pins.py`` (closed forms, library routines, brute-force
full-sequence recomputation, invariants).  Agreement with a trained pi0.5
policy is unpinned: no checkpoint exists here.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# Timestep conditioning (precomputed tables; report Sec. 5.1 / Sec. 5.5)
# ---------------------------------------------------------------------------

def sinusoidal_embedding(t: float, dim: int, min_period: float = 4e-3,
                         max_period: float = 4.0) -> np.ndarray:
    """Sinusoidal embedding of a scalar timestep.

    Reading (the pages name precomputed timestep tables but not the formula):
    half = dim/2 geometric periods from min_period to max_period,
    period_i = min_period * (max_period/min_period)^(i/(half-1)), and
    e = [sin(2 pi t / period_i) for i] ++ [cos(2 pi t / period_i) for i].
    """
    half = dim // 2
    i = np.arange(half, dtype=F64)
    frac = i / (half - 1) if half > 1 else np.zeros(1, dtype=F64)
    period = min_period * (max_period / min_period) ** frac
    ang = 2.0 * math.pi * F64(t) / period
    return np.concatenate([np.sin(ang), np.cos(ang)])


def swish(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def time_conditioning(t: float, p: "OracleParams") -> np.ndarray:
    """c(t) = swish(W_t2 swish(W_t1 e(t) + b_t1) + b_t2)  (reading: a two-layer
    MLP with swish after each layer)."""
    e = sinusoidal_embedding(t, p.D)
    z = swish(p.w_t1 @ e + p.b_t1)
    return swish(p.w_t2 @ z + p.b_t2)


@dataclasses.dataclass
class StepTables:
    """Modulation for one Euler step: per layer, for the attention norm
    (j = 0) and the MLP norm (j = 1), the (scale, shift, gate) vectors; the
    final norm's (scale, shift); and dt."""
    scale: np.ndarray    # [L][2][D]
    shift: np.ndarray    # [L][2][D]
    gate: np.ndarray     # [L][2][D]
    scale_f: np.ndarray  # [D]
    shift_f: np.ndarray  # [D]
    dt: float


def modulation_tables(t_grid: Sequence[float], p: "OracleParams") -> List[StepTables]:
    """Build the per-step tables once for a timestep grid (K+1 points).

    For step k: c = c(t_k); (scale, shift, gate) = split3(W_mod[l, j] c +
    b_mod[l, j]) for every layer l and norm j; (scale_f, shift_f) =
    split2(W_modf c + b_modf); dt_k = t_{k+1} - t_k.
    """
    out = []
    D, L = p.D, p.L
    for k in range(len(t_grid) - 1):
        c = time_conditioning(float(t_grid[k]), p)
        m = (p.w_mod.reshape(-1, D) @ c).reshape(2 * L, 3 * D) + p.b_mod   # [2L][3D]
        m = m.reshape(L, 2, 3, D)
        f = p.w_modf @ c + p.b_modf
        out.append(StepTables(scale=m[:, :, 0, :].copy(), shift=m[:, :, 1, :].copy(),
                              gate=m[:, :, 2, :].copy(), scale_f=f[:D].copy(),
                              shift_f=f[D:].copy(),
                              dt=float(t_grid[k + 1]) - float(t_grid[k])))
    return out


# ---------------------------------------------------------------------------
# Layer pieces
# ---------------------------------------------------------------------------

def ada_rms_norm(h: np.ndarray, scale: np.ndarray, shift: np.ndarray,
                 eps: float) -> np.ndarray:
    """Adaptive RMSNorm (reading: no learned gain):
    y = h / sqrt(mean(h^2) + eps) * (1 + scale) + shift, over the last axis."""
    r = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)
    return h * r * (1.0 + scale) + shift


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def rope(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotary position embedding of per-head vectors x [T][H][d] at integer
    positions [T].

    Reading (the pages do not print it; the vla.cpp abstract on page 1 only
    warns that positional-index precision matters): the rotate-half form, in
    which channel i < d/2 pairs with channel i + d/2 and the pair turns by
    angle pos * base^(-2i/d):
      out_i       = x_i cos(a_i) - x_{i+d/2} sin(a_i)
      out_{i+d/2} = x_{i+d/2} cos(a_i) + x_i sin(a_i).
    Angles are formed in float64 from the integer positions.
    """
    d = x.shape[-1]
    half = d // 2
    inv_freq = base ** (-2.0 * np.arange(half, dtype=F64) / d)          # [half]
    ang = np.asarray(positions, dtype=F64)[:, None] * inv_freq[None, :]  # [T][half]
    c = np.cos(ang)[:, None, :]
    sn = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * sn, x2 * c + x1 * sn], axis=-1)


def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
              mask: Optional[np.ndarray] = None, return_probs: bool = False):
    """Grouped-query attention, one request.

    q [T][Hq][d]; keys, values [S][Hkv][d]; query head h reads KV head
    h // (Hq/Hkv).  s = q . k / sqrt(d); p = softmax over the keys allowed by
    ``mask`` ([T][S] booleans, True = visible; None = all visible);
    o = p . v.  Returns o [T][Hq][d] (and p [Hq][T][S] when asked).
    """
    T, Hq, d = q.shape
    S, Hkv, _ = keys.shape
    grp = Hq // Hkv
    o = np.zeros((T, Hq, d), dtype=F64)
    probs = np.zeros((Hq, T, S), dtype=F64) if return_probs else None
    for h in range(Hq):
        g = h // grp
        s = (q[:, h, :] @ keys[:, g, :].T) / math.sqrt(d)              # [T][S]
        if mask is not None:
            s = np.where(mask, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        e = np.exp(s - m)
        pr = e / np.sum(e, axis=1, keepdims=True)
        o[:, h, :] = pr @ values[:, g, :]
        if return_probs:
            probs[h] = pr
    return (o, probs) if return_probs else o


@dataclasses.dataclass
class OracleParams:
    """Float64 copies of the exact parameter values the kernels see."""
    L: int
    D: int
    Hq: int
    Hkv: int
    d: int
    F: int
    A: int
    eps: float
    w_in: np.ndarray
    b_in: np.ndarray
    w_out: np.ndarray
    b_out: np.ndarray
    w_t1: np.ndarray
    b_t1: np.ndarray
    w_t2: np.ndarray
    b_t2: np.ndarray
    w_mod: np.ndarray   # [2L][3D][D]
    b_mod: np.ndarray   # [2L][3D]
    w_modf: np.ndarray  # [2D][D]
    b_modf: np.ndarray  # [2D]
    w_qkv: List[np.ndarray]
    w_o: List[np.ndarray]
    w_gate: List[np.ndarray]
    w_up: List[np.ndarray]
    w_down: List[np.ndarray]
    rope_base: float = 0.0  # 0: no rotary embedding; else its base (positions P_b + i)


def params_from_weights(cfg, W) -> OracleParams:
    """Wrap generator output (float32 / int4 records) as float64 arrays."""
    def f(a):
        return np.asarray(a, dtype=F64)

    def mat(name, l):
        m = W[name][l]
        if hasattr(m, "codes"):   # int4 record: value = code * group scale
            grp = m.codes.shape[1] // m.scales.shape[1]
            return m.codes.astype(F64) * np.repeat(m.scales.astype(F64), grp, axis=1)
        return f(m)

    L = cfg.layers
    return OracleParams(
        L=L, D=cfg.width, Hq=cfg.n_q_heads, Hkv=cfg.n_kv_heads, d=cfg.head_dim,
        F=cfg.mlp_dim, A=cfg.action_dim, eps=float(cfg.rms_eps),
        w_in=f(W["w_in"]), b_in=f(W["b_in"]), w_out=f(W["w_out"]), b_out=f(W["b_out"]),
        w_t1=f(W["w_t1"]), b_t1=f(W["b_t1"]), w_t2=f(W["w_t2"]), b_t2=f(W["b_t2"]),
        w_mod=f(W["w_mod"]), b_mod=f(W["b_mod"]), w_modf=f(W["w_modf"]),
        b_modf=f(W["b_modf"]),
        w_qkv=[mat("w_qkv", l) for l in range(L)], w_o=[mat("w_o", l) for l in range(L)],
        w_gate=[mat("w_gate", l) for l in range(L)], w_up=[mat("w_up", l) for l in range(L)],
        w_down=[mat("w_down", l) for l in range(L)],
        rope_base=float(getattr(cfg, "rope_base", 0.0)))


def expert_layer(h: np.ndarray, l: int, tab: StepTables, p: OracleParams,
                 k_pre: np.ndarray, v_pre: np.ndarray, trace: Optional[dict] = None):
    """One expert layer over the H action tokens of one request.

    h [H][D] residual stream; k_pre, v_pre [P][Hkv][d] this layer's cached
    prefix K/V.  Attention block: y = adaRMSNorm(h; attention modulation),
    [q|k|v] = y W_qkv^T, every action token attends to all P prefix keys and
    to all H action keys (no mask inside the action block; reading),
    h += gate_a * (o W_o^T).  MLP block: y = adaRMSNorm(h; MLP modulation),
    h += gate_m * ((gelu_tanh(y W_gate^T) * (y W_up^T)) W_down^T).
    Attention and MLP carry no biases (reading).  With p.rope_base set, q and
    the action keys are rotated at positions P + i (the cached prefix keys
    already carry their own positions 0..P-1).
    """
    H = h.shape[0]
    Hq, Hkv, d = p.Hq, p.Hkv, p.d
    y = ada_rms_norm(h, tab.scale[l, 0], tab.shift[l, 0], p.eps)
    qkv = y @ p.w_qkv[l].T
    q = qkv[:, :Hq * d].reshape(H, Hq, d)
    k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(H, Hkv, d)
    v = qkv[:, (Hq + Hkv) * d:].reshape(H, Hkv, d)
    if p.rope_base:
        # action token i of a request with a P-token prefix sits at position P + i
        pos = k_pre.shape[0] + np.arange(H)
        q = rope(q, pos, p.rope_base)
        k = rope(k, pos, p.rope_base)
    keys = np.concatenate([k_pre, k], axis=0)
    vals = np.concatenate([v_pre, v], axis=0)
    if trace is not None:
        o, pr = attention(q, keys, vals, return_probs=True)
        trace.setdefault("probs", []).append(pr)
    else:
        o = attention(q, keys, vals)
    h = h + tab.gate[l, 0] * (o.reshape(H, Hq * d) @ p.w_o[l].T)
    y = ada_rms_norm(h, tab.scale[l, 1], tab.shift[l, 1], p.eps)
    u = gelu_tanh(y @ p.w_gate[l].T) * (y @ p.w_up[l].T)
    h = h + tab.gate[l, 1] * (u @ p.w_down[l].T)
    if trace is not None:
        trace.setdefault("h", []).append(h.copy())
    return h


def velocity(x: np.ndarray, tab: StepTables, p: OracleParams,
             k_pre: Sequence[np.ndarray], v_pre: Sequence[np.ndarray],
             trace: Optional[dict] = None) -> np.ndarray:
    """Velocity field of one request at one step: h = x W_in^T + b_in, the L
    expert layers, then v = adaRMSNorm(h; final modulation) W_out^T + b_out
    (the final norm has no gate)."""
    h = x @ p.w_in.T + p.b_in
    for l in range(p.L):
        h = expert_layer(h, l, tab, p, k_pre[l], v_pre[l], trace)
    y = ada_rms_norm(h, tab.scale_f, tab.shift_f, p.eps)
    return y @ p.w_out.T + p.b_out


def denoise_row(x0: np.ndarray, tables: Sequence[StepTables], p: OracleParams,
                k_pre: Sequence[np.ndarray], v_pre: Sequence[np.ndarray],
                trace: Optional[dict] = None) -> np.ndarray:
    """Euler integration of one request: x_{k+1} = x_k + dt_k v(x_k, t_k),
    with the prefix K/V fixed across all steps (report Sec. 5.1)."""
    x = np.asarray(x0, dtype=F64).copy()
    for tab in tables:
        x = x + tab.dt * velocity(x, tab, p, k_pre, v_pre, trace)
    return x


def denoise(x0: np.ndarray, t_grid: Sequence[float], p: OracleParams,
            k_pre_rows, v_pre_rows, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Batched denoise: rows are independent requests (report Sec. 5.5,
    "Distribute the appropriate unit of work").  ``k_pre_rows[b][l]`` is
    [P_b][Hkv][d].  ``rows`` selects a subset of rows to evaluate."""
    tables = modulation_tables(t_grid, p)
    sel = range(x0.shape[0]) if rows is None else rows
    return np.stack([denoise_row(x0[b], tables, p, [np.asarray(a, F64) for a in k_pre_rows[b]],
                                 [np.asarray(a, F64) for a in v_pre_rows[b]])
                     for b in sel])


# ---------------------------------------------------------------------------
# Brute force: the whole [prefix | action] sequence recomputed every step.
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PrefixStack:
    """Weights of a stand-in vision-language stack that produces the prefix:
    per layer a plain RMSNorm, a QKV projection, an output projection and a
    GeGLU MLP.  Only used to check that caching the prefix K/V is exact."""
    w_qkv: List[np.ndarray]
    w_o: List[np.ndarray]
    w_gate: List[np.ndarray]
    w_up: List[np.ndarray]
    w_down: List[np.ndarray]


def _rms(h, eps):
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def prefix_stack_kv(z: np.ndarray, ps: PrefixStack, p: OracleParams):
    """Run the prefix stack alone on prefix hidden states z [P][Dp] and return
    its per-layer K/V (lists of [P][Hkv][d]): the cache a runner keeps.  The
    stack's width Dp is z's; with p.rope_base its queries and keys sit at
    positions 0..P-1."""
    ks, vs, _ = _prefix_stack_run(z, ps, p)
    return ks, vs


def prefix_stack_hidden(z: np.ndarray, ps: PrefixStack, p: OracleParams) -> List[np.ndarray]:
    """The input hidden state of every layer of the prefix stack ([P][Dp] per
    layer; layer 0's is z): what a runner holds when it produces the cache
    layer by layer."""
    return _prefix_stack_run(z, ps, p)[2]


def _prefix_stack_run(z, ps, p):
    P = z.shape[0]
    Hq, Hkv, d = p.Hq, p.Hkv, p.d
    ks, vs, hs = [], [], []
    h = np.asarray(z, dtype=F64).copy()
    pos = np.arange(P)
    for l in range(p.L):
        hs.append(h.copy())
        y = _rms(h, p.eps)
        qkv = y @ ps.w_qkv[l].T
        q = qkv[:, :Hq * d].reshape(P, Hq, d)
        k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(P, Hkv, d)
        v = qkv[:, (Hq + Hkv) * d:].reshape(P, Hkv, d)
        if p.rope_base:
            q = rope(q, pos, p.rope_base)
            k = rope(k, pos, p.rope_base)
        ks.append(k)
        vs.append(v)
        o = attention(q, k, v)
        h = h + o.reshape(P, Hq * d) @ ps.w_o[l].T
        y = _rms(h, p.eps)
        h = h + (gelu_tanh(y @ ps.w_gate[l].T) * (y @ ps.w_up[l].T)) @ ps.w_down[l].T
    return ks, vs, hs


def prefix_kv_from_hidden(hs: Sequence[np.ndarray], w_kv: Sequence[np.ndarray], p: OracleParams):
    """The prefix production step: per layer l, the cached keys and values of
    a P-token prefix from that layer's input hidden state hs[l] [P][Dp].

    y = h / sqrt(mean(h^2) + eps) (a plain RMSNorm, no gain); [k | v] = y W_kv[l]^T
    where W_kv[l] [2 Hkv d][Dp] holds the layer's key rows then its value rows;
    with p.rope_base the keys are rotated at positions 0..P-1 (the prefix comes
    first in the joint sequence).  Returns lists of [P][Hkv][d].  PhyAI report
    Sec. 5.1: the prefix is computed once per observation and its per-layer K/V
    is cached."""
    Hkv, d = p.Hkv, p.d
    ks, vs = [], []
    for l, h in enumerate(hs):
        h = np.asarray(h, dtype=F64)
        P = h.shape[0]
        y = h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + p.eps)
        kv = y @ np.asarray(w_kv[l], dtype=F64).T
        k = kv[:, :Hkv * d].reshape(P, Hkv, d)
        v = kv[:, Hkv * d:].reshape(P, Hkv, d)
        if p.rope_base:
            k = rope(k, np.arange(P), p.rope_base)
        ks.append(k)
        vs.append(v)
    return ks, vs


def brute_force_denoise_row(x0: np.ndarray, t_grid: Sequence[float], p: OracleParams,
                            z: np.ndarray, ps: PrefixStack) -> np.ndarray:
    """Every Euler step recomputes the joint [prefix | action] sequence under a
    block-causal mask: prefix tokens see only prefix tokens, action tokens see
    everything.  Prefix tokens use the prefix stack's weights (width Dp, z's),
    action tokens the expert's.  With p.rope_base every query and key is
    rotated at its position in the joint sequence.  No cache is kept between
    steps."""
    tables = modulation_tables(t_grid, p)
    Hq, Hkv, d = p.Hq, p.Hkv, p.d
    P = z.shape[0]
    x = np.asarray(x0, dtype=F64).copy()
    H = x.shape[0]
    S = P + H
    mask = np.zeros((S, S), dtype=bool)
    mask[:P, :P] = True
    mask[P:, :] = True
    for tab in tables:
        hp = z.copy()
        ha = x @ p.w_in.T + p.b_in
        for l in range(p.L):
            yp = _rms(hp, p.eps)
            ya = ada_rms_norm(ha, tab.scale[l, 0], tab.shift[l, 0], p.eps)
            qkv = np.concatenate([yp @ ps.w_qkv[l].T, ya @ p.w_qkv[l].T], axis=0)
            q = qkv[:, :Hq * d].reshape(S, Hq, d)
            k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(S, Hkv, d)
            v = qkv[:, (Hq + Hkv) * d:].reshape(S, Hkv, d)
            if p.rope_base:
                q = rope(q, np.arange(S), p.rope_base)
                k = rope(k, np.arange(S), p.rope_base)
            o = attention(q, k, v, mask=mask).reshape(S, Hq * d)
            hp = hp + o[:P] @ ps.w_o[l].T
            ha = ha + tab.gate[l, 0] * (o[P:] @ p.w_o[l].T)
            yp = _rms(hp, p.eps)
            hp = hp + (gelu_tanh(yp @ ps.w_gate[l].T) * (yp @ ps.w_up[l].T)) @ ps.w_down[l].T
            ya = ada_rms_norm(ha, tab.scale[l, 1], tab.shift[l, 1], p.eps)
            ha = ha + tab.gate[l, 1] * (
                (gelu_tanh(ya @ p.w_gate[l].T) * (ya @ p.w_up[l].T)) @ p.w_down[l].T)
        y = ada_rms_norm(ha, tab.scale_f, tab.shift_f, p.eps)
        x = x + tab.dt * (y @ p.w_out.T + p.b_out)
    return x
