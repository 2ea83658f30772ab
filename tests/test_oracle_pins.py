"""Pins for the float64 oracle, against things other than itself.

Each test ties an oracle function to a closed form, to a library routine that
implements the textbook definition (PyTorch CPU float64: silu, gelu, rms_norm,
scaled_dot_product_attention), to brute-force recomputation, or to an
invariant the mathematics fixes.  They are chosen so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import oracle
from oracle.expert import PrefixStack, StepTables
import workloads as wl

F64 = np.float64


def _tiny(**kw):
    return wl.TINY_FP32.replace(**kw)


def _params(cfg, seed=None):
    return oracle.params_from_weights(cfg, wl.make_weights(cfg, seed=seed))


def _prefix(cfg, lengths=None, seed=None, std=1.0):
    ks, vs = wl.make_prefix(cfg, lengths=lengths, seed=seed, std=std)
    return ([[a.astype(F64) for a in r] for r in ks], [[a.astype(F64) for a in r] for r in vs])


# --------------------------------------------------------------------------
# Timestep embedding and time MLP
# --------------------------------------------------------------------------

def test_sinusoidal_closed_form_dim4():
    # dim 4 -> two periods, 4e-3 and 4.0 (the end points of the geometric ladder)
    for t in (0.0, 0.5, 1.0, 0.3):
        e = oracle.sinusoidal_embedding(t, 4)
        want = [math.sin(2 * math.pi * t / 4e-3), math.sin(2 * math.pi * t / 4.0),
                math.cos(2 * math.pi * t / 4e-3), math.cos(2 * math.pi * t / 4.0)]
        np.testing.assert_allclose(e, want, rtol=0, atol=1e-12)
    e0 = oracle.sinusoidal_embedding(0.0, 256)
    np.testing.assert_array_equal(e0[:128], 0.0)
    np.testing.assert_array_equal(e0[128:], 1.0)


def test_sinusoidal_periods_geometric_and_unit_norm():
    dim = 64
    t = 0.37
    e = oracle.sinusoidal_embedding(t, dim)
    # sin^2 + cos^2 = 1 per frequency
    np.testing.assert_allclose(e[:32] ** 2 + e[32:] ** 2, 1.0, atol=1e-13)
    # recover the angles at a tiny t (no wrap) and check the period ladder
    ts = 1e-6
    e = oracle.sinusoidal_embedding(ts, dim)
    ang = np.arctan2(e[:32], e[32:])
    period = 2 * math.pi * ts / ang
    np.testing.assert_allclose(period[0], 4e-3, rtol=1e-9)
    np.testing.assert_allclose(period[-1], 4.0, rtol=1e-9)
    ratio = period[1:] / period[:-1]
    np.testing.assert_allclose(ratio, (4.0 / 4e-3) ** (1 / 31), rtol=1e-9)


def test_swish_matches_library():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(oracle.swish(x), Fn.silu(torch.tensor(x)).numpy(), rtol=1e-14,
                               atol=1e-300)


def test_gelu_tanh_matches_library():
    x = np.linspace(-12, 12, 2001)
    want = Fn.gelu(torch.tensor(x), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.gelu_tanh(x), want, rtol=1e-12, atol=1e-15)
    # and it stays within the known 1e-3 band of the erf form
    exact = Fn.gelu(torch.tensor(x)).numpy()
    assert np.max(np.abs(oracle.gelu_tanh(x) - exact)) < 1e-3


def test_time_conditioning_zero_weight_closed_form():
    cfg = _tiny()
    p = _params(cfg)
    p.w_t1[:] = 0
    p.w_t2[:] = 0
    c = oracle.time_conditioning(0.42, p)
    want = Fn.silu(torch.tensor(p.b_t2)).numpy()
    np.testing.assert_allclose(c, want, rtol=1e-14)


def _swish(x: float) -> float:
    return x / (1.0 + math.exp(-x))


def test_time_conditioning_one_hot_closed_form():
    # W_t1 with one 1 at [j][i] routes embedding channel i into hidden unit j;
    # W_t2 = identity, b_t2 = 0.  Then c_j = swish(swish(e_i(t) + b1_j)) and
    # every other c_m = swish(swish(b1_m)).  Channel i = half - 1 is sin(2 pi t / 4),
    # which is 1 at t = 1 and 0 at t = 0, so a grid read backwards (1 - t) fails,
    # a dropped inner swish fails, and j != i makes a transposed W_t1 fail.
    cfg = _tiny()
    p = _params(cfg)
    D = cfg.width
    half = D // 2
    i, j = half - 1, 3
    p.w_t1[:] = 0
    p.w_t1[j, i] = 1.0
    p.b_t1[:] = np.linspace(-0.5, 0.7, D)
    p.w_t2[:] = np.eye(D)
    p.b_t2[:] = 0
    for t, e_i in ((1.0, 1.0), (0.0, 0.0), (0.5, math.sin(math.pi / 4))):
        c = oracle.time_conditioning(t, p)
        assert c[j] == pytest.approx(_swish(_swish(e_i + p.b_t1[j])), abs=1e-14)
        others = [m for m in range(D) if m != j]
        want = np.array([_swish(_swish(p.b_t1[m])) for m in others])
        np.testing.assert_allclose(c[others], want, rtol=0, atol=1e-14)


def test_time_conditioning_second_layer_closed_form():
    # W_t1 = 0 makes the hidden layer z = swish(b_t1), a known vector; a W_t2
    # with one 1 at [a][b] (a != b) gives c_a = swish(z_b + b2_a) and
    # c_m = swish(b2_m) elsewhere, so a transposed W_t2 or a dropped outer
    # swish fails.
    cfg = _tiny()
    p = _params(cfg)
    D = cfg.width
    a, b = 10, 200
    p.w_t1[:] = 0
    p.b_t1[:] = np.linspace(-2.0, 3.0, D)
    p.w_t2[:] = 0
    p.w_t2[a, b] = 1.0
    p.b_t2[:] = np.linspace(0.4, -0.3, D)
    c = oracle.time_conditioning(0.25, p)
    z_b = _swish(p.b_t1[b])
    assert c[a] == pytest.approx(_swish(z_b + p.b_t2[a]), abs=1e-14)
    others = [m for m in range(D) if m != a]
    np.testing.assert_allclose(c[others], [_swish(p.b_t2[m]) for m in others], rtol=0, atol=1e-14)


def test_time_conditioning_and_tables_against_library():
    # Random non-zero weights (large enough that both swishes are non-linear),
    # several timesteps: PyTorch float64 linear / silu over an embedding built
    # from the closed form, then the modulation rows through linear again.
    cfg = _tiny()
    p = _params(cfg)
    g = np.random.default_rng(11)
    D, L = cfg.width, cfg.layers
    p.w_t1[:] = g.standard_normal((D, D)) * 0.2
    p.w_t2[:] = g.standard_normal((D, D)) * 0.2
    p.b_t1[:] = g.standard_normal(D) * 0.5
    p.b_t2[:] = g.standard_normal(D) * 0.5
    half = D // 2
    period = 4e-3 * (4.0 / 4e-3) ** (torch.arange(half, dtype=torch.float64) / (half - 1))
    grid = [1.0, 0.7, 0.3, 0.05, 0.0]
    tabs = oracle.modulation_tables(grid, p)
    T = lambda a: torch.tensor(a, dtype=torch.float64)  # noqa: E731
    for k, t in enumerate(grid):
        ang = 2 * math.pi * t / period
        e = torch.cat([torch.sin(ang), torch.cos(ang)])
        c = Fn.silu(Fn.linear(Fn.silu(Fn.linear(e, T(p.w_t1), T(p.b_t1))), T(p.w_t2), T(p.b_t2)))
        # the fast embedding channels reach angles of ~1.6e3 rad: allow round-off there
        np.testing.assert_allclose(oracle.time_conditioning(t, p), c.numpy(), rtol=1e-10, atol=1e-12)
        if k == len(grid) - 1:
            break
        m = Fn.linear(c, T(p.w_mod.reshape(-1, D)), T(p.b_mod.reshape(-1))).reshape(L, 2, 3, D).numpy()
        f = Fn.linear(c, T(p.w_modf), T(p.b_modf)).numpy()
        tab = tabs[k]
        np.testing.assert_allclose(tab.scale, m[:, :, 0], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(tab.shift, m[:, :, 1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(tab.gate, m[:, :, 2], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(tab.scale_f, f[:D], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(tab.shift_f, f[D:], rtol=1e-10, atol=1e-12)
        assert tab.dt == pytest.approx(grid[k + 1] - t, abs=1e-15)


def test_tables_chunk_order_and_dt():
    cfg = _tiny()
    p = _params(cfg)
    p.w_mod[:] = 0
    p.w_modf[:] = 0
    grid = wl.uniform_grid(cfg.steps)
    tabs = oracle.modulation_tables(grid, p)
    D = cfg.width
    assert len(tabs) == cfg.steps
    for tab in tabs:
        assert tab.dt == pytest.approx(-1.0 / cfg.steps, abs=1e-15)
        for l in range(cfg.layers):
            for j in range(2):
                b = p.b_mod[2 * l + j]
                np.testing.assert_array_equal(tab.scale[l, j], b[:D])
                np.testing.assert_array_equal(tab.shift[l, j], b[D:2 * D])
                np.testing.assert_array_equal(tab.gate[l, j], b[2 * D:])
        np.testing.assert_array_equal(tab.scale_f, p.b_modf[:D])
        np.testing.assert_array_equal(tab.shift_f, p.b_modf[D:])


def test_tables_one_hot_modulation_row():
    # W_mod with a single 1 at [2l+j][r][i] copies c_i into output r
    cfg = _tiny()
    p = _params(cfg)
    p.w_mod[:] = 0
    p.b_mod[:] = 0
    D = cfg.width
    p.w_mod[3, 2 * D + 5, 7] = 1.0   # layer 1, MLP norm, gate channel 5 <- c[7]
    tab = oracle.modulation_tables([0.8, 0.4], p)[0]
    c = oracle.time_conditioning(0.8, p)
    assert tab.gate[1, 1, 5] == pytest.approx(c[7], abs=1e-15)
    assert np.count_nonzero(tab.gate) == 1
    assert np.count_nonzero(tab.scale) == 0 and np.count_nonzero(tab.shift) == 0


# --------------------------------------------------------------------------
# Normalisation and attention against library routines
# --------------------------------------------------------------------------

def test_ada_rms_norm_against_library():
    g = np.random.default_rng(5)
    h = g.standard_normal((7, 96)) * 3.0
    sc = g.standard_normal(96) * 0.1
    sh = g.standard_normal(96) * 0.1
    eps = 1e-6
    base = Fn.rms_norm(torch.tensor(h), (96,), eps=eps).numpy()
    np.testing.assert_allclose(oracle.ada_rms_norm(h, 0 * sc, 0 * sh, eps), base, rtol=1e-13)
    np.testing.assert_allclose(oracle.ada_rms_norm(h, sc, sh, eps), base * (1 + sc) + sh,
                               rtol=1e-13, atol=1e-15)
    # eps keeps a zero row finite (zero-weight closed forms rely on it)
    z = oracle.ada_rms_norm(np.zeros((1, 8)), np.zeros(8), np.full(8, 0.5), eps)
    np.testing.assert_array_equal(z, 0.5)


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (4, 4)])
def test_attention_against_sdpa(Hq, Hkv):
    g = np.random.default_rng(Hq * 10 + Hkv)
    T, S, d = 9, 23, 16
    q = g.standard_normal((T, Hq, d))
    k = g.standard_normal((S, Hkv, d)) * 2.0
    v = g.standard_normal((S, Hkv, d))
    o = oracle.attention(q, k, v)
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(k).permute(1, 0, 2)[None]
    vt = torch.tensor(v).permute(1, 0, 2)[None]
    ref = Fn.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_attention_mask_against_sdpa_and_sharp_softmax():
    g = np.random.default_rng(11)
    T, S, d, Hq = 6, 30, 32, 4
    q = g.standard_normal((T, Hq, d))
    k = g.standard_normal((S, 1, d)) * 8.0        # "sharp" logits
    v = g.standard_normal((S, 1, d))
    mask = g.random((T, S)) < 0.6
    mask[:, 0] = True
    o = oracle.attention(q, k, v, mask=mask)
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(k).permute(1, 0, 2)[None]
    vt = torch.tensor(v).permute(1, 0, 2)[None]
    ref = Fn.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(mask),
                                          enable_gqa=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_invariants():
    g = np.random.default_rng(3)
    T, S, d, Hq = 5, 17, 8, 4
    q = g.standard_normal((T, Hq, d))
    k = g.standard_normal((S, 1, d))
    v = g.standard_normal((S, 1, d))
    o, pr = oracle.attention(q, k, v, return_probs=True)
    np.testing.assert_allclose(pr.sum(axis=-1), 1.0, atol=1e-14)
    assert np.all(pr > 0)
    # a single key returns its value
    o1 = oracle.attention(q, k[:1], v[:1])
    np.testing.assert_allclose(o1, np.broadcast_to(v[:1, 0][None], (T, Hq, d)), atol=1e-15)
    # Hkv = Hq with the KV head replicated equals GQA with one KV head
    kr = np.repeat(k, Hq, axis=1)
    vr = np.repeat(v, Hq, axis=1)
    np.testing.assert_allclose(oracle.attention(q, kr, vr), o, atol=1e-14)
    # identical keys -> plain mean of values
    ku = np.repeat(k[:1], S, axis=0)
    np.testing.assert_allclose(oracle.attention(q, ku, v),
                               np.broadcast_to(v[:, 0].mean(axis=0), (T, Hq, d)), atol=1e-13)


# --------------------------------------------------------------------------
# Whole-loop closed forms
# --------------------------------------------------------------------------

def test_zero_weights_velocity_is_output_bias():
    """All matrices zero, biases nonzero: v = b_out, so x_K = x_0 + (t_K - t_0) b_out."""
    cfg = _tiny()
    p = _params(cfg)
    for name in ("w_in", "w_out", "w_t1", "w_t2", "w_mod", "w_modf"):
        getattr(p, name)[:] = 0
    for lst in (p.w_qkv, p.w_o, p.w_gate, p.w_up, p.w_down):
        for m in lst:
            m[:] = 0
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)
    for K in (1, 3, 4, 10):
        out = oracle.denoise(x0, wl.uniform_grid(K), p, ks, vs)
        np.testing.assert_allclose(out, x0 - p.b_out, rtol=0, atol=1e-14)
    out = oracle.denoise(x0, [1.0, 0.7, 0.55, 0.1], p, ks, vs)
    np.testing.assert_allclose(out, x0 - 0.9 * p.b_out, rtol=0, atol=1e-14)


def test_zero_output_projection_constant_velocity():
    """Only W_out zero (everything else random): the velocity is the constant
    b_out, so K steps of -1/K equal one step of -1."""
    cfg = _tiny()
    p = _params(cfg)
    p.w_out[:] = 0
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)
    one = oracle.denoise(x0, wl.uniform_grid(1), p, ks, vs)
    many = oracle.denoise(x0, wl.uniform_grid(7), p, ks, vs)
    np.testing.assert_allclose(many, one, rtol=0, atol=1e-12)
    np.testing.assert_allclose(one, x0 - p.b_out, rtol=0, atol=1e-14)


def test_gates_zero_makes_layers_identity():
    """Gate chunks zero: every layer leaves h unchanged, so the velocity is the
    final modulated norm of the input projection (independently restated with
    library routines)."""
    cfg = _tiny()
    p = _params(cfg)
    D = cfg.width
    p.w_mod[:, 2 * D:, :] = 0
    p.b_mod[:, 2 * D:] = 0
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)
    grid = wl.uniform_grid(2)
    tabs = oracle.modulation_tables(grid, p)
    x = torch.tensor(x0[0])
    for tab in tabs:
        h = Fn.linear(x, torch.tensor(p.w_in), torch.tensor(p.b_in))
        y = Fn.rms_norm(h, (D,), eps=p.eps) * (1 + torch.tensor(tab.scale_f)) + torch.tensor(
            tab.shift_f)
        x = x + tab.dt * Fn.linear(y, torch.tensor(p.w_out), torch.tensor(p.b_out))
    out = oracle.denoise(x0, grid, p, ks, vs)
    np.testing.assert_allclose(out[0], x.numpy(), rtol=1e-12, atol=1e-13)


def _torch_velocity(x, tab, p, kpre, vpre):
    """The expert velocity restated with PyTorch float64 library routines
    (linear, rms_norm, scaled_dot_product_attention, gelu).  Used only to pin
    the oracle's composition (q/k/v split, head mapping, gate placement)."""
    T = lambda a: torch.tensor(np.asarray(a))  # noqa: E731
    D, Hq, Hkv, d = p.D, p.Hq, p.Hkv, p.d
    H = x.shape[0]
    h = Fn.linear(T(x), T(p.w_in), T(p.b_in))
    for l in range(p.L):
        y = Fn.rms_norm(h, (D,), eps=p.eps) * (1 + T(tab.scale[l, 0])) + T(tab.shift[l, 0])
        qkv = Fn.linear(y, T(p.w_qkv[l]))
        q, k, v = torch.split(qkv, [Hq * d, Hkv * d, Hkv * d], dim=-1)
        q = q.reshape(H, Hq, d).permute(1, 0, 2)
        k = torch.cat([T(kpre[l]), k.reshape(H, Hkv, d)], 0).permute(1, 0, 2)
        v = torch.cat([T(vpre[l]), v.reshape(H, Hkv, d)], 0).permute(1, 0, 2)
        o = Fn.scaled_dot_product_attention(q[None], k[None], v[None], enable_gqa=True)[0]
        o = o.permute(1, 0, 2).reshape(H, Hq * d)
        h = h + T(tab.gate[l, 0]) * Fn.linear(o, T(p.w_o[l]))
        y = Fn.rms_norm(h, (D,), eps=p.eps) * (1 + T(tab.scale[l, 1])) + T(tab.shift[l, 1])
        u = Fn.gelu(Fn.linear(y, T(p.w_gate[l])), approximate="tanh") * Fn.linear(y, T(p.w_up[l]))
        h = h + T(tab.gate[l, 1]) * Fn.linear(u, T(p.w_down[l]))
    y = Fn.rms_norm(h, (D,), eps=p.eps) * (1 + T(tab.scale_f)) + T(tab.shift_f)
    return Fn.linear(y, T(p.w_out), T(p.b_out)).numpy()


@pytest.mark.parametrize("Hkv", [1, 2])
def test_velocity_against_library_restatement(Hkv):
    cfg = _tiny(n_kv_heads=Hkv)
    p = _params(cfg)
    # large modulation so that a misplaced scale/shift/gate shows
    p.b_mod *= 20.0
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)[0]
    tab = oracle.modulation_tables([0.6, 0.3], p)[0]
    v = oracle.velocity(x0, tab, p, ks[0], vs[0])
    ref = _torch_velocity(x0, tab, p, ks[0], vs[0])
    np.testing.assert_allclose(v, ref, rtol=1e-10, atol=1e-12)


def test_w4a16_dequantised_values():
    """int4 records: code * scale, low nibble = even k, codes clamp to [-8, 7]."""
    cfg = _tiny(dtype=wl.W4A16)
    W = wl.make_weights(cfg)
    p = oracle.params_from_weights(cfg, W)
    m = W["w_qkv"][0]
    assert m.codes.min() >= -8 and m.codes.max() <= 7
    lo = (m.packed & 0xF).astype(np.int16)
    hi = (m.packed >> 4).astype(np.int16)
    lo = np.where(lo > 7, lo - 16, lo)
    hi = np.where(hi > 7, hi - 16, hi)
    np.testing.assert_array_equal(lo, m.codes[:, 0::2])
    np.testing.assert_array_equal(hi, m.codes[:, 1::2])
    r, c = 5, 200
    assert p.w_qkv[0][r, c] == float(m.codes[r, c]) * float(m.scales[r, c // 128])


# --------------------------------------------------------------------------
# Cached prefix = brute-force joint sequence; splitting; independence
# --------------------------------------------------------------------------

def _prefix_stack(cfg, seed):
    g = np.random.default_rng(seed)
    D, F, L = cfg.width, cfg.mlp_dim, cfg.layers
    qkv = cfg.qkv_dim
    n = lambda *s: g.standard_normal(s) * 0.05  # noqa: E731
    return PrefixStack(w_qkv=[n(qkv, D) for _ in range(L)], w_o=[n(D, cfg.attn_dim) for _ in range(L)],
                       w_gate=[n(F, D) for _ in range(L)], w_up=[n(F, D) for _ in range(L)],
                       w_down=[n(D, F) for _ in range(L)])


@pytest.mark.parametrize("P,Hkv", [(64, 1), (13, 2), (0, 1)])
def test_cached_prefix_equals_brute_force(P, Hkv):
    cfg = _tiny(n_kv_heads=Hkv)
    p = _params(cfg)
    p.b_mod *= 5.0
    ps = _prefix_stack(cfg, 99)
    z = np.random.default_rng(7).standard_normal((P, cfg.width))
    x0 = wl.make_noise(cfg).astype(F64)[0]
    grid = wl.uniform_grid(cfg.steps)
    if P > 0:
        ks, vs = oracle.prefix_stack_kv(z, ps, p)
    else:
        ks = [np.zeros((0, Hkv, cfg.head_dim))] * cfg.layers
        vs = ks
    cached = oracle.denoise_row(x0, oracle.modulation_tables(grid, p), p, ks, vs)
    brute = oracle.brute_force_denoise_row(x0, grid, p, z, ps)
    np.testing.assert_allclose(cached, brute, rtol=0, atol=1e-11)
    # the cache does matter: a different prefix changes the result
    if P > 0:
        ks2 = [k * 1.5 for k in ks]
        other = oracle.denoise_row(x0, oracle.modulation_tables(grid, p), p, ks2, vs)
        assert np.max(np.abs(other - cached)) > 1e-6


def test_step_split_invariance():
    cfg = _tiny()
    p = _params(cfg)
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)
    grid = wl.uniform_grid(4)
    full = oracle.denoise(x0, grid, p, ks, vs)
    half = oracle.denoise(x0, grid[:3], p, ks, vs)
    split = oracle.denoise(half, grid[2:], p, ks, vs)
    np.testing.assert_array_equal(full, split)


def test_rows_independent_and_ragged():
    cfg = _tiny(batch=3)
    p = _params(cfg)
    lens = [64, 5, 33]
    ks, vs = _prefix(cfg, lengths=lens)
    x0 = wl.make_noise(cfg).astype(F64)
    grid = wl.uniform_grid(cfg.steps)
    allrows = oracle.denoise(x0, grid, p, ks, vs)
    for b in range(3):
        alone = oracle.denoise(x0[b:b + 1], grid, p, [ks[b]], [vs[b]])
        np.testing.assert_array_equal(allrows[b], alone[0])
    # reordering the batch permutes the result
    perm = [2, 0, 1]
    re = oracle.denoise(x0[perm], grid, p, [ks[i] for i in perm], [vs[i] for i in perm])
    np.testing.assert_array_equal(re, allrows[perm])


def test_attention_rows_sum_to_one_in_trace():
    cfg = _tiny()
    p = _params(cfg)
    ks, vs = _prefix(cfg)
    x0 = wl.make_noise(cfg).astype(F64)[0]
    tr = {}
    oracle.denoise_row(x0, oracle.modulation_tables(wl.uniform_grid(2), p), p, ks[0], vs[0], tr)
    assert len(tr["probs"]) == 2 * cfg.layers
    for pr in tr["probs"]:
        assert pr.shape == (cfg.n_q_heads, cfg.chunk, cfg.prefix + cfg.chunk)
        np.testing.assert_allclose(pr.sum(-1), 1.0, atol=1e-13)


# --------------------------------------------------------------------------
# Rotary position embedding (vla.cpp abstract, page 1: positional-index
# precision matters) and the prefix production step
# --------------------------------------------------------------------------

def test_rope_closed_forms():
    base = 10000.0
    g = np.random.default_rng(21)
    x = g.standard_normal((5, 3, 64))
    # position 0 is the identity
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(5, int), base), x)
    # d = 2: one pair turned by the plain angle pos (base^0 = 1)
    v = np.array([[[0.3, -1.2]]])
    for pos in (1, 7, 1000):
        got = oracle.rope(v, np.array([pos]), base)[0, 0]
        c, s_ = math.cos(pos), math.sin(pos)
        np.testing.assert_allclose(got, [0.3 * c + 1.2 * s_, -1.2 * c + 0.3 * s_], rtol=0, atol=1e-13)
    # a one-hot channel i at position p lands on (cos, sin) of p * base^(-2i/d) in channels i, i + d/2
    d = 64
    for i in (0, 5, 31):
        e = np.zeros((1, 1, d))
        e[0, 0, i] = 1.0
        ang = 37 * math.pow(base, -2.0 * i / d)
        out = oracle.rope(e, np.array([37]), base)[0, 0]
        want = np.zeros(d)
        want[i] = math.cos(ang)
        want[i + d // 2] = math.sin(ang)
        np.testing.assert_allclose(out, want, rtol=0, atol=1e-13)


def test_rope_complex_rotation_norm_and_relative_positions():
    base = 10000.0
    g = np.random.default_rng(22)
    d = 256
    x = g.standard_normal((7, 2, d))
    pos = np.array([0, 1, 5, 50, 968, 1017, 3])
    # pairs (i, i + d/2) as complex numbers, multiplied by e^{j a}
    z = x[..., :d // 2] + 1j * x[..., d // 2:]
    a = pos[:, None, None] * base ** (-np.arange(d // 2) * 2.0 / d)[None, None, :]
    zr = z * np.exp(1j * a)
    out = oracle.rope(x, pos, base)
    np.testing.assert_allclose(out, np.concatenate([zr.real, zr.imag], axis=-1), rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # q . k depends only on the position difference
    q, k = g.standard_normal((1, 1, d)), g.standard_normal((1, 1, d))
    def dot(m, n):
        return float(np.sum(oracle.rope(q, np.array([m]), base) * oracle.rope(k, np.array([n]), base)))
    for m, n, sh in ((3, 10, 100), (968, 0, 37), (50, 50, 900)):
        assert dot(m, n) == pytest.approx(dot(m + sh, n + sh), abs=1e-10)
    assert abs(dot(3, 10) - dot(3, 11)) > 1e-6


def _prefix_stack_w(cfg, seed, Dp=None):
    g = np.random.default_rng(seed)
    D = cfg.width if Dp is None else Dp
    L, F = cfg.layers, cfg.mlp_dim
    n = lambda *s: g.standard_normal(s) * 0.05  # noqa: E731
    return PrefixStack(w_qkv=[n(cfg.qkv_dim, D) for _ in range(L)], w_o=[n(D, cfg.attn_dim) for _ in range(L)],
                       w_gate=[n(F, D) for _ in range(L)], w_up=[n(F, D) for _ in range(L)],
                       w_down=[n(D, F) for _ in range(L)])


@pytest.mark.parametrize("P,Hkv,Dp", [(64, 1, None), (13, 2, None), (0, 1, None), (40, 1, 384)])
def test_cached_prefix_equals_brute_force_with_rope(P, Hkv, Dp):
    # every query and key rotated at its place in the joint [prefix | action]
    # sequence: the cached path must rotate action tokens at P_b + i
    cfg = _tiny(n_kv_heads=Hkv)
    p = _params(cfg)
    p.rope_base = 10000.0
    p.b_mod *= 5.0
    ps = _prefix_stack_w(cfg, 99, Dp)
    z = np.random.default_rng(7).standard_normal((P, cfg.width if Dp is None else Dp))
    x0 = wl.make_noise(cfg).astype(F64)[0]
    grid = wl.uniform_grid(cfg.steps)
    if P > 0:
        ks, vs = oracle.prefix_stack_kv(z, ps, p)
    else:
        ks = [np.zeros((0, Hkv, cfg.head_dim))] * cfg.layers
        vs = ks
    cached = oracle.denoise_row(x0, oracle.modulation_tables(grid, p), p, ks, vs)
    brute = oracle.brute_force_denoise_row(x0, grid, p, z, ps)
    np.testing.assert_allclose(cached, brute, rtol=0, atol=1e-11)
    # the rotation matters for the result
    p0 = oracle.params_from_weights(cfg, wl.make_weights(cfg))
    p0.b_mod *= 5.0
    if P > 0:
        ks0, vs0 = oracle.prefix_stack_kv(z, ps, p0)
        plain = oracle.denoise_row(x0, oracle.modulation_tables(grid, p0), p0, ks0, vs0)
        assert np.max(np.abs(plain - cached)) > 1e-6


@pytest.mark.parametrize("rope_base,Dp", [(0.0, None), (10000.0, None), (10000.0, 384)])
def test_prefix_kv_from_hidden_matches_prefix_stack(rope_base, Dp):
    # the production step (norm + key/value rows + rotation of the keys) gives
    # the cache the whole stack gives, layer by layer
    cfg = _tiny(n_kv_heads=2)
    p = _params(cfg)
    p.rope_base = rope_base
    ps = _prefix_stack_w(cfg, 5, Dp)
    P = 30
    z = np.random.default_rng(8).standard_normal((P, cfg.width if Dp is None else Dp)) * 2.0
    ks, vs = oracle.prefix_stack_kv(z, ps, p)
    hs = oracle.prefix_stack_hidden(z, ps, p)
    assert len(hs) == cfg.layers and np.array_equal(hs[0], z)
    qd = cfg.n_q_heads * cfg.head_dim
    w_kv = [w[qd:] for w in ps.w_qkv]
    k2, v2 = oracle.prefix_kv_from_hidden(hs, w_kv, p)
    for l in range(cfg.layers):
        np.testing.assert_allclose(k2[l], ks[l], rtol=0, atol=1e-12)
        np.testing.assert_allclose(v2[l], vs[l], rtol=0, atol=1e-12)
    # against a library restatement for one layer: torch rms_norm, then linear
    y = Fn.rms_norm(torch.tensor(hs[1]), (hs[1].shape[1],), eps=p.eps)
    kv = Fn.linear(y, torch.tensor(w_kv[1])).numpy()
    np.testing.assert_allclose(v2[1].reshape(P, -1), kv[:, 2 * cfg.head_dim:], rtol=1e-12, atol=1e-13)
    if not rope_base:
        np.testing.assert_allclose(k2[1].reshape(P, -1), kv[:, :2 * cfg.head_dim], rtol=1e-12, atol=1e-13)
