"""Rotary position embedding and prefix production on the GPU, against the
oracle on the same seeded inputs, through the C ABI.

Rotation: every query head and every action key is turned at its position in
the joint [prefix | action] sequence, P_b + i (the vla.cpp abstract on page 1
warns that positional-index precision changes the actions).  Prefix
production: pae_set_prefix_hidden normalises each layer's prefix hidden states,
projects them onto the key/value rows (keys rotated at 0..P-1) and writes the
results straight into the request's slot (PhyAI report Sec. 5.1: the prefix
is computed once per observation and its per-layer K/V cached).
"""
import numpy as np
import pytest

import flow_matching_action_pi0_b200 as fm
import oracle
import workloads as wl
from tests.helpers import assert_bf16_slot_close, assert_parity, build_expert, max_abs, oracle_rows, run_gpu, set_prefixes
from workloads import device as wd

pytestmark = pytest.mark.gpu

ROPE = 10000.0


def _run_case(cfg, lengths=None):
    ex, W = build_expert(cfg)
    try:
        ks, vs = wl.make_prefix(cfg, lengths=lengths)
        set_prefixes(ex, cfg, ks, vs)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        out = run_gpu(ex, noise)
        ref = oracle_rows(cfg, W, ks, vs, noise, grid)
        assert_parity(out, ref, cfg.dtype, cfg.name)
        return out, ref
    finally:
        ex.close()


def test_tiny_fp32_rope():
    out, ref = _run_case(wl.TINY_FP32.replace(name="tiny_fp32_rope", rope_base=ROPE))
    # the rotation is not a no-op: the plain oracle differs by far more than the tolerance
    cfg = wl.TINY_FP32
    ks, vs = wl.make_prefix(cfg)
    plain = oracle_rows(cfg, wl.make_weights(cfg), ks, vs, wl.make_noise(cfg), wl.uniform_grid(cfg.steps))
    assert max_abs(plain, ref) > 1e-3


def test_tiny_bf16_rope_ragged():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_rope_b5", dtype=wl.BF16, batch=5, rope_base=ROPE)
    _run_case(cfg, lengths=[64, 0, 17, 63, 1])


def test_tiny_bf16_rope_gqa2_many_tokens():
    # Hkv = 2 (two rotated key heads), 300 tokens: token tiles with a ragged tail
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_rope_gqa2", dtype=wl.BF16, n_kv_heads=2, batch=20, chunk=15,
                               rope_base=ROPE)
    _run_case(cfg, lengths=[(7 * b) % 65 for b in range(20)])


def test_tiny_bf16_rope_head_dim_256():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_rope_d256", dtype=wl.BF16, n_q_heads=2, head_dim=256,
                               rope_base=ROPE, batch=2)
    _run_case(cfg, lengths=[64, 9])


def test_tiny_w4a16_rope():
    _run_case(wl.TINY_FP32.replace(name="tiny_w4a16_rope", dtype=wl.W4A16, rope_base=ROPE, batch=3),
              lengths=[64, 7, 0])


@pytest.mark.slow
def test_pi05_bf16_bs1_rope():
    _run_case(wl.PI05_BF16_BS1.replace(name="pi05_bf16_bs1_rope", rope_base=ROPE))


# ------------------------------------------------------------ prefix production
def _slots(ex, cfg, max_batch, max_prefix):
    """Keys and values of every layer / row as float64 [L][B][Hkv][Ptot][d]."""
    H = cfg.chunk
    shp = (cfg.layers, max_batch, cfg.n_kv_heads, max_prefix + H, cfg.head_dim)

    def conv(raw):
        if cfg.dtype == wl.FP32:
            return np.frombuffer(raw.tobytes(), dtype=np.float32).reshape(shp).astype(np.float64)
        u = np.frombuffer(raw.tobytes(), dtype=np.uint16).astype(np.uint32) << 16
        return u.view(np.float32).reshape(shp).astype(np.float64)
    return conv(ex.debug_copy("kcache")), conv(ex.debug_copy("vcache"))


def _prefix_case(cfg, lengths, brute=False):
    """Rows get their prefix from pae_set_prefix_hidden; slots and final
    actions are compared with the oracle's production step."""
    W = wl.make_weights(cfg)
    pms = [wl.make_prefix_model(cfg, prefix_len=n, seed=50 + b) for b, n in enumerate(lengths)]
    W = dict(W)
    W["w_prefix_kv"] = pms[0]["w_prefix_kv"]       # the model's weights: the same for every row
    for pm in pms[1:]:
        pm["w_qkv"], pm["w_o"], pm["w_gate"], pm["w_up"], pm["w_down"] = (
            pms[0]["w_qkv"], pms[0]["w_o"], pms[0]["w_gate"], pms[0]["w_up"], pms[0]["w_down"])
    p = oracle.params_from_weights(cfg, W)
    stack = oracle.expert.PrefixStack(w_qkv=[np.float64(w) for w in pms[0]["w_qkv"]],
                                      w_o=[np.float64(w) for w in pms[0]["w_o"]],
                                      w_gate=[np.float64(w) for w in pms[0]["w_gate"]],
                                      w_up=[np.float64(w) for w in pms[0]["w_up"]],
                                      w_down=[np.float64(w) for w in pms[0]["w_down"]])
    ex, _ = build_expert(cfg, W=W)
    try:
        ks_ref, vs_ref, hs_rows = [], [], []
        for b, n in enumerate(lengths):
            z = np.float64(pms[b]["z"])
            hs = oracle.prefix_stack_hidden(z, stack, p) if n > 0 else [np.zeros((0, cfg.prefix_width))] * cfg.layers
            # the hidden states the GPU is given, in its activation dtype
            hs = [wl.round_bf16(h) if cfg.dtype != wl.FP32 else np.float32(h) for h in hs]
            hs_rows.append(hs)
            k, v = oracle.prefix_kv_from_hidden(hs, [np.float64(w) for w in W["w_prefix_kv"]], p)
            ks_ref.append(k)
            vs_ref.append(v)
            hd = [wd.to_dev(h, wd.act_dtype(cfg)) for h in hs]
            ex.set_prefix_hidden(b, hd, n)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        out = run_gpu(ex, noise)
        kc, vc = _slots(ex, cfg, cfg.batch, cfg.prefix)
        for b, n in enumerate(lengths):
            for l in range(cfg.layers):
                gk = kc[l, b, :, :n, :].transpose(1, 0, 2)
                gv = vc[l, b, :, :n, :].transpose(1, 0, 2)
                if cfg.dtype == wl.FP32:
                    assert max_abs(gk, ks_ref[b][l]) <= 1e-4, f"row {b} layer {l}: keys"
                    assert max_abs(gv, vs_ref[b][l]) <= 1e-4, f"row {b} layer {l}: values"
                else:
                    assert_bf16_slot_close(gk, ks_ref[b][l], f"row {b} layer {l}: keys")
                    assert_bf16_slot_close(gv, vs_ref[b][l], f"row {b} layer {l}: values")
        ref = oracle.denoise(noise.astype(np.float64), grid, p, ks_ref, vs_ref)
        assert_parity(out, ref, cfg.dtype, cfg.name)
        if brute:
            # the whole joint sequence recomputed every step, no cache anywhere
            for b, n in enumerate(lengths):
                bf = oracle.brute_force_denoise_row(noise[b].astype(np.float64), grid, p, np.float64(pms[b]["z"]),
                                                    stack)
                assert_parity(out[b], bf, cfg.dtype, cfg.name + f" row {b} vs brute force")
    finally:
        ex.close()


def test_prefix_production_tiny_fp32_brute_force():
    cfg = wl.TINY_FP32.replace(name="tiny_fp32_prefix", prefix_width=384, batch=2)
    _prefix_case(cfg, [64, 23], brute=True)


def test_prefix_production_tiny_fp32_rope_brute_force():
    cfg = wl.TINY_FP32.replace(name="tiny_fp32_prefix_rope", prefix_width=384, batch=2, rope_base=ROPE)
    _prefix_case(cfg, [64, 5], brute=True)


def test_prefix_production_tiny_bf16_rope_ragged():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_prefix_rope", dtype=wl.BF16, prefix_width=384, batch=3,
                               rope_base=ROPE, n_kv_heads=2)
    _prefix_case(cfg, [64, 0, 37])


def test_prefix_production_replaces_set_prefix():
    # a row first cached with pae_set_prefix, then produced from hidden states,
    # follows the new prefix (invalidation), and pae_set_prefix_hidden on a
    # context without prefix production is a state error
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_prefix_swap", dtype=wl.BF16, prefix_width=128)
    W = dict(wl.make_weights(cfg))
    pm = wl.make_prefix_model(cfg, prefix_len=40)
    W["w_prefix_kv"] = pm["w_prefix_kv"]
    ex, _ = build_expert(cfg, W=W)
    try:
        ks, vs = wl.make_prefix(cfg)
        set_prefixes(ex, cfg, ks, vs)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        first = run_gpu(ex, noise)
        hs = [wl.round_bf16(np.random.default_rng(l).standard_normal((40, 128))) for l in range(cfg.layers)]
        ex.set_prefix_hidden(0, [wd.to_dev(h, wd.act_dtype(cfg)) for h in hs], 40)
        second = run_gpu(ex, noise)
        p = oracle.params_from_weights(cfg, W)
        k, v = oracle.prefix_kv_from_hidden([np.float64(h) for h in hs], [np.float64(w) for w in W["w_prefix_kv"]],
                                            p)
        assert_parity(second, oracle.denoise(noise.astype(np.float64), grid, p, [k], [v]), cfg.dtype, cfg.name)
        assert max_abs(first, second) > 1e-3
    finally:
        ex.close()
    cfg0 = wl.TINY_FP32.replace(name="tiny_bf16_noprefix", dtype=wl.BF16)
    ex0, _ = build_expert(cfg0)
    try:
        with pytest.raises(fm.PaeError) as e:
            ex0.set_prefix_hidden(0, [wd.to_dev(np.zeros((4, 256), np.float32), wd.act_dtype(cfg0))] * cfg0.layers, 4)
        assert e.value.status == fm.PAE_ERR_STATE
    finally:
        ex0.close()


@pytest.mark.slow
def test_prefix_production_pi05_bs1_width2048():
    # full size: 18 layers, 968 prefix tokens, hidden width 2048 (a Gemma-2B-like
    # prefix model); per-layer hidden states drawn directly (the stack itself
    # is not needed for the production step)
    cfg = wl.PI05_BF16_BS1.replace(name="pi05_prefix_w2048", prefix_width=2048, rope_base=ROPE)
    W = dict(wl.make_weights(cfg))
    g = np.random.default_rng(77)
    L, P = cfg.layers, cfg.prefix
    W["w_prefix_kv"] = [wl.round_bf16(g.standard_normal((2 * cfg.head_dim, 2048)) * 0.02) for _ in range(L)]
    hs = [wl.round_bf16(g.standard_normal((P, 2048))) for _ in range(L)]
    p = oracle.params_from_weights(cfg, W)
    k, v = oracle.prefix_kv_from_hidden([np.float64(h) for h in hs], [np.float64(w) for w in W["w_prefix_kv"]], p)
    ex, _ = build_expert(cfg, W=W)
    try:
        ex.set_prefix_hidden(0, [wd.to_dev(h, wd.act_dtype(cfg)) for h in hs], P)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        out = run_gpu(ex, noise)
        kc, vc = _slots(ex, cfg, 1, P)
        for l in range(L):
            assert_bf16_slot_close(kc[l, 0, :, :P].transpose(1, 0, 2), k[l], f"layer {l}: keys")
            assert_bf16_slot_close(vc[l, 0, :, :P].transpose(1, 0, 2), v[l], f"layer {l}: values")
        assert_parity(out, oracle.denoise(noise.astype(np.float64), grid, p, [k], [v]), cfg.dtype, cfg.name)
    finally:
        ex.close()
