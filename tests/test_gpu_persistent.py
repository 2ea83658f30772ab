"""The persistent loop (one launch per call, grid barriers between phases) on
the GPU, through the C ABI: parity with the oracle on the same seeded inputs,
agreement with the captured-graph path, and the shapes that take its other
branches (head_dim 256 with P over the K buffer, several query tiles, GQA
groups, key ranges of more than one 64-key chunk per CTA, empty prefixes)."""
import numpy as np
import pytest

import flow_matching_action_pi0_b200 as fm
import workloads as wl
from tests.helpers import assert_parity, build_expert, oracle_rows, run_gpu, set_prefixes

pytestmark = pytest.mark.gpu

TINY_BF16 = wl.TINY_FP32.replace(name="tiny_bf16_p", dtype=wl.BF16)


def _both_paths(cfg, lengths=None, max_prefix=None):
    """(persistent output, graph output, oracle) on the same context and inputs."""
    ex, W = build_expert(cfg, max_prefix=max_prefix)
    try:
        ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
        ks, vs = wl.make_prefix(cfg, lengths=lengths)
        set_prefixes(ex, cfg, ks, vs)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        assert ex.query(fm.PAE_Q_PERSISTENT, cfg.batch) == 1
        per = run_gpu(ex, noise)
        ex.set_option(fm.PAE_OPT_PERSISTENT, 0)
        assert ex.query(fm.PAE_Q_PERSISTENT, cfg.batch) == 0
        gra = run_gpu(ex, noise)
        ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
        again = run_gpu(ex, noise)
        np.testing.assert_array_equal(per, again)  # bitwise reproducible
        ref = oracle_rows(cfg, W, ks, vs, noise, grid)
        return per, gra, ref
    finally:
        ex.close()


def _check(cfg, **kw):
    per, gra, ref = _both_paths(cfg, **kw)
    assert_parity(per, ref, cfg.dtype, cfg.name + " persistent")
    assert_parity(gra, ref, cfg.dtype, cfg.name + " graph")
    assert_parity(per, gra, cfg.dtype, cfg.name + " persistent vs graph")


def test_eligibility():
    cfg = TINY_BF16.replace(batch=5)
    ex, _ = build_expert(cfg)
    try:
        assert ex.query(fm.PAE_Q_PERSISTENT, 1) == 0   # off by default
        ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
        assert ex.query(fm.PAE_Q_PERSISTENT, 1) == 1   # 16 tokens
        assert ex.query(fm.PAE_Q_PERSISTENT, 4) == 1   # 64 tokens
        assert ex.query(fm.PAE_Q_PERSISTENT, 5) == 0   # 80 tokens: graph of kernels
        ex.set_option(fm.PAE_OPT_PERSISTENT, 0)
        assert ex.query(fm.PAE_Q_PERSISTENT, 1) == 0
    finally:
        ex.close()
    for c in (wl.TINY_FP32, wl.TINY_FP32.replace(name="tiny_w4_p", dtype=wl.W4A16)):
        ex, _ = build_expert(c)
        try:
            ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
            assert ex.query(fm.PAE_Q_PERSISTENT, 1) == 0
        finally:
            ex.close()


def test_tiny_bf16_batch1():
    _check(TINY_BF16)


def test_tiny_bf16_batch4_ragged_with_empty_prefix():
    # 64 tokens, four requests, one with no prefix at all
    _check(TINY_BF16.replace(name="tiny_bf16_p4", batch=4), lengths=[64, 0, 33, 1])


def test_head_dim_256_two_query_heads():
    # head_dim 256: P overlays the K chunk; two key splits merged through the workspace
    cfg = TINY_BF16.replace(name="tiny_bf16_d256", n_q_heads=2, head_dim=256, batch=2)
    _check(cfg, lengths=[64, 20])


def test_two_query_tiles():
    # 8 query heads x 32 tokens = 256 query rows per KV head: two 128-row tiles
    cfg = TINY_BF16.replace(name="tiny_bf16_qt2", n_q_heads=8, chunk=32, batch=2)
    _check(cfg, lengths=[64, 17])


def test_gqa2_long_prefix_two_chunks_per_cta():
    # 4 requests x 2 KV heads = 8 groups; 2064 keys = 33 chunks > 148 / 8, so
    # every CTA walks two 64-key chunks (online softmax across chunks)
    cfg = TINY_BF16.replace(name="tiny_bf16_gqa2_long", n_q_heads=8, n_kv_heads=2, batch=4, prefix=2048)
    _check(cfg, lengths=[2048, 1500, 700, 64])


@pytest.mark.slow
def test_pi05_bf16_bs1_persistent():
    """The persistent kernel at the full pi0.5 batch-1 size (the graph is the default there)."""
    cfg = wl.PI05_BF16_BS1
    ex, W = build_expert(cfg)
    try:
        ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
        ks, vs = wl.make_prefix(cfg)
        set_prefixes(ex, cfg, ks, vs)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        out = run_gpu(ex, noise)
        assert_parity(out, oracle_rows(cfg, W, ks, vs, noise, grid), cfg.dtype, "pi05 bs1 persistent")
    finally:
        ex.close()


def test_persistent_wait_timeout_reports_status():
    """With a 1 microsecond wait limit the persistent kernel's first grid barrier
    runs out: the CTA that times out raises the launch-wide abort flag, every
    other CTA's bounded wait sees it, each CTA drains its copies and MMAs and
    frees TMEM, and the call reports PAE_ERR_TIMEOUT.  After pae_clear_error the
    context gives the same result as before, bitwise."""
    import torch
    cfg = TINY_BF16.replace(name="tiny_bf16_pto")
    ex, W = build_expert(cfg)
    try:
        ex.set_option(fm.PAE_OPT_PERSISTENT, 1)
        ks, vs = wl.make_prefix(cfg)
        set_prefixes(ex, cfg, ks, vs)
        ex.precompute_tables(wl.uniform_grid(cfg.steps))
        noise = wl.make_noise(cfg)
        good = run_gpu(ex, noise)
        ex.set_option(fm.PAE_OPT_WAIT_LIMIT_US, 1)
        hit = False
        for _ in range(20):
            x = torch.from_numpy(noise).cuda()
            try:
                ex.denoise(x)
                ex.sync()
            except fm.PaeError as e:
                assert e.status == fm.PAE_ERR_TIMEOUT
                hit = True
                break
        fm.pae_clear_error(ex.ctx)
        ex.set_option(fm.PAE_OPT_WAIT_LIMIT_US, 2_000_000)
        again = run_gpu(ex, noise)
        np.testing.assert_array_equal(again, good)
        if not hit:
            pytest.skip("no wait ran out at a 1 us limit on this run")
    finally:
        ex.close()
