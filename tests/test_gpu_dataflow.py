"""The dataflow loop: all Euler steps of a call as one launch of thread-block
clusters whose stages wait on per-tile counters (batches of at most 64 action
tokens), against the oracle on the same seeded inputs and against the graph of
per-stage kernels, through the C ABI."""
import numpy as np
import pytest
import torch

import flow_matching_action_pi0_b200 as fm
import workloads as wl
from tests.helpers import assert_parity, build_expert, max_abs, oracle_rows, run_gpu, set_prefixes

pytestmark = pytest.mark.gpu


def _case(cfg, lengths=None, cluster=0, graph_too=True):
    ex, W = build_expert(cfg)
    try:
        ex.set_option(fm.PAE_OPT_DATAFLOW, 1)
        if cluster:
            ex.set_option(fm.PAE_OPT_DATAFLOW_CLUSTER, cluster)
        ks, vs = wl.make_prefix(cfg, lengths=lengths)
        set_prefixes(ex, cfg, ks, vs)
        grid = wl.uniform_grid(cfg.steps)
        ex.precompute_tables(grid)
        noise = wl.make_noise(cfg)
        C = ex.query(fm.PAE_Q_DATAFLOW, cfg.batch)
        assert C > 0 and (not cluster or C == cluster)
        out = run_gpu(ex, noise)
        np.testing.assert_array_equal(run_gpu(ex, noise), out)  # bitwise reproducible
        ref = oracle_rows(cfg, W, ks, vs, noise, grid)
        assert_parity(out, ref, cfg.dtype, f"{cfg.name} dataflow C={C}")
        if graph_too:
            ex.set_option(fm.PAE_OPT_DATAFLOW, 0)
            assert ex.query(fm.PAE_Q_DATAFLOW, cfg.batch) == 0
            graph = run_gpu(ex, noise)
            assert_parity(graph, ref, cfg.dtype, f"{cfg.name} graph")
        return out, ref
    finally:
        ex.close()


def test_tiny_bf16_batch1():
    _case(wl.TINY_FP32.replace(name="tiny_bf16_df", dtype=wl.BF16))


def test_tiny_bf16_batch4_ragged_64_tokens():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_df_b4", dtype=wl.BF16, batch=4)
    _case(cfg, lengths=[64, 0, 17, 1])


def test_tiny_bf16_gqa2_rope_batch3():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_df_gqa2", dtype=wl.BF16, batch=3, n_kv_heads=2, rope_base=10000.0)
    _case(cfg, lengths=[64, 30, 5])


def test_tiny_bf16_head_dim_256_cluster_sizes():
    # head_dim 256 (four 64-wide boxes per row), several key chunks per rank with 2-CTA clusters
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_df_d256", dtype=wl.BF16, n_q_heads=2, head_dim=256, batch=2)
    a, ref = _case(cfg, lengths=[64, 40], cluster=2, graph_too=False)
    b, _ = _case(cfg, lengths=[64, 40], cluster=4)
    assert max_abs(a, b) < 2e-2


def test_tiny_w4a16_batch3_rope():
    # int4 weights: packed blocks dequantised by the weight producer warp
    cfg = wl.TINY_FP32.replace(name="tiny_w4a16_df", dtype=wl.W4A16, batch=3, rope_base=10000.0)
    _case(cfg, lengths=[64, 9, 0])


def test_step_split_bitwise_and_host_buffers():
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_df_split", dtype=wl.BF16, batch=2)
    ex, W = build_expert(cfg)
    try:
        ex.set_option(fm.PAE_OPT_DATAFLOW, 1)
        ks, vs = wl.make_prefix(cfg, lengths=[64, 33])
        set_prefixes(ex, cfg, ks, vs)
        ex.precompute_tables(wl.uniform_grid(cfg.steps))
        noise = wl.make_noise(cfg)
        full = run_gpu(ex, noise)
        x = torch.from_numpy(noise).cuda()
        mid = torch.empty_like(x)
        end = torch.empty_like(x)
        ex.denoise_steps(x, mid, 0, 1)
        ex.denoise_steps(mid, mid, 1, 3)
        ex.denoise_steps(mid, end, 3, cfg.steps)
        ex.sync()
        np.testing.assert_array_equal(end.cpu().numpy(), full)
        nh = torch.from_numpy(noise).pin_memory()
        oh = torch.empty_like(nh).pin_memory()
        ex.denoise_host(nh, oh)
        ex.sync()
        np.testing.assert_array_equal(oh.numpy(), full)
    finally:
        ex.close()


def test_dataflow_wait_timeout_reports_status():
    """A bounded wait of the dataflow loop that runs out (1 us limit) returns
    PAE_ERR_TIMEOUT; every CTA unwinds, drains and meets its cluster, and the
    context is usable again after pae_clear_error."""
    cfg = wl.TINY_FP32.replace(name="tiny_bf16_df_to", dtype=wl.BF16)
    ex, W = build_expert(cfg)
    try:
        ex.set_option(fm.PAE_OPT_DATAFLOW, 1)
        ks, vs = wl.make_prefix(cfg)
        set_prefixes(ex, cfg, ks, vs)
        ex.precompute_tables(wl.uniform_grid(cfg.steps))
        noise = wl.make_noise(cfg)
        assert ex.query(fm.PAE_Q_DATAFLOW, 1) > 0
        good = run_gpu(ex, noise)
        ex.set_option(fm.PAE_OPT_WAIT_LIMIT_US, 1)
        hit = False
        for _ in range(20):
            try:
                ex.denoise(torch.from_numpy(noise).cuda())
                ex.sync()
            except fm.PaeError as e:
                assert e.status == fm.PAE_ERR_TIMEOUT
                hit = True
                break
        fm.pae_clear_error(ex.ctx)
        ex.set_option(fm.PAE_OPT_WAIT_LIMIT_US, 2_000_000)
        np.testing.assert_array_equal(run_gpu(ex, noise), good)
        assert hit, "no wait ran out at a 1 us limit"
    finally:
        ex.close()


@pytest.mark.slow
@pytest.mark.parametrize("cluster", [16, 8])
def test_pi05_bf16_bs1_dataflow(cluster):
    _case(wl.PI05_BF16_BS1.replace(name=f"pi05_bf16_bs1_df{cluster}"), cluster=cluster, graph_too=cluster == 16)


@pytest.mark.slow
def test_pi05_w4a16_bs1_dataflow():
    _case(wl.PI05_W4A16_BS1.replace(name="pi05_w4a16_bs1_df"), graph_too=False)


@pytest.mark.slow
def test_pi05_bf16_bs1_dataflow_rope():
    _case(wl.PI05_BF16_BS1.replace(name="pi05_bf16_bs1_df_rope", rope_base=10000.0), graph_too=False)
