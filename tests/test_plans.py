"""The launch planners (host arithmetic, no device): split-K factors, token
tiles and split-KV counts through pae_plan_query, pinned at the pi0.5 shape to
the plans the GPU contexts report, and checked for the rules they follow at
every batch size."""
import pytest

import flow_matching_action_pi0_b200 as fm
import workloads as wl
from workloads.device import abi_config

SMS = 148


def _cfg(c, max_batch=None):
    return fm.make_config(**abi_config(c, max_batch=max_batch))


def _splits(cfg, batch):
    v = fm.pae_plan_query(cfg, fm.PAE_Q_SPLITS, batch)
    return tuple((v >> (8 * i)) & 0xFF for i in range(4))  # QKV, O, gate/up, down


def test_pi05_plans_match_the_gpu_contexts():
    cfg = _cfg(wl.PI05_BF16_BS32)
    assert _splits(cfg, 1) == (4, 8, 4, 8)
    assert fm.pae_plan_query(cfg, fm.PAE_Q_TOKEN_TILE, 1) == 64
    assert fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_SPLITS, 1) == 8
    assert fm.pae_plan_query(cfg, fm.PAE_Q_FUSED_NORM, 1) == 0  # norm kernels by default
    assert _splits(cfg, 32) == (1, 2, 1, 2)
    assert fm.pae_plan_query(cfg, fm.PAE_Q_FUSED_NORM, 32) == 0
    assert fm.pae_plan_query(cfg, fm.PAE_Q_TOKEN_TILE, 32) == 240
    assert fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_SPLITS, 32) == 1
    # 128 keys per split at batch 1 run as two 64-key chunks, the whole slot
    # at batch 32 as 128-key chunks
    assert fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_CHUNK, 1) == 64
    assert fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_CHUNK, 32) == 128
    assert fm.pae_plan_query(_cfg(wl.RAGGED_BF16_BS16), fm.PAE_Q_ATTN_CHUNK, 16) == 128
    w4 = _cfg(wl.PI05_W4A16_BS1)
    assert _splits(w4, 1) == (4, 8, 4, 8)


def test_fp32_mode_has_no_tensor_core_plan():
    cfg = _cfg(wl.TINY_FP32)
    for q in (fm.PAE_Q_SPLITS, fm.PAE_Q_TOKEN_TILE, fm.PAE_Q_ATTN_SPLITS, fm.PAE_Q_ATTN_CHUNK, fm.PAE_Q_FUSED_NORM):
        assert fm.pae_plan_query(cfg, q, 1) == 0


@pytest.mark.parametrize("base", [wl.PI05_BF16_BS32, wl.PI05_W4A16_BS1, wl.TINY_FP32.replace(dtype=wl.BF16)])
def test_plan_rules_at_every_batch(base):
    """Split-K factors are powers of two that divide the K blocks; a batch of
    one token tile takes the padded token count; larger batches take tiles of
    128..256 tokens; at <= 64 tokens every projection stays within two CTAs
    per SM, and QKV / gate-up within one when they follow a norm kernel (norm
    not factored into the epilogues); split-KV is a power of two <= 16 that
    only multiplies a launch still under one wave."""
    c = base.replace(batch=min(40, 4096 // base.chunk))
    cfg = _cfg(c)
    D, F, qd = c.width, c.mlp_dim, c.n_q_heads * c.head_dim
    qkv_rows = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim
    ks = (D // 64, qd // 64, D // 64, F // 64)                      # K blocks per projection
    tiles = (-(-qkv_rows // 128), -(-D // 128), -(-F // 128), -(-D // 128))  # 128-feature output tiles
    for B in range(1, c.batch + 1):
        M = B * c.chunk
        sp = _splits(cfg, B)
        tn = fm.pae_plan_query(cfg, fm.PAE_Q_TOKEN_TILE, B)
        for s, k in zip(sp, ks):
            assert s >= 1 and s & (s - 1) == 0 and s <= 16 and k % s == 0, (B, sp)
        assert tn % 16 == 0 and 16 <= tn <= 256
        if M <= 256:
            assert tn == max(16, -(-M // 16) * 16), (B, tn)
        else:
            assert 128 <= tn <= 256, (B, tn)
        if tn <= 64:
            ntok = -(-M // tn)
            per_sm = 2 if fm.pae_plan_query(cfg, fm.PAE_Q_FUSED_NORM, B) == 2 else 1
            assert tiles[0] * ntok * sp[0] <= per_sm * SMS and tiles[2] * ntok * sp[2] <= per_sm * SMS, (B, sp)
            assert tiles[1] * ntok * sp[1] <= 2 * SMS and tiles[3] * ntok * sp[3] <= 2 * SMS, (B, sp)
        a = fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_SPLITS, B)
        assert a >= 1 and a & (a - 1) == 0 and a <= 16
        assert fm.pae_plan_query(cfg, fm.PAE_Q_ATTN_CHUNK, B) in (64, 128)
        qtiles = -(-(c.n_q_heads // c.n_kv_heads) * c.chunk // 128)
        if a > 1:
            assert B * c.n_kv_heads * qtiles * a <= SMS


def test_plan_query_rejects_bad_arguments():
    cfg = _cfg(wl.PI05_BF16_BS1)
    for batch in (0, 2):
        with pytest.raises(fm.PaeError) as e:
            fm.pae_plan_query(cfg, fm.PAE_Q_SPLITS, batch)
        assert e.value.status == fm.PAE_ERR_ARG
    with pytest.raises(fm.PaeError) as e:
        fm.pae_plan_query(cfg, fm.PAE_Q_GRAPH_KERNELS, 1)
    assert e.value.status == fm.PAE_ERR_ARG
    bad = _cfg(wl.PI05_BF16_BS1)
    bad.head_dim = 96
    with pytest.raises(fm.PaeError) as e:
        fm.pae_plan_query(bad, fm.PAE_Q_SPLITS, 1)
    assert e.value.status == fm.PAE_ERR_UNSUPPORTED
