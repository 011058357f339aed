"""Pins of the oracle's rotary embedding (the library's RoPE reading: the
Llama rotate-half form) against things other than the oracle: the
transformers Llama implementation (a library routine), closed forms and
invariants that a sign, pairing or frequency mistake breaks.
"""
import numpy as np
import pytest
import torch

import oracle


def test_rope_matches_transformers_llama():
    from transformers import LlamaConfig
    from transformers.models.llama import modeling_llama as m
    d, H, n = 128, 3, 40
    cfg = LlamaConfig(hidden_size=H * d, num_attention_heads=H, head_dim=d, rope_theta=10000.0,
                      max_position_embeddings=32768)
    rot = m.LlamaRotaryEmbedding(cfg)
    g = np.random.default_rng(0)
    q = g.standard_normal((n, H, d))
    k = g.standard_normal((n, H, d))
    pos = np.sort(g.choice(2048, n, replace=False))
    qt = torch.tensor(q).permute(1, 0, 2)[None]  # [1, H, n, d]
    kt = torch.tensor(k).permute(1, 0, 2)[None]
    cos, sin = rot(qt, torch.tensor(pos)[None])
    qr, kr = m.apply_rotary_pos_emb(qt, kt, cos.double(), sin.double())
    # transformers forms the angles from float32 frequencies: ~1e-4 rad at 2k
    assert np.max(np.abs(qr[0].permute(1, 0, 2).numpy() - oracle.rope(q, pos))) < 2e-3
    assert np.max(np.abs(kr[0].permute(1, 0, 2).numpy() - oracle.rope(k, pos))) < 2e-3


def test_rope_closed_forms():
    # position 0 is the identity
    x = np.random.default_rng(1).standard_normal((5, 2, 64))
    assert np.array_equal(oracle.rope(x, np.zeros(5)), x)
    # d = 2: the frequency is 1, e1 turns to (cos p, sin p), e2 to (-sin p, cos p)
    p = np.array([0.3, 2.0, -1.0, 1000.0])
    e1 = np.tile([1.0, 0.0], (4, 1))
    e2 = np.tile([0.0, 1.0], (4, 1))
    assert np.allclose(oracle.rope(e1, p), np.stack([np.cos(p), np.sin(p)], 1), atol=1e-15)
    assert np.allclose(oracle.rope(e2, p), np.stack([-np.sin(p), np.cos(p)], 1), atol=1e-15)
    # pair i turns at theta^(-2i/d): with theta = 16, d = 4, pair 1 turns at 1/4
    y = oracle.rope(np.array([[0.0, 1.0, 0.0, 0.0]]), [2.0], theta=16.0)
    assert np.allclose(y, [[0.0, np.cos(0.5), 0.0, np.sin(0.5)]], atol=1e-15)


def test_rope_is_a_rotation_with_relative_scores():
    g = np.random.default_rng(2)
    q, k = g.standard_normal((1, 128)), g.standard_normal((1, 128))
    # norms of each pair are kept
    r = oracle.rope(q, [123.0])
    assert np.allclose(np.hypot(r[0, :64], r[0, 64:]), np.hypot(q[0, :64], q[0, 64:]), rtol=1e-13)
    # the score depends on the position difference only
    for m_, n_, s in [(5, 2, 100), (1000, 7, 31000), (40, 40, 12345)]:
        a = oracle.rope(q, [m_]) @ oracle.rope(k, [n_]).T
        b = oracle.rope(q, [m_ + s]) @ oracle.rope(k, [n_ + s]).T
        assert abs(a - b) < 1e-9


def test_rope_positions_policies():
    assert oracle.rope_position("absolute", 100, 0, 8) == 100
    assert oracle.rope_position("absolute", 100, 9, 8) == 109
    assert oracle.rope_position("slot", 100, 9, 8) == 101
    assert oracle.rope_position("slot", 100, 7, 8) == 107
