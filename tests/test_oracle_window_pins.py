"""Pins of the oracle's standard sliding-window prefill (the contrast mode):
torch's float64 scaled_dot_product_attention with a banded mask (a library
routine), the full causal oracle when the window covers the prompt, and the
W = 1 closed form (each token sees only itself)."""
import numpy as np
import torch

import oracle


def _qkv(P=40, H=2, d=16, seed=0):
    g = np.random.default_rng(seed)
    return g.standard_normal((3, P, H, d))


def test_window_prefill_matches_sdpa_band():
    q, k, v = _qkv()
    P, W, scale = q.shape[0], 7, 0.25
    i = np.arange(P)
    band = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)  # [query, key]
    t = lambda x: torch.tensor(x).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=torch.tensor(band), scale=scale)[0].permute(1, 0, 2).numpy()
    assert np.max(np.abs(oracle.prefill_window(q, k, v, scale, W) - ref)) < 1e-12


def test_window_prefill_special_cases():
    q, k, v = _qkv(P=25, seed=1)
    # a window as long as the prompt is plain causal attention
    assert np.max(np.abs(oracle.prefill_window(q, k, v, 0.3, 25) - oracle.prefill(q, k, v, 0.3))) < 1e-12
    # W = 1: each token sees only itself
    assert np.array_equal(oracle.prefill_window(q, k, v, 0.3, 1), v)
