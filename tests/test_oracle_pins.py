"""Pins for the FP64 oracle against things other than itself.

Every check here compares the oracle with an independent statement of the same
result: torch's float64 scaled_dot_product_attention (a library routine), closed
forms, brute force over the union key set the pages define, the transformers
no-repeat-ngram processor, and hand-worked fixtures under tests/golden/.

Method source: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.1 (ring
sliding-window attention) and §2.3 (windowed no-repeat n-gram ban).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL64 = 1e-12


def sdpa64(q, k, v, scale, causal=False):
    """torch float64 SDPA; q [m, d], k/v [n, d] -> [m, d]."""
    q = torch.as_tensor(np.asarray(q, dtype=np.float64))[None, None]
    k = torch.as_tensor(np.asarray(k, dtype=np.float64))[None, None]
    v = torch.as_tensor(np.asarray(v, dtype=np.float64))[None, None]
    return F.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale)[0, 0].numpy()


def rng(s):
    return np.random.default_rng(s)


# --------------------------------------------------------------------------
# attention of one query
# --------------------------------------------------------------------------
@pytest.mark.parametrize("n,d", [(1, 64), (7, 64), (300, 128), (1217, 128)])
def test_attend_matches_sdpa(oracle, n, d):
    r = rng(n * 31 + d)
    q, k, v = r.standard_normal(d), r.standard_normal((n, d)), r.standard_normal((n, d))
    s = 1.0 / math.sqrt(d)
    got = oracle.attend(q, k, v, s)
    ref = sdpa64(q[None], k, v, s)[0]
    assert np.max(np.abs(got - ref)) < TOL64


def test_attend_closed_forms(oracle):
    r = rng(1)
    d = 16
    # identical keys: uniform weights, output is the mean of the values
    k = np.tile(r.standard_normal(d), (9, 1))
    v = r.standard_normal((9, d))
    out = oracle.attend(r.standard_normal(d), k, v, 0.7)
    assert np.max(np.abs(out - v.mean(0))) < 1e-14
    # one key: output is its value exactly
    out = oracle.attend(r.standard_normal(d), k[:1], v[:1], 0.3)
    assert np.array_equal(out, v[0])
    # one dominant key: weights of the others are below exp(-700)
    k = np.eye(d)[:5]
    q = 1000.0 * k[3]
    out = oracle.attend(q, k, v[:5], 1.0)
    assert np.max(np.abs(out - v[3])) < 1e-300 + 1e-15
    # scale enters multiplicatively: scale 0 gives the plain mean
    out = oracle.attend(r.standard_normal(d), r.standard_normal((6, d)), v[:6], 0.0)
    assert np.max(np.abs(out - v[:6].mean(0))) < 1e-14


def test_attend_permutation_invariant(oracle):
    r = rng(2)
    q, k, v = r.standard_normal(32), r.standard_normal((50, 32)), r.standard_normal((50, 32))
    p = r.permutation(50)
    a = oracle.attend(q, k, v, 0.2)
    b = oracle.attend(q, k[p], v[p], 0.2)
    assert np.max(np.abs(a - b)) < TOL64


# --------------------------------------------------------------------------
# prefill (full causal attention, §2.1)
# --------------------------------------------------------------------------
def test_prefill_matches_causal_sdpa(oracle):
    r = rng(3)
    P, H, d = 37, 3, 16
    q, k, v = (r.standard_normal((P, H, d)) for _ in range(3))
    s = 0.25
    out = oracle.prefill(q, k, v, s)
    for h in range(H):
        ref = sdpa64(q[:, h], k[:, h], v[:, h], s, causal=True)
        assert np.max(np.abs(out[:, h] - ref)) < TOL64
    # row 0 attends to itself only
    assert np.array_equal(out[0], v[0])


def test_prefill_row_range(oracle):
    r = rng(4)
    P, H, d = 20, 2, 8
    q, k, v = (r.standard_normal((P, H, d)) for _ in range(3))
    full = oracle.prefill(q, k, v, 0.5)
    part = oracle.prefill(q, k, v, 0.5, 5, 11)
    assert np.array_equal(part[5:11], full[5:11])
    assert np.isnan(part[:5]).all() and np.isnan(part[11:]).all()


# --------------------------------------------------------------------------
# ring indices and cache size (§2.1 three phases)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("P,W", [(0, 1), (5, 1), (5, 3), (64, 8), (3, 128)])
def test_ring_slots_closed_form(oracle, P, W):
    H, d = 1, 2
    ring = oracle.Ring(P, W, H, d)
    ring.prefill(np.zeros((P, H, d)), np.zeros((P, H, d)))
    z = np.zeros((H, d))
    for t in range(5 * W + 3):
        _, slot, n = ring.step(z, z, z, 1.0)
        assert slot == P + (t % W)
        assert n == P + min(t + 1, W)
        if t >= W - 1:
            assert n == P + W  # constant-size invariant
        assert ring.ring_pos == ((t + 1) % W if t >= W else 0)


def test_ring_step_before_prefill_is_rejected(oracle):
    ring = oracle.Ring(4, 2, 1, 2)
    z = np.zeros((1, 2))
    with pytest.raises(ValueError):
        ring.step(z, z, z, 1.0)


def _ring_run(oracle, P, W, H, d, steps, seed):
    r = rng(seed)
    pk, pv = r.standard_normal((P, H, d)), r.standard_normal((P, H, d))
    qs, ks, vs = (r.standard_normal((steps, H, d)) for _ in range(3))
    ring = oracle.Ring(P, W, H, d)
    ring.prefill(pk, pv)
    s = 1.0 / math.sqrt(d)
    outs = np.stack([ring.step(qs[t], ks[t], vs[t], s)[0] for t in range(steps)])
    return pk, pv, qs, ks, vs, outs, ring, s


@pytest.mark.parametrize("P,W,steps", [(64, 8, 40), (64, 1, 10), (0, 3, 12), (64, 64, 40)])
def test_ring_equals_union_every_step(oracle, P, W, steps):
    """Brute-force pin: step t attends to all prefill tokens plus the generated
    tokens s with max(0, t-W+1) <= s <= t, rebuilt from the step inputs."""
    H, d = 2, 64
    pk, pv, qs, ks, vs, outs, _, s = _ring_run(oracle, P, W, H, d, steps, seed=P + 7 * W)
    for t in range(steps):
        lo = max(0, t - W + 1)
        for h in range(H):
            kk = np.concatenate([pk[:, h], ks[lo:t + 1, h]])
            vv = np.concatenate([pv[:, h], vs[lo:t + 1, h]])
            ref = sdpa64(qs[t, h][None], kk, vv, s)[0]
            assert np.max(np.abs(outs[t, h] - ref)) < TOL64, (t, h)


def test_ring_W_at_least_steps_is_full_cache(oracle):
    """With W >= number of steps the ring never wraps: plain full-cache decode."""
    P, W, H, d, steps = 16, 32, 2, 8, 20
    pk, pv, qs, ks, vs, outs, _, s = _ring_run(oracle, P, W, H, d, steps, seed=11)
    for t in range(steps):
        for h in range(H):
            kk = np.concatenate([pk[:, h], ks[:t + 1, h]])
            vv = np.concatenate([pv[:, h], vs[:t + 1, h]])
            assert np.max(np.abs(outs[t, h] - sdpa64(qs[t, h][None], kk, vv, s)[0])) < TOL64


def test_ring_W1_is_prefill_plus_self(oracle):
    P, W, H, d, steps = 10, 1, 1, 8, 6
    pk, pv, qs, ks, vs, outs, _, s = _ring_run(oracle, P, W, H, d, steps, seed=12)
    for t in range(steps):
        kk = np.concatenate([pk[:, 0], ks[t:t + 1, 0]])
        vv = np.concatenate([pv[:, 0], vs[t:t + 1, 0]])
        assert np.max(np.abs(outs[t, 0] - sdpa64(qs[t, 0][None], kk, vv, s)[0])) < TOL64


def test_ring_cache_contents(oracle):
    """Slot P + (s mod W) holds the latest generated s with that residue; the
    prefill slots never change."""
    P, W, H, d, steps = 12, 5, 2, 4, 23
    pk, pv, qs, ks, vs, _, ring, _ = _ring_run(oracle, P, W, H, d, steps, seed=13)
    kc, vc, n = ring.snapshot()
    assert n == P + W
    assert np.array_equal(kc[:P], pk) and np.array_equal(vc[:P], pv)
    for j in range(W):
        latest = max(s for s in range(steps) if s % W == j)
        assert np.array_equal(kc[P + j], ks[latest])
        assert np.array_equal(vc[P + j], vs[latest])


# --------------------------------------------------------------------------
# windowed no-repeat n-gram ban (§2.3)
# --------------------------------------------------------------------------
def _load_golden():
    with open(os.path.join(GOLDEN, "ngram_handbuilt.json")) as f:
        return json.load(f)


def _row(case, pad_default=0):
    hist = case["history"]
    window = case.get("window", len(hist))
    pad = case.get("pad", pad_default)
    row = list(hist) + [pad] * (window - len(hist))
    return np.array([row], dtype=np.int32), window, case.get("hist_len", len(hist))


@pytest.mark.parametrize("case", _load_golden()["cases"], ids=lambda c: c["id"])
def test_ngram_handbuilt(oracle, case):
    vocab = _load_golden()["vocab"]
    hist, window, h = _row(case)
    logits = np.random.default_rng(5).standard_normal((1, vocab)).astype(np.float32)
    before = logits.copy()
    assert oracle.ngram_ban(logits, hist, np.array([h], np.int32), case["n"], window) == 0
    banned = sorted(int(i) for i in np.nonzero(np.isneginf(logits[0]))[0])
    assert banned == sorted(case["banned"])
    keep = ~np.isneginf(logits[0])
    assert np.array_equal(logits[0][keep].view(np.uint32), before[0][keep].view(np.uint32))
    assert (logits[0][~keep].view(np.uint32) == np.uint32(0xFF800000)).all()


@pytest.mark.parametrize("case", _load_golden()["bad_rows"], ids=lambda c: c["id"])
def test_ngram_bad_rows_untouched(oracle, case):
    vocab = _load_golden()["vocab"]
    hist, window, h = _row(case)
    logits = np.random.default_rng(6).standard_normal((1, vocab)).astype(np.float32)
    before = logits.copy()
    assert oracle.ngram_ban(logits, hist, np.array([h], np.int32), case["n"], window) == -1
    assert np.array_equal(logits.view(np.uint32), before.view(np.uint32))


def _brute_ngram(hist, n):
    """All n-grams present in hist, then every x with (suffix, x) among them."""
    h = len(hist)
    if h < n:
        return set()
    grams = {tuple(hist[i:i + n]) for i in range(h - n + 1)}
    suffix = tuple(hist[h - n + 1:]) if n > 1 else tuple()
    return {g[-1] for g in grams if g[:-1] == suffix}


@pytest.mark.parametrize("n", [1, 2, 3, 5, 35])
def test_ngram_vs_hf_and_bruteforce(oracle, n):
    from transformers.generation.logits_process import NoRepeatNGramLogitsProcessor

    r = rng(100 + n)
    rows, window, vocab = 24, 128, 50
    hist = r.integers(0, vocab if n > 3 else 6, (rows, window)).astype(np.int32)
    hl = r.integers(0, window + 1, rows).astype(np.int32)
    hl[:4] = window
    hl[0:rows:2] = np.maximum(hl[0:rows:2], min(window, 2 * n + 1))
    # plant a repeat of the (n-1)-suffix of the held history in half of the rows
    for i in range(0, rows, 2):
        m, h = n - 1, int(hl[i])
        if m and h - 2 * m - 1 >= 0:
            st = int(r.integers(0, h - 2 * m))
            hist[i, st:st + m] = hist[i, h - m:h]
    logits = r.standard_normal((rows, vocab)).astype(np.float32)
    ours = logits.copy()
    assert oracle.ngram_ban(ours, hist, hl, n, window) == 0
    proc = NoRepeatNGramLogitsProcessor(n)
    planted_hits = 0
    for i in range(rows):
        h = int(hl[i])
        want = _brute_ngram(hist[i, :h].tolist(), n)
        got = set(np.nonzero(np.isneginf(ours[i]))[0].tolist())
        assert got == want, i
        if h > 0:
            hf = proc(torch.as_tensor(hist[i:i + 1, :h].astype(np.int64)),
                      torch.as_tensor(logits[i:i + 1].copy()))[0].numpy()
            assert set(np.nonzero(np.isneginf(hf))[0].tolist()) == got, i
        planted_hits += bool(got)
    assert planted_hits >= rows // 4


def test_ngram_noop_cases(oracle):
    logits = np.ones((2, 10), np.float32)
    hist = np.array([[1, 2, 1, 2], [3, 3, 3, 3]], np.int32)
    # window shorter than n: valid, bans nothing
    assert oracle.ngram_ban(logits, hist, None, 5, 4) == 0
    assert (logits == 1).all()
    # zero rows
    assert oracle.ngram_ban(np.ones((0, 10), np.float32), np.zeros((0, 4), np.int32), None, 2, 4) == 0


def test_constants_match_pages():
    from ring_sliding_window_b200 import synth
    with open(os.path.join(GOLDEN, "constants.json")) as f:
        c = json.load(f)
    for item in c["constants"]:
        assert getattr(synth, item["name"]) == item["value"], item
    for w in synth.workloads()[1:]:
        assert w.layers == c["lm_shape"]["layers"]
        assert w.heads * w.head_dim == c["lm_shape"]["hidden"]
        assert w.window == synth.RING_WINDOW
        assert max(w.prefill_lens) + w.window <= synth.MAX_POSITIONS
