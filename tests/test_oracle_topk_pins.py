"""Pins of the oracle's fused n-gram ban + top-k selection and its sampling
rule, against things other than the oracle itself: hand-worked fixtures,
numpy's argmax and stable argsort (library routines reached by a different
path than the oracle's lexsort), and closed forms of the sampling CDF.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.3.
"""
import json
import os

import numpy as np
import pytest

import oracle
from ring_sliding_window_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "topk_handbuilt.json")


def _f(v):
    return float(v)  # also parses "nan", "-inf"


def _cases():
    return json.load(open(GOLDEN))["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_topk_handbuilt(oracle, case):
    logits = np.array([[_f(x) for x in case["logits"]]], dtype=np.float32)
    hist = np.array([case["history"]], dtype=np.int32)
    idx, val, _, bad = oracle.ngram_topk(logits, hist, np.array([case["hist_len"]], np.int32),
                                         case["n"], case["window"], case["k"])
    assert idx[0].tolist() == case["expect_idx"]
    want = np.array([_f(x) for x in case["expect_val"]], dtype=np.float32)
    assert np.array_equal(val[0], want, equal_nan=True)
    assert bad[0] == (case["expect_idx"][0] == -1)


def _random_rows(seed, rows=6, vocab=3000, n=4, window=64):
    logits, hist, _ = synth.ngram_inputs(rows, vocab, n, window, seed)
    logits = logits.numpy().copy()
    hist = hist.numpy().copy()
    # the follower of the planted repeat gets the row's largest value, so the
    # ban decides the top-1 (a dropped ban fails below)
    h = window
    for r in range(rows):
        suffix = hist[r, h - (n - 1):]
        for i in range(h - n + 1):
            if np.array_equal(hist[r, i:i + n - 1], suffix):
                logits[r, hist[r, i + n - 1]] = 50.0
    return logits, hist


def test_top1_is_argmax_of_masked(oracle):
    logits, hist = _random_rows(7)
    idx, val, masked, bad = oracle.ngram_topk(logits, hist, None, 4, 64, 1)
    assert not bad.any()
    assert (masked == -np.inf).any(axis=1).all()  # every row banned something
    assert np.array_equal(idx[:, 0], np.argmax(masked, axis=1))
    assert np.all(val[:, 0] < 50.0)


def test_full_order_is_stable_argsort(oracle):
    logits, hist = _random_rows(8, rows=3, vocab=500)
    logits[0, 10:20] = 1.25  # ties
    logits[1, 5] = np.nan
    idx, val, masked, _ = oracle.ngram_topk(logits, hist, None, 4, 64, 500)
    for r in range(3):
        x = masked[r].astype(np.float64)
        x[np.isnan(x)] = -np.inf
        want = np.argsort(-x, kind="stable")
        assert np.array_equal(idx[r], want)
        assert np.array_equal(val[r], x[want].astype(np.float32))


def test_sampling_cdf_closed_forms(oracle):
    k = 8
    # equal values: p uniform, so u in [i/k, (i+1)/k) draws i
    for i in range(k):
        for u in (i / k + 1e-9, (i + 0.5) / k):
            assert oracle.topk_sample_cdf(np.zeros(k), u, 1.0)[0] == i
    # geometric values x_i = -i T ln 2: p_i = 2^-i, c_i = 2 - 2^-i
    T = 0.7
    x = -np.arange(k) * T * np.log(2.0)
    _, c, _ = oracle.topk_sample_cdf(x, 0.3, T)
    assert np.allclose(c, 2.0 - 2.0 ** -np.arange(k), rtol=1e-14)
    # -inf candidates never drawn
    x = np.array([1.0, -np.inf, 0.5, -np.inf])
    for u in np.linspace(0, 0.999, 50):
        assert oracle.topk_sample_cdf(x, u, 1.0)[0] in (0, 2)
    # a tiny temperature is greedy
    assert oracle.topk_sample_cdf(np.array([3.0, 2.9, 1.0]), 0.999, 1e-3)[0] == 0
