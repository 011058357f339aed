"""N-gram ban parity, bit-exact against the oracle.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.3 -- inside the
history window every token that would repeat an n-gram gets -inf; defaults
no_repeat_ngram_size 35, ngram_window 128.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_mask(logits_np, hist_np, hl_np, n, window, vocab=None):
    from ring_sliding_window_b200 import rswa
    lg = torch.from_numpy(logits_np.copy()).cuda()
    hist = torch.from_numpy(np.ascontiguousarray(hist_np, dtype=np.int32)).cuda()
    hl = None if hl_np is None else torch.from_numpy(np.asarray(hl_np, dtype=np.int32)).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rswa.rswa_ngram_mask(lg, hist, hl, n, window, device_error=err, vocab=vocab)
    torch.cuda.synchronize()
    return lg.cpu().numpy(), int(err.item())


def _bits(a):
    return a.view(np.uint32)


def test_ngram_full_size_planted():
    """64 rows x 129,280 vocab, n = 35, window = 128, one planted repeat per row."""
    rows, V, n, W = 64, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW
    logits, hist, starts = synth.ngram_inputs(rows, V, n, W, synth.seed(5, 0, 700_000))
    lg, hi = logits.numpy(), hist.numpy()
    want = lg.copy()
    assert oracle.ngram_ban(want, hi, None, n, W) == 0
    got, err = _gpu_mask(lg, hi, None, n, W)
    assert err == 0
    assert np.array_equal(_bits(got), _bits(want))
    for r in range(rows):  # the planted ban is there
        assert np.isneginf(got[r, hi[r, int(starts[r]) + n - 1]])


@pytest.mark.parametrize("n", [1, 2, 3, 4, 7, 35, 128])
def test_ngram_random_dense_matches(n):
    """Small alphabets make many repeats; ragged hist_len including 0 and window."""
    rng = np.random.default_rng(n)
    rows, V, W = 96, 300, 128
    hist = rng.integers(0, 4, (rows, W)).astype(np.int32)
    hl = rng.integers(0, W + 1, rows).astype(np.int32)
    hl[0], hl[1], hl[2] = 0, W, n
    logits = rng.standard_normal((rows, V)).astype(np.float32)
    want = logits.copy()
    assert oracle.ngram_ban(want, hist, hl, n, W) == 0
    got, err = _gpu_mask(logits, hist, hl, n, W)
    assert err == 0
    assert np.array_equal(_bits(got), _bits(want))


def test_ngram_golden_cases():
    g = json.load(open(os.path.join(GOLDEN, "ngram_handbuilt.json")))
    V = g["vocab"]
    for case in g["cases"]:
        hist = case["history"]
        window = case.get("window", len(hist))
        row = np.array([list(hist) + [case.get("pad", 0)] * (window - len(hist))], np.int32)
        logits = np.random.default_rng(1).standard_normal((1, V)).astype(np.float32)
        got, err = _gpu_mask(logits, row, [len(hist)], case["n"], window)
        assert err == 0, case["id"]
        banned = sorted(np.nonzero(np.isneginf(got[0]))[0].tolist())
        assert banned == sorted(case["banned"]), case["id"]


def test_ngram_bad_rows_flagged_and_untouched():
    g = json.load(open(os.path.join(GOLDEN, "ngram_handbuilt.json")))
    V = g["vocab"]
    from ring_sliding_window_b200 import rswa
    for case in g["bad_rows"]:
        hist = case["history"]
        window = case.get("window", len(hist))
        row = np.array([hist + [0] * (window - len(hist))], np.int32)
        h = case.get("hist_len", len(hist))
        logits = np.random.default_rng(2).standard_normal((1, V)).astype(np.float32)
        got, err = _gpu_mask(logits, row, [h], case["n"], window)
        assert np.array_equal(_bits(got), _bits(logits)), case["id"]
        expect = rswa.RSWA_DEVERR_BAD_LENGTH if h > window else rswa.RSWA_DEVERR_BAD_TOKEN
        assert err == expect, case["id"]


def test_ngram_strided_logits_and_noops():
    from ring_sliding_window_b200 import rswa
    rng = np.random.default_rng(3)
    V, W = 50, 16
    base = torch.randn(4, 64, device="cuda")
    lg = base[:, :V]  # ld = 64 > vocab
    hist = torch.tensor(rng.integers(0, 3, (4, W)), dtype=torch.int32, device="cuda")
    want = lg.cpu().numpy().copy()
    full = base.cpu().numpy().copy()
    oracle.ngram_ban(want, hist.cpu().numpy(), None, 2, W)
    rswa.rswa_ngram_mask(lg, hist, None, 2, W)
    torch.cuda.synchronize()
    got = base.cpu().numpy()
    assert np.array_equal(_bits(got[:, :V]), _bits(want))
    assert np.array_equal(_bits(got[:, V:]), _bits(full[:, V:]))  # padding untouched
    # window < n bans nothing
    before = base.clone()
    rswa.rswa_ngram_mask(lg, hist, None, W + 1, W)
    torch.cuda.synchronize()
    assert torch.equal(before, base)
    # zero rows is a no-op
    rswa.rswa_ngram_mask(torch.empty(0, V, device="cuda"), torch.empty(0, W, dtype=torch.int32, device="cuda"),
                         None, 2, W)
