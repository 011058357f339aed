"""The seeded input generators: the same seed gives the same bits, and the
n-gram inputs carry the planted repeat their recipe states (the pages'
windowed no-repeat ban, "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘"
§2.3: 64 rows over the 129,280-token vocabulary, n = 35, window 128)."""
import numpy as np
import torch

import oracle
from ring_sliding_window_b200 import synth


def test_seed_formula_and_determinism():
    assert synth.seed(3, 2, 7) == 3 * 1_000_003 + 2 * 10_007 + 7
    a = synth.normal((4, 5), 123, torch.bfloat16)
    b = synth.normal((4, 5), 123, torch.bfloat16)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a, synth.normal((4, 5), 124, torch.bfloat16))
    # bf16 is the RNE cast of the fp32 draw
    assert torch.equal(a, synth.normal((4, 5), 123, torch.float32).to(torch.bfloat16))


def test_ngram_inputs_plant_one_repeat_per_row():
    rows, vocab, n, window = 64, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW
    logits, hist, starts = synth.ngram_inputs(rows, vocab, n, window, 17)
    assert logits.shape == (rows, vocab) and logits.dtype == torch.float32
    assert hist.shape == (rows, window) and hist.dtype == torch.int32
    h = hist.numpy()
    m = n - 1
    assert (h >= 0).all() and (h < vocab).all()
    for r in range(rows):
        i = int(starts[r])
        assert 0 <= i <= window - 2 * m - 1          # 0 .. 59 at the pages' sizes
        assert np.array_equal(h[r, i:i + m], h[r, window - m:])
        assert i + m < window - m                    # the follower lies before the suffix
    # the oracle bans at least the planted follower of every row
    _, _, masked, bad = oracle.ngram_topk(logits.numpy(), h, None, n, window, 1)
    assert not bad.any()
    for r in range(rows):
        assert masked[r, h[r, int(starts[r]) + m]] == -np.inf
