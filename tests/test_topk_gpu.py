"""Fused n-gram ban + top-k (+ sampling) on the GPU against the oracle.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.3.  Selection
is comparisons only, so indices, values and the in-place masked logits must
match the oracle bit for bit; a sampled token must be a valid inverse-CDF
draw of the FP64 probabilities (the two sides sum in different orders).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "topk_handbuilt.json")


def _rswa():
    from ring_sliding_window_b200 import rswa
    return rswa


def _run(logits, hist, hist_len, n, window, k, mask_in_place=False, uniform=None, temperature=1.0):
    rswa = _rswa()
    lg = logits.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, val, tok = rswa.rswa_ngram_topk(
        lg, hist.cuda(), None if hist_len is None else hist_len.cuda(), n, window, k,
        mask_in_place=mask_in_place, uniform=None if uniform is None else uniform.cuda(),
        temperature=temperature, device_error=err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), tok.cpu().numpy(), lg.cpu().numpy(), int(err.item())


def _check(logits, hist, hist_len, n, window, k, mask_in_place):
    lg_np = logits.numpy()
    want_idx, want_val, masked, bad = oracle.ngram_topk(
        lg_np, hist.numpy(), None if hist_len is None else hist_len.numpy(), n, window, k)
    idx, val, tok, lg_after, err = _run(logits, hist, hist_len, n, window, k, mask_in_place)
    assert np.array_equal(idx, want_idx)
    assert np.array_equal(val, want_val, equal_nan=True)
    assert np.array_equal(tok, np.where(bad, -1, want_idx[:, 0]))
    if mask_in_place:
        assert np.array_equal(lg_after.view(np.uint32), masked.view(np.uint32))
    else:
        assert np.array_equal(lg_after.view(np.uint32), lg_np.view(np.uint32))
    assert (err != 0) == bool(bad.any())
    return idx


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_topk_handbuilt(case):
    logits = torch.tensor([[float(x) for x in case["logits"]]], dtype=torch.float32)
    # ld must be a multiple of 4: pad the row
    ld = (logits.shape[1] + 3) // 4 * 4
    padded = torch.zeros(1, ld)
    padded[:, :logits.shape[1]] = logits
    hist = torch.tensor([case["history"]], dtype=torch.int32)
    hl = torch.tensor([case["hist_len"]], dtype=torch.int32)
    rswa = _rswa()
    lg = padded.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, val, tok = rswa.rswa_ngram_topk(lg, hist.cuda(), hl.cuda(), case["n"], case["window"],
                                         case["k"], device_error=err, vocab=logits.shape[1])
    assert idx.cpu().tolist()[0] == case["expect_idx"]
    want = np.array([float(x) for x in case["expect_val"]], dtype=np.float32)
    assert np.array_equal(val.cpu().numpy()[0], want, equal_nan=True)
    assert (err.item() != 0) == (case["expect_idx"][0] == -1)


@pytest.mark.parametrize("k", [1, 2, 8, 64])
@pytest.mark.parametrize("mask_in_place", [False, True])
def test_topk_full_vocab_vs_oracle(k, mask_in_place):
    """The pages' sizes: 64 rows over the 129,280-token vocabulary, n=35, window=128."""
    logits, hist, _ = synth.ngram_inputs(64, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW,
                                         synth.seed(5, 0, 800_000 + k))
    # push each row's banned follower to the top so the ban decides the selection
    for r in range(64):
        h = hist[r]
        suffix = h[-(synth.NGRAM_SIZE - 1):]
        for i in range(synth.NGRAM_WINDOW - synth.NGRAM_SIZE + 1):
            if torch.equal(h[i:i + synth.NGRAM_SIZE - 1], suffix):
                logits[r, h[i + synth.NGRAM_SIZE - 1]] = 100.0
    idx = _check(logits, hist, None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW, k, mask_in_place)
    assert (idx >= 0).all()


@pytest.mark.parametrize("vocab", [1, 3, 1000, 16384, 16385, 40000, 262144])
def test_topk_vocab_sizes_and_clusters(vocab):
    """One to sixteen CTAs per row, ragged last CTA, k up to min(64, vocab)."""
    rows = 5
    g = torch.Generator().manual_seed(vocab)
    logits = torch.randn(rows, (vocab + 3) // 4 * 4, generator=g)
    hist = torch.randint(0, vocab, (rows, 16), generator=g, dtype=torch.int32)
    hist[:, 8:11] = hist[:, 13:16]  # a repeat of the last 3 tokens (n = 4)
    for k in sorted({1, min(7, vocab), min(64, vocab)}):
        lg = logits[:, :vocab].contiguous() if (vocab % 4 == 0) else None
        if lg is None:  # keep ld a multiple of 4
            lg = logits
        rswa = _rswa()
        want_idx, want_val, _, _ = oracle.ngram_topk(lg[:, :vocab].contiguous().numpy(), hist.numpy(),
                                                     None, 4, 16, k)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        idx, val, tok = rswa.rswa_ngram_topk(lg.cuda(), hist.cuda(), None, 4, 16, k,
                                             device_error=err, vocab=vocab)
        assert np.array_equal(idx.cpu().numpy(), want_idx), (vocab, k)
        assert np.array_equal(val.cpu().numpy(), want_val), (vocab, k)
        assert err.item() == 0


@pytest.mark.parametrize("rows,vocab", [(300, 16), (513, 1000), (64, 4100)])
def test_topk_many_short_rows_per_cta(rows, vocab):
    """Many short rows (one to two CTAs each) and a row of 4,100 columns over
    one cluster of CTAs; a repeat planted in every history, k and
    mask_in_place over their range."""
    g = torch.Generator().manual_seed(rows * 7 + vocab)
    logits = torch.randn(rows, vocab, generator=g)
    window, n = 12, 3
    hist = torch.randint(0, vocab, (rows, window), generator=g, dtype=torch.int32)
    hist[:, 3:5] = hist[:, window - 2:]  # the last 2 tokens also at 3..4: bans hist[5]
    for k in sorted({1, 5, min(64, vocab)}):
        for mask_in_place in (False, True):
            _check(logits, hist, None, n, window, k, mask_in_place)


def test_topk_ties_nan_inf_and_ragged_histories():
    vocab, rows, n, window = 5000, 8, 3, 32
    g = torch.Generator().manual_seed(11)
    logits = torch.randn(rows, vocab, generator=g)
    logits[0] = 0.5                       # every column ties
    logits[1, ::3] = float("nan")
    logits[2, :] = float("-inf")          # every column -inf
    logits[3, 100:200] = 7.0              # 100-way tie at the top
    logits[4, 17] = float("inf")
    logits[5, :4000] = -0.0
    logits[5, 4000:] = 0.0
    hist = torch.randint(0, vocab, (rows, window), generator=g, dtype=torch.int32)
    hist[:, 5:7] = hist[:, 30:32]
    hist_len = torch.tensor([32, 0, 1, 2, 3, 31, 32, 17], dtype=torch.int32)
    for k in (1, 5, 64):
        _check(logits, hist, hist_len, n, window, k, True)


def test_topk_bad_rows_flagged_and_left_out():
    vocab, rows, window = 256, 4, 8
    logits = torch.randn(rows, vocab, generator=torch.Generator().manual_seed(3))
    hist = torch.randint(0, vocab, (rows, window), dtype=torch.int32,
                         generator=torch.Generator().manual_seed(4))
    hist[1, 2] = vocab          # token out of range
    hist_len = torch.tensor([8, 8, 9, 8], dtype=torch.int32)  # row 2: longer than the window
    idx, val, tok, lg_after, err = _run(logits, hist, hist_len, 2, window, 3, mask_in_place=True)
    rswa = _rswa()
    assert err & rswa.RSWA_DEVERR_BAD_TOKEN and err & rswa.RSWA_DEVERR_BAD_LENGTH
    for r in (1, 2):
        assert (idx[r] == -1).all() and np.isnan(val[r]).all() and tok[r] == -1
        assert np.array_equal(lg_after[r], logits[r].numpy())
    want_idx, _, _, _ = oracle.ngram_topk(logits.numpy(), hist.numpy(), hist_len.numpy(), 2, window, 3)
    assert np.array_equal(idx[[0, 3]], want_idx[[0, 3]])


@pytest.mark.parametrize("temperature", [0.3, 1.0, 4.0])
def test_topk_sampling_is_a_valid_inverse_cdf_draw(temperature):
    rows, k = 64, 64
    logits, hist, _ = synth.ngram_inputs(rows, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW,
                                         synth.seed(5, 1, 810_000))
    u = torch.rand(rows, generator=torch.Generator().manual_seed(9))
    u[0], u[1] = 0.0, float(np.nextafter(np.float32(1.0), np.float32(0.0)))
    idx, val, tok, _, err = _run(logits, hist, None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW, k,
                                 uniform=u, temperature=temperature)
    assert err == 0
    want_idx, want_val, _, _ = oracle.ngram_topk(logits.numpy(), hist.numpy(), None,
                                                 synth.NGRAM_SIZE, synth.NGRAM_WINDOW, k)
    assert np.array_equal(idx, want_idx)
    for r in range(rows):
        pos = int(np.nonzero(idx[r] == tok[r])[0][0])
        _, c, target = oracle.topk_sample_cdf(want_val[r], float(u[r]), temperature)
        lo = c[pos - 1] if pos else 0.0
        slack = 1e-5 * c[-1]
        assert lo - slack <= target <= c[pos] + slack, (r, pos, target, lo, c[pos])


def test_topk_rejects_bad_arguments():
    rswa = _rswa()
    lg = torch.zeros(2, 8, device="cuda")
    hist = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    out = torch.empty(2, 64, dtype=torch.int32, device="cuda")
    lib = rswa.lib
    args = lambda **kw: dict(dict(ld=8, rows=2, vocab=8, n=2, window=4, k=1, uniform=None, temp=1.0), **kw)
    def call(a):
        return lib.rswa_ngram_topk(lg.data_ptr(), a["ld"], hist.data_ptr(), 4, None, a["rows"],
                                   a["vocab"], a["n"], a["window"], a["k"], 0, a["uniform"],
                                   a["temp"], out.data_ptr(), None, None, None, None)
    assert call(args()) == rswa.RSWA_OK
    for bad in (args(k=0), args(k=9), args(k=65), args(ld=6), args(ld=7, vocab=7), args(n=0),
                args(rows=-1), args(vocab=262145, ld=262148),
                args(uniform=lg.data_ptr(), temp=0.0)):
        assert call(bad) == rswa.RSWA_EINVAL, bad
    torch.cuda.synchronize()


def _two_ban_history(window, n, bans, vocab, seed):
    """A history of `window` tokens whose (n-1)-suffix also precedes each token
    of `bans`, so exactly those tokens are banned (other tokens avoid the suffix)."""
    g = torch.Generator().manual_seed(seed)
    suffix = [vocab - 1, vocab - 2][: n - 1]
    h = torch.randint(0, vocab - 3, (window,), generator=g, dtype=torch.int32)
    pos = 0
    for t in bans:
        h[pos:pos + n - 1] = torch.tensor(suffix, dtype=torch.int32)
        h[pos + n - 1] = t
        pos += n + 2
    h[window - (n - 1):] = torch.tensor(suffix, dtype=torch.int32)
    return h


@pytest.mark.parametrize("k", [1, 2, 64])
def test_topk_two_banned_in_one_thread_and_banned_lone_maximum(k):
    """Columns 1000 and 2024 are held by the same thread of the greedy kernel:
    with both banned and both the largest, that thread must look past both.
    Row 1: the only finite value is banned, so every column ranks -inf and the
    lowest column wins."""
    vocab, n, window = 5000, 3, 32
    g = torch.Generator().manual_seed(21)
    logits = torch.randn(3, vocab, generator=g)
    logits[0, 1000], logits[0, 2024] = 100.0, 99.0
    logits[1] = float("-inf")
    logits[1, 1000] = 5.0
    logits[2, 1000], logits[2, 2024] = 100.0, 99.0  # not banned in row 2
    hist = torch.stack([_two_ban_history(window, n, [1000, 2024], vocab, 1),
                        _two_ban_history(window, n, [1000], vocab, 2),
                        _two_ban_history(window, n, [7], vocab, 3)])
    idx = _check(logits, hist, None, n, window, k, False)
    assert idx[0, 0] not in (1000, 2024) and idx[1, 0] == 0 and idx[2, 0] == 1000


@pytest.mark.parametrize("tied", [False, True], ids=["distinct", "tied"])
def test_topk_many_candidates_in_few_threads(tied):
    """More than 256 candidates reach the leader (the radix-select branch of
    the final selection), and threads hold more than two keys >= T (the
    reread branch): every column of five threads' strided ranges (thread t of
    the CTA at column offset 16,384 rho reads columns
    16,384 rho + 4 (t + 256 i) + u, i < 16, u < 4) gets a value far above the
    rest, so the threshold from the thread maxima lets 320 of them through."""
    rows, k = 3, 64
    logits, hist, _ = synth.ngram_inputs(rows, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW,
                                         synth.seed(5, 0, 900_000 + int(tied)))
    cols = []
    for rho, t in ((1, 0), (1, 37), (2, 100), (5, 200), (7, 255)):
        for i in range(16):
            for u in range(4):
                c = 16384 * rho + 4 * (t + 256 * i) + u
                if c < synth.VOCAB:
                    cols.append(c)
    cols = torch.tensor(cols)
    planted = torch.full((len(cols),), 50.0) if tied else 50.0 + 0.001 * torch.arange(len(cols))
    logits[:, cols] = planted
    idx = _check(logits, hist, None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW, k, False)
    # the k chosen are planted columns (a banned follower may have taken one out)
    assert np.isin(idx, cols.numpy()).all()
