"""Scores whose running maximum keeps jumping: the online-softmax rescale paths.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.1 (prefill keeps
full attention; each decode step attends to the prompt plus the ring).  The
definition is plain softmax attention, so the FP64 oracle is unchanged; what
these inputs add is magnitude.  With N(0, 1) inputs a row's maximum settles
in its first key tile, so the paths that rescale the running output when a
later tile raises the maximum (the tensor-core prefill rescales O in TMEM
when a warp's maximum grows by more than 2^8; the decode kernel rescales at
every tile; the split-K merge combines partials whose maxima differ by many
orders of magnitude) would otherwise hardly run.

Key magnitudes grow (or shrink) by tile of 128 positions, so consecutive
tiles' row maxima differ by about 2^11 in the softmax's base-2 units.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu

TILE = 128


def _ramp(P, grow):
    t = np.arange(P) // TILE
    if not grow:
        t = t.max(initial=0) - t
    return torch.tensor(1.0 + 1.5 * t, dtype=torch.float64)


def _tol(dtype, q, k, v, scale):
    """bf16: the suite's bound.  fp32: the suite's bound plus what rounding
    of the scores alone allows at these magnitudes.  A fp32 dot product of
    length d is off by at most d u sum|q_i k_i| (u = 2^-24, the standard
    forward error bound), and a softmax average moves by at most
    2 max|v| per unit of score error, so the outputs may differ from the
    exact ones by 2 max|v| d u max sum|q_i k_i| scale."""
    if dtype == torch.bfloat16:
        return tol_for(dtype)
    q, k, v = (np.abs(x.reshape(-1, x.shape[-2], x.shape[-1])) for x in (q, k, v))
    smax = max(float(np.max(q[:, h] @ k[:, h].T)) for h in range(q.shape[1])) * scale
    d = q.shape[-1]
    return tol_for(dtype) + 2.0 * float(v.max()) * d * 2.0 ** -24 * smax


def _rescale_fraction(q, k, scale, thresh=8.0):
    """Fraction of (row, head) whose causal running maximum, in base-2 units,
    rises by more than `thresh` at some key tile after the first: the rows
    on which the tensor-core prefill has to rescale O."""
    P, H, _ = q.shape
    hits = 0
    for h in range(H):
        s = (q[:, h] @ k[:, h].T) * scale / np.log(2.0)
        s[np.triu_indices(P, 1)] = -np.inf
        run = np.full(P, -np.inf)
        hit = np.zeros(P, bool)
        for j0 in range(0, P, TILE):
            m = np.maximum(run, s[:, j0:j0 + TILE].max(axis=1))
            if j0:
                hit |= m > run + thresh
            run = m
        hits += hit[TILE:].sum()
    return hits / (H * (P - TILE))


def _prompt(lens, H, d, dtype, grow, seed):
    tot = sum(lens)
    q = synth.normal((tot, H, d), synth.seed(seed, 0, 1), torch.float32, "cpu") * 2.0
    k = synth.normal((tot, H, d), synth.seed(seed, 0, 2), torch.float32, "cpu")
    v = synth.normal((tot, H, d), synth.seed(seed, 0, 3), torch.float32, "cpu")
    for sl, P in zip(seq_slices(lens), lens):
        k[sl] *= _ramp(P, grow).to(torch.float32)[:, None, None]
    return tuple(x.to(dtype).cuda() for x in (q, k, v))


# (dtype, d, prompt lengths, heads): the tensor-core prefill runs two query
# tiles per CTA once the batch has at least one tile pair per SM (the 16-head
# case), one tile per CTA below that; fp32 takes the SIMT kernel
SHAPES = [(torch.bfloat16, 128, [2200, 0, 300], 16), (torch.bfloat16, 128, [700, 0, 300], 2),
          (torch.float32, 64, [700, 0, 300], 2)]


@pytest.mark.parametrize("dtype,d,lens,H", SHAPES,
                         ids=["bf16_tile_pairs", "bf16_single_tiles", "fp32_simt"])
@pytest.mark.parametrize("grow", [True, False], ids=["growing", "shrinking"])
def test_prefill_growing_scores_all_rows(dtype, d, lens, H, grow):
    from ring_sliding_window_b200 import rswa
    st = rswa.State(len(lens), 1, H, d, 8, lens, dtype=dtype)
    q, k, v = _prompt(lens, H, d, dtype, grow, 61)
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    torch.cuda.synchronize()
    assert st.check() == 0
    scale = 1.0 / np.sqrt(d)
    for b, sl in enumerate(seq_slices(lens)):
        if not lens[b]:
            continue
        qq, kk, vv = f64(q[sl]), f64(k[sl]), f64(v[sl])
        if grow and lens[b] > 2 * TILE:
            assert _rescale_fraction(qq, kk, scale) > 0.5
        ref = oracle.prefill(qq, kk, vv, scale)
        err = np.max(np.abs(f64(out[sl]) - ref))
        assert err <= _tol(dtype, qq, kk, vv, scale), (b, err)
    st.close()


@pytest.mark.parametrize("split", ["streamk", "cluster"])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_growing_generated_keys(split, dtype, d, monkeypatch):
    """Every generated key is larger than the last, so the ring's newest
    slots dominate a cache whose prompt is long: the split-K pieces over the
    prompt carry maxima far below the piece holding the ring."""
    from ring_sliding_window_b200 import rswa
    monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    lens, H, W, steps = [900, 40], 2, 8, 14
    st = rswa.State(len(lens), 1, H, d, W, lens, dtype=dtype)
    q, k, v = _prompt(lens, H, d, dtype, False, 62)
    st.prefill(0, q, k, v, torch.empty_like(q))
    rings = [oracle.Ring(P, W, H, d) for P in lens]
    for r, sl in zip(rings, seq_slices(lens)):
        r.prefill(f64(k[sl]), f64(v[sl]))
    scale = 1.0 / np.sqrt(d)
    keys = [[f64(k[sl])] for sl in seq_slices(lens)]
    vals = [[f64(v[sl])] for sl in seq_slices(lens)]
    for t in range(steps):
        qs, kn, vn = (synth.normal((len(lens), H, d), synth.seed(63, t, i), torch.float32, "cpu")
                      for i in range(3))
        kn = kn * (1.0 + 0.75 * t)
        qs, kn, vn = (x.to(dtype).cuda() for x in (qs * 2.0, kn, vn))
        out = torch.empty_like(qs)
        st.decode_step(0, qs, kn, vn, out)
        for b, r in enumerate(rings):
            ref, _, _ = r.step(f64(qs[b]), f64(kn[b]), f64(vn[b]), scale)
            err = np.max(np.abs(f64(out[b]) - ref))
            keys[b].append(f64(kn[b])[None])
            vals[b].append(f64(vn[b])[None])
            tol = _tol(dtype, f64(qs[b])[None], np.concatenate(keys[b]), np.concatenate(vals[b]),
                       scale)
            assert err <= tol, (t, b, err, tol)
        st.advance()
    assert st.check() == 0
    st.close()
