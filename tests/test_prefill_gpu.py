"""Prefill parity: causal attention over the prompt and the cache fill.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.1 -- the prefill
segment keeps full attention; every prompt K/V stays in the cache.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


def _state(w):
    from ring_sliding_window_b200 import rswa
    return rswa.State(w.batch, w.layers, w.heads, w.head_dim, w.window, w.prefill_lens, dtype=w.dtype)


SMALL = [
    synth.Workload("p_fp32_d64", 21, torch.float32, 1, 1, 2, 64, 8, (64,), 0),
    synth.Workload("p_fp32_d128_ragged", 22, torch.float32, 3, 1, 2, 128, 8, (1, 130, 257), 0),
    synth.Workload("p_bf16_d128_ragged", 23, torch.bfloat16, 4, 1, 3, 128, 16, (129, 5, 383, 256), 0),
    synth.Workload("p_bf16_d64", 24, torch.bfloat16, 2, 1, 2, 64, 4, (200, 64), 0),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_prefill_small_all_rows(w):
    st = _state(w)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    torch.cuda.synchronize()
    sl = seq_slices(w.prefill_lens)
    for b in range(w.batch):
        ref = oracle.prefill(f64(q[sl[b]]), f64(k[sl[b]]), f64(v[sl[b]]), w.scale)
        err = np.max(np.abs(f64(out[sl[b]]) - ref)) if w.prefill_lens[b] else 0.0
        assert err <= tol_for(w.dtype), (b, err)
        # cache fill: slots [0, P_b) hold the prompt K/V bit for bit
        for h in range(w.heads):
            P = w.prefill_lens[b]
            assert torch.equal(st.cache_view(0, "k", b, h)[:P], k[sl[b], h])
            assert torch.equal(st.cache_view(0, "v", b, h)[:P], v[sl[b], h])
    assert st.check() == 0


def _sample_rows(P, rng, tile=128):
    rows = {0, 1, P - 1, P // 2}
    for t in range(tile, P, tile * 7):
        rows |= {t - 1, t}
    rows |= set(int(x) for x in rng.integers(0, P, 6))
    return sorted(r for r in rows if 0 <= r < P)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["single_page_decode", "multi_page_decode", "near_max_context"])
def test_prefill_full_size_sampled_rows(name):
    """Full-size prompts (P = 1,088 / 8,256 / 32,640), one layer: sampled rows
    (first, last, tile boundaries, random) of sampled heads and sequences."""
    w = synth.workload(name)
    w1 = synth.Workload(w.name, w.cfg_id, w.dtype, w.batch, 1, w.heads, w.head_dim, w.window,
                        w.prefill_lens, 0)
    st = _state(w1)
    q, k, v = synth.prefill_qkv(w1, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    torch.cuda.synchronize()
    assert st.check() == 0
    rng = np.random.default_rng(7)
    sl = seq_slices(w1.prefill_lens)
    for b in sorted({0, w1.batch - 1}):
        P = w1.prefill_lens[b]
        for h in (0, w1.heads - 1):
            kk, vv = f64(k[sl[b], h]), f64(v[sl[b], h])
            for i in _sample_rows(P, rng):
                ref = oracle.attend(f64(q[sl[b].start + i, h]), kk[:i + 1], vv[:i + 1], w1.scale)
                err = np.max(np.abs(f64(out[sl[b].start + i, h]) - ref))
                assert err <= tol_for(w1.dtype), (b, h, i, err)
        kc = st.cache_view(0, "k", b, 0)
        assert torch.equal(kc[:P], k[sl[b], 0])


@pytest.mark.slow
def test_prefill_ragged_long_prompts_cache_fill_and_sampled_rows():
    """Long ragged prompts as in the ragged-serving mix (lengths drawn from
    [1,024, 16,384], none a multiple of 128), 10 heads x 128, bf16: enough
    blocks for the tensor-core kernel's tile pairs.  The cache's prompt slots
    [0, P_b) of every (b, h) ring hold the prompt's K and V bit for bit (the
    fill is fused into the prefill: whole tiles by TMA store, the ragged last
    tile row by row), and sampled rows match the oracle."""
    from ring_sliding_window_b200 import rswa
    lens = (1031, 16383, 4097, 9001, 2053, 12289)
    w = synth.Workload("ragged_long", 27, torch.bfloat16, len(lens), 1, 10, 128, 128, lens, 0)
    st = _state(w)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    torch.cuda.synchronize()
    assert st.check() == 0
    sl = seq_slices(lens)
    for b, P in enumerate(lens):
        for h in range(w.heads):
            assert torch.equal(st.cache_view(0, "k", b, h)[:P], k[sl[b], h]), (b, h)
            assert torch.equal(st.cache_view(0, "v", b, h)[:P], v[sl[b], h]), (b, h)
    rng = np.random.default_rng(11)
    for b in (0, 1, 3):
        P = lens[b]
        h = int(rng.integers(0, w.heads))
        kk, vv = f64(k[sl[b], h]), f64(v[sl[b], h])
        rows = sorted({0, P - 1, (P // 128) * 128, (P // 128) * 128 - 1, int(rng.integers(0, P))})
        for i in rows:
            ref = oracle.attend(f64(q[sl[b].start + i, h]), kk[:i + 1], vv[:i + 1], w.scale)
            err = np.max(np.abs(f64(out[sl[b].start + i, h]) - ref))
            assert err <= tol_for(w.dtype), (b, h, i, err)
    st.close()
