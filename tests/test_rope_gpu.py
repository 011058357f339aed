"""RoPE at cache-write time (rswa_state_set_rope) against the FP64 oracle.

The oracle composes its rotary embedding (pinned to the transformers Llama
implementation) with the ring simulation: keys are rotated at their
positions before they enter the oracle's cache, queries at theirs.  The
position policies: prompt token i at i; generated token t at P + t
('absolute') or at its cache slot P + (t mod W) ('slot').
Outputs within the usual tolerances; V cache contents bit-exact; rotated K
contents within one rounding of the cache's type (the two sides rotate in
different precisions).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu

POLICIES = {"absolute": 1, "slot": 2}


@pytest.mark.parametrize("policy", ["absolute", "slot"])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64),
                                     (torch.bfloat16, 64)])
@pytest.mark.parametrize("split", ["streamk", "cluster"])
def test_rope_prefill_and_decode_vs_oracle(policy, dtype, d, split, monkeypatch):
    from ring_sliding_window_b200 import rswa
    monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    B, L, H, W, P, steps, theta = 2, 2, 2, 8, (200, 37), 20, 10000.0
    w = synth.Workload("rope", 61, dtype, B, L, H, d, W, P, steps)
    st = rswa.State(B, L, H, d, W, P, dtype=dtype)
    st.set_rope(POLICIES[policy], theta)
    tol = tol_for(dtype)
    sl = seq_slices(P)
    model = oracle.RingModel(P, W, L, H, d)
    for l in range(L):
        q, k, v = synth.prefill_qkv(w, l, "cuda")
        out = torch.empty_like(q)
        st.prefill(l, q, k, v, out)
        for b in range(B):
            pos = np.arange(P[b])
            qr, kr = oracle.rope(f64(q[sl[b]]), pos, theta), oracle.rope(f64(k[sl[b]]), pos, theta)
            ref = oracle.prefill(qr, kr, f64(v[sl[b]]), w.scale)
            assert np.max(np.abs(f64(out[sl[b]]) - ref)) <= tol, (l, b)
            model.prefill(l, b, kr, f64(v[sl[b]]))
    for t in range(steps):
        for l in range(L):
            q, kn, vn = synth.decode_qkv(w, l, t, "cuda")
            out = torch.empty_like(q)
            st.decode_step(l, q, kn, vn, out)
            for b in range(B):
                p = [oracle.rope_position(policy, P[b], t, W)]
                ref, _, _ = model.rings[l][b].step(oracle.rope(f64(q[b])[None], p, theta)[0],
                                                   oracle.rope(f64(kn[b])[None], p, theta)[0],
                                                   f64(vn[b]), w.scale)
                err = np.max(np.abs(f64(out[b]) - ref))
                assert err <= tol, (t, l, b, err)
        st.advance()
    # caches: V exact, rotated K within one rounding of the cache type
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -23
    for l in range(L):
        for b in range(B):
            kc, vc, held = model.rings[l][b].snapshot()
            for h in range(H):
                assert np.array_equal(f64(st.cache_view(l, "v", b, h)[:held]), vc[:held, h])
                gk = f64(st.cache_view(l, "k", b, h)[:held])
                assert np.all(np.abs(gk - kc[:held, h]) <= rel * np.abs(kc[:held, h]) + 1e-6)
    assert st.check() == 0


@pytest.mark.slow
@pytest.mark.parametrize("policy", ["absolute", "slot"])
def test_rope_long_prompt_sampled_rows_and_ring_wrap(policy):
    """A 32,640-token prompt (the near-max length): rotation angles up to
    ~3.3e4 radians, where the reduction of the angle matters.  Sampled query
    rows of the prefill against the oracle, sampled rotated cache rows within
    one bf16 rounding, then W + 3 decode steps (one ring wrap) step by step."""
    from ring_sliding_window_b200 import rswa
    B, L, H, d, W, theta = 1, 1, 2, 128, 128, 10000.0
    P = (32640,)
    w = synth.Workload("rope_long", 62, torch.bfloat16, B, L, H, d, W, P, W + 3)
    st = rswa.State(B, L, H, d, W, P, dtype=torch.bfloat16)
    st.set_rope(POLICIES[policy], theta)
    tol = tol_for(torch.bfloat16)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    pos = np.arange(P[0])
    qr, kr, vv = oracle.rope(f64(q), pos, theta), oracle.rope(f64(k), pos, theta), f64(v)
    for r in (0, 1, 127, 128, 4095, 16383, 16384, 32511, 32639):
        ref = oracle.prefill(qr[:r + 1], kr[:r + 1], vv[:r + 1], w.scale, r, r + 1)[r]
        assert np.max(np.abs(f64(out[r]) - ref)) <= tol, r
    rows = np.array([0, 1, 8191, 16384, 30000, 32639])
    for h in range(H):
        gk = f64(st.cache_view(0, "k", 0, h)[rows])
        assert np.all(np.abs(gk - kr[rows, h]) <= 2.0 ** -8 * np.abs(kr[rows, h]) + 1e-6), h
    model = oracle.RingModel(P, W, L, H, d)
    model.prefill(0, 0, kr, vv)
    for t in range(W + 3):
        qd, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        o = torch.empty_like(qd)
        st.decode_step(0, qd, kn, vn, o)
        p = [oracle.rope_position(policy, P[0], t, W)]
        ref, _, _ = model.rings[0][0].step(oracle.rope(f64(qd[0])[None], p, theta)[0],
                                           oracle.rope(f64(kn[0])[None], p, theta)[0],
                                           f64(vn[0]), w.scale)
        assert np.max(np.abs(f64(o[0]) - ref)) <= tol, t
        st.advance()
    assert st.check() == 0


def test_rope_reset_and_policy_errors():
    from ring_sliding_window_b200 import rswa
    st = rswa.State(1, 1, 2, 128, 8, [64], dtype=torch.bfloat16)
    for pol, th in [(3, 10000.0), (-1, 10000.0), (1, 0.0), (1, float("nan")), (2, -5.0)]:
        with pytest.raises(rswa.RswaError) as e:
            st.set_rope(pol, th)
        assert e.value.status == rswa.RSWA_EINVAL
    # reset_ring puts the position table back with the counters: a replay of
    # the same steps after a reset gives the same outputs
    w = synth.Workload("rope_reset", 62, torch.bfloat16, 1, 1, 2, 128, 8, (64,), 12)
    st.set_rope(1, 10000.0)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    st.prefill(0, q, k, v, torch.empty_like(q))
    runs = []
    for _ in range(2):
        outs = []
        for t in range(12):
            a, b_, c = synth.decode_qkv(w, 0, t, "cuda")
            o = torch.empty_like(a)
            st.decode_step(0, a, b_, c, o)
            st.advance()
            outs.append(o)
        runs.append(torch.stack(outs))
        st.reset_ring()
    assert torch.equal(runs[0], runs[1])
    assert st.check() == 0
