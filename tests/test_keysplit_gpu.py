"""Key-range split of one sequence's cache, on one GPU: G shares each hold
their slice of the prompt as an ordinary state (the last one also the ring),
produce partials with rswa_decode_step_partial, and rswa_combine_partials
merges them.  Every step is compared with the FP64 ring oracle over the whole
prompt.  The shares run one after another on the same device (no kernel
waits on another), standing in for one process per device; the exchange
itself is covered by the gloo test.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shares", [1, 2, 3])
@pytest.mark.parametrize("split", ["auto", "streamk"])
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_keysplit_shares_vs_oracle(shares, split, dtype, d, monkeypatch):
    from ring_sliding_window_b200 import rswa
    from ring_sliding_window_b200.keysplit import share_bounds
    if split != "auto":
        monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    H, W, P, steps, L = 2, 8, 1000, 14, 1
    w = synth.Workload("keysplit", 81, dtype, 1, L, H, d, W, (P,), steps)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    model = oracle.RingModel((P,), W, L, H, d)
    model.prefill(0, 0, f64(k), f64(v))
    bounds = share_bounds(P, shares)
    states = []
    for g, (lo, hi) in enumerate(bounds):
        st = rswa.State(1, L, H, d, W, [hi - lo], dtype=dtype)
        st.prefill(0, q[lo:hi], k[lo:hi], v[lo:hi], torch.empty_like(q[lo:hi]))
        states.append(st)
    ml = torch.empty(shares, 1, H, 2, dtype=torch.float32, device="cuda")
    o = torch.empty(shares, 1, H, d, dtype=torch.float32, device="cuda")
    tol = tol_for(dtype)
    for t in range(steps):
        qs, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        for g, st in enumerate(states):
            lo, hi = bounds[g]
            # the last share attends to its slice and the ring; the others to their slice
            key_hi = (hi - lo) + (W if g == shares - 1 else 0)
            st.decode_step_partial(0, qs, kn, vn, 0, key_hi, ml[g], o[g])
        out = torch.empty_like(qs)
        rswa.rswa_combine_partials(ml, o, out)
        ref = model.step(0, f64(qs), f64(kn), f64(vn), w.scale)
        err = np.max(np.abs(f64(out) - ref))
        assert err <= tol, (t, err)
        for st in states:
            st.advance()
    # only the last share wrote ring slots, and its ring matches the oracle's
    kc, vc, held = model.rings[0][0].snapshot()
    last = states[-1]
    lo = bounds[-1][0]
    for h in range(H):
        ring_k = f64(last.cache_view(0, "k", 0, h)[P - lo:P - lo + W])
        assert np.array_equal(ring_k, kc[P:P + W, h])
    for st in states:
        assert st.check() == 0
        st.close()


@pytest.mark.slow
@pytest.mark.parametrize("shares", [2, 4])
def test_keysplit_near_max_length_across_a_ring_wrap(shares):
    """The near-max sequence (32,640 prompt tokens, 10 heads x 128, W = 128)
    split over 2 and 4 shares, W + 2 decode steps (one ring wrap), every step
    against the FP64 ring oracle over the whole cache."""
    from ring_sliding_window_b200 import rswa
    from ring_sliding_window_b200.keysplit import share_bounds
    H, d, W, P, L = 10, 128, 128, 32640, 1
    steps = W + 2
    w = synth.Workload("keysplit_long", 83, torch.bfloat16, 1, L, H, d, W, (P,), steps)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    model = oracle.RingModel((P,), W, L, H, d)
    model.prefill(0, 0, f64(k), f64(v))
    bounds = share_bounds(P, shares)
    states = []
    for lo, hi in bounds:
        st = rswa.State(1, L, H, d, W, [hi - lo], dtype=torch.bfloat16)
        st.prefill(0, q[lo:hi], k[lo:hi], v[lo:hi], torch.empty_like(q[lo:hi]))
        states.append(st)
    del q, k, v
    ml = torch.empty(shares, 1, H, 2, dtype=torch.float32, device="cuda")
    o = torch.empty(shares, 1, H, d, dtype=torch.float32, device="cuda")
    for t in range(steps):
        qs, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        for g, st in enumerate(states):
            lo, hi = bounds[g]
            key_hi = (hi - lo) + (W if g == shares - 1 else 0)
            st.decode_step_partial(0, qs, kn, vn, 0, key_hi, ml[g], o[g])
        out = torch.empty_like(qs)
        rswa.rswa_combine_partials(ml, o, out)
        ref = model.step(0, f64(qs), f64(kn), f64(vn), w.scale)
        assert np.max(np.abs(f64(out) - ref)) <= tol_for(torch.bfloat16), t
        for st in states:
            st.advance()
    for st in states:
        assert st.check() == 0
        st.close()


def test_partial_ranges_of_one_state_match_the_full_step():
    """Two calls over [0, a) and [a, end) of the same state merge to the
    output of rswa_decode_step (the second call performs the ring write)."""
    from ring_sliding_window_b200 import rswa
    H, d, W, P = 3, 128, 8, (300, 77)
    w = synth.Workload("keysplit1", 82, torch.bfloat16, 2, 1, H, d, W, P, 10)
    full = rswa.State(2, 1, H, d, W, P, dtype=w.dtype)
    part = rswa.State(2, 1, H, d, W, P, dtype=w.dtype)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    for st in (full, part):
        st.prefill(0, q, k, v, torch.empty_like(q))
    ml = torch.empty(2, 2, H, 2, device="cuda")
    o = torch.empty(2, 2, H, d, device="cuda")
    for t in range(10):
        qs, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        ref = torch.empty_like(qs)
        full.decode_step(0, qs, kn, vn, ref)
        part.decode_step_partial(0, qs, kn, vn, 0, 50, ml[0], o[0])
        part.decode_step_partial(0, qs, kn, vn, 50, 1 << 40, ml[1], o[1])
        got = torch.empty_like(qs)
        rswa.rswa_combine_partials(ml, o, got)
        assert (got.float() - ref.float()).abs().max().item() <= 2e-2, t
        full.advance()
        part.advance()
    for b in range(2):
        for h in range(H):
            assert torch.equal(full.cache_view(0, "k", b, h), part.cache_view(0, "k", b, h))
    assert full.check() == 0 and part.check() == 0
