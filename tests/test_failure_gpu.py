"""Failure detection on the GPU without a fault: a test-only flag makes the
decode kernel's producer issue no copies (or the prefill's producers no tile
loads), so every bounded wait in the kernel runs out (about one second).  The
kernel records the timeout in the state's device error word and returns; the
host reads RSWA_ETIMEOUT; the context and the state stay usable, and the next
call is correct again."""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


def test_decode_wait_timeout_is_reported_and_recoverable():
    from ring_sliding_window_b200 import rswa
    w = synth.Workload("timeout_case", 41, torch.bfloat16, 2, 1, 2, 128, 8, (300, 70), 3)
    st = rswa.State(w.batch, 1, w.heads, w.head_dim, w.window, w.prefill_lens, dtype=w.dtype)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    st.prefill(0, q, k, v, torch.empty_like(q))
    sl = seq_slices(w.prefill_lens)
    model = oracle.RingModel(w.prefill_lens, w.window, 1, w.heads, w.head_dim)
    for b in range(w.batch):
        model.prefill(0, b, f64(k[sl[b]]), f64(v[sl[b]]))

    # step 0: normal
    qn, kn, vn = synth.decode_qkv(w, 0, 0, "cuda")
    out = torch.empty_like(qn)
    st.decode_step(0, qn, kn, vn, out)
    assert np.max(np.abs(f64(out) - model.step(0, f64(qn), f64(kn), f64(vn), w.scale))) <= tol_for(w.dtype)
    st.advance()
    assert st.check() == rswa.RSWA_OK

    # step 1 with the copies dropped: the waits run out, the status says so
    rswa.rswa_debug_inject_fault(st.handle, rswa.RSWA_FAULT_DROP_DECODE_COPIES)
    qn, kn, vn = synth.decode_qkv(w, 0, 1, "cuda")
    st.decode_step(0, qn, kn, vn, torch.empty_like(qn))
    assert st.check() == rswa.RSWA_ETIMEOUT
    assert st.check() == rswa.RSWA_OK  # reading the word clears it

    # back to normal: the same step (no advance in between) again is correct;
    # the failed step's ring write put the same k_new/v_new in the same slot
    rswa.rswa_debug_inject_fault(st.handle, 0)
    out = torch.empty_like(qn)
    st.decode_step(0, qn, kn, vn, out)
    torch.cuda.synchronize()
    ref = model.step(0, f64(qn), f64(kn), f64(vn), w.scale)
    assert np.max(np.abs(f64(out) - ref)) <= tol_for(w.dtype)
    assert st.check() == rswa.RSWA_OK
    st.close()


def test_prefill_wait_timeout_is_reported_and_recoverable():
    """The tensor-core prefill's timeout path: with its tile loads dropped
    every bounded wait runs out; the kernel records the timeout, frees its
    tensor memory and returns, and the same prefill afterwards is correct
    (outputs against the oracle, the cache's prompt slots bit-exact) and the
    state decodes normally."""
    from ring_sliding_window_b200 import rswa
    w = synth.Workload("prefill_timeout", 42, torch.bfloat16, 2, 1, 2, 128, 8, (300, 70), 1)
    st = rswa.State(w.batch, 1, w.heads, w.head_dim, w.window, w.prefill_lens, dtype=w.dtype)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    rswa.rswa_debug_inject_fault(st.handle, rswa.RSWA_FAULT_DROP_PREFILL_LOADS)
    st.prefill(0, q, k, v, out)
    assert st.check() == rswa.RSWA_ETIMEOUT
    assert st.check() == rswa.RSWA_OK  # reading the word clears it

    rswa.rswa_debug_inject_fault(st.handle, 0)
    st.prefill(0, q, k, v, out)
    torch.cuda.synchronize()
    assert st.check() == rswa.RSWA_OK
    sl = seq_slices(w.prefill_lens)
    model = oracle.RingModel(w.prefill_lens, w.window, 1, w.heads, w.head_dim)
    for b in range(w.batch):
        ref = oracle.prefill(f64(q[sl[b]]), f64(k[sl[b]]), f64(v[sl[b]]), w.scale)
        assert np.max(np.abs(f64(out[sl[b]]) - ref)) <= tol_for(w.dtype)
        for h in range(w.heads):
            P = w.prefill_lens[b]
            assert torch.equal(st.cache_view(0, "k", b, h)[:P], k[sl[b], h])
            assert torch.equal(st.cache_view(0, "v", b, h)[:P], v[sl[b], h])
        model.prefill(0, b, f64(k[sl[b]]), f64(v[sl[b]]))
    qn, kn, vn = synth.decode_qkv(w, 0, 0, "cuda")
    o1 = torch.empty_like(qn)
    st.decode_step(0, qn, kn, vn, o1)
    torch.cuda.synchronize()
    ref = model.step(0, f64(qn), f64(kn), f64(vn), w.scale)
    assert np.max(np.abs(f64(o1) - ref)) <= tol_for(w.dtype)
    assert st.check() == rswa.RSWA_OK
    st.close()
