"""Failure detection on the GPU without a fault: a test-only flag makes the
decode kernel's producer issue no copies, so every bounded wait in the kernel
runs out (about one second).  The kernel records the timeout in the state's
device error word and returns; the host reads RSWA_ETIMEOUT; the context and
the state stay usable, and the next step is correct again."""
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
