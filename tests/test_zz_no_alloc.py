"""The allocation-free decode entry point against the workspace-based one.

rswa_decode_step_noalloc is for callers that cannot give the library a
workspace (a plugin inside another runtime that may not allocate device
memory of its own, or a serving loop that keeps cudaMalloc/cudaFree off its
hot path).  It takes its scratch from a static device array inside the
library.  These tests call it through the C ABI and compare it with
rswa_decode_step on two calls in a row, at the tolerance the other decode
tests use.  The file sorts last so that a failure here stops a -x run only
after every other test has run.
"""
import numpy as np
import pytest
import torch

from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def _tol(dtype):
    return 2e-2 if dtype == torch.bfloat16 else 1e-5


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_noalloc_matches_workspace_path_two_calls(dtype, d):
    from ring_sliding_window_b200 import rswa
    B, H, W, P = 3, 4, 8, (300, 17, 1000)
    w = synth.Workload("noalloc", 31, dtype, B, 1, H, d, W, P, 2)
    st = rswa.State(B, 1, H, d, W, P, dtype=dtype)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    st.prefill(0, q, k, v, torch.empty_like(q))
    # the no-alloc path works on its own copy of the same cache
    kc, vc = st.k_cache[0].clone(), st.v_cache[0].clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cfg = rswa.make_config(B, 1, H, d, W, dtype)
    for t in range(2):
        qn, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        ref = torch.empty_like(qn)
        st.decode_step(0, qn, kn, vn, ref)
        st.advance()
        got = torch.empty_like(qn)
        rswa.rswa_decode_step_noalloc(cfg, P, [t] * B, kc, vc, qn, kn, vn, got, device_error=err)
        torch.cuda.synchronize()
        diff = (got.double() - ref.double()).abs().max().item()
        assert diff <= _tol(dtype), (t, diff)
        # bit patterns: slots not yet written hold whatever the allocator left (maybe NaN)
        assert torch.equal(_bits(kc), _bits(st.k_cache[0])), t
        assert torch.equal(_bits(vc), _bits(st.v_cache[0])), t
    assert int(err.item()) == 0
    assert st.check() == 0
    st.close()


def test_noalloc_rejects_batches_beyond_the_scratch_limit():
    from ring_sliding_window_b200 import rswa
    # enough (b, h) rings that the split-K partials alone exceed the array
    B, H, d, W = 512, 32, 128, 8
    cfg = rswa.make_config(B, 1, H, d, W, torch.bfloat16)
    plens = [16] * B
    assert rswa.rswa_workspace_bytes(cfg, plens) > rswa.RSWA_NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rswa.RswaError) as e:
        rswa.rswa_decode_step_noalloc(cfg, plens, [0] * B, dummy, dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == rswa.RSWA_ENOMEM
    # missing arguments are rejected on the host, before anything is enqueued
    assert rswa.lib.rswa_decode_step_noalloc(None, None, None, None, None, None, None, None,
                                             None, None, None) == rswa.RSWA_EINVAL
    with pytest.raises(rswa.RswaError) as e:
        rswa.rswa_decode_step_noalloc(cfg, plens, [-1] + [0] * (B - 1), dummy, dummy, dummy,
                                      dummy, dummy, dummy)
    assert e.value.status == rswa.RSWA_EINVAL
