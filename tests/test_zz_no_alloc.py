"""The allocation-free decode entry point against the workspace-based one.

rswa_decode_step_noalloc is for callers that cannot give the library a
workspace (a plugin inside another runtime that may not allocate device
memory of its own, or a serving loop that keeps cudaMalloc/cudaFree off its
hot path).  It takes its scratch from a static device array inside the
library.  These tests call it through the C ABI across two wraps of the
ring and compare every call with the FP64 oracle and with rswa_decode_step,
at the tolerance the other decode tests use.  The file sorts last so that a failure here stops a -x run only
after every other test has run.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def _tol(dtype):
    return 2e-2 if dtype == torch.bfloat16 else 1e-5


def _ring_view(buf, plens, W, H, d, b, h):
    """[P_b + W, d] rows of ring (b, h) in a cache laid out request after
    request, each request's slots head-major (the layout rswa_cache_offset
    reports for a state created without a pool)."""
    base = sum(p + W for p in plens[:b]) * H * d
    n = (plens[b] + W) * d
    off = base + h * n
    return buf[off:off + n].view(plens[b] + W, d)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_noalloc_matches_oracle_and_workspace_path_across_wraps(dtype, d):
    """2W + 3 steps with W = 8: the ring fills (warm-up appends), then wraps
    twice, so steps t >= W overwrite slot P_b + (t mod W) and attend over
    exactly P_b + W keys.  Every step is checked against the FP64 oracle's
    ring simulation (attention within tolerance, the cache bit-exact) and
    against rswa_decode_step on a state over the same inputs.  The ring
    position is passed explicitly as n_generated = t."""
    from ring_sliding_window_b200 import rswa
    B, H, W, P = 3, 4, 8, (300, 17, 1000)
    steps = 2 * W + 3
    w = synth.Workload("noalloc", 31, dtype, B, 1, H, d, W, P, steps)
    st = rswa.State(B, 1, H, d, W, P, dtype=dtype)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    st.prefill(0, q, k, v, torch.empty_like(q))
    for b in range(B):
        for h in range(H):
            assert _ring_view(st.k_cache[0], P, W, H, d, b, h).data_ptr() == \
                st.cache_view(0, "k", b, h).data_ptr()
    model = oracle.RingModel(P, W, 1, H, d)
    base = 0
    for b in range(B):
        model.prefill(0, b, f64(k[base:base + P[b]]), f64(v[base:base + P[b]]))
        base += P[b]
    # the no-alloc path works on its own copy of the same cache
    kc, vc = st.k_cache[0].clone(), st.v_cache[0].clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cfg = rswa.make_config(B, 1, H, d, W, dtype)
    tol = _tol(dtype)
    for t in range(steps):
        qn, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        ref = torch.empty_like(qn)
        st.decode_step(0, qn, kn, vn, ref)
        st.advance()
        got = torch.empty_like(qn)
        rswa.rswa_decode_step_noalloc(cfg, P, [t] * B, kc, vc, qn, kn, vn, got, device_error=err)
        torch.cuda.synchronize()
        want = model.step(0, f64(qn), f64(kn), f64(vn), w.scale)
        diff_oracle = float(np.max(np.abs(f64(got) - want)))
        assert diff_oracle <= tol, (t, diff_oracle)
        diff_ws = (got.double() - ref.double()).abs().max().item()
        assert diff_ws <= tol, (t, diff_ws)
        for b in range(B):
            ok, ov, held = model.rings[0][b].snapshot()
            assert held == P[b] + min(t + 1, W)
            for h in range(H):
                gk = f64(_ring_view(kc, P, W, H, d, b, h)[:held])
                gv = f64(_ring_view(vc, P, W, H, d, b, h)[:held])
                assert np.array_equal(gk, ok[:held, h]), (t, b, h)
                assert np.array_equal(gv, ov[:held, h]), (t, b, h)
        # and bit for bit the same cache as the workspace path
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
