"""Standard sliding-window mode (rswa_state_set_attention) against the FP64
oracle: the contrast the pages draw in "开源5天Star破万之后：百度Unlimited-OCR
的爆火路径复盘" §2.1 -- a standard window also cuts the prompt.

Prompt query i attends to keys (i - W, i]; generated token t (position
P + t) to positions (P + t - W, P + t], taken here by brute force from the
token history (not from any cache).  The ring writes are the same as in
R-SWA mode, so the caches still match the ring oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("split", ["auto", "streamk"])
@pytest.mark.parametrize("W", [8, 130])
def test_standard_swa_prefill_and_decode(dtype, d, split, W, monkeypatch):
    from ring_sliding_window_b200 import rswa
    if split != "auto":
        monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    B, L, H, P, steps = 2, 2, 2, (200, 37), 20 if W == 8 else 140
    w = synth.Workload("swa", 71 + W, dtype, B, L, H, d, W, P, steps)
    st = rswa.State(B, L, H, d, W, P, dtype=dtype)
    st.set_attention(rswa.RSWA_ATTN_STANDARD_SWA)
    grid, csize = st.decode_launch_shape()
    assert (csize == 0) == (split == "streamk")
    tol = tol_for(dtype)
    sl = seq_slices(P)
    model = oracle.RingModel(P, W, L, H, d)
    hist_k = [[None] * B for _ in range(L)]
    hist_v = [[None] * B for _ in range(L)]
    for l in range(L):
        q, k, v = synth.prefill_qkv(w, l, "cuda")
        out = torch.empty_like(q)
        st.prefill(l, q, k, v, out)
        for b in range(B):
            ref = oracle.prefill_window(f64(q[sl[b]]), f64(k[sl[b]]), f64(v[sl[b]]), w.scale, W)
            assert np.max(np.abs(f64(out[sl[b]]) - ref)) <= tol, (l, b)
            hist_k[l][b], hist_v[l][b] = list(f64(k[sl[b]])), list(f64(v[sl[b]]))
            model.prefill(l, b, f64(k[sl[b]]), f64(v[sl[b]]))
    for t in range(steps):
        for l in range(L):
            q, kn, vn = synth.decode_qkv(w, l, t, "cuda")
            out = torch.empty_like(q)
            st.decode_step(l, q, kn, vn, out)
            for b in range(B):
                model.rings[l][b].step(f64(q[b]), f64(kn[b]), f64(vn[b]), w.scale)
                hist_k[l][b].append(f64(kn[b]))
                hist_v[l][b].append(f64(vn[b]))
                K = np.stack(hist_k[l][b][-W:])  # the last W positions, this token included
                V = np.stack(hist_v[l][b][-W:])
                for h in range(H):
                    ref = oracle.attend(f64(q[b, h]), K[:, h], V[:, h], w.scale)
                    err = np.max(np.abs(f64(out[b, h]) - ref))
                    assert err <= tol, (t, l, b, h, err)
        st.advance()
    for l in range(L):
        for b in range(B):
            kc, vc, held = model.rings[l][b].snapshot()
            for h in range(H):
                assert np.array_equal(f64(st.cache_view(l, "k", b, h)[:held]), kc[:held, h])
                assert np.array_equal(f64(st.cache_view(l, "v", b, h)[:held]), vc[:held, h])
    assert st.check() == 0


@pytest.mark.slow
@pytest.mark.parametrize("W", [128, 300])
def test_standard_swa_long_prompt_sampled_rows(W):
    """An 8,256-token prompt (the multi-page length) in standard-SWA mode:
    every query tile reads only the key tiles of its window.  Sampled rows at
    tile and window boundaries against the windowed attention of the oracle."""
    from ring_sliding_window_b200 import rswa
    B, L, H, d = 1, 1, 2, 128
    P = (8256,)
    w = synth.Workload("swa_long", 75, torch.bfloat16, B, L, H, d, W, P, 0)
    st = rswa.State(B, L, H, d, W, P, dtype=torch.bfloat16)
    st.set_attention(rswa.RSWA_ATTN_STANDARD_SWA)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    qq, kk, vv, oo = f64(q), f64(k), f64(v), f64(out)
    for i in (0, 1, 127, 128, W - 1, W, 255, 256, 300, 4000, 8063, 8064, 8191, 8192, 8255):
        lo = max(0, i - W + 1)
        for h in range(H):
            ref = oracle.attend(qq[i, h], kk[lo:i + 1, h], vv[lo:i + 1, h], w.scale)
            assert np.max(np.abs(oo[i, h] - ref)) <= tol_for(torch.bfloat16), (i, h)
    assert st.check() == 0


def test_attention_mode_switch_and_errors():
    from ring_sliding_window_b200 import rswa
    st = rswa.State(1, 1, 2, 128, 8, [64], dtype=torch.bfloat16)
    for bad in (2, -1):
        with pytest.raises(rswa.RswaError) as e:
            st.set_attention(bad)
        assert e.value.status == rswa.RSWA_EINVAL
    ring_shape = st.decode_launch_shape()
    st.set_attention(rswa.RSWA_ATTN_STANDARD_SWA)
    assert st.decode_launch_shape()[1] == 1  # ceil(8 / 64) CTAs per ring
    st.set_attention(rswa.RSWA_ATTN_RING)
    assert st.decode_launch_shape() == ring_shape


@pytest.mark.parametrize("policy", [1, 2])
def test_standard_swa_with_rope(policy):
    """The two options compose: rotated keys in the cache, a window over them."""
    from ring_sliding_window_b200 import rswa
    dtype, d, B, H, W, P, steps, theta = torch.bfloat16, 128, 2, 2, 8, (200, 37), 14, 10000.0
    w = synth.Workload("swa_rope", 91 + policy, dtype, B, 1, H, d, W, P, steps)
    st = rswa.State(B, 1, H, d, W, P, dtype=dtype)
    st.set_attention(rswa.RSWA_ATTN_STANDARD_SWA)
    st.set_rope(policy, theta)
    pol = "absolute" if policy == 1 else "slot"
    tol = tol_for(dtype)
    sl = seq_slices(P)
    q, k, v = synth.prefill_qkv(w, 0, "cuda")
    out = torch.empty_like(q)
    st.prefill(0, q, k, v, out)
    hk, hv = [], []
    for b in range(B):
        pos = np.arange(P[b])
        qr, kr = oracle.rope(f64(q[sl[b]]), pos, theta), oracle.rope(f64(k[sl[b]]), pos, theta)
        ref = oracle.prefill_window(qr, kr, f64(v[sl[b]]), w.scale, W)
        assert np.max(np.abs(f64(out[sl[b]]) - ref)) <= tol, b
        hk.append(list(kr))
        hv.append(list(f64(v[sl[b]])))
    for t in range(steps):
        qs, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
        o = torch.empty_like(qs)
        st.decode_step(0, qs, kn, vn, o)
        for b in range(B):
            p = [oracle.rope_position(pol, P[b], t, W)]
            hk[b].append(oracle.rope(f64(kn[b])[None], p, theta)[0])
            hv[b].append(f64(vn[b]))
            K, V = np.stack(hk[b][-W:]), np.stack(hv[b][-W:])
            qr = oracle.rope(f64(qs[b])[None], p, theta)[0]
            for h in range(H):
                ref = oracle.attend(qr[h], K[:, h], V[:, h], w.scale)
                assert np.max(np.abs(f64(o[b, h]) - ref)) <= tol, (t, b, h)
        st.advance()
    assert st.check() == 0
