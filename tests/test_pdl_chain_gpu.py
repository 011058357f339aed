"""Layers chained through their outputs under programmatic dependent launch.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.1 (each layer's
decode step attends to its own cache).  A model feeds layer l's attention
output (through its projections) into layer l+1; here layer l's output
buffer is layer l+1's q directly.  The decode kernel lets the next one start
early and pulls that row toward L2 before its grid-dependency wait, so this
is the case where a kernel reads what the kernel right before it wrote.
The output buffers are filled with NaN before every replay: a read ahead of
the write would surface as NaN.

The oracle chains its own outputs (layer l+1's query is the oracle's layer-l
output), so the GPU's layer l+1 sees a query that differs from the oracle's
by layer l's rounding; the bound below adds that propagated difference.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, seq_slices, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("split", ["cluster", "streamk"])
def test_layers_chained_through_outputs_in_a_graph(split, monkeypatch):
    from ring_sliding_window_b200 import rswa
    monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    lens, L, H, d, W, steps = [300, 40], 3, 2, 128, 8, 12
    B = len(lens)
    dtype = torch.bfloat16
    scale = 1.0 / np.sqrt(d)
    st = rswa.State(B, L, H, d, W, lens, dtype=dtype)
    rings = [[oracle.Ring(P, W, H, d) for P in lens] for _ in range(L)]
    tot = sum(lens)
    for l in range(L):
        q, k, v = (synth.normal((tot, H, d), synth.seed(71, l, i), dtype, "cuda") for i in range(3))
        st.prefill(l, q, k, v, torch.empty_like(q))
        for b, sl in enumerate(seq_slices(lens)):
            rings[l][b].prefill(f64(k[sl]), f64(v[sl]))
    # inputs of the graph: layer 0's q and every layer's k_new / v_new
    q0 = torch.empty(B, H, d, dtype=dtype, device="cuda")
    kn = torch.empty(L, B, H, d, dtype=dtype, device="cuda")
    vn = torch.empty_like(kn)
    outs = torch.empty(L, B, H, d, dtype=dtype, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for l in range(L):
            st.decode_step(l, q0 if l == 0 else outs[l - 1], kn[l], vn[l], outs[l], stream=s)
        st.advance(stream=s)
    torch.cuda.synchronize()
    for t in range(steps):
        q0.copy_(synth.normal((B, H, d), synth.seed(72, 0, t), dtype, "cuda"))
        for l in range(L):
            kn[l].copy_(synth.normal((B, H, d), synth.seed(73, l, t), dtype, "cuda"))
            vn[l].copy_(synth.normal((B, H, d), synth.seed(74, l, t), dtype, "cuda"))
        outs.fill_(float("nan"))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = f64(outs)
        assert np.isfinite(got).all(), t
        for b in range(B):
            q_or = f64(q0[b])
            err_prev = 0.0
            for l in range(L):
                ref, _, _ = rings[l][b].step(q_or, f64(kn[l, b]), f64(vn[l, b]), scale)
                err = np.max(np.abs(got[l, b] - ref))
                # the query differs from the oracle's by the previous layer's
                # error; a softmax average moves by at most
                # 2 max|v| |dq| sum|k| scale for a query change dq
                kk, vv, held = rings[l][b].snapshot()
                kmax = np.max(np.sum(np.abs(kk[:held]), axis=-1))
                vmax = np.max(np.abs(vv[:held]))
                bound = tol_for(dtype) + 2.0 * vmax * err_prev * kmax * scale
                assert err <= bound, (t, b, l, err, bound)
                err_prev = err
                q_or = ref
    assert st.check() == 0
    del g
    st.close()
