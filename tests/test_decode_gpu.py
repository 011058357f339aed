"""Decode-step parity: the CUDA path (through the C ABI) against the FP64 oracle.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.1 -- each
generated token's K/V lands in slot prefill_len + ring_pos (append during
warm-up, overwrite in steady state) and the token attends to the whole cache.
Ring indices and cache contents must match bit for bit; attention outputs
within 1e-5 (fp32 inputs) or 2e-2 (bf16 inputs) max-abs.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import StepInputs, f64, seq_slices, tol_for, union_expect
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu


def _state(w, n_generated=None):
    from ring_sliding_window_b200 import rswa
    return rswa.State(w.batch, w.layers, w.heads, w.head_dim, w.window, w.prefill_lens,
                      dtype=w.dtype, n_generated=n_generated)


def _prefill_all(st, w):
    outs, ins = [], []
    for l in range(w.layers):
        q, k, v = synth.prefill_qkv(w, l, "cuda")
        out = torch.empty_like(q)
        st.prefill(l, q, k, v, out)
        outs.append(out)
        ins.append((q, k, v))
    return ins, outs


def _small(name, dtype, batch, layers, heads, d, window, plens, steps, cfg_id):
    return synth.Workload(name, cfg_id, dtype, batch, layers, heads, d, window, tuple(plens), steps)


# ------------------------------------------------------------------ full runs
FULL_RUN_CASES = [
    synth.workload("tiny_ring_fp32"),
    _small("ragged_bf16_d128", torch.bfloat16, 3, 2, 2, 128, 8, (100, 37, 1), 30, 11),
    _small("ragged_fp32_d128", torch.float32, 2, 1, 3, 128, 5, (70, 0), 17, 12),
    _small("bf16_d64_W1", torch.bfloat16, 2, 1, 2, 64, 1, (65, 3), 6, 13),
    _small("bf16_long_tail", torch.bfloat16, 1, 1, 1, 128, 16, (1000,), 40, 14),
]


@pytest.mark.parametrize("split", ["streamk", "cluster"])
@pytest.mark.parametrize("w", FULL_RUN_CASES, ids=lambda w: w.name)
def test_decode_full_run_vs_oracle_ring(w, split, monkeypatch):
    """Every step of the run against the oracle's three-phase ring simulation;
    ring counters and cache contents bit-exact after every step.  Both decode
    splits run: stream-K ranges merged through the workspace, and one cluster
    per ring merged through distributed shared memory."""
    monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    st = _state(w)
    grid, csize = st.decode_launch_shape()
    if split == "streamk":
        assert csize == 0
    else:
        assert csize >= 2 and grid == w.batch * w.heads * csize
    ins, _ = _prefill_all(st, w)
    sl = seq_slices(w.prefill_lens)
    model = oracle.RingModel(w.prefill_lens, w.window, w.layers, w.heads, w.head_dim)
    for l in range(w.layers):
        _, k, v = ins[l]
        for b in range(w.batch):
            model.prefill(l, b, f64(k[sl[b]]), f64(v[sl[b]]))
    tol = tol_for(w.dtype)
    for t in range(w.decode_steps):
        for l in range(w.layers):
            q, kn, vn = synth.decode_qkv(w, l, t, "cuda")
            out = torch.empty_like(q)
            st.decode_step(l, q, kn, vn, out)
            ref = model.step(l, f64(q), f64(kn), f64(vn), w.scale)
            err = np.max(np.abs(f64(out) - ref))
            assert err <= tol, (t, l, err)
        st.advance()
        n, rp, cl = st.ring()
        for b in range(w.batch):
            rg = model.rings[0][b]
            assert n[b] == t + 1
            assert rp[b] == rg.ring_pos, (t, b)
            assert cl[b] == rg.length == w.prefill_lens[b] + min(t + 1, w.window)
        # cache contents bit-exact against the oracle's cache
        for l in range(w.layers):
            for b in range(w.batch):
                kc, vc, held = model.rings[l][b].snapshot()
                for h in range(w.heads):
                    gk = f64(st.cache_view(l, "k", b, h)[:held])
                    gv = f64(st.cache_view(l, "v", b, h)[:held])
                    assert np.array_equal(gk, kc[:held, h]), (t, l, b, h)
                    assert np.array_equal(gv, vc[:held, h]), (t, l, b, h)
    assert st.check() == 0


# --------------------------------------------------- full-size sampled checks
def _sampled_decode(w, steps, check_steps, heads_to_check, layers_to_check, seqs_to_check):
    st = _state(w)
    ins, _ = _prefill_all(st, w)
    sl = seq_slices(w.prefill_lens)
    inputs = StepInputs(w, steps)
    outs = {}
    for t in range(steps):
        for l in range(w.layers):
            q, kn, vn = inputs.get(t, l)
            out = torch.empty_like(q)
            st.decode_step(l, q, kn, vn, out)
            if t in check_steps and l in layers_to_check:
                outs[(t, l)] = out
        st.advance()
    torch.cuda.synchronize()
    assert st.check() == 0
    tol = tol_for(w.dtype)
    worst = 0.0
    for (t, l), out in outs.items():
        _, k, v = ins[l]
        for b in seqs_to_check:
            for h in heads_to_check:
                pk, pv = f64(k[sl[b], h]), f64(v[sl[b], h])
                gen_k = {s: f64(inputs.get(s, l)[1][b, h]) for s in range(max(0, t - w.window + 1), t + 1)}
                gen_v = {s: f64(inputs.get(s, l)[2][b, h]) for s in gen_k}
                q = f64(inputs.get(t, l)[0][b, h])
                ref = union_expect(pk, pv, gen_k, gen_v, q, t, w.window, w.scale)
                err = np.max(np.abs(f64(out[b, h]) - ref))
                worst = max(worst, err)
                assert err <= tol, (t, l, b, h, err)
    n, rp, cl = st.ring()
    assert all(x == steps for x in n)
    assert all(c == p + w.window for c, p in zip(cl, w.prefill_lens)) or steps < w.window
    return worst


@pytest.mark.slow
def test_decode_single_page_full_run():
    """Single-page workload at full size: all 4,096 steps x 12 layers run; sampled
    steps across warm-up, the first wrap and the end are checked."""
    w = synth.workload("single_page_decode")
    W = w.window
    checks = {0, 1, W - 2, W - 1, W, W + 1, 2 * W, 3 * W + 7, w.decode_steps - 1}
    _sampled_decode(w, w.decode_steps, checks, heads_to_check=[0, 3, 9],
                    layers_to_check={0, 5, 11}, seqs_to_check=[0])


@pytest.mark.slow
@pytest.mark.parametrize("name", ["multi_page_decode", "near_max_context"])
def test_decode_large_sampled(name):
    """Full-size caches (P = 8,256 or 32,640); 2W + 3 steps cover warm-up and
    two wraps (the kernel's work does not change after the first wrap)."""
    w = synth.workload(name)
    W = w.window
    steps = 2 * W + 3
    checks = {0, W - 1, W, 2 * W + 2}
    _sampled_decode(w, steps, checks, heads_to_check=[0, 9], layers_to_check={0, 11},
                    seqs_to_check=[0, w.batch - 1])


@pytest.mark.slow
def test_decode_ragged_serving_snapshot():
    """64 requests, P_b in [1024, 16384], ring fill f_b in [0, 128]: the caches are
    written directly by torch (a resumed batch), then one step runs on all 12
    layers.  Oracle keys: slots [0, P_b + min(f_b + 1, W)) of the cache as
    written, with slot P_b + (f_b mod W) replaced by this step's k_new/v_new."""
    w = synth.workload("ragged_serving")
    st = _state(w, n_generated=list(w.n_generated))
    for l in range(w.layers):
        st.k_cache[l].copy_(synth.normal(st.k_cache[l].shape, synth.seed(5, l, 500_000), w.dtype, "cuda"))
        st.v_cache[l].copy_(synth.normal(st.v_cache[l].shape, synth.seed(5, l, 600_000), w.dtype, "cuda"))
    layers = [0, 7, 11]
    before = {}
    for l in layers:
        for b in (0, 17, 31, 63):
            for h in (0, 9):
                before[(l, b, h)] = (f64(st.cache_view(l, "k", b, h)), f64(st.cache_view(l, "v", b, h)))
    outs = {}
    qkv = {}
    for l in range(w.layers):
        q, kn, vn = synth.decode_qkv(w, l, 0, "cuda")
        out = torch.empty_like(q)
        st.decode_step(l, q, kn, vn, out)
        outs[l], qkv[l] = out, (q, kn, vn)
    st.advance()
    torch.cuda.synchronize()
    assert st.check() == 0
    for (l, b, h), (kc, vc) in before.items():
        P, f = w.prefill_lens[b], w.n_generated[b]
        slot = P + f % w.window
        n = P + min(f + 1, w.window)
        kk, vv = kc[:n].copy(), vc[:n].copy()
        q, kn, vn = qkv[l]
        kk[slot], vv[slot] = f64(kn[b, h]), f64(vn[b, h])
        ref = oracle.attend(f64(q[b, h]), kk, vv, w.scale)
        assert np.max(np.abs(f64(outs[l][b, h]) - ref)) <= tol_for(w.dtype), (l, b, h)
        # the ring write landed, bit-exact, and nothing else in the ring moved
        gk = f64(st.cache_view(l, "k", b, h))
        assert np.array_equal(gk[slot], f64(kn[b, h]))
        assert np.array_equal(np.delete(gk, slot, axis=0), np.delete(kc, slot, axis=0))
    n, rp, cl = st.ring()
    assert n == [f + 1 for f in w.n_generated]


# ------------------------------------------------------------ graph capture
def test_decode_step_graph_capture_matches_eager():
    """A whole token (all layers + advance) captured once and replayed gives the
    same outputs as eager calls, because the ring counters live on the device."""
    w = _small("graph_case", torch.bfloat16, 2, 3, 2, 128, 8, (300, 130), 20, 15)
    outs_e, outs_g = [], []
    for mode in ("eager", "graph"):
        st = _state(w)
        _prefill_all(st, w)
        q = [torch.empty(w.batch, w.heads, w.head_dim, dtype=w.dtype, device="cuda") for _ in range(w.layers)]
        kn = [torch.empty_like(x) for x in q]
        vn = [torch.empty_like(x) for x in q]
        out = [torch.empty_like(x) for x in q]
        s = torch.cuda.Stream()

        def token():
            for l in range(w.layers):
                st.decode_step(l, q[l], kn[l], vn[l], out[l], stream=s)
            st.advance(stream=s)

        graph = None
        if mode == "graph":
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=s):
                token()
        res = []
        for t in range(w.decode_steps):
            for l in range(w.layers):
                a, b_, c = synth.decode_qkv(w, l, t, "cuda")
                q[l].copy_(a); kn[l].copy_(b_); vn[l].copy_(c)
            torch.cuda.synchronize()
            if graph is None:
                token()
            else:
                graph.replay()
            s.synchronize()
            res.append(torch.stack([o.clone() for o in out]))
        (outs_e if mode == "eager" else outs_g).append(torch.stack(res))
        assert st.check() == 0
    assert torch.equal(outs_e[0], outs_g[0])


def test_reset_ring_restarts_generation():
    w = _small("reset_case", torch.bfloat16, 1, 1, 2, 128, 4, (50,), 6, 16)
    st = _state(w)
    _prefill_all(st, w)
    runs = []
    for _ in range(2):
        outs = []
        for t in range(w.decode_steps):
            q, kn, vn = synth.decode_qkv(w, 0, t, "cuda")
            out = torch.empty_like(q)
            st.decode_step(0, q, kn, vn, out)
            st.advance()
            outs.append(out)
        runs.append(torch.stack(outs))
        st.reset_ring()
        assert st.ring()[0] == [0]
    assert torch.equal(runs[0], runs[1])
