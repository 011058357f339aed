"""Continuous batching over a token pool, against the FP64 oracle.

Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §三 (serving
with a page size of one token) and §2.1 (each request's cache is its
prefill plus a ring of W generated tokens, P + W slots for its whole life).
Requests are independent, so the oracle is one ring per (request, layer).

A schedule of joins and leaves runs on one pool whose capacity forces the
allocator to reuse freed ranges: a joining request lands on slots that held
another request's keys, and its prefill must overwrite them.  After every
step: outputs within tolerance of the oracle, each live request's cache
bit-exact against its oracle ring at the pool location the allocator gave it,
and the ring counters equal to the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f64, tol_for
from ring_sliding_window_b200 import synth

pytestmark = pytest.mark.gpu

# step -> (requests leaving, requests joining as (id, prefill_len))
SCHEDULE = {
    0: ([], [("A", 100), ("B", 37), ("C", 1)]),
    4: (["A"], [("D", 60), ("E", 30)]),
    9: (["C", "B"], [("F", 120)]),
    12: (["E"], [("G", 0)]),
}
STEPS = 16
CAPACITY = 240
IDS = {name: i for i, name in enumerate("ABCDEFG")}


def _seed(req, layer, step, what):
    return synth.seed(40 + IDS[req], layer, 3 * step + what)


@pytest.mark.parametrize("dtype,d,split", [(torch.bfloat16, 128, "streamk"),
                                           (torch.bfloat16, 128, "cluster"),
                                           (torch.float32, 64, "auto")])
def test_continuous_batching_vs_oracle(dtype, d, split, monkeypatch):
    from ring_sliding_window_b200 import rswa
    if split != "auto":
        monkeypatch.setenv("RSWA_DECODE_SPLIT", split)
    L, H, W = 2, 2, 8
    scale = 1.0 / np.sqrt(d)
    pool = rswa.TokenPool(CAPACITY, L, H, d, W, dtype=dtype)
    live = []  # dicts: id, P, base, t, rings[layer]
    expect_base = {}
    st = None
    tol = tol_for(dtype)
    for step in range(STEPS):
        leaving, joining = SCHEDULE.get(step, ([], []))
        if leaving or joining:
            if st is not None:
                n, _, _ = st.ring()
                assert n == [r["t"] for r in live]
                st.close()
                st = None
            for name in leaving:
                r = next(r for r in live if r["id"] == name)
                pool.free(r["base"])
                live.remove(r)
            new = []
            for name, P in joining:
                base = pool.alloc(P)
                new.append({"id": name, "P": P, "base": base, "t": 0,
                            "rings": [oracle.Ring(P, W, H, d) for _ in range(L)]})
                expect_base[name] = base
            # the joining requests' prompts, through a state over them alone
            pst = pool.state([r["P"] for r in new], [r["base"] for r in new])
            for l in range(L):
                ks, vs, qs = [], [], []
                for r in new:
                    k = synth.normal((r["P"], H, d), _seed(r["id"], l, 10_000, 0), dtype, "cuda")
                    v = synth.normal((r["P"], H, d), _seed(r["id"], l, 10_000, 1), dtype, "cuda")
                    ks.append(k)
                    vs.append(v)
                    qs.append(torch.zeros_like(k))
                    r["rings"][l].prefill(f64(k), f64(v))
                q, k, v = torch.cat(qs), torch.cat(ks), torch.cat(vs)
                pst.prefill(l, q, k, v, torch.empty_like(q))
            pst.close()
            live.extend(new)
            st = pool.state([r["P"] for r in live], [r["base"] for r in live],
                            n_generated=[r["t"] for r in live])
        for l in range(L):
            q, kn, vn = (torch.stack([synth.normal((H, d), _seed(r["id"], l, step, i), dtype, "cuda")
                                      for r in live]) for i in range(3))
            out = torch.empty_like(q)
            st.decode_step(l, q, kn, vn, out)
            for b, r in enumerate(live):
                ref, _, _ = r["rings"][l].step(f64(q[b]), f64(kn[b]), f64(vn[b]), scale)
                err = np.max(np.abs(f64(out[b]) - ref))
                assert err <= tol, (step, l, r["id"], err)
        st.advance()
        for r in live:
            r["t"] += 1
        n, rp, cl = st.ring()
        for b, r in enumerate(live):
            ring = r["rings"][0]
            assert n[b] == r["t"] and rp[b] == ring.ring_pos and cl[b] == ring.length
            for l in range(L):
                kc, vc, held = r["rings"][l].snapshot()
                for h in range(H):
                    assert np.array_equal(f64(st.cache_view(l, "k", b, h)[:held]), kc[:held, h])
                    assert np.array_equal(f64(st.cache_view(l, "v", b, h)[:held]), vc[:held, h])
    assert st.check() == 0
    st.close()
    # first fit: D reuses A's range, F lands on the merged hole B and C left
    assert expect_base["A"] == 0 and expect_base["D"] == 0
    assert expect_base["E"] == 68 and expect_base["F"] == 106
    pool.close()


@pytest.mark.slow
def test_continuous_batching_serving_sizes():
    """Ragged-serving sizes on one pool: 8 requests with prompts of 1,024 to
    16,384 tokens, W = 128, 10 heads x 128; 2 leave and 2 join at step 60 (the
    joiners land in freed ranges) and again at step 133, after the first
    requests' rings have wrapped.  Every step's outputs against the oracle;
    every live cache bit-exact at the end."""
    from ring_sliding_window_b200 import rswa
    L, H, d, W, steps = 1, 10, 128, 128, 140
    dtype = torch.bfloat16
    scale = 1.0 / np.sqrt(d)
    rng = np.random.default_rng(7)
    plen = {i: int(rng.integers(1024, 16385)) for i in range(12)}
    schedule = {0: ([], list(range(8))), 60: ([1, 5], [8, 9]), 133: ([0, 8], [10, 11])}
    capacity = int(1.25 * sum(plen[i] + W for i in range(8))) + 2 * (16384 + W)
    pool = rswa.TokenPool(capacity, L, H, d, W, dtype=dtype)
    seed = lambda req, step, what: synth.seed(90 + req, 0, 3 * step + what)  # noqa: E731
    live, st = [], None
    for step in range(steps):
        leaving, joining = schedule.get(step, ([], []))
        if leaving or joining:
            if st is not None:
                st.close()
            for rid in leaving:
                r = next(r for r in live if r["id"] == rid)
                pool.free(r["base"])
                live.remove(r)
            new = []
            for rid in joining:
                P = plen[rid]
                new.append({"id": rid, "P": P, "base": pool.alloc(P), "t": 0,
                            "ring": oracle.Ring(P, W, H, d)})
            pst = pool.state([r["P"] for r in new], [r["base"] for r in new])
            ks, vs = [], []
            for r in new:
                ks.append(synth.normal((r["P"], H, d), seed(r["id"], 10_000, 0), dtype, "cuda"))
                vs.append(synth.normal((r["P"], H, d), seed(r["id"], 10_000, 1), dtype, "cuda"))
                r["ring"].prefill(f64(ks[-1]), f64(vs[-1]))
            k, v = torch.cat(ks), torch.cat(vs)
            pst.prefill(0, torch.zeros_like(k), k, v, torch.empty_like(k))
            pst.close()
            del k, v, ks, vs
            live.extend(new)
            st = pool.state([r["P"] for r in live], [r["base"] for r in live],
                            n_generated=[r["t"] for r in live])
        q, kn, vn = (torch.stack([synth.normal((H, d), seed(r["id"], step, i), dtype, "cuda")
                                  for r in live]) for i in range(3))
        out = torch.empty_like(q)
        st.decode_step(0, q, kn, vn, out)
        for b, r in enumerate(live):
            ref, _, _ = r["ring"].step(f64(q[b]), f64(kn[b]), f64(vn[b]), scale)
            assert np.max(np.abs(f64(out[b]) - ref)) <= tol_for(dtype), (step, r["id"])
        st.advance()
        for r in live:
            r["t"] += 1
    n, _, _ = st.ring()
    assert n == [r["t"] for r in live]
    for b, r in enumerate(live):
        kc, vc, held = r["ring"].snapshot()
        for h in range(H):
            assert np.array_equal(f64(st.cache_view(0, "k", b, h)[:held]), kc[:held, h])
            assert np.array_equal(f64(st.cache_view(0, "v", b, h)[:held]), vc[:held, h])
    assert st.check() == 0
    st.close()
    pool.close()
