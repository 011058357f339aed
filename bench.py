#!/usr/bin/env python
"""R-SWA decode benchmark on B200: decode steps/s, KV-read GB/s vs HBM, prefill TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--also NAMES|none] [--cpu-seconds S]

A timed step is one generated token of the whole batch: for every layer the
fused ring write + split-K attention + combine (rswa_decode_step), then the
ring advance and the windowed n-gram ban over the batch's logits -- one CUDA
graph replay.  The prefill (cache fill + causal attention) is a once-per-batch
phase; it is timed in the same run and reported under "prefill".

Timing: CUDA events on the launching stream, L2 flushed (256 MiB write)
before every timed step, outside the events; with N > 1 GPUs every rank runs
its own replica of the workload (weak scaling) and the time is the max over
ranks.  rank 0 prints one JSON line.

--impl reference times the FP64 CPU oracle (the only other implementation of
the method: the pages publish no code) on the host cores, on a bounded
sample of the same workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from ring_sliding_window_b200 import synth  # noqa: E402

METRIC = "R-SWA decode steps/s and KV-read GB/s vs HBM peak; prefill TFLOP/s (1xB200)"
UNIT = "decode steps/s"
DATASHEET_HBM_GBS = 8000.0
L2_BYTES = 126e6  # B200 L2 (nominal)
DATASHEET_BF16_TFLOPS = 2250.0
FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"unavailable": "nvidia-smi not runnable"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"unavailable": "no samples"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# the decode kernel's device code (the host-side headers change for unrelated
# reasons; a change to the kernel itself or its PTX helpers voids the record)
DECODE_KERNEL_SOURCES = ("decode.cu", "ptx.cuh")


def kernel_source_hash(files=DECODE_KERNEL_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "ring_sliding_window_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes per decode-kernel launch from the committed ncu record, or
    None when the kernel sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "decode_split_kernel_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_sha256") != kernel_source_hash() or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


def max_over_ranks(x: float) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return float(x)


def aggregate_rate(steps_per_rank: int, max_total_ms: float, world: int) -> float:
    """Whole-job rate: every rank ran `steps_per_rank` steps of its own replica
    (weak scaling); the job took as long as its slowest rank."""
    return world * steps_per_rank / (max_total_ms / 1e3)


def kv_bytes_per_layer(w: synth.Workload, t_list):
    """Algorithmic bytes of one rswa_decode_step (one layer): K and V rows of
    every valid slot, q, k_new/v_new read, ring write, output write."""
    e = w.elem_bytes
    row = w.heads * w.head_dim * e
    total = 0
    for b, P in enumerate(w.prefill_lens):
        t = t_list[b]
        total += 2 * (P + min(t + 1, w.window)) * row + row + 2 * row + 2 * row + row
    return total


def prefill_flops_per_layer(w: synth.Workload):
    return sum(4 * w.heads * w.head_dim * P * (P + 1) // 2 for P in w.prefill_lens)


# --------------------------------------------------------------------------
class DecodeRig:
    """State, graph-captured token step and its I/O buffers for one workload."""

    def __init__(self, w: synth.Workload, start_t: int, fill: str, stream: torch.cuda.Stream,
                 rope: int = 0):
        from ring_sliding_window_b200 import rswa
        self.w, self.s = w, stream
        L, B, H, d = w.layers, w.batch, w.heads, w.head_dim
        ng = None if fill == "prefill" else [start_t] * B
        if w.n_generated is not None and fill != "prefill":
            ng = list(w.n_generated)
        self.st = rswa.State(B, L, H, d, w.window, w.prefill_lens, dtype=w.dtype, n_generated=ng)
        if rope:
            self.st.set_rope(rope, 10000.0, stream=stream)
        # q, k_new, v_new of all layers in one buffer: one host copy per step
        self.qkv = torch.empty(3, L, B, H, d, dtype=w.dtype, device="cuda")
        self.q, self.kn, self.vn = self.qkv[0], self.qkv[1], self.qkv[2]
        self.out = torch.empty_like(self.q)
        for l in range(L):
            a, b_, c = synth.decode_qkv(w, l, 0, "cuda")
            self.q[l].copy_(a)
            self.kn[l].copy_(b_)
            self.vn[l].copy_(c)
        rows = B
        logits, hist, _ = synth.ngram_inputs(rows, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW,
                                             synth.seed(w.cfg_id, 0, 800_000))
        self.logits = logits.cuda()
        self.hist = hist.cuda()
        self.prefill_ms = None
        if fill == "random":
            for l in range(L):
                g = torch.Generator(device="cuda").manual_seed(synth.seed(w.cfg_id, l, 900_000))
                self.st.k_cache[l].normal_(generator=g)
                self.st.v_cache[l].normal_(generator=g)
        self.graph = None

    def prefill_all(self, flush, time_it=True):
        """Run rswa_prefill on every layer (this fills the caches); then time
        each layer's call replayed from a CUDA graph after an L2 flush, so the
        host side of the call (argument checks, tensor-map encoding, Python
        marshalling) stays outside the events and the inputs are cold.
        Returns per-layer event times (ms)."""
        w = self.w
        q, k, v = synth.prefill_qkv(w, 0, "cuda")
        out = torch.empty_like(q)
        with torch.cuda.stream(self.s):
            for l in range(w.layers):
                self.st.prefill(l, q, k, v, out, stream=self.s)
        self.s.synchronize()
        if not time_it:
            return []
        graphs = []
        for l in range(w.layers):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.s):
                self.st.prefill(l, q, k, v, out, stream=self.s)
            graphs.append(g)
        times = []
        with torch.cuda.stream(self.s):
            for g in graphs:
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(self.s)
                g.replay()
                e1.record(self.s)
                times.append((e0, e1))
        self.s.synchronize()
        res = [a.elapsed_time(b) for a, b in times]
        del graphs
        return res

    def token(self):
        from ring_sliding_window_b200 import rswa
        w = self.w
        for l in range(w.layers):
            self.st.decode_step(l, self.q[l], self.kn[l], self.vn[l], self.out[l], stream=self.s)
        self.st.advance(stream=self.s)
        rswa.rswa_ngram_mask(self.logits, self.hist, None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW,
                             stream=self.s)

    def capture(self):
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.s):
            self.token()
        # the same token without the n-gram ban, for the end-to-end run (the
        # ban waits there for the logits copied in meanwhile)
        self.graph_dec = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_dec, stream=self.s):
            for l in range(self.w.layers):
                self.st.decode_step(l, self.q[l], self.kn[l], self.vn[l], self.out[l], stream=self.s)
            self.st.advance(stream=self.s)
        torch.cuda.synchronize()

    def launches_per_token(self):
        return self.w.layers + 2  # one decode kernel per layer, advance, n-gram mask

    def ring_t(self):
        n, _, _ = self.st.ring(stream=self.s)
        return n


def _barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()


def timed_tokens(rig: DecodeRig, steps: int, warmup: int, flush, sampler=None):
    """Replay the token graph; returns (per-step ms list, per-step t lists)."""
    s = rig.s
    with torch.cuda.stream(s):
        for _ in range(warmup):
            flush.zero_()
            rig.graph.replay()
    s.synchronize()
    t0 = rig.ring_t()
    _barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    if sampler:
        sampler.start()
    with torch.cuda.stream(s):
        for i in range(steps):
            flush.zero_()
            evs[i][0].record(s)
            rig.graph.replay()
            evs[i][1].record(s)
    s.synchronize()
    _barrier()
    clocks = sampler.stop() if sampler else None
    ms = [a.elapsed_time(b) for a, b in evs]
    ts = [[t + i for t in t0] for i in range(steps)]
    return ms, ts, clocks


def fill_ring(rig: DecodeRig):
    """Replay the token graph until every ring holds W generated entries (the
    method's warm-up phase); untimed."""
    need = rig.w.window - min(rig.ring_t())
    with torch.cuda.stream(rig.s):
        for _ in range(max(0, need)):
            rig.graph.replay()
    rig.s.synchronize()


def timed_decode_launches(rig: DecodeRig, reps: int, flush):
    """Average duration of one decode_split_kernel launch (one rswa_decode_step)
    in the bench's launch configuration: a CUDA graph of the layers' decode
    steps only (no advance, so every replay sees the same ring position),
    replayed after an L2 flush and bracketed by events on the stream; the
    replay time divided by the layer count."""
    w, s = rig.w, rig.s
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for l in range(w.layers):
            rig.st.decode_step(l, rig.q[l], rig.kn[l], rig.vn[l], rig.out[l], stream=s)
    torch.cuda.synchronize()
    t0 = rig.ring_t()
    evs = []
    with torch.cuda.stream(s):
        g.replay()
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            g.replay()
            e1.record(s)
            evs.append((e0, e1))
    s.synchronize()
    ms = [a.elapsed_time(b) / w.layers for a, b in evs]
    del g
    return ms, t0


def e2e_tokens(rig: DecodeRig, steps: int, warmup: int, flush):
    """Token steps through the public API with host buffers, run the way a
    serving loop runs them.  Every step copies its q/k_new/v_new (all layers),
    logits and history in from pinned host memory, runs the decode layers,
    the ring advance and the n-gram ban, and copies all layers' outputs and
    the masked logits back.  Two sets of device and host buffers alternate,
    and the copies in and out run on streams of their own, so one step's
    copies overlap its neighbours' compute (a step's input copy waits until
    the step two back has finished with that buffer set).  Timed as one
    region, from the first step's first copy in to the last step's last copy
    back.  Each step reads the whole KV cache; when that is less than four
    times the L2, an L2 flush runs before each step's decode, inside the
    region.  Returns ([total ms], H2D bytes per step, D2H bytes per step)."""
    from ring_sliding_window_b200 import rswa
    w, s = rig.w, rig.s
    hq = [rig.qkv.cpu().pin_memory() for _ in range(2)]
    hl = [rig.logits.cpu().pin_memory() for _ in range(2)]
    hh = [rig.hist.cpu().pin_memory() for _ in range(2)]
    ho = [torch.empty(rig.out.shape, dtype=rig.out.dtype, pin_memory=True) for _ in range(2)]
    hlo = [torch.empty_like(hl[0], pin_memory=True) for _ in range(2)]
    h2d = hq[0].numel() * hq[0].element_size() + hl[0].numel() * 4 + hh[0].numel() * 4
    d2h = ho[0].numel() * ho[0].element_size() + hlo[0].numel() * 4
    # device buffer sets: the rig's own (with its captured decode graph) and a second one
    dq = [rig.qkv, torch.empty_like(rig.qkv)]
    dout = [rig.out, torch.empty_like(rig.out)]
    dl = [rig.logits, torch.empty_like(rig.logits)]
    dh = [rig.hist, torch.empty_like(rig.hist)]
    torch.cuda.synchronize()
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=s):
        for l in range(w.layers):
            rig.st.decode_step(l, dq[1][0][l], dq[1][1][l], dq[1][2][l], dout[1][l], stream=s)
        rig.st.advance(stream=s)
    graphs = [rig.graph_dec, g1]
    torch.cuda.synchronize()
    t_now = min(rig.ring_t())
    flush_each = kv_bytes_per_layer(w, [t_now] * w.batch) * w.layers < 4 * L2_BYTES
    hs, ds = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        p = i % 2
        if i >= 2:
            hs.wait_event(out_done[p])  # the step two back is done with set p
        with torch.cuda.stream(hs):
            dq[p].copy_(hq[p], non_blocking=True)
            dl[p].copy_(hl[p], non_blocking=True)
            dh[p].copy_(hh[p], non_blocking=True)
            in_ready[p].record(hs)
        s.wait_event(in_ready[p])
        with torch.cuda.stream(s):
            if flush_each:
                flush.zero_()
            graphs[p].replay()
            rswa.rswa_ngram_mask(dl[p], dh[p], None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW, stream=s)
            comp_done[p].record(s)
        ds.wait_event(comp_done[p])
        with torch.cuda.stream(ds):
            ho[p].copy_(dout[p], non_blocking=True)
            hlo[p].copy_(dl[p], non_blocking=True)
            out_done[p].record(ds)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    _barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(hs)
    for i in range(steps):
        step(i)
    ds.wait_event(comp_done[(steps - 1) % 2])
    e1.record(ds)
    torch.cuda.synchronize()
    _barrier()
    total = e0.elapsed_time(e1)
    del g1
    return [total], h2d, d2h


# --------------------------------------------------------------------------
def host_cpu():
    """(logical CPUs this process may use, CPU model name) of this host."""
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 0
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return n, model


class OracleSample:
    """The oracle as it stands, on this host's cores, over a bounded sample of
    a workload: `layers` layers of the sequences `seqs`, with `heads` of the
    heads (all by default; heads are independent), prefilled with N(0,1) keys
    and values, then decoded from t = 0.  A step runs the sampled layers' ring
    steps and the n-gram ban of the whole batch (n = 35, window = 128).  The
    attention part is scaled to the whole model by its key count (sampled keys
    / all keys of all layers and heads), the ban is counted once per step, so
    `rate()` is full-model decode steps per second."""

    def __init__(self, w: synth.Workload, layers: int, seqs, heads: int = 0):
        import numpy as np

        import oracle
        self.w, self.layers, self.seqs = w, layers, list(seqs)
        self.heads = heads if heads > 0 else w.heads
        H = self.heads
        rng = np.random.default_rng(0)
        plens = [w.prefill_lens[b] for b in self.seqs]
        self.model = oracle.RingModel(plens, w.window, layers, H, w.head_dim)
        for l in range(layers):
            for i, P in enumerate(plens):
                self.model.prefill(l, i, rng.standard_normal((P, H, w.head_dim)),
                                   rng.standard_normal((P, H, w.head_dim)))
        nb = len(plens)
        self.qkv = [rng.standard_normal((3, nb, H, w.head_dim)) for _ in range(layers)]
        logits, hist, _ = synth.ngram_inputs(w.batch, synth.VOCAB, synth.NGRAM_SIZE,
                                             synth.NGRAM_WINDOW, 1)
        self.lg, self.hi = logits.numpy(), hist.numpy()
        keys = lambda ps: sum(P + w.window for P in ps)  # noqa: E731 (steady-state keys)
        self.fraction = layers * H * keys(plens) / (w.layers * w.heads * keys(w.prefill_lens))
        self.steps, self.attn_s, self.ban_s = 0, 0.0, 0.0

    def run(self, seconds: float = 0.0, max_steps=None):
        import oracle
        w = self.w
        t_start = time.perf_counter()
        n = 0
        while True:
            t0 = time.perf_counter()
            for l in range(self.layers):
                q, kn, vn = self.qkv[l]
                self.model.step(l, q, kn, vn, w.scale)
            t1 = time.perf_counter()
            oracle.ngram_ban(self.lg, self.hi, None, synth.NGRAM_SIZE, synth.NGRAM_WINDOW)
            t2 = time.perf_counter()
            self.attn_s += t1 - t0
            self.ban_s += t2 - t1
            self.steps += 1
            n += 1
            if max_steps is not None and n >= max_steps:
                break
            if max_steps is None and time.perf_counter() - t_start >= seconds and n >= 2:
                break
        return n

    def reset_timers(self):
        self.steps, self.attn_s, self.ban_s = 0, 0.0, 0.0

    def rate(self) -> float:
        per_step = self.attn_s / self.steps / self.fraction + self.ban_s / self.steps
        return 1.0 / per_step

    def describe(self) -> str:
        w = self.w
        heads = f"all {w.heads}" if self.heads == w.heads else f"{self.heads} of {w.heads}"
        return (f"{self.steps} decode steps of {self.layers} of {w.layers} layers x "
                f"{len(self.seqs)} of {w.batch} sequences ({heads} heads) of {w.name} "
                f"from t = 0, plus the n-gram ban of the batch; {self.attn_s + self.ban_s:.1f} s. "
                f"Attention scaled to the whole model by its key count "
                f"(sample = {self.fraction:.4f} of the keys); the first W steps attend over "
                f"fewer keys than steady state ({w.window} of "
                f"{min(w.prefill_lens) + w.window} at most)")


def oracle_prefill_sample(w: synth.Workload, seconds: float) -> dict:
    """The oracle's causal prefill on this host's cores, over a bounded sample
    of the workload's prefill: blocks of 64 consecutive query rows of one head
    of the first sequence, at evenly spaced positions of its prompt (N(0,1)
    q, k, v), run until `seconds` have passed.  A row i costs 4*d*(i + 1)
    FLOPs (causal keys only, as the GPU figure counts them), so the rate is
    FLOP/s of the same work and the full prefill time is extrapolated from
    it."""
    import numpy as np

    import oracle
    P, d = w.prefill_lens[0], w.head_dim
    rng = np.random.default_rng(1)
    q, k, v = (rng.standard_normal((P, 1, d)) for _ in range(3))
    block = min(64, P)
    starts = [min(P - block, (P * j) // 8) for j in range(8)]
    flops, rows, spent, j = 0, 0, 0.0, 0
    while spent < seconds or j < len(starts):
        lo = starts[j % len(starts)]
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, w.scale, lo, lo + block)
        spent += time.perf_counter() - t0
        flops += sum(4 * d * (i + 1) for i in range(lo, lo + block))
        rows += block
        j += 1
    rate = flops / spent
    nproc, model = host_cpu()
    full = prefill_flops_per_layer(w) * w.layers
    return {"value": rate / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "nproc": nproc, "cpu_model": model,
            "sample": f"{rows} query rows of 1 of {w.heads} heads of sequence 0 "
                      f"(P = {P}) in blocks of {block} at 8 evenly spaced positions; "
                      f"{spent:.1f} s",
            "extrapolated_full_prefill_s": full / rate}


def cpu_baseline_block(sample: OracleSample) -> dict:
    import oracle
    nproc, model = host_cpu()
    return {"value": sample.rate(), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "nproc": nproc, "cpu_model": model, "sample": sample.describe()}


# --------------------------------------------------------------------------
def _workload(args):
    import dataclasses
    w = synth.workload(args.workload)
    if args.layers:
        w = dataclasses.replace(w, layers=args.layers)
    return w


def run_ours(args, rank, world, local_rank):
    hbm_peak, tc_peak, peak_src = measured_peaks()
    w = _workload(args)
    dev = torch.cuda.current_device()
    s = torch.cuda.Stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    # ---- prefill (fills the caches of the main workload), then the ring's
    # warm-up: W tokens appended after the prompt (untimed), so that every
    # timed token overwrites the oldest ring entry and attends over exactly
    # P_b + W keys (steady state)
    rig = DecodeRig(w, 0, "prefill", s)
    pf_ms = rig.prefill_all(flush)
    rig.capture()
    fill_ring(rig)
    sampler = ClockSampler(dev if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[dev]))
    ms, ts, clocks = timed_tokens(rig, args.steps, args.warmup, flush, sampler)
    decode_from_t = min(ts[0])
    total_ms = max_over_ranks(sum(ms))
    value = aggregate_rate(args.steps, total_ms, world)
    kv_bytes = sum(w.layers * kv_bytes_per_layer(w, t) for t in ts)
    kv_gbs = kv_bytes / (sum(ms) / 1e3) / 1e9

    # ---- dominant kernel: decode_split_kernel (one per rswa_decode_step)
    launch_ms, t_at = timed_decode_launches(rig, 16, flush)
    per_launch_bytes = kv_bytes_per_layer(w, t_at)
    dur = statistics.mean(launch_ms) / 1e3
    achieved = per_launch_bytes / dur / 1e9

    # ---- e2e through the public API with host buffers
    e2e_ms, h2d, d2h = e2e_tokens(rig, args.steps, args.warmup, flush)
    e2e_total = max_over_ranks(sum(e2e_ms))
    e2e_value = aggregate_rate(args.steps, e2e_total, world)
    pf_flops = prefill_flops_per_layer(w)
    pf_mean = statistics.mean(pf_ms) / 1e3
    assert rig.st.check() == 0, "device error word set during the run"
    dec_grid, dec_cluster = rig.st.decode_launch_shape()
    rig.st.close()
    del rig
    torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded N(0,1) q/k/v; random histories with a planted repeat)",
        "config": {"workload": w.name, "batch": w.batch, "layers": w.layers, "heads": w.heads,
                   "head_dim": w.head_dim, "prefill_len": list(w.prefill_lens)[:4],
                   "window": w.window, "decode_steps_timed": args.steps,
                   "decode_from_t": decode_from_t, "steady_state": decode_from_t >= w.window,
                   "step": "one token: all layers' rswa_decode_step + "
                   "rswa_advance + rswa_ngram_mask (n=35, window=128) as one CUDA graph",
                   "l2": "flushed before every timed step (256 MiB write, outside the events)",
                   "parallelism": f"replicas x{world}",
                   "decode_launch": {"grid": dec_grid, "cluster_size": dec_cluster,
                                     "split": "cluster per ring (DSMEM merge)" if dec_cluster
                                     else "stream-K (workspace merge)"}},
        "kv_read_gbs": kv_gbs,
        "roofline": {"kernel": "decode_split_kernel (rswa_decode_step: ring write + split-K "
                               "attention + in-kernel combine)",
                     "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_source": peak_src,
                     "frac_of_datasheet_8000": achieved / DATASHEET_HBM_GBS,
                     "algorithmic_bytes_per_launch": per_launch_bytes,
                     "avg_launch_us": dur * 1e6, "traffic": measured_traffic(w.name)},
        "prefill": {"workload": w.name, "tflops": pf_flops / pf_mean / 1e12, "unit": "TFLOP/s",
                    "peak": tc_peak, "frac": pf_flops / pf_mean / 1e12 / tc_peak,
                    "frac_of_datasheet_2250": pf_flops / pf_mean / 1e12 / DATASHEET_BF16_TFLOPS,
                    "ms_per_layer": pf_mean * 1e3, "flops_per_layer": pf_flops},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "timing": "one region over all steps: every step's inputs in from pinned host "
                          "memory and its outputs back, two buffer sets, copies on their own "
                          "streams overlapping the neighbouring steps' compute"},
        "gpu_launches": args.steps * (w.layers + 2),
        "clocks": clocks,
    }

    # ---- the bandwidth-bound workloads, steady state (t >= W), decode only
    also = []
    if world == 1 and args.also != "none":
        for name in args.also.split(","):
            if name == w.name:
                continue  # the headline already measured it
            if name == "continuous_batching":
                also.append(run_continuous_batching(args, s, hbm_peak))
            elif name == "ngram_topk":
                also.append(run_ngram_topk(args, flush, s, hbm_peak))
            elif name == "rope":
                also.append(run_rope(args, flush, s, hbm_peak, tc_peak))
            elif name == "standard_swa":
                also.append(run_swa(args, flush, s, hbm_peak))
            elif name == "keysplit":
                also.append(run_keysplit(args, flush, s, hbm_peak))
            else:
                also.append(run_also(synth.workload(name), args, flush, s, hbm_peak, tc_peak))
            torch.cuda.empty_cache()
        line["also"] = also

    # ---- CPU oracle on this host (rank 0, N = 1)
    if world == 1 and rank == 0 and args.cpu_seconds > 0:
        sample = OracleSample(w, 1, range(w.batch))
        sample.run(seconds=args.cpu_seconds)
        line["cpu_baseline"] = cpu_baseline_block(sample)
        line["prefill"]["cpu_baseline"] = oracle_prefill_sample(w, args.cpu_seconds / 2)
    return line


def run_continuous_batching(args, s, hbm_peak, steps=64, churn_every=8, churn=4):
    """Continuous batching on one token pool: the ragged-serving batch (64
    requests, prefill_len U{1024..16384}, ring fill U{0..128}) placed in a
    pool with 25 % headroom; every `churn_every` steps `churn` random requests
    leave and as many new ones (same distributions) join, and the decode state
    is rebuilt over the live requests.  Joining requests' caches hold random
    values (their prefill is not timed: the prefill figures are measured
    elsewhere).  Timed with CUDA events around the whole run, rebuilds
    included; every input is larger than L2."""
    import random
    from ring_sliding_window_b200 import rswa
    w = synth.workload("ragged_serving")
    L, H, d, W = w.layers, w.heads, w.head_dim, w.window
    rng = random.Random(synth.seed(w.cfg_id, 0, 950_000))
    capacity = int(sum(P + W for P in w.prefill_lens) * 1.25)
    pool = rswa.TokenPool(capacity, L, H, d, W, dtype=w.dtype)
    for l in range(L):
        g = torch.Generator(device="cuda").manual_seed(synth.seed(w.cfg_id, l, 950_001))
        pool.k_cache[l].normal_(generator=g)
        pool.v_cache[l].normal_(generator=g)
    live = []  # [prefill_len, base, t]
    order = list(range(w.batch))
    rng.shuffle(order)
    for b in order:
        live.append([w.prefill_lens[b], pool.alloc(w.prefill_lens[b]), w.n_generated[b]])
    bmax = w.batch
    q = torch.randn(L, bmax, H, d, device="cuda").to(w.dtype)
    kn, vn, out = torch.randn_like(q), torch.randn_like(q), torch.empty_like(q)

    def build():
        return pool.state([r[0] for r in live], [r[1] for r in live], n_generated=[r[2] for r in live],
                          stream=s)

    def step_bytes():
        row = H * d * w.elem_bytes
        return L * sum(2 * (P + min(t + 1, W)) * row + 6 * row for P, _, t in live)

    def run(n_steps, st, record):
        nbytes, rebuild_ms, skipped = 0, [], 0
        for i in range(n_steps):
            if i and i % churn_every == 0:
                n, _, _ = st.ring(stream=s)  # waits for the queued steps
                t0 = time.perf_counter()
                for r, t in zip(live, n):
                    r[2] = t
                st.close()
                for _ in range(churn):
                    r = live.pop(rng.randrange(len(live)))
                    pool.free(r[1])
                for _ in range(churn):
                    P = rng.randint(1024, 16384)
                    try:
                        live.append([P, pool.alloc(P), rng.randint(0, 128)])
                    except rswa.RswaError:
                        skipped += 1
                st = build()
                rebuild_ms.append((time.perf_counter() - t0) * 1e3)
            B = len(live)
            if record:
                nbytes += step_bytes()
            with torch.cuda.stream(s):
                for l in range(L):
                    st.decode_step(l, q[l, :B], kn[l, :B], vn[l, :B], out[l, :B], stream=s)
                st.advance(stream=s)
            for r in live:
                r[2] += 1
        return st, nbytes, rebuild_ms, skipped

    st = build()
    st, _, _, _ = run(max(args.warmup, churn_every + 1), st, False)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    st, nbytes, rebuild_ms, skipped = run(steps, st, True)
    e1.record(s)
    s.synchronize()
    ms = e0.elapsed_time(e1)
    assert st.check() == 0
    free, largest, n_free, n_alloc = pool.stats()
    st.close()
    pool.close()
    return {"workload": "continuous_batching (ragged_serving requests in one token pool)",
            "decode_steps_per_s": steps / (ms / 1e3), "ms_per_step": ms / steps,
            "kv_read_gbs": nbytes / (ms / 1e3) / 1e9,
            "frac_of_measured_hbm": nbytes / (ms / 1e3) / 1e9 / hbm_peak,
            "steps_timed": steps, "churn": f"{churn} leave + {churn} join every {churn_every} steps",
            "rebuilds": len(rebuild_ms),
            "rebuild_host_ms_mean": statistics.mean(rebuild_ms),
            "rebuild_host_ms_max": max(rebuild_ms),
            "rebuild": "frees, allocations, rswa_state_create_pooled (plan + table upload, "
                       "synchronous), after the ring counters are read back",
            "joins_refused_for_space": skipped,
            "pool": {"capacity_slots": capacity, "free_slots": free, "largest_free": largest,
                     "free_ranges": n_free, "requests": n_alloc}}


def run_ngram_topk(args, flush, s, hbm_peak, reps=5, calls=16, nbuf=4):
    """rswa_ngram_topk on the pages' sampling shape: 64 rows over the
    129,280-token vocabulary, n = 35, window = 128 (the n-gram inputs of the
    decode step), k = 1 (greedy) and k = 64 (with sampling).  Timed as a CUDA
    graph of `calls` launches rotating over `nbuf` logits buffers (4 x 33 MB,
    more than L2), events on the stream, median of `reps` replays: per-call
    time.  Algorithmic bytes per call: the logits read once (rows x vocab x 4),
    the histories and the outputs.  For context, one eager launch after an L2
    flush, and the unfused pair rswa_ngram_mask + torch.topk timed the same
    way, are reported too."""
    from ring_sliding_window_b200 import rswa
    rows, V, n, win = 64, synth.VOCAB, synth.NGRAM_SIZE, synth.NGRAM_WINDOW
    logits, hist, _ = synth.ngram_inputs(rows, V, n, win, synth.seed(5, 0, 820_000))
    bufs = [logits.cuda() for _ in range(nbuf)]
    hist = hist.cuda()
    u = torch.rand(rows, device="cuda")
    out = {}

    def graph_us(fn):
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for j in range(calls):
                fn(bufs[j % nbuf])
        torch.cuda.synchronize()
        ms = []
        with torch.cuda.stream(s):
            for _ in range(3):
                g.replay()
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                g.replay()
                e1.record(s)
                ms.append((e0, e1))
        s.synchronize()
        del g
        return statistics.median(a.elapsed_time(b) for a, b in ms) * 1e3 / calls

    def eager_us(fn):
        ms = []
        with torch.cuda.stream(s):
            for _ in range(3):
                fn(bufs[0])
            for _ in range(reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                fn(bufs[0])
                e1.record(s)
                ms.append((e0, e1))
        s.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ms) * 1e3

    for k in (1, 64):
        idx = torch.empty(rows, k, dtype=torch.int32, device="cuda")
        val = torch.empty(rows, k, device="cuda")
        tok = torch.empty(rows, dtype=torch.int32, device="cuda")
        samp = u if k > 1 else None
        fused = lambda lg: rswa.rswa_ngram_topk(lg, hist, None, n, win, k, uniform=samp,
                                                top_idx=idx, top_val=val, token=tok, stream=s)
        unfused = lambda lg: (rswa.rswa_ngram_mask(lg, hist, None, n, win, stream=s),
                              torch.topk(lg, k, dim=1))
        us = graph_us(fused)
        nbytes = rows * V * 4 + hist.numel() * 4 + rows * k * 8 + rows * 4
        gbs = nbytes / (us * 1e-6) / 1e9
        out[f"k{k}"] = {"us_per_call": us, "algorithmic_bytes": nbytes, "gbs": gbs,
                        "frac_of_measured_hbm": gbs / hbm_peak,
                        "eager_after_l2_flush_us": eager_us(fused),
                        "sampling": "inverse CDF at a uniform per row" if samp is not None else "greedy",
                        "unfused_mask_plus_torch_topk_us": graph_us(unfused)}
    return {"workload": "ngram_topk (64 rows x 129,280 vocab, n=35, window=128)",
            "timing": f"CUDA graph of {calls} calls over {nbuf} logits buffers (> L2)", **out}


def run_rope(args, flush, s, hbm_peak, tc_peak, steps=512):
    """RoPE at cache-write time (absolute positions, theta = 10000) on the
    single-page decode workload (the headline step with rotation on) and on
    the multi-page prefill (2 layers; the rotation pre-pass is inside the
    timed prefill).  The same measurements without RoPE sit beside them."""
    w = synth.workload("single_page_decode")
    res = {"workload": "rope (absolute positions, theta 10000)"}
    for rope in (0, 1):
        rig = DecodeRig(w, 0, "random", s, rope=rope)
        rig.capture()
        ms, _, _ = timed_tokens(rig, steps, args.warmup, flush)
        launch_ms, t_at = timed_decode_launches(rig, 8, flush)
        key = "rope" if rope else "no_rope"
        res[f"single_page_{key}"] = {"decode_steps_per_s": steps / (sum(ms) / 1e3),
                                     "avg_decode_launch_us": statistics.mean(launch_ms) * 1e3}
        assert rig.st.check() == 0
        rig.st.close()
        del rig
        torch.cuda.empty_cache()
    wm = synth.workload("multi_page_decode")
    w1 = synth.Workload(wm.name, wm.cfg_id, wm.dtype, wm.batch, 2, wm.heads, wm.head_dim,
                        wm.window, wm.prefill_lens, 0)
    for rope in (0, 1):
        rig = DecodeRig(w1, 0, "prefill", s, rope=rope)
        pf_ms = rig.prefill_all(flush)
        f = prefill_flops_per_layer(w1) / (statistics.mean(pf_ms) / 1e3) / 1e12
        res[f"multi_page_prefill_{'rope' if rope else 'no_rope'}"] = {
            "tflops": f, "frac": f / tc_peak, "ms_per_layer": statistics.mean(pf_ms)}
        rig.st.close()
        del rig
        torch.cuda.empty_cache()
    return res


def run_swa(args, flush, s, hbm_peak):
    """Standard sliding-window contrast mode on the multi-page workload
    (batch 8, prefill_len 8,256, W = 128): a decode step reads only the last
    W positions of each ring; the prefill attends within the window.  Decode
    per launch (steady state) and the 2-layer prefill, each beside the same
    measurement in R-SWA mode."""
    from ring_sliding_window_b200 import rswa
    w = synth.workload("multi_page_decode")
    res = {"workload": "standard_swa contrast (multi_page_decode shapes, W = 128)"}
    row = w.heads * w.head_dim * w.elem_bytes
    for mode in (rswa.RSWA_ATTN_RING, rswa.RSWA_ATTN_STANDARD_SWA):
        rig = DecodeRig(w, w.window, "random", s)
        rig.st.set_attention(mode)
        rig.capture()
        launch_ms, t_at = timed_decode_launches(rig, 8, flush)
        us = statistics.mean(launch_ms) * 1e3
        if mode == rswa.RSWA_ATTN_RING:
            nbytes = kv_bytes_per_layer(w, t_at)
        else:  # W keys per ring (t >= W - 1), plus q/k_new/v_new, ring write, out
            nbytes = w.batch * (2 * w.window * row + 6 * row)
        key = "ring" if mode == rswa.RSWA_ATTN_RING else "standard_swa"
        res[f"decode_{key}"] = {"avg_launch_us": us, "algorithmic_bytes": nbytes,
                                "gbs": nbytes / (us * 1e-6) / 1e9}
        assert rig.st.check() == 0
        rig.st.close()
        del rig
        torch.cuda.empty_cache()
    w1 = synth.Workload(w.name, w.cfg_id, w.dtype, w.batch, 2, w.heads, w.head_dim, w.window,
                        w.prefill_lens, 0)
    rig = DecodeRig(w1, 0, "prefill", s)
    rig.st.set_attention(rswa.RSWA_ATTN_STANDARD_SWA)
    pf_ms = rig.prefill_all(flush)
    flops = sum(4 * w.heads * w.head_dim * sum(min(i + 1, w.window) for i in range(P))
                for P in w.prefill_lens)
    res["prefill_standard_swa"] = {"ms_per_layer": statistics.mean(pf_ms),
                                   "tflops": flops / (statistics.mean(pf_ms) / 1e3) / 1e12,
                                   "kernel": "prefill_tc_kernel, key tiles of each window only"}
    rig.st.close()
    del rig
    torch.cuda.empty_cache()
    return res


def run_keysplit(args, flush, s, hbm_peak, reps=20):
    """Key-range split of one near-max sequence (prefill_len 32,640, W = 128,
    10 heads x 128) into G shares, run here one after another on one device:
    per layer, G partial decode launches plus the merge, against one full
    decode launch.  On G devices the shares run side by side and only the
    partials (G x H x (d + 2) floats) cross between them; here the numbers
    show the split's own cost.  Steady state, L2 flushed before each rep."""
    from ring_sliding_window_b200 import rswa
    from ring_sliding_window_b200.keysplit import share_bounds
    P, W, H, d = 127 * synth.TOKENS_PER_PAGE + 128, 128, 10, 128
    row = H * d * 2
    res = {"workload": "keysplit (one sequence, prefill_len 32,640)"}
    q = torch.randn(1, H, d, device="cuda").to(torch.bfloat16)
    kn, vn = torch.randn_like(q), torch.randn_like(q)

    def timed(fn):
        ms = []
        with torch.cuda.stream(s):
            for _ in range(3):
                fn()
            for _ in range(reps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(s)
                fn()
                e1.record(s)
                ms.append((e0, e1))
        s.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ms) * 1e3

    for G in (1, 2, 4):
        bounds = share_bounds(P, G)
        states = []
        for g, (lo, hi) in enumerate(bounds):
            st = rswa.State(1, 1, H, d, W, [hi - lo], dtype=torch.bfloat16, n_generated=[W])
            gen = torch.Generator(device="cuda").manual_seed(950_100 + g)
            st.k_cache[0].normal_(generator=gen)
            st.v_cache[0].normal_(generator=gen)
            states.append(st)
        ml = torch.empty(G, 1, H, 2, device="cuda")
        o = torch.empty(G, 1, H, d, device="cuda")
        out = torch.empty_like(q)

        def step():
            for g, st in enumerate(states):
                lo, hi = bounds[g]
                st.decode_step_partial(0, q, kn, vn, 0, (hi - lo) + (W if g == G - 1 else 0),
                                       ml[g], o[g], stream=s)
            rswa.rswa_combine_partials(ml, o, out, stream=s)

        if G == 1:
            full = rswa.State(1, 1, H, d, W, [P], dtype=torch.bfloat16, n_generated=[W])
            full_us = timed(lambda: full.decode_step(0, q, kn, vn, out, stream=s))
            res["full_decode_us"] = full_us
            full.close()
        us = timed(step)
        nbytes = 2 * (P + W) * row
        res[f"G{G}"] = {"us_per_layer_all_shares": us, "kv_gbs": nbytes / (us * 1e-6) / 1e9,
                        "partial_floats_exchanged": G * H * (d + 2)}
        for st in states:
            st.close()
        torch.cuda.empty_cache()
    return res


def run_also(w, args, flush, s, hbm_peak, tc_peak):
    steps = args.also_steps
    rig = DecodeRig(w, w.window, "random", s)
    rig.capture()
    ms, ts, _ = timed_tokens(rig, steps, args.warmup, flush)
    kv_bytes = sum(w.layers * kv_bytes_per_layer(w, t) for t in ts)
    launch_ms, t_at = timed_decode_launches(rig, 8, flush)
    per_launch = kv_bytes_per_layer(w, t_at)
    ach = per_launch / (statistics.mean(launch_ms) / 1e3) / 1e9
    res = {"workload": w.name, "decode_steps_per_s": steps / (sum(ms) / 1e3),
           "ms_per_step": sum(ms) / steps, "kv_read_gbs": kv_bytes / (sum(ms) / 1e3) / 1e9,
           "decode_step_launch_gbs": ach, "frac_of_measured_hbm": ach / hbm_peak,
           "frac_of_datasheet_8000": ach / DATASHEET_HBM_GBS, "avg_launch_us": statistics.mean(launch_ms) * 1e3,
           "steps_timed": steps, "from_t": w.window if w.n_generated is None else "n_generated"}
    assert rig.st.check() == 0
    rig.st.close()
    del rig
    torch.cuda.empty_cache()
    if w.name in ("multi_page_decode", "near_max_context") and not args.skip_prefill_also:
        w1 = synth.Workload(w.name, w.cfg_id, w.dtype, w.batch, 2, w.heads, w.head_dim, w.window,
                            w.prefill_lens, 0)
        rig = DecodeRig(w1, 0, "prefill", s)
        pf_ms = rig.prefill_all(flush)
        f = prefill_flops_per_layer(w1) / (statistics.mean(pf_ms) / 1e3) / 1e12
        res["prefill_tflops"] = f
        res["prefill_frac"] = f / tc_peak
        res["prefill_frac_of_datasheet_2250"] = f / DATASHEET_BF16_TFLOPS
        rig.st.close()
        del rig
    return res


def reference_sample(w: synth.Workload, steps_total: int, budget_s: float,
                     mem_cap: float = 4e9) -> OracleSample:
    """The largest sample of (layer, sequence) units whose `steps_total` steps
    fit in `budget_s` seconds and whose FP64 caches fit in `mem_cap` bytes:
    one unit is timed first, then the sample is built once.  When even one
    unit is too slow, the sample keeps only some of its heads."""
    longest = int(max(range(w.batch), key=lambda b: w.prefill_lens[b]))
    probe = OracleSample(w, 1, [longest])
    probe.run(max_steps=1)
    unit_attn, unit_ban = probe.attn_s, probe.ban_s
    del probe
    by_time = int(budget_s / max((unit_attn + unit_ban) * steps_total, 1e-9))
    by_mem = int(mem_cap // (16 * (max(w.prefill_lens) + w.window) * w.heads * w.head_dim))
    units = min(by_time, by_mem, w.layers * w.batch)
    if units < 1:
        # one layer of one sequence, as many heads as the budget allows
        per_head = unit_attn / w.heads
        heads = int((budget_s / steps_total - unit_ban) / max(per_head, 1e-9))
        return OracleSample(w, 1, [longest], heads=max(1, min(w.heads, heads)))
    seqs = min(w.batch, units)
    layers = max(1, min(w.layers, units // seqs))
    return OracleSample(w, layers, range(seqs))


def run_reference(args):
    w = _workload(args)
    sample = reference_sample(w, args.steps + args.warmup, args.reference_budget)
    if args.warmup:
        sample.run(max_steps=args.warmup)
    sample.reset_timers()
    sample.run(max_steps=args.steps)
    rate = sample.rate()
    return {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / rate,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "batch": w.batch, "layers": w.layers,
                                        "heads": w.heads, "head_dim": w.head_dim,
                                        "prefill_len": list(w.prefill_lens)[:4], "window": w.window},
        "cpu_baseline": cpu_baseline_block(sample),
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2048)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="near_max_context")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (small profiling runs)")
    ap.add_argument("--also", default="single_page_decode,multi_page_decode,ragged_serving,"
                                      "continuous_batching,ngram_topk,rope,standard_swa,"
                                      "keysplit")
    ap.add_argument("--also-steps", type=int, default=40)
    ap.add_argument("--skip-prefill-also", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-budget", type=float, default=120.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        dist.barrier()
    line = run_ours(args, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
