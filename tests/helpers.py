"""Shared test plumbing: run the CUDA path step by step and compute oracle
expectations from the same seeded inputs (never from CUDA-path outputs)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from ring_sliding_window_b200 import synth

BF16_TOL = 2e-2   # max-abs, bf16 inputs (attention outputs)
F32_TOL = 1e-5    # max-abs, fp32 inputs


def tol_for(dtype) -> float:
    return BF16_TOL if dtype == torch.bfloat16 else F32_TOL


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def seq_slices(prefill_lens):
    out, base = [], 0
    for p in prefill_lens:
        out.append(slice(base, base + p))
        base += p
    return out


def union_expect(pk, pv, gen_k, gen_v, q, t, W, scale):
    """Oracle attention of one (b, h) query at step t over the union key set:
    all prefill keys plus generated keys s in [max(0, t-W+1), t].
    pk, pv: [P, d]; gen_k, gen_v: sequence of [d] arrays indexed by step."""
    lo = max(0, t - W + 1)
    kk = np.concatenate([pk, np.stack([gen_k[s] for s in range(lo, t + 1)])])
    vv = np.concatenate([pv, np.stack([gen_v[s] for s in range(lo, t + 1)])])
    return oracle.attend(q, kk, vv, scale)


class StepInputs:
    """All decode-step inputs of a run, generated on the GPU: [steps][L][3] of [B, H, d]."""

    def __init__(self, w: synth.Workload, steps: int, device="cuda"):
        self.w, self.steps = w, steps
        self.qkv = [[synth.decode_qkv(w, l, s, device) for l in range(w.layers)]
                    for s in range(steps)]

    def get(self, step, layer):
        return self.qkv[step][layer]
