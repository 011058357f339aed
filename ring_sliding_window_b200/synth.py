"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module draws random numbers and describes workload shapes; it holds none of
the method's arithmetic (no attention, no ring indexing, no n-gram logic beyond
planting a repeated suffix into a random history, which is input construction).

Workload shapes follow the facts the pages give ("开源5天Star破万之后：百度
Unlimited-OCR的爆火路径复盘"): ring window 128 (§2.1), about 256 image tokens
per 1024x1024 page and 32,768 positions (§2.1), 12 LM layers with hidden size
1280 (§2.2/§2.4), vocabulary 129,280 (§2.4), n-gram size 35 and window 128 (§2.3).
Heads x head_dim = 10 x 128 is an assumption (the pages give hidden 1280 only).

Seeds: seed(cfg, layer, step) = cfg * 1_000_003 + layer * 10_007 + step.
Every tensor is drawn in float32 from N(0, 1) with a torch.Generator and cast to
the workload dtype with round-to-nearest-even; both sides receive the same bits.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

NGRAM_SIZE = 35       # §2.3 default no_repeat_ngram_size
NGRAM_WINDOW = 128    # §2.3 default ngram_window
RING_WINDOW = 128     # §2.1 sliding_window_size
VOCAB = 129_280       # §2.4 vocabulary
MAX_POSITIONS = 32_768  # §2.1 max_position_embeddings
TOKENS_PER_PAGE = 256   # §2.1: 16 x 16 image tokens per 1024x1024 page


def seed(cfg: int, layer: int, step: int) -> int:
    return cfg * 1_000_003 + layer * 10_007 + step


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    dtype: torch.dtype
    batch: int
    layers: int
    heads: int
    head_dim: int
    window: int
    prefill_lens: tuple
    decode_steps: int
    n_generated: Optional[tuple] = None  # ragged ring fill (serving snapshot)
    ngram_rows: int = 0

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == torch.bfloat16 else 4

    @property
    def scale(self) -> float:
        return self.head_dim ** -0.5


def _ragged_lens(n: int, lo: int, hi: int, s: int):
    g = torch.Generator().manual_seed(s)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


def workloads() -> List[Workload]:
    """The five workloads, smallest first."""
    rag_p = _ragged_lens(64, 1024, 16384, seed(5, 0, 900_001))
    rag_f = _ragged_lens(64, 0, 128, seed(5, 0, 900_002))
    return [
        Workload("tiny_ring_fp32", 1, torch.float32, 1, 1, 2, 64, 8, (64,), 40),
        Workload("single_page_decode", 2, torch.bfloat16, 1, 12, 10, 128, 128,
                 (4 * TOKENS_PER_PAGE + 64,), 4096),
        Workload("multi_page_decode", 3, torch.bfloat16, 8, 12, 10, 128, 128,
                 (32 * TOKENS_PER_PAGE + 64,) * 8, 8192),
        Workload("near_max_context", 4, torch.bfloat16, 4, 12, 10, 128, 128,
                 (127 * TOKENS_PER_PAGE + 128,) * 4, 20000),
        Workload("ragged_serving", 5, torch.bfloat16, 64, 12, 10, 128, 128, rag_p, 1,
                 n_generated=rag_f, ngram_rows=64),
    ]


def workload(name_or_id) -> Workload:
    for w in workloads():
        if w.name == name_or_id or w.cfg_id == name_or_id:
            return w
    raise KeyError(name_or_id)


def normal(shape, s: int, dtype: torch.dtype, device="cpu") -> torch.Tensor:
    """N(0,1) drawn in float32 from a generator seeded with `s`, cast to dtype."""
    g = torch.Generator(device=device).manual_seed(int(s))
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return x.to(dtype)


def prefill_qkv(w: Workload, layer: int, device="cpu"):
    """Packed varlen prefill inputs q, k, v: [sum P_b, H, d] for one layer."""
    tot = sum(w.prefill_lens)
    shape = (tot, w.heads, w.head_dim)
    return tuple(normal(shape, seed(w.cfg_id, layer, 100_000_000 + i), w.dtype, device)
                 for i in range(3))


def decode_qkv(w: Workload, layer: int, step: int, device="cpu"):
    """Per-step decode inputs q, k_new, v_new: [B, H, d] for one layer."""
    shape = (w.batch, w.heads, w.head_dim)
    return tuple(normal(shape, seed(w.cfg_id, layer, 3 * step + i), w.dtype, device)
                 for i in range(3))


def ngram_inputs(rows: int, vocab: int, n: int, window: int, s: int, device="cpu"):
    """fp32 N(0,1) logits [rows, vocab] and int32 histories [rows, window].

    Each history is uniform over the vocabulary; its last n-1 tokens are copied
    to a random earlier start i in [0, window - 2(n-1) - 1] so that at least one
    n-gram repeats inside the window.  Returns (logits, history, starts).
    """
    g = torch.Generator().manual_seed(int(s))
    logits = torch.randn((rows, vocab), generator=g, dtype=torch.float32)
    hist = torch.randint(0, vocab, (rows, window), generator=g, dtype=torch.int64)
    m = n - 1
    hi = window - 2 * m - 1
    starts = torch.randint(0, max(hi, 0) + 1, (rows,), generator=g)
    if m > 0 and hi >= 0:
        for r in range(rows):
            i = int(starts[r])
            hist[r, i:i + m] = hist[r, window - m:].clone()
    return logits.to(device), hist.to(torch.int32).to(device), starts
