"""R-SWA CPU oracle (FP64) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding in ``ring_sliding_window_b200``) never imports, links or executes
anything here, and this package imports nothing from it.

The arithmetic lives in ``oracle.c`` (plain C, double precision); this module
only marshals numpy arrays through ctypes and keeps per-(layer, sequence) ring
objects for multi-layer, multi-sequence runs.

Method source, by page title and section:
  "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §2.1 (ring
  sliding-window attention: prefill kept whole, warm-up append, steady-state
  ring overwrite of slot prefill_len + ring_pos) and §2.3 (no-repeat n-gram ban
  restricted to a sliding window).

Pins (in tests/): float64 SDPA from torch, closed forms, brute force over the
union key set, the transformers no-repeat-ngram processor, hand-built n-gram
fixtures under tests/golden/.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ORC_OK, ORC_EINVAL, ORC_ENOMEM, ORC_ESTATE, ORC_EDATA = 0, 1, 2, 4, 6


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (OpenMP when available)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + ".tmp"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_ip = ctypes.POINTER(ctypes.c_int32)
_lp = ctypes.POINTER(ctypes.c_int64)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # ORACLE_LIB_OVERRIDE points the pins at a deliberately broken build of
    # oracle.c (tests/test_oracle_mutants.py), to show that they catch it.
    lib = ctypes.CDLL(os.environ.get("ORACLE_LIB_OVERRIDE") or build())
    lib.oracle_attend.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_double, _dp]
    lib.oracle_attend.restype = ctypes.c_int
    lib.oracle_prefill.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_double, ctypes.c_int64, ctypes.c_int64, _dp]
    lib.oracle_prefill.restype = ctypes.c_int
    lib.oracle_ring_create.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
    lib.oracle_ring_create.restype = ctypes.c_void_p
    lib.oracle_ring_destroy.argtypes = [ctypes.c_void_p]
    lib.oracle_ring_destroy.restype = None
    lib.oracle_ring_prefill.argtypes = [ctypes.c_void_p, _dp, _dp]
    lib.oracle_ring_prefill.restype = ctypes.c_int
    lib.oracle_ring_step.argtypes = [ctypes.c_void_p, _dp, _dp, _dp, ctypes.c_double, _dp, _lp, _lp]
    lib.oracle_ring_step.restype = ctypes.c_int
    lib.oracle_ring_snapshot.argtypes = [ctypes.c_void_p, _dp, _dp]
    lib.oracle_ring_snapshot.restype = ctypes.c_int64
    lib.oracle_ring_ring_pos.argtypes = [ctypes.c_void_p]
    lib.oracle_ring_ring_pos.restype = ctypes.c_int64
    lib.oracle_ring_len.argtypes = [ctypes.c_void_p]
    lib.oracle_ring_len.restype = ctypes.c_int64
    lib.oracle_ngram_ban.argtypes = [_fp, ctypes.c_int64, _ip, ctypes.c_int64, _ip, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.oracle_ngram_ban.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def attend(q, k, v, scale: float) -> np.ndarray:
    """Softmax attention of one query q[d] over keys k[n, d] and values v[n, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    n, d = k.shape
    out = np.empty(d, dtype=np.float64)
    rc = _load().oracle_attend(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), n, d, d, float(scale),
                               _ptr(out, _dp))
    if rc != ORC_OK:
        raise ValueError(f"oracle_attend failed ({rc})")
    return out


def prefill(q, k, v, scale: float, row_lo: int = 0, row_hi: int | None = None) -> np.ndarray:
    """Causal prefill attention of one sequence; q, k, v: [P, H, d].

    Returns out[P, H, d]; rows outside [row_lo, row_hi) are left as NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    P, H, d = q.shape
    row_hi = P if row_hi is None else row_hi
    out = np.full((P, H, d), np.nan, dtype=np.float64)
    rc = _load().oracle_prefill(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), P, H, d, float(scale),
                                row_lo, row_hi, _ptr(out, _dp))
    if rc != ORC_OK:
        raise ValueError(f"oracle_prefill failed ({rc})")
    return out


class Ring:
    """One (layer, sequence) R-SWA cache simulated by the oracle."""

    def __init__(self, prefill_len: int, window: int, heads: int, head_dim: int):
        lib = _load()
        self._h = lib.oracle_ring_create(prefill_len, window, heads, head_dim)
        if not self._h:
            raise ValueError("oracle_ring_create failed")
        self.P, self.W, self.H, self.d = prefill_len, window, heads, head_dim

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.oracle_ring_destroy(h)

    def prefill(self, k, v) -> None:
        k = _f64(k).reshape(self.P, self.H, self.d)
        v = _f64(v).reshape(self.P, self.H, self.d)
        rc = _lib.oracle_ring_prefill(self._h, _ptr(k, _dp), _ptr(v, _dp))
        if rc != ORC_OK:
            raise ValueError(f"oracle_ring_prefill failed ({rc})")

    def step(self, q, k_new, v_new, scale: float):
        """Write one generated token and attend.  Returns (out[H, d], slot, len)."""
        q = _f64(q).reshape(self.H, self.d)
        k_new = _f64(k_new).reshape(self.H, self.d)
        v_new = _f64(v_new).reshape(self.H, self.d)
        out = np.empty((self.H, self.d), dtype=np.float64)
        slot = ctypes.c_int64(-1)
        n = ctypes.c_int64(-1)
        rc = _lib.oracle_ring_step(self._h, _ptr(q, _dp), _ptr(k_new, _dp), _ptr(v_new, _dp),
                                   float(scale), _ptr(out, _dp), ctypes.byref(slot), ctypes.byref(n))
        if rc != ORC_OK:
            raise ValueError(f"oracle_ring_step failed ({rc})")
        return out, int(slot.value), int(n.value)

    def snapshot(self):
        """(k[P+W, H, d], v[P+W, H, d], entries held)."""
        shape = (self.P + self.W, self.H, self.d)
        k = np.empty(shape, dtype=np.float64)
        v = np.empty(shape, dtype=np.float64)
        n = _lib.oracle_ring_snapshot(self._h, _ptr(k, _dp), _ptr(v, _dp))
        return k, v, int(n)

    @property
    def ring_pos(self) -> int:
        return int(_lib.oracle_ring_ring_pos(self._h))

    @property
    def length(self) -> int:
        return int(_lib.oracle_ring_len(self._h))


def ngram_ban(logits: np.ndarray, history: np.ndarray, hist_len, n: int, window: int) -> int:
    """Apply the windowed no-repeat n-gram ban in place.

    logits: float32 [rows, vocab] (C-contiguous), history: int32 [rows, >=window],
    hist_len: int32 [rows] or None (every row holds `window` tokens).
    Returns 0, or minus the number of rows rejected as bad data (left untouched).
    """
    if logits.dtype != np.float32 or not logits.flags.c_contiguous:
        raise TypeError("logits must be C-contiguous float32")
    history = np.ascontiguousarray(history, dtype=np.int32)
    rows, vocab = logits.shape
    hl = None if hist_len is None else np.ascontiguousarray(hist_len, dtype=np.int32)
    rc = _load().oracle_ngram_ban(
        _ptr(logits, _fp), vocab, _ptr(history, _ip), history.shape[1] if rows else window,
        None if hl is None else _ptr(hl, _ip), rows, vocab, n, window)
    if rc > 0:
        raise ValueError(f"oracle_ngram_ban rejected its arguments ({rc})")
    return int(rc)


def attend_partial(q, k, v, scale: float):
    """The share of softmax attention over one part of a key set, in FP64:
    m = max_j s_j with s_j = scale * log2(e) * q.k_j (log2 units),
    l = sum_j 2^(s_j - m), o = sum_j 2^(s_j - m) v_j.  An empty part gives
    (-inf, 0, 0).  q: [d]; k, v: [n, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if k.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(q.shape[-1])
    s = (k @ q) * float(scale) / np.log(2.0)
    m = float(np.max(s))
    p = np.exp2(s - m)
    return m, float(p.sum()), p @ v


def combine_partials(parts):
    """Log-sum-exp merge of (m, l, o) shares: sum 2^(m_g - M) o_g over
    sum 2^(m_g - M) l_g, M = max m_g; equals attention over the union of the
    parts (the key-range split of the decode step)."""
    M = max(m for m, _, _ in parts)
    w = [0.0 if m == -np.inf else 2.0 ** (m - M) for m, _, _ in parts]
    L = sum(wi * l for wi, (_, l, _) in zip(w, parts))
    return sum(wi * o for wi, (_, _, o) in zip(w, parts)) / L


def prefill_window(q, k, v, scale: float, window: int) -> np.ndarray:
    """Standard sliding-window prefill, the contrast of "开源5天Star破万之后：
    百度Unlimited-OCR的爆火路径复盘" §2.1 (a standard window would cut the
    prompt's K/V too): query i of each head attends to keys
    max(0, i - window + 1) .. i.  q, k, v: [P, H, d]; returns [P, H, d]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    P, H, d = q.shape
    out = np.empty((P, H, d), dtype=np.float64)
    for i in range(P):
        lo = max(0, i - window + 1)
        for h in range(H):
            out[i, h] = attend(q[i, h], k[lo:i + 1, h], v[lo:i + 1, h], scale)
    return out


def rope(x, pos, theta: float = 10000.0) -> np.ndarray:
    """Rotary position embedding, rotate-half form, in FP64.

    The pages give the model's max_position_embeddings (32768, §2.1) and name
    Llama-style attention but define no position encoding; the reading here
    is the Llama one: for i < d/2 the pair (x_i, x_{i+d/2}) turns by the angle
    pos * theta^(-2i/d).  x: [n, ..., d]; pos: [n] positions of the n rows.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    inv_freq = float(theta) ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64).reshape((-1,) + (1,) * (x.ndim - 2) + (1,)) * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_position(policy: str, prefill_len: int, t: int, window: int) -> int:
    """Position of generated token t (0-based) of a request with prefill_len
    prompt tokens: 'absolute' -> P + t; 'slot' -> the cache slot it is
    written to, P + (t mod W) (the ring slot of the pages' §2.1)."""
    return prefill_len + t if policy == "absolute" else prefill_len + t % window


def ngram_topk(logits: np.ndarray, history: np.ndarray, hist_len, n: int, window: int, k: int):
    """Windowed n-gram ban, then the k best columns of the masked row.

    Method: "开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘" §2.3 -- the
    banned tokens score -inf and the next token is chosen from the masked
    scores (greedy decoding takes the best one).  The selection order is
    stated here: masked value descending (NaN counts as -inf), the lower
    column first among equal values; a library sort does the ordering.
    Returns (top_idx int32 [rows, k], top_val float32 [rows, k],
    masked float32 [rows, vocab] (the logits after the ban, NaN untouched),
    bad bool [rows]).  Rows whose history is invalid keep -1 / NaN outputs.
    """
    rows, vocab = logits.shape
    masked = np.array(logits, dtype=np.float32, copy=True, order="C")
    bad = np.zeros(rows, dtype=bool)
    for r in range(rows):
        hl = None if hist_len is None else np.asarray(hist_len)[r:r + 1]
        bad[r] = ngram_ban(masked[r:r + 1], np.asarray(history)[r:r + 1], hl, n, window) < 0
    top_idx = np.full((rows, k), -1, dtype=np.int32)
    top_val = np.full((rows, k), np.nan, dtype=np.float32)
    cols = np.arange(vocab)
    for r in range(rows):
        if bad[r]:
            continue
        x = masked[r].astype(np.float64)
        x[np.isnan(x)] = -np.inf
        order = np.lexsort((cols, -x))[:k]  # primary key -x, then column
        top_idx[r] = order
        top_val[r] = x[order].astype(np.float32)
    return top_idx, top_val, masked, bad


def topk_sample_cdf(top_val: np.ndarray, u: float, temperature: float):
    """Inverse-CDF sampling among k ordered candidates (FP64).

    p_i = exp((x_i - x_0) / T) (0 where x_i = -inf), c_i = p_0 + ... + p_i;
    the draw is the first i with c_i > u * c_{k-1}.  Returns (i, c, u * c_{k-1}).
    """
    x = np.asarray(top_val, dtype=np.float64)
    if not np.isfinite(x[0]):
        return 0, np.zeros_like(x), 0.0
    p = np.where(np.isneginf(x), 0.0, np.exp((x - x[0]) / temperature))
    c = np.cumsum(p)
    target = u * c[-1]
    i = int(np.argmax(c > target))
    return i, c, target


class RingModel:
    """Oracle state for a whole batch: one Ring per (layer, sequence)."""

    def __init__(self, prefill_lens, window: int, layers: int, heads: int, head_dim: int):
        self.P = [int(p) for p in prefill_lens]
        self.W, self.L, self.H, self.d = window, layers, heads, head_dim
        self.rings = [[Ring(p, window, heads, head_dim) for p in self.P] for _ in range(layers)]

    def prefill(self, layer: int, b: int, k, v) -> None:
        self.rings[layer][b].prefill(k, v)

    def step(self, layer: int, q, k_new, v_new, scale: float) -> np.ndarray:
        """q, k_new, v_new: [B, H, d] for one layer; returns out[B, H, d]."""
        outs = [self.rings[layer][b].step(q[b], k_new[b], v_new[b], scale)[0]
                for b in range(len(self.P))]
        return np.stack(outs)
