"""Thin ctypes binding of librswa (include/rswa.h), same names as the C ABI.

Functions here only marshal arguments: torch tensors become raw device
pointers, the current torch CUDA stream becomes the ``stream`` argument, and a
non-zero status becomes an ``RswaError``.  All computation happens in the CUDA
kernels of librswa.so; if that library is missing this module raises at import.

``State`` is a convenience owner of the device memory a batch needs (one K and
one V cache per layer, and the workspace), allocated through torch, plus the
opaque ``rswa_state``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# RSWA_LIBRARY may point at another build of the same library (e.g. one built
# with different compile-time tuning); the default is the in-tree build.
_LIB_PATH = os.environ.get("RSWA_LIBRARY") or os.path.join(_PKG, "librswa.so")

RSWA_OK, RSWA_EINVAL, RSWA_ENOMEM, RSWA_ECUDA, RSWA_ESTATE, RSWA_ETIMEOUT, RSWA_EDEVICE = range(7)
RSWA_F32, RSWA_BF16 = 0, 1
RSWA_DEVERR_TIMEOUT, RSWA_DEVERR_BAD_TOKEN, RSWA_DEVERR_BAD_LENGTH = 1, 2, 4

EXPORTED = (
    "rswa_cache_bytes", "rswa_workspace_bytes", "rswa_state_create", "rswa_state_destroy",
    "rswa_cache_offset", "rswa_prefill", "rswa_decode_step", "rswa_advance", "rswa_reset_ring",
    "rswa_ngram_mask", "rswa_get_ring", "rswa_check_device_error", "rswa_status_string",
    "rswa_decode_step_noalloc", "rswa_last_cuda_error", "rswa_debug_inject_fault",
    "rswa_decode_launch_shape", "rswa_pool_create", "rswa_pool_destroy", "rswa_pool_alloc",
    "rswa_pool_free", "rswa_pool_stats", "rswa_pool_capacity", "rswa_pool_cache_bytes",
    "rswa_state_create_pooled", "rswa_ngram_topk", "rswa_state_set_rope",
    "rswa_state_set_attention", "rswa_decode_step_partial", "rswa_combine_partials",
    "rswa_debug_prefill_plan",
)
RSWA_ATTN_RING, RSWA_ATTN_STANDARD_SWA = 0, 1
RSWA_ROPE_NONE, RSWA_ROPE_ABSOLUTE, RSWA_ROPE_SLOT = 0, 1, 2
RSWA_TOPK_MAX, RSWA_TOPK_MAX_VOCAB = 64, 262144
RSWA_FAULT_DROP_DECODE_COPIES = 1
RSWA_FAULT_DROP_PREFILL_LOADS = 2
RSWA_NOALLOC_SCRATCH_BYTES = 4 << 20


class RswaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)} ({status})"
        if status == RSWA_ECUDA:
            msg += f": {lib.rswa_last_cuda_error().decode()}"
        super().__init__(msg)


class rswa_config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_layers", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("window", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


if not os.path.exists(_LIB_PATH):
    raise ImportError(f"librswa.so is missing at {_LIB_PATH}; build it with "
                      "`python -m ring_sliding_window_b200.build` (needs nvcc)")

lib = ctypes.CDLL(_LIB_PATH)

_vp = ctypes.c_void_p
_cfgp = ctypes.POINTER(rswa_config)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)

lib.rswa_cache_bytes.argtypes = [_cfgp, _i64p]
lib.rswa_cache_bytes.restype = ctypes.c_size_t
lib.rswa_workspace_bytes.argtypes = [_cfgp, _i64p]
lib.rswa_workspace_bytes.restype = ctypes.c_size_t
lib.rswa_state_create.argtypes = [_cfgp, _i64p, _i64p, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                  _vp, ctypes.c_size_t, _vp, ctypes.POINTER(_vp)]
lib.rswa_state_destroy.argtypes = [_vp]
lib.rswa_cache_offset.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64]
lib.rswa_cache_offset.restype = ctypes.c_int64
lib.rswa_prefill.argtypes = [_vp, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp]
lib.rswa_decode_step.argtypes = [_vp, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp]
lib.rswa_advance.argtypes = [_vp, _vp]
lib.rswa_reset_ring.argtypes = [_vp, _vp]
lib.rswa_ngram_mask.argtypes = [_vp, ctypes.c_int64, _vp, ctypes.c_int64, _vp, ctypes.c_int32,
                                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp, _vp]
lib.rswa_get_ring.argtypes = [_vp, _i64p, _i32p, _i64p, _vp]
lib.rswa_check_device_error.argtypes = [_vp, _vp]
lib.rswa_decode_launch_shape.argtypes = [_vp, _i32p, _i32p]
lib.rswa_state_set_rope.argtypes = [_vp, ctypes.c_int32, ctypes.c_float, _vp]
lib.rswa_state_set_attention.argtypes = [_vp, ctypes.c_int32]
lib.rswa_decode_step_partial.argtypes = [_vp, ctypes.c_int32, _vp, _vp, _vp, ctypes.c_int64,
                                         ctypes.c_int64, _vp, _vp, _vp]
lib.rswa_combine_partials.argtypes = [_vp, _vp, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int32, _vp, _vp]
lib.rswa_ngram_topk.argtypes = [_vp, ctypes.c_int64, _vp, ctypes.c_int64, _vp, ctypes.c_int32,
                                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                ctypes.c_int32, _vp, ctypes.c_float, _vp, _vp, _vp, _vp, _vp]
lib.rswa_pool_create.argtypes = [ctypes.c_int64, ctypes.POINTER(_vp)]
lib.rswa_pool_destroy.argtypes = [_vp]
lib.rswa_pool_alloc.argtypes = [_vp, ctypes.c_int64, _i64p]
lib.rswa_pool_free.argtypes = [_vp, ctypes.c_int64]
lib.rswa_pool_stats.argtypes = [_vp, _i64p, _i64p, _i32p, _i32p]
lib.rswa_pool_capacity.argtypes = [_vp]
lib.rswa_pool_capacity.restype = ctypes.c_int64
lib.rswa_pool_cache_bytes.argtypes = [_cfgp, ctypes.c_int64]
lib.rswa_pool_cache_bytes.restype = ctypes.c_size_t
lib.rswa_state_create_pooled.argtypes = [_cfgp, _i64p, _i64p, _i64p, ctypes.c_int64,
                                         ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp,
                                         ctypes.c_size_t, _vp, ctypes.POINTER(_vp)]
lib.rswa_decode_step_noalloc.argtypes = [_cfgp, _i64p, _i64p, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.rswa_decode_step_noalloc.restype = ctypes.c_int
lib.rswa_debug_inject_fault.argtypes = [_vp, ctypes.c_int32, _vp]
lib.rswa_debug_inject_fault.restype = ctypes.c_int
lib.rswa_debug_prefill_plan.argtypes = [_vp, _vp, ctypes.c_int32, _vp, ctypes.c_int64]
lib.rswa_debug_prefill_plan.restype = ctypes.c_int64
lib.rswa_last_cuda_error.argtypes = []
lib.rswa_last_cuda_error.restype = ctypes.c_char_p
lib.rswa_status_string.argtypes = [ctypes.c_int]
lib.rswa_status_string.restype = ctypes.c_char_p
for _n in ("rswa_state_create", "rswa_state_destroy", "rswa_prefill", "rswa_decode_step",
           "rswa_advance", "rswa_reset_ring", "rswa_ngram_mask", "rswa_get_ring",
           "rswa_check_device_error", "rswa_decode_launch_shape", "rswa_pool_create",
           "rswa_pool_destroy", "rswa_pool_alloc", "rswa_pool_free", "rswa_pool_stats",
           "rswa_state_create_pooled", "rswa_ngram_topk", "rswa_state_set_rope",
           "rswa_state_set_attention", "rswa_decode_step_partial", "rswa_combine_partials"):
    getattr(lib, _n).restype = ctypes.c_int


def status_string(status: int) -> str:
    return lib.rswa_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != RSWA_OK:
        raise RswaError(status, what)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _i64(vals: Sequence[int]):
    return (ctypes.c_int64 * len(vals))(*[int(x) for x in vals])


def make_config(batch, num_layers, num_heads, head_dim, window, dtype, scale=0.0) -> rswa_config:
    d = RSWA_BF16 if dtype in (torch.bfloat16, RSWA_BF16, "bf16") else RSWA_F32
    return rswa_config(batch, num_layers, num_heads, head_dim, window, d, float(scale))


# ----------------------------------------------------------------- C names
def rswa_cache_bytes(cfg: rswa_config, prefill_len: Sequence[int]) -> int:
    return int(lib.rswa_cache_bytes(ctypes.byref(cfg), _i64(prefill_len)))


def rswa_workspace_bytes(cfg: rswa_config, prefill_len: Sequence[int]) -> int:
    return int(lib.rswa_workspace_bytes(ctypes.byref(cfg), _i64(prefill_len)))


def rswa_state_create(cfg, prefill_len, n_generated, k_cache, v_cache, workspace,
                      workspace_size, stream=None) -> ctypes.c_void_p:
    kp = (ctypes.c_void_p * len(k_cache))(*[_ptr(t).value for t in k_cache])
    vp = (ctypes.c_void_p * len(v_cache))(*[_ptr(t).value for t in v_cache])
    out = ctypes.c_void_p()
    st = lib.rswa_state_create(ctypes.byref(cfg), _i64(prefill_len),
                               None if n_generated is None else _i64(n_generated), kp, vp,
                               _ptr(workspace), int(workspace_size), _stream(stream),
                               ctypes.byref(out))
    _check(st, "rswa_state_create")
    return out


def rswa_state_create_pooled(cfg, prefill_len, n_generated, slot_base, pool_slots, k_cache,
                             v_cache, workspace, workspace_size, stream=None) -> ctypes.c_void_p:
    kp = (ctypes.c_void_p * len(k_cache))(*[_ptr(t).value for t in k_cache])
    vp = (ctypes.c_void_p * len(v_cache))(*[_ptr(t).value for t in v_cache])
    out = ctypes.c_void_p()
    st = lib.rswa_state_create_pooled(ctypes.byref(cfg), _i64(prefill_len),
                                      None if n_generated is None else _i64(n_generated),
                                      None if slot_base is None else _i64(slot_base),
                                      int(pool_slots), kp, vp, _ptr(workspace),
                                      int(workspace_size), _stream(stream), ctypes.byref(out))
    _check(st, "rswa_state_create_pooled")
    return out


def rswa_pool_cache_bytes(cfg: rswa_config, pool_slots: int) -> int:
    return int(lib.rswa_pool_cache_bytes(ctypes.byref(cfg), int(pool_slots)))


def rswa_pool_create(capacity: int) -> ctypes.c_void_p:
    out = ctypes.c_void_p()
    _check(lib.rswa_pool_create(int(capacity), ctypes.byref(out)), "rswa_pool_create")
    return out


def rswa_pool_destroy(pool) -> None:
    _check(lib.rswa_pool_destroy(pool), "rswa_pool_destroy")


def rswa_pool_alloc(pool, slots: int) -> int:
    base = ctypes.c_int64(0)
    _check(lib.rswa_pool_alloc(pool, int(slots), ctypes.byref(base)), "rswa_pool_alloc")
    return int(base.value)


def rswa_pool_free(pool, base: int) -> None:
    _check(lib.rswa_pool_free(pool, int(base)), "rswa_pool_free")


def rswa_pool_stats(pool):
    """(free_slots, largest_free_range, n_free_ranges, n_allocated)."""
    f, lg = ctypes.c_int64(0), ctypes.c_int64(0)
    nf, na = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.rswa_pool_stats(pool, ctypes.byref(f), ctypes.byref(lg), ctypes.byref(nf),
                               ctypes.byref(na)), "rswa_pool_stats")
    return int(f.value), int(lg.value), int(nf.value), int(na.value)


def rswa_pool_capacity(pool) -> int:
    return int(lib.rswa_pool_capacity(pool))


def rswa_state_destroy(state) -> None:
    _check(lib.rswa_state_destroy(state), "rswa_state_destroy")


def rswa_cache_offset(state, b: int, h: int, slot: int) -> int:
    return int(lib.rswa_cache_offset(state, b, h, slot))


def rswa_prefill(state, layer, q, k, v, out, stream=None) -> None:
    _check(lib.rswa_prefill(state, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _stream(stream)),
           "rswa_prefill")


def rswa_decode_step(state, layer, q, k_new, v_new, out, stream=None) -> None:
    _check(lib.rswa_decode_step(state, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                _stream(stream)), "rswa_decode_step")


def rswa_advance(state, stream=None) -> None:
    _check(lib.rswa_advance(state, _stream(stream)), "rswa_advance")


def rswa_reset_ring(state, stream=None) -> None:
    _check(lib.rswa_reset_ring(state, _stream(stream)), "rswa_reset_ring")


def rswa_ngram_mask(logits, history, hist_len, n: int, window: int, device_error=None,
                    stream=None, vocab: Optional[int] = None) -> None:
    """logits: cuda float32 [rows, ld]; history: cuda int32 [rows, hist_ld]."""
    rows = logits.shape[0]
    ld = logits.stride(0) if rows else logits.shape[1]
    vocab = logits.shape[1] if vocab is None else vocab
    hist_ld = history.stride(0) if rows else window
    _check(lib.rswa_ngram_mask(_ptr(logits), ld, _ptr(history), hist_ld, _ptr(hist_len), rows,
                               vocab, n, window, _ptr(device_error), _stream(stream)),
           "rswa_ngram_mask")


def rswa_ngram_topk(logits, history, hist_len, n: int, window: int, k: int, mask_in_place=False,
                    uniform=None, temperature: float = 1.0, top_idx=None, top_val=None,
                    token=None, device_error=None, stream=None, vocab: Optional[int] = None):
    """Fused n-gram ban + top-k (+ sampling).  logits: cuda float32 [rows, ld];
    history: cuda int32 [rows, hist_ld].  Outputs are allocated when not given;
    returns (top_idx [rows, k] int32, top_val [rows, k] float32, token [rows] int32)."""
    rows = logits.shape[0]
    ld = logits.stride(0) if rows else logits.shape[1]
    vocab = logits.shape[1] if vocab is None else vocab
    hist_ld = history.stride(0) if rows else window
    dev = logits.device
    if top_idx is None:
        top_idx = torch.empty(rows, k, dtype=torch.int32, device=dev)
    if top_val is None:
        top_val = torch.empty(rows, k, dtype=torch.float32, device=dev)
    if token is None:
        token = torch.empty(rows, dtype=torch.int32, device=dev)
    _check(lib.rswa_ngram_topk(_ptr(logits), ld, _ptr(history), hist_ld, _ptr(hist_len), rows,
                               vocab, n, window, k, int(bool(mask_in_place)), _ptr(uniform),
                               float(temperature), _ptr(top_idx), _ptr(top_val), _ptr(token),
                               _ptr(device_error), _stream(stream)), "rswa_ngram_topk")
    return top_idx, top_val, token


def rswa_get_ring(state, batch: int, stream=None):
    """Returns (n_generated[B], ring_pos[B], cache_len[B]) as Python lists."""
    n = (ctypes.c_int64 * batch)()
    rp = (ctypes.c_int32 * batch)()
    cl = (ctypes.c_int64 * batch)()
    _check(lib.rswa_get_ring(state, n, rp, cl, _stream(stream)), "rswa_get_ring")
    return list(n), list(rp), list(cl)


def rswa_state_set_rope(state, policy: int, theta: float = 10000.0, stream=None) -> None:
    _check(lib.rswa_state_set_rope(state, int(policy), float(theta), _stream(stream)),
           "rswa_state_set_rope")


def rswa_state_set_attention(state, mode: int) -> None:
    _check(lib.rswa_state_set_attention(state, int(mode)), "rswa_state_set_attention")


def rswa_decode_step_partial(state, layer, q, k_new, v_new, key_lo, key_hi, part_ml, part_o,
                             stream=None) -> None:
    """Decode over cache slots [key_lo, key_hi): part_ml float32 [B, H, 2] (m, l),
    part_o float32 [B, H, d] (unnormalised)."""
    _check(lib.rswa_decode_step_partial(state, layer, _ptr(q), _ptr(k_new), _ptr(v_new),
                                        int(key_lo), int(key_hi), _ptr(part_ml), _ptr(part_o),
                                        _stream(stream)), "rswa_decode_step_partial")


def rswa_combine_partials(part_ml, part_o, out, stream=None) -> None:
    """part_ml [G, B, H, 2], part_o [G, B, H, d] (float32) -> out [B, H, d]."""
    G = part_ml.shape[0]
    rings = part_ml[0].numel() // 2
    d = part_o.shape[-1]
    dt = RSWA_BF16 if out.dtype == torch.bfloat16 else RSWA_F32
    _check(lib.rswa_combine_partials(_ptr(part_ml), _ptr(part_o), G, rings, d, dt, _ptr(out),
                                     _stream(stream)), "rswa_combine_partials")


def rswa_decode_launch_shape(state):
    """(grid, cluster_size) of this state's decode launches; cluster_size 0 = stream-K split."""
    g, c = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.rswa_decode_launch_shape(state, ctypes.byref(g), ctypes.byref(c)),
           "rswa_decode_launch_shape")
    return int(g.value), int(c.value)


def rswa_check_device_error(state, stream=None) -> int:
    """Returns the status (does not raise): RSWA_OK, RSWA_ETIMEOUT or RSWA_EDEVICE."""
    return int(lib.rswa_check_device_error(state, _stream(stream)))


def rswa_decode_step_noalloc(cfg: rswa_config, prefill_len, n_generated, k_cache, v_cache,
                             q, k_new, v_new, out, device_error=None, stream=None) -> None:
    """One layer's decode step with scratch in the library's static device array
    (for callers that cannot allocate a workspace); t_b passed explicitly."""
    _check(lib.rswa_decode_step_noalloc(ctypes.byref(cfg), _i64(prefill_len), _i64(n_generated),
                                        _ptr(k_cache), _ptr(v_cache), _ptr(q), _ptr(k_new),
                                        _ptr(v_new), _ptr(out), _ptr(device_error),
                                        _stream(stream)), "rswa_decode_step_noalloc")


def rswa_debug_prefill_plan(batch, num_heads, head_dim, window, dtype, prefill_lens,
                            num_sms: int):
    """Test-only: the tensor-core prefill's blocks for this batch on a part
    with `num_sms` SMs, in launch order, as a list of (b, h, first query tile,
    query tiles).  Host only."""
    import numpy as np
    cfg = make_config(batch, 1, num_heads, head_dim, window, dtype)
    pl = (ctypes.c_int64 * batch)(*[int(p) for p in prefill_lens])
    n = lib.rswa_debug_prefill_plan(ctypes.byref(cfg), pl, int(num_sms), None, 0)
    if n < 0:
        raise RswaError(RSWA_EINVAL, "rswa_debug_prefill_plan")
    out = np.zeros((max(int(n), 1), 4), dtype=np.int32)
    lib.rswa_debug_prefill_plan(ctypes.byref(cfg), pl, int(num_sms), out.ctypes.data, int(n))
    return [tuple(int(x) for x in row) for row in out[:n]]


def rswa_debug_inject_fault(state, flags: int, stream=None) -> None:
    """Test-only: make this state's decode kernels drop their copies (their
    bounded waits then run out and report RSWA_ETIMEOUT); 0 restores."""
    _check(lib.rswa_debug_inject_fault(state, int(flags), _stream(stream)), "rswa_debug_inject_fault")


# ---------------------------------------------------------- owning helper
class State:
    """A batch's caches + workspace (torch-allocated) and its rswa_state."""

    def __init__(self, batch, num_layers, num_heads, head_dim, window, prefill_lens,
                 dtype=torch.bfloat16, n_generated=None, scale=0.0, device="cuda", stream=None,
                 pool=None, slot_base=None):
        self.cfg = make_config(batch, num_layers, num_heads, head_dim, window, dtype, scale)
        self.dtype = torch.bfloat16 if self.cfg.dtype == RSWA_BF16 else torch.float32
        self.prefill_lens = [int(p) for p in prefill_lens]
        self.B, self.L, self.H, self.d, self.W = batch, num_layers, num_heads, head_dim, window
        wb = rswa_workspace_bytes(self.cfg, self.prefill_lens)
        if wb == 0:
            raise RswaError(RSWA_EINVAL, "rswa_workspace_bytes")
        self.workspace = torch.empty(wb, dtype=torch.uint8, device=device)
        if pool is not None:
            # requests placed in a TokenPool's caches at the given slot bases
            self.k_cache, self.v_cache = pool.k_cache, pool.v_cache
            self.slot_base = [int(x) for x in slot_base]
            self.handle = rswa_state_create_pooled(self.cfg, self.prefill_lens, n_generated,
                                                   self.slot_base, pool.capacity, self.k_cache,
                                                   self.v_cache, self.workspace, wb, stream)
            return
        cb = rswa_cache_bytes(self.cfg, self.prefill_lens)
        if cb == 0:
            raise RswaError(RSWA_EINVAL, "rswa_cache_bytes")
        elems = cb // (2 if self.dtype == torch.bfloat16 else 4)
        self.k_cache = [torch.empty(elems, dtype=self.dtype, device=device) for _ in range(num_layers)]
        self.v_cache = [torch.empty(elems, dtype=self.dtype, device=device) for _ in range(num_layers)]
        self.handle = rswa_state_create(self.cfg, self.prefill_lens, n_generated, self.k_cache,
                                        self.v_cache, self.workspace, wb, stream)

    def close(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            rswa_state_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def cache_view(self, layer: int, which: str, b: int, h: int) -> torch.Tensor:
        """[P_b + W, d] view of one (b, h) ring of a layer's K or V cache."""
        off = rswa_cache_offset(self.handle, b, h, 0)
        n = (self.prefill_lens[b] + self.W) * self.d
        buf = (self.k_cache if which == "k" else self.v_cache)[layer]
        return buf[off:off + n].view(self.prefill_lens[b] + self.W, self.d)

    def prefill(self, layer, q, k, v, out, stream=None):
        rswa_prefill(self.handle, layer, q, k, v, out, stream)

    def decode_step(self, layer, q, k_new, v_new, out, stream=None):
        rswa_decode_step(self.handle, layer, q, k_new, v_new, out, stream)

    def advance(self, stream=None):
        rswa_advance(self.handle, stream)

    def reset_ring(self, stream=None):
        rswa_reset_ring(self.handle, stream)

    def ring(self, stream=None):
        return rswa_get_ring(self.handle, self.B, stream)

    def check(self, stream=None) -> int:
        return rswa_check_device_error(self.handle, stream)

    def decode_launch_shape(self):
        return rswa_decode_launch_shape(self.handle)

    def set_rope(self, policy: int, theta: float = 10000.0, stream=None):
        rswa_state_set_rope(self.handle, policy, theta, stream)

    def set_attention(self, mode: int):
        rswa_state_set_attention(self.handle, mode)

    def decode_step_partial(self, layer, q, k_new, v_new, key_lo, key_hi, part_ml, part_o,
                            stream=None):
        rswa_decode_step_partial(self.handle, layer, q, k_new, v_new, key_lo, key_hi, part_ml,
                                 part_o, stream)


class TokenPool:
    """One K/V pool per layer (torch-allocated) and the slot-range allocator:
    requests join with `alloc(prefill_len)` and leave with `free(base)`; a
    `State` over any set of live requests is built with `state(...)`."""

    def __init__(self, capacity, num_layers, num_heads, head_dim, window, dtype=torch.bfloat16,
                 device="cuda"):
        self.capacity = int(capacity)
        self.L, self.H, self.d, self.W = num_layers, num_heads, head_dim, window
        self.dtype = dtype
        cfg = make_config(1, num_layers, num_heads, head_dim, window, dtype)
        cb = rswa_pool_cache_bytes(cfg, self.capacity)
        if cb == 0:
            raise RswaError(RSWA_EINVAL, "rswa_pool_cache_bytes")
        elems = cb // (2 if dtype == torch.bfloat16 else 4)
        self.k_cache = [torch.empty(elems, dtype=dtype, device=device) for _ in range(num_layers)]
        self.v_cache = [torch.empty(elems, dtype=dtype, device=device) for _ in range(num_layers)]
        self.handle = rswa_pool_create(self.capacity)

    def alloc(self, prefill_len: int) -> int:
        return rswa_pool_alloc(self.handle, int(prefill_len) + self.W)

    def free(self, base: int) -> None:
        rswa_pool_free(self.handle, base)

    def stats(self):
        return rswa_pool_stats(self.handle)

    def state(self, prefill_lens, slot_bases, n_generated=None, stream=None, scale=0.0) -> State:
        return State(len(prefill_lens), self.L, self.H, self.d, self.W, prefill_lens,
                     dtype=self.dtype, n_generated=n_generated, scale=scale, stream=stream,
                     pool=self, slot_base=slot_bases)

    def close(self):
        h, self.handle = getattr(self, "handle", None), None
        if h:
            rswa_pool_destroy(h)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
