"""The C ABI: the library loads, exports every call include/rswa.h declares,
and the host-side checks reject bad arguments before anything is launched."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rswa.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rswa_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def rswa():
    from ring_sliding_window_b200 import build
    build.build()
    from ring_sliding_window_b200 import rswa as mod
    return mod


def test_exports_every_declared_symbol(rswa):
    declared = _declared()
    assert len(declared) >= 13
    for name in declared:
        assert hasattr(rswa.lib, name), name
    assert set(declared) == set(rswa.EXPORTED)


def test_status_strings(rswa):
    for s in range(7):
        assert rswa.status_string(s)
    assert rswa.status_string(99) == "unknown status"


def test_cache_bytes_host_only(rswa):
    cfg = rswa.make_config(2, 12, 10, 128, 128, torch.bfloat16)
    assert rswa.rswa_cache_bytes(cfg, [1088, 10]) == (1088 + 128 + 10 + 128) * 10 * 128 * 2
    cfg32 = rswa.make_config(1, 1, 2, 64, 8, torch.float32)
    assert rswa.rswa_cache_bytes(cfg32, [64]) == 72 * 2 * 64 * 4


@pytest.mark.parametrize("field,value", [("batch", 0), ("num_layers", 0), ("num_heads", 0),
                                         ("head_dim", 96), ("window", 0), ("dtype", 7),
                                         ("scale", -1.0)])
def test_bad_config_rejected(rswa, field, value):
    cfg = rswa.make_config(1, 1, 2, 64, 8, torch.float32)
    setattr(cfg, field, value)
    assert rswa.rswa_cache_bytes(cfg, [64]) == 0
    assert rswa.rswa_workspace_bytes(cfg, [64]) == 0
    with pytest.raises(rswa.RswaError) as e:
        rswa.rswa_state_create(cfg, [64], None, [1 << 20], [1 << 20], 1 << 20, 1 << 20, 0)
    assert e.value.status == rswa.RSWA_EINVAL


def test_bad_lengths_rejected(rswa):
    cfg = rswa.make_config(2, 1, 2, 64, 8, torch.float32)
    assert rswa.rswa_cache_bytes(cfg, [64, -1]) == 0
    assert rswa.rswa_cache_bytes(cfg, [64, (1 << 31) - 8]) == 0


def test_null_and_misaligned_pointers_rejected(rswa):
    cfg = rswa.make_config(1, 2, 2, 64, 8, torch.float32)
    for kp, vp, ws in [([0, 4096], [4096, 4096], 1 << 20), ([4096, 4096], [4096, 4104], 1 << 20),
                       ([4096, 4096], [4096, 4096], 0), ([4096, 4096], [4096, 4096], (1 << 20) + 16)]:
        with pytest.raises(rswa.RswaError) as e:
            rswa.rswa_state_create(cfg, [64], None, kp, vp, ws, 1 << 20, 0)
        assert e.value.status == rswa.RSWA_EINVAL
    with pytest.raises(rswa.RswaError) as e:
        rswa.rswa_state_create(cfg, [64], [-1], [4096, 4096], [4096, 4096], 1 << 20, 1 << 20, 0)
    assert e.value.status == rswa.RSWA_EINVAL


def test_null_state_and_ngram_args_rejected(rswa):
    lib = rswa.lib
    assert lib.rswa_prefill(None, 0, None, None, None, None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_decode_step(None, 0, None, None, None, None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_advance(None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_reset_ring(None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_check_device_error(None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_decode_launch_shape(None, None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_state_destroy(None) == rswa.RSWA_EINVAL
    assert lib.rswa_cache_offset(None, 0, 0, 0) == -1
    # rows < 0, vocab < 1, n < 1, ld < vocab, hist_ld < window, null logits
    bad = [(-1, 10, 2, 10, 4), (1, 0, 2, 10, 4), (1, 10, 0, 10, 4), (1, 10, 2, 9, 4)]
    for rows, vocab, n, ld, w in bad:
        assert lib.rswa_ngram_mask(4096, ld, 4096, w, None, rows, vocab, n, w, None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_ngram_mask(4096, 10, 4096, 3, None, 1, 10, 2, 4, None, None) == rswa.RSWA_EINVAL
    assert lib.rswa_ngram_mask(None, 10, 4096, 4, None, 1, 10, 2, 4, None, None) == rswa.RSWA_EINVAL
    # zero rows: valid no-op, nothing launched
    assert lib.rswa_ngram_mask(None, 10, None, 4, None, 0, 10, 2, 4, None, None) == rswa.RSWA_OK


def test_topk_combine_and_setter_args_rejected(rswa):
    """The later entry points check their arguments on the host and return
    RSWA_EINVAL before any launch (or RSWA_OK for an empty call)."""
    lib = rswa.lib
    E, OK = rswa.RSWA_EINVAL, rswa.RSWA_OK
    A = 4096  # a 16-byte-aligned stand-in address: never dereferenced on these paths

    def topk(logits=A, ld=16, hist=A, hist_ld=4, rows=1, vocab=16, n=2, window=4, k=2,
             uniform=None, temperature=1.0, top_idx=A):
        return lib.rswa_ngram_topk(logits, ld, hist, hist_ld, None, rows, vocab, n, window, k, 0,
                                   uniform, temperature, top_idx, None, None, None, None)

    for kw in (dict(rows=-1), dict(vocab=0), dict(vocab=rswa.RSWA_TOPK_MAX_VOCAB + 1, ld=1 << 20),
               dict(n=0), dict(window=-1), dict(k=0), dict(k=rswa.RSWA_TOPK_MAX + 1, vocab=128, ld=128),
               dict(k=17), dict(ld=15), dict(ld=18), dict(hist_ld=3), dict(window=8193, hist_ld=8193),
               dict(uniform=A, temperature=0.0), dict(uniform=A, temperature=float("inf")),
               dict(logits=None), dict(logits=A + 4), dict(top_idx=None), dict(hist=None)):
        assert topk(**kw) == E, kw
    assert topk(rows=0, logits=None, top_idx=None) == OK  # empty: nothing launched

    def combine(ml=A, o=A, shares=2, rings=3, d=128, dtype=rswa.RSWA_BF16, out=A):
        return lib.rswa_combine_partials(ml, o, shares, rings, d, dtype, out, None)

    for kw in (dict(shares=0), dict(rings=-1), dict(d=96), dict(dtype=7), dict(ml=None),
               dict(o=None), dict(out=None)):
        assert combine(**kw) == E, kw
    assert combine(rings=0, ml=None, o=None, out=None) == OK

    assert lib.rswa_state_set_rope(None, 1, 10000.0, None) == E
    assert lib.rswa_state_set_attention(None, 1) == E
    assert lib.rswa_decode_step_partial(None, 0, A, A, A, 0, 10, A, A, None) == E
