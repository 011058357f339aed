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
