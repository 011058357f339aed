"""The software exp2 of the prefill softmax (FMA pipe): its constants are the
ones the Remez derivation in csrc/gen_exp2_poly.py produces, and the whole
function (range reduction + polynomial + exponent add), emulated in float32
with the kernel's operation order, stays within its stated error bound."""
import os
import re

import numpy as np

from ring_sliding_window_b200.csrc import gen_exp2_poly as gen

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "ring_sliding_window_b200", "csrc", "tcgen05.cuh")


def _kernel_constants():
    src = open(HDR).read()
    vals = {}
    for i in range(4):
        m = re.search(rf"kExp2C{i}\s*=\s*([0-9a-fx.p+-]+)f;", src)
        vals[i] = np.float32(float.fromhex(m.group(1)))
    return np.array([vals[i] for i in range(4)], dtype=np.float32)


def test_constants_match_remez_derivation():
    c32, err = gen.coefficients()
    assert np.array_equal(_kernel_constants().view(np.uint32), c32.view(np.uint32))
    assert err < 1e-4


def _exp2_fma_emulated(x):
    """float32 emulation of tc::exp2_fma (same operations, same order)."""
    c = _kernel_constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = gen.eval_kernel_order(c, f)
    ji = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (ji << 23)).view(np.float32)


def test_software_exp2_error_bound():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001), np.arange(-125, 9, 0.5)]).astype(np.float32)
    y = _exp2_fma_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() < 1e-4, rel.max()


def test_software_exp2_masked_inputs_are_negligible():
    y = _exp2_fma_emulated(np.array([-np.inf, -1e30, -200.0, -126.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y <= np.float32(2.0 ** -124))
