"""The FMA-pipe exp2 used for a share of the softmax, emulated in float32.

The kernel's constants are read from its source, so this checks the very
coefficients the kernel uses: range reduction x = n + f (n = round(x) via the
1.5 * 2^23 trick), the fitted cubic for 2^f, and 2^n applied through the
exponent bits.  Bound: 1.2e-4 relative error on [-126, 8], far below the
2^-9 relative rounding that P receives when it is stored as bf16.
"""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_threshold_b200", "csrc", "ptx.cuh")


def _constants():
    text = open(SRC).read()
    body = text[text.index("exp2_fma_pair"):]
    get = lambda name: float(re.search(name + r"\s*=\s*([0-9.eE+-]+)f", body).group(1))
    return get("kMagic"), get("kC1"), get("kC2"), get("kC3")


def _emulate(x):
    f32 = np.float32
    magic, c1, c2, c3 = (f32(v) for v in _constants())
    xc = np.maximum(x, f32(-126))
    t = (xc + magic).astype(f32)
    r = (t + (-magic)).astype(f32)
    f = (r * f32(-1) + xc).astype(f32)
    q = (c3 * f + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + f32(1)).astype(f32)
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(f32), f


def test_fma_exp2_error_bound():
    x = np.linspace(-126, 8, 1_000_001, dtype=np.float32)
    p, f = _emulate(x)
    assert f.min() >= -0.5 and f.max() <= 0.5
    rel = np.abs(p.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4


def test_fma_exp2_exact_at_integers_and_clamped_below():
    x = np.arange(-126, 9, dtype=np.float32)
    p, _ = _emulate(x)
    assert np.array_equal(p, np.exp2(x.astype(np.float64)).astype(np.float32))
    tiny, _ = _emulate(np.array([-1000.0, -np.inf], dtype=np.float32))
    assert np.all(tiny == np.float32(2.0 ** -126))


def test_fit_script_reproduces_the_constants():
    import importlib.util
    path = os.path.join(os.path.dirname(SRC), "fit_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c = mod.fit()
    _, c1, c2, c3 = _constants()
    assert np.allclose(c, [c1, c2, c3], rtol=1e-6)
    assert mod.max_rel_error(c) < 1.2e-4
