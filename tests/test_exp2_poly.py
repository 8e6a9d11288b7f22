"""CPU check of the FMA-pipe exp2 used for a quarter of the softmax exponentials in
the tensor-core attention kernel: the same float32 operation sequence as the kernel
(round-to-nearest split through the 1.5 * 2^23 shift, cubic on [-1/2, 1/2], exponent
add), with the kernel's own constants read from its source, against numpy's exp2."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_chunk_ring_b200", "csrc", "attn_sm100.cu")


def _coeffs():
    text = open(SRC).read()
    m = re.search(r"kExpC1 = ([0-9.e-]+)f, kExpC2 = ([0-9.e-]+)f, kExpC3 = ([0-9.e-]+)f", text)
    return [np.float32(float(x)) for x in m.groups()]


def ex2_fma_f32(x):
    c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    f = (x - (t - shift)).astype(np.float32)
    p = (np.float32(1.0) + f * (c1 + f * (c2 + f * c3))).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-120.0, 8.0, 400001).astype(np.float32)
    y = ex2_fma_f32(x)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.2e-4          # below bf16's 2^-9 relative rounding of P


def test_integers_exact_and_masked_zero():
    n = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(ex2_fma_f32(n), np.exp2(n))
    z = ex2_fma_f32(np.array([-np.inf, -127.0, -1000.0], np.float32))
    assert np.all(z == 0.0)
