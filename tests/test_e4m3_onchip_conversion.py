"""The integer e4m3 -> fp32 step the on-chip weight converters use (CPU).

The converters of the e4m3-weight GEMMs (mla_set_e4m3_weight_conversion) turn
a code c into fp32 bits ((c & 0x80) << 24) | ((c & 0x7F) << 20), read them as
a float, and multiply by 2^120 and the block scale. This checks that step
against the oracle's e4m3 decode for every finite code, subnormals and both
zeros included, in numpy float32 arithmetic (the GPU path is checked bit for
bit against the dequantising path in tests/test_gpu_parity.py). The format's
two NaN codes are outside a saturating quantizer's output and are excluded.
"""
import math

import numpy as np

import oracle


def _converted(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.uint32)
    bits = ((c & np.uint32(0x80)) << np.uint32(24)) | ((c & np.uint32(0x7F)) << np.uint32(20))
    return bits.view(np.float32) * np.float32(2.0 ** 120)


def test_every_finite_code_converts_exactly():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    got = _converted(codes).astype(np.float64)
    want = np.array([oracle.e4m3_to_double(int(c)) for c in codes])
    assert np.all(got == want), [(int(c), g, w) for c, g, w in zip(codes, got, want) if g != w][:5]
    # signs of the zeros survive
    assert math.copysign(1.0, float(_converted(np.array([0x80], dtype=np.uint8))[0])) == -1.0


def test_scaled_product_rounds_like_the_dequantised_copy():
    # bf16(code * s) with the fp32 product rounded once: the same value the
    # dequantising kernel stores, for random codes and scales.
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, 4096).astype(np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]
    scales = (rng.uniform(0.5, 2.0, codes.size) * 2.0 ** rng.integers(-20, 4, codes.size)).astype(np.float32)
    conv = _converted(codes) * scales  # float32 multiply
    ref = np.array([oracle.e4m3_to_double(int(c)) for c in codes]).astype(np.float32) * scales
    assert np.array_equal(conv.view(np.uint32), ref.view(np.uint32))
