"""Accuracy of the attention kernel's FMA-pipe exponential (exp2_poly in
k_umma_attn.cu): Cody-Waite style range reduction, 2^y = 2^j * 2^f with j = round(y)
taken by the 1.5 * 2^23 shift and f in [-1/2, 1/2], then a degree-3 polynomial for
2^f.  The steps are replayed here in float32 with the coefficients read from the
kernel source, over the argument range the softmax uses, against float64 2^y."""
import pathlib
import re

import numpy as np

SRC = pathlib.Path(__file__).resolve().parents[1] / "linear_attention_paged_b200" / "csrc" / "k_umma_attn.cu"


def _coefficients():
    body = SRC.read_text()
    body = body[body.index("float2 exp2_poly(float2 y)"):]
    body = body[:body.index("return make_float2")]
    nums = [float(x) for x in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    nums = [x for x in nums if x != 12582912.0]   # the rounding shift, not a coefficient
    # Horner order in the source: c3, c2, then c1, then c0
    assert len(nums) == 4, nums
    return nums


def _exp2_poly(y):
    f32 = np.float32
    c3, c2, c1, c0 = (f32(c) for c in _coefficients())
    y = np.maximum(y.astype(f32), f32(-125.0))
    t = (y + f32(12582912.0)).astype(f32)
    jf = (t + f32(-12582912.0)).astype(f32)
    f = (y - jf).astype(f32)
    q = (c3 * f + c2).astype(f32)
    q = (q * f + c1).astype(f32)
    q = (q * f + c0).astype(f32)
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error():
    # the softmax evaluates 2^(s * log2(e)/sqrt(d) - m) with the stale max m at most
    # 2^8 below the true one, so arguments lie in (-inf, 8]; below -125 the result
    # is clamped to 2^-125 (about 2e-38, zero for every later use)
    y = np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float64).astype(np.float32)
    got = _exp2_poly(y).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4          # bf16 keeps 8 bits: P's own rounding is 2^-9
    assert np.all(got > 0)


def test_exp2_poly_integers_and_clamp():
    y = np.arange(-125, 9, dtype=np.float32)
    got = _exp2_poly(y).astype(np.float64)
    assert np.allclose(got, np.exp2(y.astype(np.float64)), rtol=1e-4, atol=0)
    far = _exp2_poly(np.array([-300.0, -1e6], dtype=np.float32))
    assert np.all(far > 0) and np.all(far < 1e-37)
