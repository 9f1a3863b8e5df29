"""Arithmetic behind the f16 activation path of the tensor engine, checked on
the CPU over every bf16 value.

The pre-pass scales each activation row by 2^sh, where sh = 141 - E (E is
the biased exponent of the row's largest finite magnitude), clamped to at
most 126, and rounds to f16.  The epilogue multiplies by 2^-sh.  The claims
(stated with the kernel) are:
  - the row maximum lands in [2^14, 2^15) unless the clamp applies;
  - every bf16 value whose scaled magnitude is at least 2^-17 converts to
    f16 exactly, and smaller ones are off by at most 2^-25;
  - both factors are normal fp32 numbers, so the scaling is exact while
    the results stay normal.
"""
import numpy as np


def bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return v[np.isfinite(v)]


def biased_exponent(x):
    return int((np.float32(x).view(np.uint32) >> 23) & 0xFF)


def shift_for(max_abs):
    """The pre-pass's rule: sh = 141 - E (E >= 1), at most 126; 0 for a zero row."""
    return 0 if max_abs == 0 else min(141 - max(biased_exponent(max_abs), 1), 126)


def test_row_maximum_lands_in_range():
    v = bf16_values()
    for m in np.unique(np.abs(v[v != 0])):
        sh = shift_for(m)
        scaled = np.float64(m) * 2.0 ** sh
        if 141 - max(biased_exponent(m), 1) <= 126:
            assert 2.0 ** 14 <= scaled < 2.0 ** 15, (m, sh)
        else:  # maxima below 2^-112: the clamp keeps 2^sh a normal fp32 number
            assert scaled < 2.0 ** 15
        # both factors 2^sh and 2^-sh are normal fp32 numbers (exact scaling)
        assert -126 <= sh <= 127 and -126 <= -sh <= 127


def test_conversion_exact_above_the_subnormal_grid():
    v = bf16_values().astype(np.float64)
    for sh in (-113, -40, -8, 0, 7, 30, 90, 126):
        s = v * 2.0 ** sh
        s = s[np.abs(s) < 65504.0]
        h = s.astype(np.float16).astype(np.float64)
        big = np.abs(s) >= 2.0 ** -17
        assert np.array_equal(h[big], s[big]), sh
        assert np.max(np.abs(h[~big] - s[~big]), initial=0.0) <= 2.0 ** -25, sh


def test_epilogue_undoes_the_scaling_exactly():
    """Exact while the product stays a normal fp32 number (a result in the
    fp32 subnormal range rounds there on either path)."""
    rng = np.random.default_rng(0)
    for sh in (-113, -20, 0, 5, 100):
        t = rng.standard_normal(1000).astype(np.float32) * np.float32(2.0 ** 10)
        inv = np.float32(2.0 ** -sh)
        back = (t * inv).astype(np.float64)
        assert np.all(np.abs(back) >= 2.0 ** -126)
        assert np.array_equal(back, t.astype(np.float64) * 2.0 ** -sh)
