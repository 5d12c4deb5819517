"""The fp16 arithmetic the tensor-core path uses to turn an int4 code and its
bf16 scale into the MMA operand q * s, checked exhaustively on the host for
every code and every bf16 scale from 2^-13 to 1: each step must be exact, so
the operand equals q * s exactly (an inexact shortcut, such as one fused
multiply-add with a -72 s addend, fails here)."""
import numpy as np


def _bf16_scales(lo_bits=0x3900, hi_bits=0x3F80):
    b = np.arange(lo_bits, hi_bits, dtype=np.uint32) << 16
    return b.view(np.float32)


def test_dequant_steps_exact_for_all_codes_and_scales():
    codes = np.arange(-8, 8)
    # the unpack's magic values: even codes as 1032 + q, odd codes as 1152 + 16 q
    t_even = (np.float16(1032) + codes.astype(np.float16))
    t_odd = (np.float16(1152) + (16 * codes).astype(np.float16))
    assert np.array_equal(t_even.astype(np.float64), 1032 + codes)
    assert np.array_equal(t_odd.astype(np.float64), 1152 + 16 * codes)
    for s in _bf16_scales():                  # 2^-13 <= s < 1
        s2 = np.float16(s)
        s16 = np.float16(np.float32(s) * np.float32(0.0625))
        assert float(s2) == float(s) and float(s16) == float(s) / 16
        v_even = (t_even - np.float16(1032)) * s2
        v_odd = (t_odd - np.float16(1152)) * s16
        ref = codes * np.float64(s)
        assert np.array_equal(v_even.astype(np.float64), ref), s
        assert np.array_equal(v_odd.astype(np.float64), ref), s


def test_single_fma_shortcut_is_not_exact():
    """fma(1152 + 16 q, s / 16, -72 s) would need -72 s exactly in fp16, which
    takes up to 12 significant bits: it fails for some scales."""
    bad = 0
    for s in _bf16_scales(0x3B00, 0x3C00):
        c72 = np.float16(-72.0 * np.float64(s))
        bad += float(c72) != -72.0 * float(s)
    assert bad > 0
