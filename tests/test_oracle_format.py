"""Oracle pins: int4 gs64 decoding against hand-packed bytes."""
import os

import numpy as np
import pytest

import oracle
from npref import bf16_bits_to_f64, dequant

GOLD = os.path.join(os.path.dirname(__file__), "golden", "int4_decode.txt")


def _golden_rows():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, s, ce, co, ve, vo = line.split()
        rows.append((int(b, 16), int(s, 16), int(ce), int(co), float(ve), float(vo)))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_hand_packed_bytes(row):
    byte, sbits, ce, co, ve, vo = row
    q = np.array([byte] * 32, dtype=np.uint8)           # one 64-element group
    s = np.array([sbits], dtype=np.uint16)
    assert list(oracle.int4_codes(q, 2)) == [ce, co]
    assert oracle.weight(q, s, 64, 0, 0) == ve
    assert oracle.weight(q, s, 64, 0, 1) == vo
    assert oracle.weight(q, s, 64, 0, 62) == ve
    assert oracle.weight(q, s, 64, 0, 63) == vo


def test_bf16_conversion_known_bits():
    assert oracle.bf16_to_double(0x3F80) == 1.0
    assert oracle.bf16_to_double(0x3F00) == 0.5
    assert oracle.bf16_to_double(0xC000) == -2.0
    assert oracle.bf16_to_double(0x3C80) == 2.0 ** -6
    assert oracle.bf16_to_double(0x0000) == 0.0
    assert np.isinf(oracle.bf16_to_double(0x7F80))
    # smallest bf16 above 1: 1 + 2^-7
    assert oracle.bf16_to_double(0x3F81) == 1.0 + 2.0 ** -7


def test_pack_unpack_roundtrip_all_bytes():
    q = np.arange(256, dtype=np.uint8)
    codes = oracle.int4_codes(q, 512)
    assert codes.min() == -8 and codes.max() == 7
    assert np.array_equal(oracle.int4_pack(codes), q)


def test_scale_group_index():
    # 2 rows x 128 elements: row 1 group 1 has its own scale; all codes = 1
    q = np.full((2, 64), 0x11, dtype=np.uint8)
    s = np.array([[0x3F80, 0x4000], [0x4040, 0x4080]], dtype=np.uint16)  # 1, 2, 3, 4
    assert oracle.weight(q, s, 128, 0, 63) == 1.0
    assert oracle.weight(q, s, 128, 0, 64) == 2.0
    assert oracle.weight(q, s, 128, 1, 0) == 3.0
    assert oracle.weight(q, s, 128, 1, 127) == 4.0


def test_matches_numpy_dequant_random():
    rng = np.random.default_rng(3)
    q = rng.integers(0, 256, size=(3, 64), dtype=np.uint8)
    s = (rng.uniform(0.005, 0.02, size=(3, 2)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    W = dequant(q, s)
    for n in range(3):
        for k in (0, 1, 2, 63, 64, 65, 127):
            assert oracle.weight(q, s, 128, n, k) == W[n, k]
    assert np.all(bf16_bits_to_f64(s) > 0)
