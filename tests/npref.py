"""Independent numpy restatement of the layer, used only to pin the oracle.

It is written separately from the C oracle (different language, vectorised
numpy, its own int4 decoding) so that a mistake in one is unlikely to be
repeated in the other.  Readings follow the C-ABI header: low nibble = even
element, two's-complement codes, one bf16 scale per 64 elements of a row.
"""
import numpy as np


def bf16_bits_to_f64(bits):
    bits = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def dequant(q, s_bits):
    """[rows][K/2] uint8 + [rows][K/64] bf16 bits -> [rows][K] float64."""
    q = np.asarray(q, dtype=np.uint8)
    lo = (q & 0x0F).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    codes = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.float64)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    scale = np.repeat(bf16_bits_to_f64(s_bits), 64, axis=1)
    return codes * scale


def swiglu_mlp(ex, x):
    """Dense SwiGLU MLP with numpy matmuls: x [..., H] float64 -> [..., H]."""
    wg = dequant(ex["gate_q"], ex["gate_s"])
    wu = dequant(ex["up_q"], ex["up_s"])
    wd = dequant(ex["down_q"], ex["down_s"])
    g = x @ wg.T
    u = x @ wu.T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ wd.T


def dequant_rows(q, s_bits):
    """Per-row int4: [rows][K/2] uint8 + [rows][1] bf16 bits -> [rows][K]."""
    q = np.asarray(q, dtype=np.uint8)
    lo = (q & 0x0F).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    codes = np.empty((q.shape[0], q.shape[1] * 2), dtype=np.float64)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    return codes * bf16_bits_to_f64(np.asarray(s_bits).reshape(-1, 1))


def swiglu_mlp_rows(ex, x):
    """Dense SwiGLU MLP of a per-row int4 expert, numpy matmuls."""
    wg = dequant_rows(ex["gate_q"], ex["gate_s"])
    wu = dequant_rows(ex["up_q"], ex["up_s"])
    wd = dequant_rows(ex["down_q"], ex["down_s"])
    g = x @ wg.T
    u = x @ wu.T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ wd.T
