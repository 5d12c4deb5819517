"""CPU oracle for the routed int4 gs64 MoE layer (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference leg may import this package.  The product path
(the CUDA library and its binding) never imports it and shares no code with it.

The arithmetic lives in ``coli_oracle.c`` (plain C, double precision, per
token); this module compiles it with gcc on first use and marshals numpy
arrays through ctypes.  See that file's header for what each function
computes and the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "coli_oracle.c")
_LIB = os.path.join(_HERE, "libcoli_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no vector or fast-math flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared", "-o", tmp,
                        _SRC, "-lm", "-lpthread"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


class Expert(ctypes.Structure):
    _fields_ = [("gate_q", ctypes.c_void_p), ("up_q", ctypes.c_void_p),
                ("down_q", ctypes.c_void_p), ("gate_s", ctypes.c_void_p),
                ("up_s", ctypes.c_void_p), ("down_s", ctypes.c_void_p),
                ("group", ctypes.c_int32)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_int4_code.argtypes = [P, ctypes.c_int64]
        L.oracle_int4_code.restype = i32
        L.oracle_int4_pack.argtypes = [P, ctypes.c_int64, P]
        L.oracle_int4_pack.restype = None
        L.oracle_weight.argtypes = [P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_weight.restype = ctypes.c_double
        L.oracle_weight_per_row.argtypes = [P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_weight_per_row.restype = ctypes.c_double
        L.oracle_route.argtypes = [i32, i32, i32, P, P, P]
        L.oracle_route.restype = i32
        L.oracle_router_logits.argtypes = [i32, i32, i32, P, P, P]
        L.oracle_router_logits.restype = None
        L.oracle_union.argtypes = [i32, i32, i32, P, P, P, P, P, P]
        L.oracle_union.restype = i32
        L.oracle_expert_ffn.argtypes = [i32, i32, ctypes.POINTER(Expert), P, P]
        L.oracle_expert_ffn.restype = None
        L.oracle_layer.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(Expert), i32, P, P, P,
                                   P, P, i32, P, i32]
        L.oracle_layer.restype = i32
        L.oracle_layer_grouped.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(Expert), i32,
                                           P, P, P, P, P, i32, P, P]
        L.oracle_layer_grouped.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- scalar formats ---------------------------------------------------------

def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(int(bits) & 0xFFFF)


def int4_codes(row: np.ndarray, n: int) -> np.ndarray:
    row = _c(row, np.uint8)
    return np.array([lib().oracle_int4_code(_p(row), k) for k in range(n)], dtype=np.int64)


def int4_pack(codes: np.ndarray) -> np.ndarray:
    codes = _c(codes, np.int8)
    out = np.zeros(codes.size // 2, dtype=np.uint8)
    lib().oracle_int4_pack(_p(codes), codes.size, _p(out))
    return out


def weight(q: np.ndarray, s_bits: np.ndarray, K: int, n: int, k: int) -> float:
    q = _c(q, np.uint8)
    s_bits = _c(s_bits, np.uint16)
    return lib().oracle_weight(_p(q), _p(s_bits), K, n, k)


def weight_per_row(q: np.ndarray, s_bits: np.ndarray, K: int, n: int, k: int) -> float:
    """W[n][k] of a per-row int4 matrix (one bf16 scale per row)."""
    q = _c(q, np.uint8)
    s_bits = _c(s_bits, np.uint16)
    return lib().oracle_weight_per_row(_p(q), _p(s_bits), K, n, k)


# ---- routing and union ------------------------------------------------------

def route(logits: np.ndarray, k: int):
    """Top-k (logit desc, lower index on ties) and renormalised softmax weights.

    Returns ``(idx int32 [T][k], w float64 [T][k])``.
    """
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    rc = lib().oracle_route(T, E, k, _p(logits), _p(idx), _p(w))
    if rc:
        raise ValueError("oracle_route: bad sizes")
    return idx, w


def router_logits(x_bf16_bits: np.ndarray, wr: np.ndarray) -> np.ndarray:
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    out = np.zeros((T, E), dtype=np.float64)
    lib().oracle_router_logits(T, E, H, _p(x), _p(wr), _p(out))
    return out


def union(idx: np.ndarray, E: int):
    """Batch-union lists.  Returns dict counts/offsets/pairs/active/n_active."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    pairs = np.zeros(max(T * k, 1), np.int32)
    active = np.zeros(E, np.int32)
    na = np.zeros(1, np.int32)
    rc = lib().oracle_union(T, E, k, _p(idx), _p(counts), _p(offsets), _p(pairs), _p(active),
                            _p(na))
    if rc:
        raise ValueError("oracle_union: index out of range")
    return dict(counts=counts, offsets=offsets, pairs=pairs[:T * k], active=active,
                n_active=int(na[0]))


# ---- FFN and layer ------------------------------------------------------------

class Experts:
    """Host expert table for the oracle: ``experts[e]`` is a dict of numpy
    arrays (gate_q, up_q, down_q uint8; gate_s, up_s, down_s uint16 bf16 bits,
    and optionally "group": 64 for gs64, the default, or 0 for one scale per
    row) or None for an expert the caller knows is never selected."""

    def __init__(self, experts: list):
        self.keep = []
        self.table = (Expert * len(experts))()
        for e, ex in enumerate(experts):
            if ex is None:
                continue
            arrs = {}
            for name in ("gate_q", "up_q", "down_q"):
                arrs[name] = _c(ex[name], np.uint8)
            for name in ("gate_s", "up_s", "down_s"):
                arrs[name] = _c(ex[name], np.uint16)
            self.keep.append(arrs)
            for name, a in arrs.items():
                setattr(self.table[e], name, a.ctypes.data)
            self.table[e].group = int(ex.get("group", 64))
        self.present = [ex is not None for ex in experts]


def expert_ffn(H: int, I: int, ex: dict, x: np.ndarray) -> np.ndarray:
    tab = Experts([ex])
    x = _c(x, np.float64)
    y = np.zeros(H, np.float64)
    lib().oracle_expert_ffn(H, I, tab.table, _p(x), _p(y))
    return y


def layer(H: int, I: int, E: int, k: int, n_shared: int, experts: Experts,
          x_bf16_bits: np.ndarray, idx: np.ndarray, w: np.ndarray, residual=None,
          sample=None, n_threads: int = 1) -> np.ndarray:
    """Per-token layer output in double for the tokens in ``sample`` (all if None)."""
    x = _c(x_bf16_bits, np.uint16)
    T = x.shape[0]
    idx = _c(idx, np.int32)
    w = _c(w, np.float64)
    sample = np.arange(T, dtype=np.int32) if sample is None else _c(sample, np.int32)
    for t in sample:
        for e in list(idx[t]) + [E + s for s in range(n_shared)]:
            if not experts.present[e]:
                raise ValueError(f"expert {e} needed by token {t} was not supplied")
    res = None if residual is None else _c(residual, np.float64)
    out = np.zeros((len(sample), H), np.float64)
    rc = lib().oracle_layer(H, I, E, k, n_shared, experts.table, T, _p(x), _p(idx), _p(w),
                            None if res is None else _p(res), _p(sample), len(sample), _p(out),
                            n_threads)
    if rc:
        raise ValueError("oracle_layer: bad arguments")
    return out


def layer_grouped(H: int, I: int, E: int, k: int, n_shared: int, experts: Experts,
                  x_bf16_bits: np.ndarray, w: np.ndarray, un: dict, residual=None) -> np.ndarray:
    x = _c(x_bf16_bits, np.uint16)
    T = x.shape[0]
    w = _c(w, np.float64)
    res = None if residual is None else _c(residual, np.float64)
    out = np.zeros((T, H), np.float64)
    lib().oracle_layer_grouped(H, I, E, k, n_shared, experts.table, T, _p(x), _p(w),
                               _p(_c(un["offsets"], np.int32)), _p(_c(un["pairs"], np.int32)),
                               _p(_c(un["active"], np.int32)), un["n_active"],
                               None if res is None else _p(res), _p(out))
    return out
