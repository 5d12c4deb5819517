"""Python binding of libcoli_moe.so (the C ABI in include/coli_moe.h).

Argument marshalling only: every function here passes device pointers,
sizes and a CUDA stream handle to the C ABI of the same name; all the work
runs in the library's kernels.  PyTorch supplies device memory and streams.

The library is loaded from this package directory; if it is missing, import
of this module raises (build it with ``python -m
int4_routed_expert_coli_b200.build``).  There is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcoli_moe.so")

# coli_status codes (include/coli_moe.h)
COLI_OK = 0
COLI_ERR_INVALID_ARG = 1
COLI_ERR_SHAPE = 2
COLI_ERR_ALIGN = 3
COLI_ERR_WORKSPACE = 4
COLI_ERR_CUDA = 5
COLI_ERR_TIMEOUT = 6
COLI_ERR_UNSUPPORTED = 7
COLI_ERR_BAD_INDEX = 8
COLI_ERR_RANGE = 9
COLI_OUT_F32 = 0
COLI_WS_LOGITS_OFFSET = 16384  # router logits left in the workspace by coli_moe_layer
COLI_WS_HEADER_BYTES = 16384
COLI_OUT_BF16 = 1
COLI_GROUP_PER_ROW = 0  # coli_moe_desc.group_size of the per-row int4 format

EXPORTS = ("coli_moe_create", "coli_moe_destroy", "coli_moe_workspace_size",
           "coli_moe_workspace_clear", "coli_moe_route", "coli_moe_union",
           "coli_moe_union_workspace_size", "coli_moe_ffn",
           "coli_moe_layer", "coli_moe_layer_noalloc", "coli_moe_combine_rows",
           "coli_moe_prefetch",
           "coli_moe_get_status",
           "coli_moe_debug_inject",
           "coli_moe_profile_enable",
           "coli_moe_profile_read", "coli_status_string")


class ColiError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class CExpert(ctypes.Structure):
    _fields_ = [("gate_q", ctypes.c_void_p), ("up_q", ctypes.c_void_p),
                ("down_q", ctypes.c_void_p), ("gate_s", ctypes.c_void_p),
                ("up_s", ctypes.c_void_p), ("down_s", ctypes.c_void_p)]


class CDesc(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_routed", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("group_size", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("experts", ctypes.POINTER(CExpert)), ("prefill_min_tokens", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m int4_routed_expert_coli_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    L.coli_moe_create.argtypes = [ctypes.POINTER(CDesc), ctypes.POINTER(P)]
    L.coli_moe_create.restype = ctypes.c_int
    L.coli_moe_destroy.argtypes = [P]
    L.coli_moe_destroy.restype = None
    L.coli_moe_workspace_size.argtypes = [P, i32]
    L.coli_moe_workspace_size.restype = sz
    L.coli_moe_workspace_clear.argtypes = [P, sz, P]
    L.coli_moe_workspace_clear.restype = ctypes.c_int
    L.coli_moe_route.argtypes = [i32, i32, i32, P, P, P, P]
    L.coli_moe_route.restype = ctypes.c_int
    L.coli_moe_union.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, sz, P]
    L.coli_moe_union.restype = ctypes.c_int
    L.coli_moe_union_workspace_size.argtypes = [i32, i32, i32]
    L.coli_moe_union_workspace_size.restype = sz
    L.coli_moe_ffn.argtypes = [P, i32, P, P, P, P, P, P, P, P, P, ctypes.c_int, P, sz, P]
    L.coli_moe_ffn.restype = ctypes.c_int
    L.coli_moe_layer.argtypes = [P, i32, P, P, P, P, P, ctypes.c_int, P, P, P, sz, P]
    L.coli_moe_layer.restype = ctypes.c_int
    L.coli_moe_layer_noalloc.argtypes = [ctypes.POINTER(CDesc), i32, P, P, P, P, ctypes.c_int, P, P]
    L.coli_moe_layer_noalloc.restype = ctypes.c_int
    L.coli_moe_combine_rows.argtypes = [i32, i32, i32, P, P, P, P, ctypes.c_int, P]
    L.coli_moe_combine_rows.restype = ctypes.c_int
    L.coli_moe_prefetch.argtypes = [P, i32, i32, P, sz, P, sz, P]
    L.coli_moe_prefetch.restype = ctypes.c_int
    L.coli_moe_get_status.argtypes = [P, P]
    L.coli_moe_get_status.restype = ctypes.c_int
    L.coli_moe_debug_inject.argtypes = [i32]
    L.coli_moe_debug_inject.restype = ctypes.c_int
    L.coli_moe_profile_enable.argtypes = [i32]
    L.coli_moe_profile_enable.restype = ctypes.c_int
    L.coli_moe_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i32)]
    L.coli_moe_profile_read.restype = ctypes.c_int
    L.coli_status_string.argtypes = [ctypes.c_int]
    L.coli_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def status_string(s: int) -> str:
    return lib.coli_status_string(int(s)).decode()


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on the CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str, raise_on_error: bool):
    if raise_on_error and status != COLI_OK:
        raise ColiError(status, where)
    return status


# ---- the ABI, one function each -------------------------------------------

def coli_moe_route(T, E, k, logits, topk_idx, topk_w, stream=None, raise_on_error=True):
    s = lib.coli_moe_route(T, E, k, _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _stream(stream))
    return _check(s, "coli_moe_route", raise_on_error)


def coli_moe_union(T, E, k, topk_idx, counts, offsets, pairs, active, n_active, ws=None,
                   stream=None, raise_on_error=True):
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    s = lib.coli_moe_union(T, E, k, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(pairs),
                           _ptr(active), _ptr(n_active), _ptr(ws), ws_bytes, _stream(stream))
    return _check(s, "coli_moe_union", raise_on_error)


def coli_moe_union_workspace_size(T, E, k):
    return int(lib.coli_moe_union_workspace_size(T, E, k))


def coli_moe_ffn(handle, T, x, topk_w, counts, offsets, pairs, active, n_active, residual, out,
                 out_dtype, ws, stream=None, raise_on_error=True):
    s = lib.coli_moe_ffn(handle, T, _ptr(x), _ptr(topk_w), _ptr(counts), _ptr(offsets),
                         _ptr(pairs), _ptr(active), _ptr(n_active), _ptr(residual), _ptr(out),
                         out_dtype, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(s, "coli_moe_ffn", raise_on_error)


def coli_moe_layer(handle, T, x, logits, router_w, residual, out, out_dtype, topk_idx_out, topk_w_out,
                   ws, stream=None, raise_on_error=True):
    s = lib.coli_moe_layer(handle, T, _ptr(x), _ptr(logits), _ptr(router_w), _ptr(residual),
                           _ptr(out), out_dtype, _ptr(topk_idx_out), _ptr(topk_w_out), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream))
    return _check(s, "coli_moe_layer", raise_on_error)


def coli_moe_layer_noalloc(desc, T, x, logits, residual, out, out_dtype, status_out=None,
                           stream=None, raise_on_error=True):
    """Layer step without handle or workspace (see include/coli_moe.h):
    `desc` is a CDesc (e.g. MoELayer.desc), T <= 8."""
    s = lib.coli_moe_layer_noalloc(ctypes.byref(desc), T, _ptr(x), _ptr(logits), _ptr(residual),
                                   _ptr(out), out_dtype, _ptr(status_out), _stream(stream))
    return _check(s, "coli_moe_layer_noalloc", raise_on_error)


def coli_moe_combine_rows(T, k, H, rows, shared, residual, out, out_dtype, stream=None,
                          raise_on_error=True):
    s = lib.coli_moe_combine_rows(T, k, H, _ptr(rows), _ptr(shared), _ptr(residual), _ptr(out),
                                  out_dtype, _stream(stream))
    return _check(s, "coli_moe_combine_rows", raise_on_error)


def coli_moe_prefetch(handle, T, k, topk_idx, max_bytes, ws=None, stream=None,
                      raise_on_error=True):
    ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    s = lib.coli_moe_prefetch(handle, T, k, _ptr(topk_idx), int(max_bytes), _ptr(ws), ws_bytes,
                              _stream(stream))
    return _check(s, "coli_moe_prefetch", raise_on_error)


def coli_moe_workspace_clear(ws, stream=None, raise_on_error=True):
    s = lib.coli_moe_workspace_clear(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(s, "coli_moe_workspace_clear", raise_on_error)


def coli_moe_get_status(ws, stream=None):
    return lib.coli_moe_get_status(_ptr(ws), _stream(stream))


COLI_INJECT_WITHHOLD_STAGE = 1
COLI_INJECT_NOT_RESIDENT = 2


def coli_moe_debug_inject(what: int):
    return lib.coli_moe_debug_inject(int(what))


def coli_moe_profile_enable(enable: bool):
    return lib.coli_moe_profile_enable(1 if enable else 0)


def coli_moe_profile_read():
    """Summed milliseconds per phase [prep, gate/up, down, combine] and the
    number of recorded calls since the last read."""
    ms = (ctypes.c_double * 4)()
    n = ctypes.c_int32()
    s = lib.coli_moe_profile_read(ms, ctypes.byref(n))
    _check(s, "coli_moe_profile_read", True)
    return list(ms), int(n.value)


# ---- handle ---------------------------------------------------------------

class MoELayer:
    """A coli_moe handle over an ExpertBank (device tensors; routed experts
    first, shared experts last)."""

    def __init__(self, bank, n_routed: int, top_k: int, n_shared: int = 1,
                 prefill_min_tokens: int = 0):
        """`bank.per_row` selects the per-row int4 format (group_size
        COLI_GROUP_PER_ROW) instead of gs64."""
        if bank.n != n_routed + n_shared:
            raise ValueError("bank holds a different number of experts")
        self.bank = bank
        self.H, self.I, self.E, self.k, self.n_shared = bank.hidden, bank.inter, n_routed, top_k, n_shared
        tab = (CExpert * bank.n)()
        for e in range(bank.n):
            for name in ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s"):
                t = getattr(bank, name)[e]
                setattr(tab[e], name, t.data_ptr())
        group = COLI_GROUP_PER_ROW if getattr(bank, "per_row", False) else 64
        desc = CDesc(bank.hidden, bank.inter, n_routed, top_k, group, n_shared, tab,
                     prefill_min_tokens)
        self._table = tab
        self.desc = desc
        h = ctypes.c_void_p()
        s = lib.coli_moe_create(ctypes.byref(desc), ctypes.byref(h))
        if s != COLI_OK:
            raise ColiError(s, "coli_moe_create")
        self.handle = h

    def workspace_size(self, max_tokens: int) -> int:
        return int(lib.coli_moe_workspace_size(self.handle, max_tokens))

    def workspace(self, max_tokens: int, device=None) -> torch.Tensor:
        """A cleared workspace for calls with up to max_tokens tokens."""
        n = self.workspace_size(max_tokens)
        ws = torch.empty(n, dtype=torch.uint8, device=device or self.bank.gate_q.device)
        coli_moe_workspace_clear(ws)
        return ws

    def layer(self, x, logits=None, router_w=None, residual=None, out=None, out_dtype=COLI_OUT_F32,
              topk_idx_out=None, topk_w_out=None, ws=None, stream=None):
        T = x.shape[0]
        if out is None:
            dt = torch.float32 if out_dtype == COLI_OUT_F32 else torch.bfloat16
            out = torch.empty(T, self.H, dtype=dt, device=x.device)
        if ws is None:
            ws = self.workspace(T, x.device)
        coli_moe_layer(self.handle, T, x, logits, router_w, residual, out, out_dtype, topk_idx_out,
                       topk_w_out, ws, stream)
        return out

    def close(self):
        if getattr(self, "handle", None):
            lib.coli_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
