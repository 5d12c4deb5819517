"""C-ABI checks that need no GPU: the library loads, exports every function
the header declares, and rejects bad arguments on the host before any CUDA
call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "coli_moe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(coli_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    names = _declared()
    for n in ("coli_moe_route", "coli_moe_union", "coli_moe_ffn", "coli_moe_layer",
              "coli_moe_create", "coli_moe_destroy", "coli_moe_workspace_size",
              "coli_moe_get_status", "coli_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from int4_routed_expert_coli_b200 import coli_moe as c
    for n in _declared():
        assert hasattr(c.lib, n), n
        assert n in c.EXPORTS, n
        assert callable(getattr(c, n, None)) or n in ("coli_moe_create", "coli_moe_destroy",
                                                      "coli_moe_workspace_size",
                                                      "coli_status_string"), n


def test_header_constants_match_binding():
    from int4_routed_expert_coli_b200 import coli_moe as c
    src = open(HEADER).read()
    for name in ("COLI_WS_LOGITS_OFFSET", "COLI_WS_HEADER_BYTES", "COLI_INJECT_WITHHOLD_STAGE",
                 "COLI_INJECT_NOT_RESIDENT", "COLI_GROUP_PER_ROW"):
        m = re.search(r"#define\s+" + name + r"\s+(\d+)", src)
        assert m and int(m.group(1)) == getattr(c, name), name
    for name, val in re.findall(r"\b(COLI_(?:OK|ERR_\w+|OUT_\w+))\s*=\s*(\d+)", src):
        assert getattr(c, name) == int(val), name


def test_status_strings():
    from int4_routed_expert_coli_b200 import coli_moe as c
    for s in range(10):
        assert c.status_string(s) and c.status_string(s) != "unknown status"
    assert c.status_string(99) == "unknown status"


def test_host_validation_without_gpu():
    from int4_routed_expert_coli_b200 import coli_moe as c
    L = c.lib
    P = ctypes.c_void_p
    # route: T < 0, k > E, k > 32, E > 1024: rejected before any CUDA call
    assert L.coli_moe_route(-1, 16, 2, None, None, None, None) == c.COLI_ERR_INVALID_ARG
    assert L.coli_moe_route(4, 4, 5, None, None, None, None) == c.COLI_ERR_SHAPE
    assert L.coli_moe_route(4, 64, 33, None, None, None, None) == c.COLI_ERR_SHAPE
    assert L.coli_moe_route(4, 1025, 2, None, None, None, None) == c.COLI_ERR_SHAPE
    assert L.coli_moe_route(4, 16, 2, None, None, None, None) == c.COLI_ERR_INVALID_ARG
    # T == 0 is a no-op
    assert L.coli_moe_route(0, 16, 2, None, None, None, None) == c.COLI_OK
    assert L.coli_moe_route(1, 16, 2, P(2), P(4), P(8), None) == c.COLI_ERR_ALIGN
    # union: missing outputs
    assert L.coli_moe_union(4, 16, 2, None, None, None, None, None, None, None, 0, None) == \
        c.COLI_ERR_INVALID_ARG
    # create: bad descriptors
    h = P()
    assert L.coli_moe_create(None, ctypes.byref(h)) == c.COLI_ERR_INVALID_ARG
    tab = (c.CExpert * 2)()
    d = c.CDesc(256, 128, 1, 1, 32, 1, tab, 0)       # group size must be 64
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_SHAPE
    d = c.CDesc(200, 128, 1, 1, 64, 1, tab, 0)       # H not a multiple of 128
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_SHAPE
    d = c.CDesc(256, 128, 1, 2, 64, 1, tab, 0)       # k > E
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_SHAPE
    d = c.CDesc(256, 128, 1, 1, 64, 1, tab, -1)      # negative tensor-core threshold
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_INVALID_ARG
    d = c.CDesc(256, 128, 1, 1, 64, 1, tab, 0)       # NULL expert pointers
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_INVALID_ARG
    for f in ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s"):
        setattr(tab[0], f, 4096)
        setattr(tab[1], f, 4096 + 8)                 # misaligned
    assert L.coli_moe_create(ctypes.byref(d), ctypes.byref(h)) == c.COLI_ERR_ALIGN
    # handle-taking calls reject a NULL handle
    assert L.coli_moe_workspace_size(None, 4) == 0
    assert L.coli_moe_layer(None, 1, None, None, None, None, None, 0, None, None, None, 0,
                            None) == c.COLI_ERR_INVALID_ARG
    assert L.coli_moe_ffn(None, 1, None, None, None, None, None, None, None, None, None, 0,
                          None, 0, None) == c.COLI_ERR_INVALID_ARG
    assert L.coli_moe_workspace_clear(None, 0, None) == c.COLI_ERR_INVALID_ARG
    # fault injection: unknown codes are refused, 0 switches it off
    assert L.coli_moe_debug_inject(12345) == c.COLI_ERR_INVALID_ARG
    assert L.coli_moe_debug_inject(0) == c.COLI_OK


def test_binding_refuses_host_tensors():
    import torch
    from int4_routed_expert_coli_b200 import coli_moe as c
    with pytest.raises(ValueError):
        c.coli_moe_route(1, 16, 2, torch.zeros(1, 16), torch.zeros(1, 2, dtype=torch.int32),
                         torch.zeros(1, 2))
