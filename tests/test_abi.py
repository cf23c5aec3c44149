"""Host-side checks of the C ABI: the library loads, exports every symbol that
include/wkv4.h declares, and rejects bad arguments before touching a GPU."""

import ctypes
import os
import re

import pytest

from rwkv_wkv_linear_b200 import wkv4

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "wkv4.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"WKV4_API\s+[\w\s\*]*?\b(wkv4_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_symbols() == sorted(wkv4.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = wkv4.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_version_and_status_strings():
    assert wkv4.version() == 100
    for code in wkv4.STATUS:
        assert wkv4.status_string(code)
    assert wkv4.status_string(12345) == "unknown status"


P = 0x7F0000000000  # fake device addresses: these calls must return before any CUDA call


def _call(B=2, T=8, C=16, w=P, u=P + 0x1000, k=P + 0x10000, v=P + 0x20000, si=None,
          y=P + 0x30000, so=None, dtype=wkv4.F32, variant=wkv4.KERNEL_AUTO):
    return wkv4.load().wkv4_forward_variant(B, T, C, w, u, k, v, si, y, so, None, dtype, variant)


def test_negative_sizes_are_rejected():
    assert _call(B=-1) == -1
    assert _call(T=-1) == -1
    assert _call(C=-5) == -1


def test_bad_dtype_and_variant():
    assert _call(dtype=7) == -2
    assert _call(variant=9) == -7
    assert _call(variant=-1) == -7


def test_empty_problems_are_noops():
    assert _call(B=0) == 0
    assert _call(C=0) == 0
    assert _call(B=0, k=None, v=None, y=None) == 0


def test_null_required_pointers():
    assert _call(k=None) == -1
    assert _call(v=None) == -1
    assert _call(y=None) == -1
    assert _call(w=None) == -1
    lib = wkv4.load()
    assert lib.wkv4_decode_step(2, 16, P, P + 0x1000, P + 0x10000, P + 0x20000, None,
                                P + 0x30000, None, 0) == -1


def test_overlapping_outputs_are_rejected():
    # y overlapping k (B*T*C*4 = 1024 bytes)
    assert _call(y=P + 0x10000 + 512) == -3
    # state_out overlapping v
    assert _call(so=P + 0x20000 + 64) == -3
    # state_out partially overlapping state_in (equal is allowed, partial is not)
    assert _call(si=P + 0x40000, so=P + 0x40000 + 4) == -3
    # y overlapping the state
    assert _call(si=P + 0x40000, y=P + 0x40000 + 8) == -3


def _slots(B=2, C=16, S=5, w=P, u=P + 0x1000, k=P + 0x10000, v=P + 0x20000, pool=P + 0x40000,
           ids=P + 0x50000, y=P + 0x30000, dtype=wkv4.F32):
    return wkv4.load().wkv4_decode_step_slots(B, C, S, w, u, k, v, pool, ids, y, None, dtype)


def test_slot_decode_argument_checks():
    assert _slots(B=-1) == -1
    assert _slots(C=-1) == -1
    assert _slots(S=-1) == -1
    assert _slots(dtype=5) == -2
    assert _slots(B=0) == 0 and _slots(C=0) == 0
    for name in ("w", "u", "k", "v", "pool", "ids", "y"):
        assert _slots(**{name: None}) == -1, name
    # y over the pool (3*5*16*4 = 960 bytes), the pool over k, the ids inside the pool
    assert _slots(y=P + 0x40000 + 256) == -3
    assert _slots(pool=P + 0x10000 + 64) == -3
    assert _slots(ids=P + 0x40000 + 512) == -3
    assert _slots(y=P + 0x50000 + 4) == -3


def _shift(B=2, T=8, C=16, x=P + 0x10000, xp=None, mk=P, mv=P + 0x1000, mr=None,
           xk=P + 0x20000, xv=P + 0x30000, xr=None, xl=None, dtype=wkv4.F32):
    return wkv4.load().wkv4_token_shift(B, T, C, x, xp, mk, mv, mr, xk, xv, xr, xl, None, dtype)


def test_token_shift_argument_checks():
    assert _shift(B=-1) == -1 and _shift(T=-1) == -1 and _shift(C=-1) == -1
    assert _shift(dtype=3) == -2
    assert _shift(B=0) == 0 and _shift(C=0) == 0
    assert _shift(T=0) == 0  # no x_last: nothing to do
    for name in ("x", "mk", "mv", "xk", "xv"):
        assert _shift(**{name: None}) == -1, name
    assert _shift(mr=P + 0x2000) == -1          # mix_r without xr
    assert _shift(B=70000) == -1                # beyond the grid's batch dimension
    # xk over x (2*8*16*4 = 1024 bytes), xv over xk, x_last over x_prev, xr over mix_r
    assert _shift(xk=P + 0x10000 + 512) == -3
    assert _shift(xv=P + 0x20000 + 4) == -3
    assert _shift(xp=P + 0x40000, xl=P + 0x40000 + 8) == -3
    assert _shift(mr=P + 0x2000, xr=P + 0x2000) == -3


def test_binding_rejects_host_tensors_and_bad_shapes():
    """The Python binding checks devices, dtypes and shapes before any CUDA
    call (host tensors, so no GPU is needed to reach these errors)."""
    import torch
    k = torch.zeros(2, 8, 16)
    w = torch.zeros(16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        wkv4.forward(k, k, w, w)
    with pytest.raises(ValueError, match="\\[B, T, C\\]"):
        wkv4.forward(k[0], k[0], w, w)
    with pytest.raises(ValueError, match="unsupported dtype"):
        wkv4.forward(k.double(), k.double(), w, w)
    with pytest.raises(ValueError, match="\\[B, C\\]"):
        wkv4.decode_step(k, k, w, w, torch.zeros(3, 2, 16))
    with pytest.raises(ValueError, match="\\[B, C\\]"):
        wkv4.decode_step_slots(k, k, w, w, torch.zeros(3, 4, 16), torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensor"):
        wkv4.decode_step_slots(k[:, 0], k[:, 0], w, w, torch.zeros(3, 4, 16),
                               torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError, match="\\[B, T, C\\]"):
        wkv4.token_shift(k[0], w, w)
    with pytest.raises(ValueError, match="CUDA tensor"):
        wkv4.token_shift(k, w, w)


def _gated(B=2, T=8, C=16, w=P, u=P + 0x1000, k=P + 0x10000, v=P + 0x20000, r=P + 0x60000,
           si=None, y=P + 0x30000, so=None, dtype=wkv4.F32, variant=wkv4.KERNEL_AUTO):
    return wkv4.load().wkv4_forward_gated_variant(B, T, C, w, u, k, v, r, si, y, so, None, dtype,
                                                  variant)


def test_gated_argument_checks():
    assert _gated(B=-1) == -1 and _gated(T=-1) == -1
    assert _gated(dtype=4) == -2 and _gated(variant=8) == -7
    assert _gated(r=None) == -1                       # the receptance is required
    assert _gated(B=0, r=None) == 0                   # ... unless there is nothing to do
    assert _gated(y=P + 0x60000 + 64) == -3           # y over r
    assert _gated(so=P + 0x60000) == -3               # the state over r
    lib = wkv4.load()
    d = lib.wkv4_decode_step_gated
    assert d(2, 16, P, P + 0x1000, P + 0x10000, P + 0x20000, None, P + 0x40000, P + 0x30000,
             None, 0) == -1                           # no r
    assert d(2, 16, P, P + 0x1000, P + 0x10000, P + 0x20000, P + 0x30000 + 8, P + 0x40000,
             P + 0x30000, None, 0) == -3              # y over r


def test_binding_requires_one_device():
    import types
    a = types.SimpleNamespace(is_cuda=True, device="cuda:0")
    b = types.SimpleNamespace(is_cuda=True, device="cuda:1")
    assert wkv4._one_device(k=a, v=a, y=None) == "cuda:0"
    with pytest.raises(ValueError, match="cuda:1"):
        wkv4._one_device(k=a, v=b)
    with pytest.raises(ValueError, match="CUDA tensor"):
        wkv4._one_device(k=types.SimpleNamespace(is_cuda=False, device="cpu"))


def _host(B=2, T=64, C=16, w=P, u=P + 0x1000, k=P + 0x100000, v=P + 0x200000, r=None, si=None,
          y=P + 0x300000, so=None, ws=P + 0x10000000, wsb=None, chunk=0, dtype=wkv4.F32):
    lib = wkv4.load()
    if wsb is None:
        wsb = lib.wkv4_forward_host_workspace(B, T, C, dtype, int(r is not None), chunk)
    return lib.wkv4_forward_host(B, T, C, w, u, k, v, r, si, y, so, ws, wsb, chunk, None, dtype)


def test_host_forward_workspace_sizes():
    lib = wkv4.load()
    ws = lib.wkv4_forward_host_workspace
    # two slots of k, v, y (gated: and r) of one chunk, and the state, each 256-byte aligned
    io = 2 * 64 * 16 * 4
    assert ws(2, 64, 16, wkv4.F32, 0, 0) == 2 * 3 * io + 512
    assert ws(2, 64, 16, wkv4.F32, 1, 0) == 2 * 4 * io + 512
    assert ws(2, 64, 16, wkv4.F32, 0, 16) == 2 * 3 * (io // 4) + 512
    assert ws(2, 64, 16, wkv4.F16, 0, 16) == 2 * 3 * 1024 + 512
    assert ws(2, 0, 16, wkv4.F32, 0, 0) == 512          # T == 0: the state only
    assert ws(0, 64, 16, wkv4.F32, 0, 0) == 0
    assert ws(2, -1, 16, wkv4.F32, 0, 0) == 0
    assert ws(2, 64, 16, 9, 0, 0) == 0
    assert ws(2, 64, 16, wkv4.F32, 0, -3) == 0
    # the default chunk: about a sixteenth of the inputs, at least 16 MB of them
    big = ws(1, 65536, 2048, wkv4.F32, 0, 0)
    assert big == 2 * 3 * 4096 * 2048 * 4 + 3 * 2048 * 4
    # 14B width (B=4, C=5120, bf16: 80 KB of inputs a step): 16 MB / 80 KB + 1 = 205 steps
    assert ws(4, 1024, 5120, wkv4.BF16, 0, 0) == 2 * 3 * 4 * 205 * 5120 * 2 + 3 * 4 * 5120 * 4


def test_host_forward_argument_checks():
    assert _host(B=-1) == -1 and _host(T=-1) == -1 and _host(C=-1) == -1
    assert _host(chunk=-1) == -1
    assert _host(dtype=4) == -2
    assert _host(B=0) == 0 and _host(C=0) == 0
    for name in ("w", "u", "k", "v", "y", "ws"):
        assert _host(**{name: None}) == -1, name
    # a workspace one byte short
    full = wkv4.load().wkv4_forward_host_workspace(2, 64, 16, wkv4.F32, 0, 0)
    assert _host(wsb=full - 1) == -1
    # y over k (2*64*16*4 = 8192 bytes), the state over y, the workspace over k
    assert _host(y=P + 0x100000 + 4096) == -3
    assert _host(so=P + 0x300000 + 64) == -3
    assert _host(ws=P + 0x100000 + 16) == -3
    # state_out partially over state_in (equal is allowed)
    assert _host(si=P + 0x400000, so=P + 0x400000 + 8) == -3
