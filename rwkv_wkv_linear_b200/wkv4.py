"""Python binding of the C ABI in include/wkv4.h (ctypes; argument marshalling only).

Every step of the computation runs in the CUDA kernels of libwkv4.so; torch
is used for device memory and streams.  There is no CPU fallback: when the
library cannot be loaded every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# WKV4_LIB selects another build of the library (e.g. one tuned differently)
LIB_PATH = os.environ.get("WKV4_LIB") or os.path.join(_PKG, "libwkv4.so")

F32, F16, BF16 = 0, 1, 2
KERNEL_AUTO, KERNEL_SEQ, KERNEL_SCAN, KERNEL_SCAN_LDG, KERNEL_STEP = 0, 1, 2, 3, 4

STATUS = {0: "OK", -1: "ERR_ARG", -2: "ERR_DTYPE", -3: "ERR_ALIAS", -4: "ERR_CUDA",
          -5: "ERR_TIMEOUT", -7: "ERR_VARIANT", -8: "ERR_SLOT"}

_DTYPES = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}

EXPORTS = ("wkv4_decode_step", "wkv4_decode_step_gated", "wkv4_decode_step_slots",
           "wkv4_device_error", "wkv4_forward", "wkv4_forward_gated", "wkv4_forward_gated_variant",
           "wkv4_forward_host", "wkv4_forward_host_workspace",
           "wkv4_forward_variant", "wkv4_state_combine", "wkv4_status_string", "wkv4_token_shift",
           "wkv4_version")

_lock = threading.Lock()
_lib = None


class Wkv4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what} failed: {STATUS.get(status, status)} ({status_string(status)})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libwkv4.so (raises OSError when it is missing: build it with
    ``python -m rwkv_wkv_linear_b200._build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise OSError(f"{path} not found: build it with python -m rwkv_wkv_linear_b200._build")
            lib = ctypes.CDLL(path)
            i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
            fwd = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, i32]
            lib.wkv4_forward.argtypes = fwd
            lib.wkv4_forward.restype = i32
            lib.wkv4_forward_variant.argtypes = fwd + [i32]
            lib.wkv4_forward_variant.restype = i32
            lib.wkv4_decode_step.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp, vp, i32]
            lib.wkv4_decode_step.restype = i32
            gfwd = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32]
            lib.wkv4_forward_gated.argtypes = gfwd
            lib.wkv4_forward_gated.restype = i32
            lib.wkv4_forward_gated_variant.argtypes = gfwd + [i32]
            lib.wkv4_forward_gated_variant.restype = i32
            lib.wkv4_decode_step_gated.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, i32]
            lib.wkv4_decode_step_gated.restype = i32
            lib.wkv4_forward_host.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                              ctypes.c_size_t, i64, vp, i32]
            lib.wkv4_forward_host.restype = i32
            lib.wkv4_forward_host_workspace.argtypes = [i64, i64, i64, i32, i32, i64]
            lib.wkv4_forward_host_workspace.restype = ctypes.c_size_t
            lib.wkv4_state_combine.argtypes = [i64, i64, vp, i64, vp, vp, vp, vp]
            lib.wkv4_state_combine.restype = i32
            lib.wkv4_decode_step_slots.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, i32]
            lib.wkv4_decode_step_slots.restype = i32
            lib.wkv4_token_shift.argtypes = [i64, i64, i64] + [vp] * 10 + [i32]
            lib.wkv4_token_shift.restype = i32
            lib.wkv4_device_error.argtypes = [i32]
            lib.wkv4_device_error.restype = i32
            lib.wkv4_status_string.argtypes = [i32]
            lib.wkv4_status_string.restype = ctypes.c_char_p
            lib.wkv4_version.argtypes = []
            lib.wkv4_version.restype = i32
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().wkv4_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device: Optional[torch.device] = None) -> ctypes.c_void_p:
    """The call's stream: `stream`, or the current stream of `device`.  A torch
    stream given for a call on `device` must belong to that device."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and isinstance(stream, torch.cuda.Stream) and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _one_device(**tensors) -> torch.device:
    """The CUDA device all given tensors live on (None entries are skipped);
    raises when they are spread over several devices.  The library launches
    on the caller's current device, so every call runs with this device made
    current."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, other arguments on {dev}")
    return dev


def _check_dev(name: str, t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def forward(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
            state_in: Optional[torch.Tensor] = None, *, y: Optional[torch.Tensor] = None,
            state_out: Optional[torch.Tensor] = None, want_state: bool = True,
            variant: int = KERNEL_AUTO, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """wkv4_forward over k, v [B, T, C] (fp32/fp16/bf16); w, u [C] fp32;
    state_in [3, B, C] fp32 or None.  Returns (y, state_out)."""
    if k.dim() != 3 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, T, C]")
    B, T, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype:
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}")
    for name, t in (("k", k), ("v", v)):
        _check_dev(name, t)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    _check_dev("state_in", state_in, torch.float32)
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    if state_in is not None and state_in.shape != (3, B, C):
        raise ValueError("state_in must be [3, B, C]")
    if y is None:
        y = torch.empty_like(k)
    _check_dev("y", y, k.dtype)
    if state_out is None and want_state:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=k.device)
    _check_dev("state_out", state_out, torch.float32)
    dev = _one_device(k=k, v=v, w=w, u=u, state_in=state_in, y=y, state_out=state_out)
    with torch.cuda.device(dev):
        rc = load().wkv4_forward_variant(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v),
                                         _ptr(state_in), _ptr(y), _ptr(state_out),
                                         _stream(stream, dev), dt, int(variant))
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_forward")
    return y, state_out


def forward_gated(k: torch.Tensor, v: torch.Tensor, r: torch.Tensor, w: torch.Tensor,
                  u: torch.Tensor, state_in: Optional[torch.Tensor] = None, *,
                  y: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                  want_state: bool = True, variant: int = KERNEL_AUTO,
                  stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """wkv4_forward_gated: y = sigmoid(r) * wkv over k, v, r [B, T, C] (one
    dtype); w, u [C] fp32; state_in [3, B, C] fp32 or None.  Returns
    (y, state_out)."""
    if k.dim() != 3 or v.shape != k.shape or r.shape != k.shape:
        raise ValueError("k, v and r must all be [B, T, C]")
    B, T, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype or r.dtype != k.dtype:
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}/{r.dtype}")
    for name, t in (("k", k), ("v", v), ("r", r)):
        _check_dev(name, t)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    _check_dev("state_in", state_in, torch.float32)
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    if state_in is not None and state_in.shape != (3, B, C):
        raise ValueError("state_in must be [3, B, C]")
    if y is None:
        y = torch.empty_like(k)
    _check_dev("y", y, k.dtype)
    if state_out is None and want_state:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=k.device)
    _check_dev("state_out", state_out, torch.float32)
    dev = _one_device(k=k, v=v, r=r, w=w, u=u, state_in=state_in, y=y, state_out=state_out)
    with torch.cuda.device(dev):
        rc = load().wkv4_forward_gated_variant(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                               _ptr(state_in), _ptr(y), _ptr(state_out),
                                               _stream(stream, dev), dt, int(variant))
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_forward_gated")
    return y, state_out


def _check_host(name: str, t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")


def host_workspace_bytes(B: int, T: int, C: int, dtype: torch.dtype, gated: bool = False,
                         chunk_steps: int = 0) -> int:
    """wkv4_forward_host_workspace: device bytes forward_host needs."""
    return int(load().wkv4_forward_host_workspace(B, T, C, _DTYPES[dtype], int(gated),
                                                  int(chunk_steps)))


def forward_host(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
                 state_in: Optional[torch.Tensor] = None, r: Optional[torch.Tensor] = None, *,
                 y: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                 want_state: bool = True, workspace: Optional[torch.Tensor] = None,
                 chunk_steps: int = 0, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """wkv4_forward_host: the forward (gated when r is given) with k, v, r,
    state_in, y and state_out in HOST memory (CPU tensors; pinned ones let the
    copies overlap the kernels) and w, u [C] fp32 on the device; workspace is
    a CUDA uint8 tensor of at least host_workspace_bytes(...) bytes (allocated
    when None).  Asynchronous on the stream: synchronise it before reading y.
    Returns (y, state_out)."""
    if k.dim() != 3 or v.shape != k.shape or (r is not None and r.shape != k.shape):
        raise ValueError("k, v (and r) must be [B, T, C]")
    B, T, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype or (r is not None and r.dtype != k.dtype):
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}")
    for name, t in (("k", k), ("v", v), ("r", r)):
        _check_host(name, t)
    _check_host("state_in", state_in, torch.float32)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    if w.shape != (C,) or u.shape != (C,):
        raise ValueError("w and u must be [C]")
    if state_in is not None and state_in.shape != (3, B, C):
        raise ValueError("state_in must be [3, B, C]")
    if y is None:
        y = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    _check_host("y", y, k.dtype)
    if state_out is None and want_state:
        state_out = torch.empty((3, B, C), dtype=torch.float32, pin_memory=True)
    _check_host("state_out", state_out, torch.float32)
    dev = _one_device(w=w, u=u, workspace=workspace)
    need = host_workspace_bytes(B, T, C, k.dtype, r is not None, chunk_steps)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check_dev("workspace", workspace)
    with torch.cuda.device(dev):
        rc = load().wkv4_forward_host(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                      _ptr(state_in), _ptr(y), _ptr(state_out), _ptr(workspace),
                                      workspace.numel(), int(chunk_steps), _stream(stream, dev), dt)
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_forward_host")
    return y, state_out


def forward_raw(B: int, T: int, C: int, w, u, k, v, state_in, y, state_out, dtype: int,
                variant: int = KERNEL_AUTO, stream=None) -> int:
    """The C call with raw device addresses (ints or None); returns the status."""
    return load().wkv4_forward_variant(B, T, C, w, u, k, v, state_in, y, state_out,
                                       _stream(stream), dtype, int(variant))


def decode_step(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
                state: torch.Tensor, *, y: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """wkv4_decode_step: k, v [B, C]; state [3, B, C] fp32 updated in place.
    Returns y [B, C]."""
    if k.dim() != 2 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, C]")
    B, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype:
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}")
    for name, t in (("k", k), ("v", v)):
        _check_dev(name, t)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    _check_dev("state", state, torch.float32)
    if state.shape != (3, B, C):
        raise ValueError("state must be [3, B, C]")
    if y is None:
        y = torch.empty_like(k)
    _check_dev("y", y, k.dtype)
    dev = _one_device(k=k, v=v, w=w, u=u, state=state, y=y)
    with torch.cuda.device(dev):
        rc = load().wkv4_decode_step(B, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(state),
                                     _ptr(y), _stream(stream, dev), dt)
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_decode_step")
    return y


def decode_step_gated(k: torch.Tensor, v: torch.Tensor, r: torch.Tensor, w: torch.Tensor,
                      u: torch.Tensor, state: torch.Tensor, *, y: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """wkv4_decode_step_gated: k, v, r [B, C]; state [3, B, C] fp32 updated in
    place.  Returns y = sigmoid(r) * wkv [B, C]."""
    if k.dim() != 2 or v.shape != k.shape or r.shape != k.shape:
        raise ValueError("k, v and r must all be [B, C]")
    B, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype or r.dtype != k.dtype:
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}/{r.dtype}")
    for name, t in (("k", k), ("v", v), ("r", r)):
        _check_dev(name, t)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    _check_dev("state", state, torch.float32)
    if state.shape != (3, B, C):
        raise ValueError("state must be [3, B, C]")
    if y is None:
        y = torch.empty_like(k)
    _check_dev("y", y, k.dtype)
    dev = _one_device(k=k, v=v, r=r, w=w, u=u, state=state, y=y)
    with torch.cuda.device(dev):
        rc = load().wkv4_decode_step_gated(B, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                           _ptr(state), _ptr(y), _stream(stream, dev), dt)
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_decode_step_gated")
    return y


def decode_step_slots(k: torch.Tensor, v: torch.Tensor, w: torch.Tensor, u: torch.Tensor,
                      state_pool: torch.Tensor, slot_ids: torch.Tensor, *,
                      y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """wkv4_decode_step_slots: k, v [B, C]; state_pool [3, S, C] fp32 whose rows
    slot_ids [B] (int32, distinct, in [0, S)) are stepped in place.  Returns y
    [B, C] (a row whose id is out of range is left as it was)."""
    if k.dim() != 2 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, C]")
    B, C = k.shape
    dt = _DTYPES.get(k.dtype)
    if dt is None or v.dtype != k.dtype:
        raise ValueError(f"unsupported dtype {k.dtype}/{v.dtype}")
    for name, t in (("k", k), ("v", v)):
        _check_dev(name, t)
    _check_dev("w", w, torch.float32)
    _check_dev("u", u, torch.float32)
    _check_dev("state_pool", state_pool, torch.float32)
    _check_dev("slot_ids", slot_ids, torch.int32)
    if state_pool.dim() != 3 or state_pool.shape[0] != 3 or state_pool.shape[2] != C:
        raise ValueError("state_pool must be [3, S, C]")
    if slot_ids.shape != (B,):
        raise ValueError("slot_ids must be [B]")
    if y is None:
        y = torch.empty_like(k)
    _check_dev("y", y, k.dtype)
    dev = _one_device(k=k, v=v, w=w, u=u, state_pool=state_pool, slot_ids=slot_ids, y=y)
    with torch.cuda.device(dev):
        rc = load().wkv4_decode_step_slots(B, C, state_pool.shape[1], _ptr(w), _ptr(u), _ptr(k),
                                           _ptr(v), _ptr(state_pool), _ptr(slot_ids), _ptr(y),
                                           _stream(stream, dev), dt)
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_decode_step_slots")
    return y


def token_shift(x: torch.Tensor, mix_k: torch.Tensor, mix_v: torch.Tensor,
                mix_r: Optional[torch.Tensor] = None, x_prev: Optional[torch.Tensor] = None, *,
                x_last: Optional[torch.Tensor] = None, stream=None):
    """wkv4_token_shift: x [B, T, C]; mixes [C] fp32; x_prev [B, C] or None.
    Returns (xk, xv, xr or None); x_last [B, C], when given, receives x[:, -1]."""
    if x.dim() != 3:
        raise ValueError("x must be [B, T, C]")
    B, T, C = x.shape
    dt = _DTYPES.get(x.dtype)
    if dt is None:
        raise ValueError(f"unsupported dtype {x.dtype}")
    _check_dev("x", x)
    for name, m in (("mix_k", mix_k), ("mix_v", mix_v), ("mix_r", mix_r)):
        _check_dev(name, m, torch.float32)
        if m is not None and m.shape != (C,):
            raise ValueError(f"{name} must be [C]")
    for name, t in (("x_prev", x_prev), ("x_last", x_last)):
        _check_dev(name, t, x.dtype)
        if t is not None and t.shape != (B, C):
            raise ValueError(f"{name} must be [B, C]")
    dev = _one_device(x=x, mix_k=mix_k, mix_v=mix_v, mix_r=mix_r, x_prev=x_prev, x_last=x_last)
    xk, xv = torch.empty_like(x), torch.empty_like(x)
    xr = torch.empty_like(x) if mix_r is not None else None
    with torch.cuda.device(dev):
        rc = load().wkv4_token_shift(B, T, C, _ptr(x), _ptr(x_prev), _ptr(mix_k), _ptr(mix_v),
                                     _ptr(mix_r), _ptr(xk), _ptr(xv), _ptr(xr), _ptr(x_last),
                                     _stream(stream, dev), dt)
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_token_shift")
    return xk, xv, xr


def state_combine(x: Optional[torch.Tensor], y: torch.Tensor, n_steps: int, w: torch.Tensor, *,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """wkv4_state_combine: the state x (or None: empty) followed by a segment
    of n_steps steps whose state from the empty state is y; x, y, out
    [3, B, C] fp32, w [C] fp32.  Returns out."""
    if y.dim() != 3 or y.shape[0] != 3 or (x is not None and x.shape != y.shape):
        raise ValueError("x and y must be [3, B, C]")
    _, B, C = y.shape
    for name, t in (("x", x), ("y", y), ("w", w)):
        _check_dev(name, t, torch.float32)
    if w.shape != (C,):
        raise ValueError("w must be [C]")
    if out is None:
        out = torch.empty_like(y)
    _check_dev("out", out, torch.float32)
    dev = _one_device(x=x, y=y, w=w, out=out)
    with torch.cuda.device(dev):
        rc = load().wkv4_state_combine(B, C, _ptr(w), int(n_steps), _ptr(x), _ptr(y), _ptr(out),
                                       _stream(stream, dev))
    if rc != 0:
        raise Wkv4Error(rc, "wkv4_state_combine")
    return out


def device_error(reset: bool = True) -> int:
    """Status of the current device's error word (0, or -5 when a bounded
    device-side wait ran out).  Synchronises the device."""
    return int(load().wkv4_device_error(1 if reset else 0))


def version() -> int:
    return int(load().wkv4_version())
