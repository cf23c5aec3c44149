"""Child process of tests/test_gpu_failure.py, run with the bounds-checked
library (WKV4_LIB pointing at libwkv4_checked.so) and, per mode, a fault
switch in the environment:

  python -m tests.failure_child clean        every entry point on small valid
                                             shapes: parity with the oracle and
                                             an empty device error word (no
                                             index outside its buffer)
  python -m tests.failure_child launch N     with WKV4_FAULT=launch:N: the
                                             N-th call's launch fails
                                             (WKV4_ERR_CUDA), every other
                                             call succeeds and is correct
  python -m tests.failure_child host         with WKV4_FAULT=launch:2: the
                                             forward from host buffers fails
                                             at its second chunk's launch
                                             (WKV4_ERR_CUDA), and the same call
                                             repeated on the same workspace and
                                             stream is correct
  python -m tests.failure_child exchange     with WKV4_FAULT=exchange: a scan
                                             call whose segment aggregates are
                                             never pushed ends with
                                             WKV4_ERR_TIMEOUT in the error
                                             word, and the next call (no
                                             exchange) is correct

Prints one line "ok" on success; any failure raises (non-zero exit).
"""

import os
import sys

import numpy as np
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity

DEV = torch.device("cuda:0")


def _dev(x):
    return {k: (t.to(DEV) if t is not None else None) for k, t in x.items()}


def _check_fwd(x, dt, y, s, what, r=None, calls=0):
    if r is None:
        y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
        ya = None if dt == "f32" else parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    else:
        y_ref, s_ref = oracle.forward_gated(x["k"], x["v"], r, x["w"], x["u"], x["state_in"])
        ya = None if dt == "f32" else parity.y_abs_gated(x["k"], x["v"], r, x["w"], x["u"],
                                                         x["state_in"])
    parity.check_y(y.cpu(), y_ref, x["v"], dt, what + " y", y_abs=ya, calls=calls)
    parity.check_state(s.cpu(), s_ref, x["v"], x["state_in"], calls=max(1, calls),
                       what=what + " state")


# one call of every entry point, on small valid shapes
def call_forward():
    x = synth.custom(2, 700, 200, "f16", seed=1, random_state=True, k_var=2.0)
    g = _dev(x)
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"])
    torch.cuda.synchronize()
    _check_fwd(x, "f16", y, s, "forward")


def call_forward_variants():
    for shape in ((1, 777, 36, "f32"), (2, 2049, 128, "f32"), (3, 517, 96, "bf16"),
                  (1, 3000, 100, "f16"), (2, 300, 5, "f32")):
        B, T, C, dt = shape
        x = synth.custom(B, T, C, dt, seed=B + T + C, random_state=True, k_var=2.0)
        g = _dev(x)
        for variant in (wkv4.KERNEL_SEQ, wkv4.KERNEL_SCAN, wkv4.KERNEL_SCAN_LDG, wkv4.KERNEL_STEP):
            y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], variant=variant)
            torch.cuda.synchronize()
            _check_fwd(x, dt, y, s, f"{shape}/{variant}")


def call_gated():
    wl = synth.Workload("custom", B=2, T=600, C=128, dtype="bf16", seed=3, random_state=True)
    x = synth.forward_inputs(wl)
    r = synth.receptance(wl)
    g = _dev(x)
    y, s = wkv4.forward_gated(g["k"], g["v"], r.to(DEV), g["w"], g["u"], g["state_in"])
    torch.cuda.synchronize()
    _check_fwd(x, "bf16", y, s, "gated", r=r)


def call_decode():
    x = synth.custom(8, 1, 256, "bf16", seed=4, random_state=True)
    g = _dev(x)
    st = g["state_in"].clone()
    y = wkv4.decode_step(g["k"][:, 0].contiguous(), g["v"][:, 0].contiguous(), g["w"], g["u"], st)
    torch.cuda.synchronize()
    _check_fwd(x, "bf16", y[:, None], st, "decode")


def call_slots():
    S, B, C = 20, 8, 128
    x = synth.custom(B, 1, C, "f32", seed=5)
    pool = torch.stack([torch.randn(S, C), torch.rand(S, C) + 0.5, torch.rand(S, C)]).float()
    ids = torch.randperm(S)[:B].to(torch.int32)
    pd = pool.to(DEV)
    y = wkv4.decode_step_slots(x["k"][:, 0].contiguous().to(DEV), x["v"][:, 0].contiguous().to(DEV),
                               x["w"].to(DEV), x["u"].to(DEV), pd, ids.to(DEV))
    torch.cuda.synchronize()
    y_ref, pool_ref, skipped = oracle.decode_slots(x["k"][:, 0], x["v"][:, 0], x["w"], x["u"],
                                                   pool.double().numpy(), ids)
    assert skipped == 0
    parity.check_y(y.cpu(), y_ref, x["v"], "f32", "slots y")


def call_shift():
    wl = synth.workload("token_shift_14b", B=2, T=40, C=256)
    x = synth.shift_inputs(wl)
    xd = x["x"].to(DEV)
    mk, mv, mr = (m.to(DEV) for m in x["mix"])
    xk, xv, xr = wkv4.token_shift(xd, mk, mv, mr, x["x_prev"].to(DEV))
    torch.cuda.synchronize()
    outs, _ = oracle.token_shift(x["x"], x["x_prev"], x["mix"])
    for got, ref in zip((xk, xv, xr), outs):
        err = np.abs(got.cpu().double().numpy() - ref)
        assert np.all(err <= 2.0 ** -7 * np.abs(ref) + 1e-6), float(err.max())


def call_combine():
    B, C = 3, 100
    w = synth.custom(1, 1, C, "f32", seed=6)["w"]
    xs = torch.stack([torch.randn(B, C), torch.rand(B, C) + 0.5, torch.rand(B, C)]).float()
    ys = torch.stack([torch.randn(B, C), torch.rand(B, C) + 0.5, torch.rand(B, C) + 3]).float()
    out = wkv4.state_combine(xs.to(DEV), ys.to(DEV), 17, w.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.combine_states(xs.double().numpy(), ys.double().numpy(), 17, w)
    parity.check_state(out.cpu(), ref, np.array([1.0]), xs, what="combine")


CALLS = [call_forward, call_gated, call_decode, call_slots, call_shift, call_combine]


def main():
    assert os.path.basename(wkv4.LIB_PATH) == "libwkv4_checked.so", wkv4.LIB_PATH
    mode = sys.argv[1]
    torch.cuda.set_device(DEV)
    wkv4.device_error(reset=True)
    if mode == "clean":
        for call in CALLS + [call_forward_variants]:
            call()
        assert wkv4.device_error(reset=True) == 0
    elif mode == "launch":
        n = int(sys.argv[2])
        assert os.environ.get("WKV4_FAULT") == f"launch:{n}"
        for i, call in enumerate(CALLS, start=1):
            if i == n:
                try:
                    call()
                except wkv4.Wkv4Error as e:
                    assert e.status == -4, e.status  # WKV4_ERR_CUDA
                else:
                    raise AssertionError(f"call {i} ({call.__name__}) did not fail")
            else:
                call()
        assert wkv4.device_error(reset=True) == 0
    elif mode == "host":
        assert os.environ.get("WKV4_FAULT") == "launch:2"
        x = synth.custom(2, 900, 128, "bf16", seed=8, random_state=True, k_var=2.0)
        w, u = x["w"].to(DEV), x["u"].to(DEV)
        kh, vh, sh = x["k"].pin_memory(), x["v"].pin_memory(), x["state_in"].pin_memory()
        ws = torch.empty(wkv4.host_workspace_bytes(2, 900, 128, torch.bfloat16, chunk_steps=300),
                         dtype=torch.uint8, device=DEV)
        try:
            wkv4.forward_host(kh, vh, w, u, sh, workspace=ws, chunk_steps=300)
        except wkv4.Wkv4Error as e:
            assert e.status == -4, e.status  # WKV4_ERR_CUDA
        else:
            raise AssertionError("the injected launch failure did not surface")
        torch.cuda.synchronize()
        y, s = wkv4.forward_host(kh, vh, w, u, sh, workspace=ws, chunk_steps=300)
        torch.cuda.synchronize()
        _check_fwd(x, "bf16", y, s, "host after the failure", calls=3)
        assert wkv4.device_error(reset=True) == 0
    elif mode == "exchange":
        assert os.environ.get("WKV4_FAULT") == "exchange"
        # one channel tile, one round of two segments (a cluster of two CTAs):
        # every wait for the peers' aggregates runs out, nothing else is in flight
        x = synth.custom(1, 512, 64, "bf16", seed=7, random_state=True)
        g = _dev(x)
        wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], variant=wkv4.KERNEL_SCAN)
        assert wkv4.device_error(reset=True) == -5  # WKV4_ERR_TIMEOUT
        assert wkv4.device_error(reset=True) == 0
        # the context still works: a call without an exchange
        y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], variant=wkv4.KERNEL_STEP)
        torch.cuda.synchronize()
        _check_fwd(x, "bf16", y, s, "after the expiry")
        assert wkv4.device_error(reset=True) == 0
    else:
        raise SystemExit(f"unknown mode {mode}")
    print("ok")


if __name__ == "__main__":
    main()
