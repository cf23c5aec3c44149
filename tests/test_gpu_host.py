"""GPU tests of the forward from host buffers (wkv4_forward_host): chunks of T
chained through the device state with the copies overlapped, against the fp64
oracle (parity, with the state re-rounded once per chunk), and bit for bit
against the same chunks run as device-buffer forward calls (the pipeline's
copies, slots and events lose or mix nothing)."""

import os

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity

pytestmark = pytest.mark.gpu

NT = os.cpu_count() or 1


@pytest.fixture(autouse=True)
def no_device_errors(cuda_device):
    yield
    assert wkv4.device_error(reset=True) == 0


def _pinned(t):
    return None if t is None else t.contiguous().pin_memory()


def _chunked_on_device(x, dev, chunk, r=None):
    """The same chunks as device-buffer forward calls chained through the state."""
    k, v = x["k"].to(dev), x["v"].to(dev)
    w, u = x["w"].to(dev), x["u"].to(dev)
    st = x["state_in"].to(dev) if x["state_in"] is not None else None
    rd = r.to(dev) if r is not None else None
    T = k.shape[1]
    ys = []
    for t0 in range(0, T, chunk):
        sl = slice(t0, min(T, t0 + chunk))
        if rd is None:
            y, st = wkv4.forward(k[:, sl].contiguous(), v[:, sl].contiguous(), w, u, st)
        else:
            y, st = wkv4.forward_gated(k[:, sl].contiguous(), v[:, sl].contiguous(),
                                       rd[:, sl].contiguous(), w, u, st)
        ys.append(y)
    torch.cuda.synchronize()
    return torch.cat(ys, dim=1).cpu(), st.cpu()


CASES = [
    # (B, T, C, dtype, random_state, chunk_steps)
    (2, 3000, 256, "f32", True, 0),
    (2, 3000, 256, "f32", False, 700),
    (3, 2100, 128, "bf16", True, 256),
    (1, 5000, 768, "f16", False, 1024),
    (4, 1024, 512, "bf16", True, 100),
    (2, 777, 100, "f16", True, 300),     # C * 2 bytes not a multiple of 16: element-wise kernels
    (1, 257, 64, "f32", True, 257),      # one chunk
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dT%dC%d_%s_rs%d_chunk%d" % c)
def test_host_forward_matches_oracle_and_device_chunks(cuda_device, case):
    B, T, C, dt, rs, chunk = case
    x = synth.custom(B, T, C, dt, seed=B * 7 + T + C, random_state=rs, k_var=2.0,
                     spike_frac=0.001)
    w, u = x["w"].to(cuda_device), x["u"].to(cuda_device)
    y, s = wkv4.forward_host(_pinned(x["k"]), _pinned(x["v"]), w, u, _pinned(x["state_in"]),
                             chunk_steps=chunk)
    torch.cuda.synchronize()
    tc = chunk
    # the library's own chunk when chunk_steps is 0: at least 16 MB of inputs
    if chunk == 0:
        es = 4 if dt == "f32" else 2
        tc = min(T, max((T + 15) // 16, (16 << 20) // (2 * B * C * es) + 1))
    nch = -(-T // tc)
    y_dev, s_dev = _chunked_on_device(x, cuda_device, tc)
    assert torch.equal(y, y_dev), "host pipeline differs from the chained device calls"
    assert torch.equal(s, s_dev)
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"], nthreads=NT)
    ya = None if dt == "f32" else parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"], NT)
    parity.check_y(y, y_ref, x["v"], dt, f"host {case} y", y_abs=ya, calls=nch)
    parity.check_state(s, s_ref, x["v"], x["state_in"], calls=nch, what=f"host {case} state")


def test_host_forward_gated(cuda_device):
    wl = synth.Workload("custom", B=2, T=1500, C=256, dtype="bf16", seed=11, random_state=True)
    x = synth.forward_inputs(wl)
    r = synth.receptance(wl)
    w, u = x["w"].to(cuda_device), x["u"].to(cuda_device)
    y, s = wkv4.forward_host(_pinned(x["k"]), _pinned(x["v"]), w, u, _pinned(x["state_in"]),
                             r=_pinned(r), chunk_steps=400)
    torch.cuda.synchronize()
    y_dev, s_dev = _chunked_on_device(x, cuda_device, 400, r=r)
    assert torch.equal(y, y_dev) and torch.equal(s, s_dev)
    y_ref, s_ref = oracle.forward_gated(x["k"], x["v"], r, x["w"], x["u"], x["state_in"])
    ya = parity.y_abs_gated(x["k"], x["v"], r, x["w"], x["u"], x["state_in"])
    parity.check_y(y, y_ref, x["v"], "bf16", "host gated y", y_abs=ya, calls=4)
    parity.check_state(s, s_ref, x["v"], x["state_in"], calls=4, what="host gated state")


def test_host_forward_in_place_state_pageable_and_back_to_back(cuda_device):
    """state_out is state_in (host, in place); pageable (unpinned) buffers;
    three calls queued back to back on one stream over one workspace, each
    continuing the last one's state: equal to one call over the joined T."""
    B, T, C = 2, 1200, 192
    x = synth.custom(B, 3 * T, C, "f32", seed=5, random_state=True)
    w, u = x["w"].to(cuda_device), x["u"].to(cuda_device)
    st = x["state_in"].clone()             # pageable, updated in place by every call
    ws = torch.empty(wkv4.host_workspace_bytes(B, T, C, torch.float32, chunk_steps=500),
                     dtype=torch.uint8, device=cuda_device)
    ys = []
    for q in range(3):
        kq = x["k"][:, q * T:(q + 1) * T].contiguous()
        vq = x["v"][:, q * T:(q + 1) * T].contiguous()
        yq = torch.empty_like(kq)
        wkv4.forward_host(kq, vq, w, u, st, y=yq, state_out=st, workspace=ws, chunk_steps=500)
        ys.append(yq)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1)
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"], nthreads=NT)
    parity.check_y(y, y_ref, x["v"], "f32", "host back to back y", calls=9)
    parity.check_state(st, s_ref, x["v"], x["state_in"], calls=9, what="host back to back state")


def test_host_forward_empty_sequence(cuda_device):
    B, C = 3, 40
    x = synth.custom(B, 1, C, "f32", seed=2, random_state=True)
    w, u = x["w"].to(cuda_device), x["u"].to(cuda_device)
    k0 = torch.empty((B, 0, C))
    # T == 0 with a state: passed through (host to host); without: the empty state
    y, s = wkv4.forward_host(k0, k0.clone(), w, u, x["state_in"])
    torch.cuda.synchronize()
    assert y.shape == (B, 0, C) and torch.equal(s, x["state_in"])
    y, s = wkv4.forward_host(k0, k0.clone(), w, u, None)
    torch.cuda.synchronize()
    assert torch.equal(s, synth.zero_state(B, C))
