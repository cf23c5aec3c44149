"""Calls of different kernels queued back to back on one stream with no host
synchronisation between them, each consuming the one before it -- the token
shift's xk, xv feeding the forward as k, v, the forward's state feeding a
decode step -- eagerly and as one CUDA graph.  Every kernel of the library is
launched so that it may start while the kernel before it is finishing, and
waits for it before its first global access; the results must equal the same
calls each followed by a device synchronisation (bit for bit) and the fp64
oracle run on the same chain."""

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity

pytestmark = pytest.mark.gpu


def _chain(x, mk, mv, mr, w, u, state, kd, vd, stream, sync):
    """token shift -> forward (from the shifted k, v) -> decode step (on the
    forward's final state, in place); returns (y, y1, state)."""
    xk, xv, xr = wkv4.token_shift(x, mk, mv, mr, stream=stream)
    if sync:
        torch.cuda.synchronize()
    y, st = wkv4.forward(xk, xv, w, u, state, stream=stream)
    if sync:
        torch.cuda.synchronize()
    y1 = wkv4.decode_step(kd, vd, w, u, st, stream=stream)
    if sync:
        torch.cuda.synchronize()
    return y, y1, st


def test_dependent_kernels_back_to_back(cuda_device):
    B, T, C = 2, 700, 512
    g = torch.Generator().manual_seed(11)
    x = torch.randn(B, T, C, generator=g).to(torch.bfloat16)
    mk, mv, mr = (torch.rand(C, generator=g) for _ in range(3))
    wl = synth.custom(B, 1, C, "bf16", seed=12, random_state=True)
    kd, vd = wl["k"][:, 0].contiguous(), wl["v"][:, 0].contiguous()
    dev = cuda_device
    args = [t.to(dev) for t in (x, mk, mv, mr, wl["w"], wl["u"], wl["state_in"], kd, vd)]
    stream = torch.cuda.Stream(dev)

    ref = _chain(*args, stream, True)
    ref = [t.clone() for t in ref]
    with torch.cuda.stream(stream):
        eager = _chain(*args, stream, False)
    torch.cuda.synchronize()
    for a, b in zip(ref, eager):
        assert torch.equal(a, b)

    # the same chain as one CUDA graph
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        out = _chain(*args, stream, False)
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(ref, out):
        assert torch.equal(a, b)

    # against the oracle: the forward over the GPU's shifted rows (the shift
    # itself is checked against the oracle in test_gpu_shift.py), then one
    # decode step from its final state
    ks = wkv4_shift_rows(args, stream, 0)
    vs = wkv4_shift_rows(args, stream, 1)
    y_ref, s_ref = oracle.forward(ks, vs, wl["w"], wl["u"], wl["state_in"])
    ya = parity.y_abs(ks, vs, wl["w"], wl["u"], wl["state_in"])
    parity.check_y(ref[0].cpu(), y_ref, vs, "bf16", "chain forward y", y_abs=ya)
    y1_ref, s1_ref = oracle.forward(kd[:, None], vd[:, None], wl["w"], wl["u"], s_ref)
    ya1 = parity.y_abs(kd[:, None], vd[:, None], wl["w"], wl["u"], s_ref)
    parity.check_y(ref[1].cpu()[:, None], y1_ref, vd[:, None], "bf16", "chain decode y", y_abs=ya1,
                   calls=1)
    parity.check_state(ref[2].cpu(), s1_ref, vs, wl["state_in"], calls=2, what="chain state")


def wkv4_shift_rows(args, stream, which=0):
    """The GPU's bf16 xk (which=0) or xv (1) of the chain's token shift, on the host."""
    x, mk, mv, mr = args[:4]
    out = wkv4.token_shift(x, mk, mv, mr, stream=stream)[which]
    torch.cuda.synchronize()
    return out.cpu()
