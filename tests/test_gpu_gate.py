"""GPU parity of the gated forward and decode step (y = sigmoid(r) * wkv, the
receptance gate of the time mix fused into the output pass) against the fp64
oracle's forward_gated / decode_gated, through the C ABI: the 169m and 14B
widths, ragged shapes on every kernel, the gate's limits, the state (which the
gate must not touch), the decode step against one step of the forward, and
misaligned pointers."""

import os

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity
from tests.test_gpu_parity import VARIANTS, VNAMES, to_dev

pytestmark = pytest.mark.gpu

NT = os.cpu_count() or 1


@pytest.fixture(autouse=True)
def no_device_errors(cuda_device):
    yield
    assert wkv4.device_error(reset=True) == 0


def gated(x, r, dev, variant=wkv4.KERNEL_AUTO):
    g = to_dev(x, dev)
    y, s = wkv4.forward_gated(g["k"], g["v"], r.to(dev), g["w"], g["u"], g["state_in"],
                              variant=variant)
    torch.cuda.synchronize()
    return y.cpu(), s.cpu()


def check_gated(x, r, dtype, y, s, what):
    y_ref, s_ref = oracle.forward_gated(x["k"], x["v"], r, x["w"], x["u"], x["state_in"],
                                        nthreads=NT)
    ya = None if dtype == "f32" else parity.y_abs_gated(x["k"], x["v"], r, x["w"], x["u"],
                                                        x["state_in"], NT)
    parity.check_y(y, y_ref, x["v"], dtype, what + " y", y_abs=ya)
    parity.check_state(s, s_ref, x["v"], x["state_in"], what=what + " state")


@pytest.mark.parametrize("name", ["rwkv4_169m_prefill", "rwkv4_14b_prefill"])
def test_gated_model_widths(cuda_device, name):
    wl = synth.workload(name)
    x = synth.forward_inputs(wl)
    r = synth.receptance(wl)
    y, s = gated(x, r, cuda_device)
    check_gated(x, r, wl.dtype, y, s, f"gated {name}")


SHAPES = [
    (2, 1000, 200, "f16", True),
    (3, 517, 96, "bf16", False),
    (1, 777, 36, "f32", True),
    (2, 2049, 128, "f32", False),    # several rounds
    (1, 3000, 100, "f16", False),    # element-wise loads
    (2, 300, 5, "f32", True),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dT%dC%d_%s" % s[:4])
@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_gated_ragged_shapes(cuda_device, shape, variant):
    B, T, C, dt, rs = shape
    wl = synth.Workload("custom", B=B, T=T, C=C, dtype=dt, seed=B * 1000 + T + C, k_var=2.0,
                        random_state=rs)
    x = synth.forward_inputs(wl)
    r = synth.receptance(wl)
    y, s = gated(x, r, cuda_device, variant)
    check_gated(x, r, dt, y, s, f"gated {shape}/{VNAMES[variant]}")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_gate_limits_and_state(cuda_device, variant, dt):
    """r = 0 halves wkv, r = +40 passes it, r = -100 and -inf give 0 (e^{-r}
    overflows), +inf passes it; the final state equals the ungated call's bit
    for bit (the gate touches only the outputs)."""
    wl = synth.Workload("custom", B=2, T=600, C=128, dtype=dt, seed=12, random_state=True)
    x = synth.forward_inputs(wl)
    g = to_dev(x, cuda_device)
    y0, s0 = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], variant=variant)
    r = torch.zeros_like(x["k"])
    r[:, :, 32:64] = 40.0
    r[:, :, 64:96] = -100.0
    r[0, :, 96:112] = float("-inf")
    r[1, :, 96:112] = float("inf")
    yg, sg = wkv4.forward_gated(g["k"], g["v"], r.to(cuda_device), g["w"], g["u"], g["state_in"],
                                variant=variant)
    torch.cuda.synchronize()
    assert torch.equal(sg, s0)
    y0, yg = y0.cpu().double(), yg.cpu().double()
    assert torch.all(yg[:, :, 64:96] == 0) and torch.all(yg[0, :, 96:112] == 0)
    ulp_rel = {"f32": 2.0 ** -20, "bf16": 2.0 ** -7}[dt]
    torch.testing.assert_close(yg[:, :, 32:64], y0[:, :, 32:64], rtol=ulp_rel, atol=0)
    torch.testing.assert_close(yg[1, :, 96:112], y0[1, :, 96:112], rtol=ulp_rel, atol=0)
    torch.testing.assert_close(yg[:, :, :32], 0.5 * y0[:, :, :32], rtol=2 * ulp_rel, atol=1e-30)
    check_gated(x, r, dt, yg.to(x["k"].dtype), sg.cpu(), f"limits/{dt}/{VNAMES[variant]}")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_gated_decode_matches_oracle_and_one_step_forward(cuda_device, dt):
    B, C, steps = 64, 640, 8
    wl = synth.Workload("custom", B=B, T=1, C=C, dtype=dt, seed=5, steps=steps)
    w, u = synth.decode_params(wl)
    gw, gu = w.to(cuda_device), u.to(cuda_device)
    state = synth.zero_state(B, C).to(cuda_device)
    ref = oracle.empty_state(B, C)
    ref_abs = oracle.empty_state(B, C)
    for step in range(steps):
        k, v = synth.decode_step_inputs(wl, step)
        r = synth.decode_receptance(wl, step)
        kd, vd, rd = k.to(cuda_device), v.to(cuda_device), r.to(cuda_device)
        before = state.clone()
        y = wkv4.decode_step_gated(kd, vd, rd, gw, gu, state)
        # the same step as a gated forward with T = 1 (the decode kernel): bit for bit
        yf, sf = wkv4.forward_gated(kd[:, None], vd[:, None], rd[:, None], gw, gu, before)
        torch.cuda.synchronize()
        assert torch.equal(yf[:, 0], y) and torch.equal(sf, state)
        y_ref, ref = oracle.decode_gated(k, v, r, w, u, ref)
        ya, ref_abs = oracle.decode(k, v.abs(), w, u, ref_abs)
        ya = oracle.sigmoid(r) * ya
        parity.check_y(y.cpu(), y_ref, v, dt, f"gated decode {dt} step {step}", y_abs=ya,
                       calls=step)
    parity.check_state(state.cpu(), ref, np.array([5.0]), None, calls=steps,
                       what=f"gated decode {dt} state")


def test_gated_misaligned_receptance_takes_elementwise_path(cuda_device):
    B, T, C = 2, 300, 64
    wl = synth.Workload("custom", B=B, T=T, C=C, dtype="f16", seed=9, random_state=True)
    x = synth.forward_inputs(wl)
    r = synth.receptance(wl)
    g = to_dev(x, cuda_device)
    rb = torch.empty(B * T * C + 1, dtype=torch.float16, device=cuda_device)
    rb[1:].copy_(r.reshape(-1))
    y = torch.empty_like(g["k"])
    so = torch.empty((3, B, C), dtype=torch.float32, device=cuda_device)
    lib = wkv4.load()
    for variant in VARIANTS:
        rc = lib.wkv4_forward_gated_variant(B, T, C, g["w"].data_ptr(), g["u"].data_ptr(),
                                            g["k"].data_ptr(), g["v"].data_ptr(),
                                            rb[1:].data_ptr(), g["state_in"].data_ptr(),
                                            y.data_ptr(), so.data_ptr(), None, wkv4.F16, variant)
        assert rc == 0
        torch.cuda.synchronize()
        check_gated(x, r, "f16", y.cpu(), so.cpu(), f"gated misaligned r/{VNAMES[variant]}")
