"""GPU parity at the full workload sizes, element by element against the fp64
oracle (all outputs and the final state):

* rwkv4_169m_prefill  B=8, T=1024, C=768, fp16, random state  (the benchmark's
  workload and launch configuration)
* rwkv4_14b_prefill   B=4, T=1024, C=5120, bf16, zero state
* long_t65536         B=1, T=65536, C=2048, fp32, 0.1% of k at +30; also as
                      16 chained calls of T=4096 with the state carried
* decode_b256         256 sequences, C=5120, 1024 decode steps in place
"""

import os

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity
from tests.test_gpu_parity import VNAMES, check, gpu_forward, to_dev

pytestmark = pytest.mark.gpu

NT = os.cpu_count() or 1


@pytest.fixture(autouse=True)
def no_device_errors(cuda_device):
    yield
    assert wkv4.device_error(reset=True) == 0


@pytest.mark.parametrize("variant", [wkv4.KERNEL_AUTO, wkv4.KERNEL_SEQ, wkv4.KERNEL_STEP],
                         ids=lambda v: VNAMES[v])
def test_rwkv4_169m_prefill(cuda_device, variant):
    wl = synth.workload("rwkv4_169m_prefill")
    x = synth.forward_inputs(wl)
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, wl.dtype, y, s, f"169m/{VNAMES[variant]}")


@pytest.mark.parametrize("variant", [wkv4.KERNEL_AUTO, wkv4.KERNEL_SEQ], ids=lambda v: VNAMES[v])
def test_rwkv4_14b_prefill(cuda_device, variant):
    wl = synth.workload("rwkv4_14b_prefill")
    x = synth.forward_inputs(wl)
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, wl.dtype, y, s, f"14b/{VNAMES[variant]}")


def test_long_t65536_single_and_chained(cuda_device):
    wl = synth.workload("long_t65536")
    x = synth.forward_inputs(wl)
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], None, nthreads=NT)
    g = to_dev(x, cuda_device)
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], None)
    torch.cuda.synchronize()
    parity.check_y(y.cpu(), y_ref, x["v"], "f32", "long y")
    parity.check_state(s.cpu(), s_ref, x["v"], None, what="long state")
    # 16 chained calls of 4096 steps, state carried on the device
    yc = torch.empty_like(g["k"])
    st = None
    for i in range(16):
        sl = slice(i * 4096, (i + 1) * 4096)
        yi, st = wkv4.forward(g["k"][:, sl].contiguous(), g["v"][:, sl].contiguous(), g["w"],
                              g["u"], st)
        yc[:, sl] = yi
    torch.cuda.synchronize()
    parity.check_y(yc.cpu(), y_ref, x["v"], "f32", "long chained y")
    parity.check_state(st.cpu(), s_ref, x["v"], None, calls=16, what="long chained state")
    parity.check_y(yc.cpu(), y.cpu().double().numpy(), x["v"], "f32", "chained vs single")


def test_decode_b256_1024_steps(cuda_device):
    """Every output of all 1024 calls and the final state against the oracle
    run call by call over the same inputs (its own fp64 state carried); the
    16-bit gate's y_abs comes from a second oracle chain on |v|."""
    wl = synth.workload("decode_b256")
    w, u = synth.decode_params(wl)
    gw, gu = w.to(cuda_device), u.to(cuda_device)
    state = synth.zero_state(wl.B, wl.C).to(cuda_device)
    ref_state = oracle.empty_state(wl.B, wl.C)
    abs_state = oracle.empty_state(wl.B, wl.C)
    vmax = 0.0
    for step in range(wl.steps):
        k, v = synth.decode_step_inputs(wl, step)
        vmax = max(vmax, float(v.abs().max()))
        y = wkv4.decode_step(k.to(cuda_device), v.to(cuda_device), gw, gu, state)
        yc = y.cpu()
        y_ref, ref_state = oracle.decode(k, v, w, u, ref_state)
        ya, abs_state = oracle.decode(k, v.abs(), w, u, abs_state)
        # the state behind call `step` passed through `step` fp32 buffers
        parity.check_y(yc, y_ref, v, "bf16", f"decode step {step} y", y_abs=ya, calls=step)
    torch.cuda.synchronize()
    parity.check_state(state.cpu(), ref_state, np.array([vmax]), None, calls=wl.steps,
                       what="decode final state")
