"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element, with the tolerances of tests/parity.py.

Small cases span several tiles and a ragged tail in T and C; the full-size
workloads (the 169m and 14B prefill widths, 1024 decode steps of 256
sequences, and the 65536-step spiked case) live in test_gpu_workloads.py.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity

pytestmark = pytest.mark.gpu

NT = os.cpu_count() or 1
VARIANTS = [wkv4.KERNEL_AUTO, wkv4.KERNEL_SEQ, wkv4.KERNEL_SCAN, wkv4.KERNEL_SCAN_LDG,
            wkv4.KERNEL_STEP]
VNAMES = {0: "auto", 1: "seq", 2: "scan", 3: "scan_ldg", 4: "step"}


def to_dev(x, dev):
    return {k: (t.to(dev) if t is not None else None) for k, t in x.items()}


def gpu_forward(x, dev, variant=wkv4.KERNEL_AUTO):
    g = to_dev(x, dev)
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], variant=variant)
    torch.cuda.synchronize()
    return y.cpu(), s.cpu()


def check(x, dtype, y, s, what, calls=1):
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"], nthreads=NT)
    ya = None if dtype == "f32" else parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"], NT)
    parity.check_y(y, y_ref, x["v"], dtype, what + " y", y_abs=ya)
    parity.check_state(s, s_ref, x["v"], x["state_in"], calls=calls, what=what + " state")


@pytest.fixture(autouse=True)
def no_device_errors(cuda_device):
    yield
    assert wkv4.device_error(reset=True) == 0


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_tiny_workload(cuda_device, variant):
    wl = synth.workload("tiny")
    x = synth.forward_inputs(wl)
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, wl.dtype, y, s, f"tiny/{VNAMES[variant]}")


SHAPES = [
    # (B, T, C, dtype, random_state): several tiles and ragged tails
    (2, 1000, 200, "f16", True),
    (3, 517, 96, "bf16", False),
    (1, 777, 36, "f32", True),
    (2, 2049, 128, "f32", False),
    (1, 4, 8, "f16", True),
    (5, 130, 1000, "bf16", True),
    (1, 3000, 100, "f16", False),   # C * 2 bytes not a multiple of 16: element-wise loads
    (2, 300, 5, "f32", True),       # C = 5: tails everywhere
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dT%dC%d_%s" % s[:4])
@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_ragged_shapes(cuda_device, shape, variant):
    B, T, C, dt, rs = shape
    x = synth.custom(B, T, C, dt, seed=B * 1000 + T + C, random_state=rs, k_var=2.0)
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, dt, y, s, f"{shape}/{VNAMES[variant]}")


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_spikes_beyond_fp32_exp_range(cuda_device, variant):
    """k up to +200 (e^200 overflows fp32): the max-trick and the per-chunk
    fallback keep every exponent in range."""
    x = synth.custom(2, 700, 64, "f32", seed=77, k_var=4.0, td_range=(-8.0, 2.0),
                     u_range=(-3.0, 3.0), spike_frac=0.01, spike_value=200.0)
    x["k"][0, 10:20, 3] = -150.0
    y, s = gpu_forward(x, cuda_device, variant)
    assert torch.isfinite(y).all() and torch.isfinite(s).all()
    check(x, "f32", y, s, f"spikes/{VNAMES[variant]}")


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_extreme_decay_and_bonus(cuda_device, variant):
    x = synth.custom(2, 600, 64, "f32", seed=5, random_state=True)
    x["w"][:16] = -1e30       # only the previous token survives
    x["w"][16:32] = 0.0       # no decay: cumulative softmax average
    x["w"][32:40] = -1e-9
    x["u"][40:48] = 40.0      # bonus dominates
    x["u"][48:56] = -60.0     # bonus vanishes
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, "f32", y, s, f"extreme/{VNAMES[variant]}")


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: VNAMES[v])
def test_lifted_state_with_fast_decay(cuda_device, variant, dt):
    """A carried state 43.5 nats above a chunk whose k spans 54.5 nats, under
    decays of 5 to 9 nats a step: the state's weight after i steps,
    e^{43.5 - i |w|}, is still comparable with the chunk's own denominator
    (about e^{-54.5}) where e^{i w} alone is below the smallest float."""
    B, T, C = 1, 96, 64
    x = synth.custom(B, T, C, dt, seed=11, random_state=True)
    x["w"][:] = -torch.linspace(5.0, 9.0, C, dtype=torch.float32)
    x["u"][:] = 0.0
    x["k"][:, :32, :] = -54.5
    x["k"][:, 0, :] = 0.0
    x["state_in"][2] = 43.5
    x["state_in"][1] = 1.3
    x["state_in"][0] = 0.9
    y, s = gpu_forward(x, cuda_device, variant)
    check(x, dt, y, s, f"lifted/{dt}/{VNAMES[variant]}")


def test_misaligned_pointers_take_elementwise_path(cuda_device):
    B, T, C = 2, 300, 64
    x = synth.custom(B, T, C, "f16", seed=9, random_state=True)
    g = to_dev(x, cuda_device)
    kb = torch.empty(B * T * C + 1, dtype=torch.float16, device=cuda_device)
    vb = torch.empty_like(kb)
    yb = torch.empty_like(kb)
    kb[1:].copy_(g["k"].reshape(-1))
    vb[1:].copy_(g["v"].reshape(-1))
    so = torch.empty((3, B, C), dtype=torch.float32, device=cuda_device)
    for variant in VARIANTS:
        rc = wkv4.forward_raw(B, T, C, g["w"].data_ptr(), g["u"].data_ptr(), kb[1:].data_ptr(),
                              vb[1:].data_ptr(), g["state_in"].data_ptr(), yb[1:].data_ptr(),
                              so.data_ptr(), wkv4.F16, variant)
        assert rc == 0
        torch.cuda.synchronize()
        check(x, "f16", yb[1:].reshape(B, T, C).cpu(), so.cpu(), f"misaligned/{VNAMES[variant]}")


def test_zero_steps_copies_state(cuda_device):
    x = synth.custom(3, 0, 40, "f32", seed=1, random_state=True)
    g = to_dev(x, cuda_device)
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"])
    assert torch.equal(s.cpu(), x["state_in"])
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], None)
    assert torch.equal(s.cpu(), synth.zero_state(3, 40))


def test_empty_batch_and_channels(cuda_device):
    for B, C in ((0, 16), (2, 0)):
        x = synth.custom(B, 5, C, "f32", seed=0)
        y, s = gpu_forward(x, cuda_device)
        assert y.numel() == 0 and s.numel() == 0


def test_in_place_state(cuda_device):
    x = synth.custom(2, 500, 128, "bf16", seed=3, random_state=True)
    g = to_dev(x, cuda_device)
    st = g["state_in"].clone()
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], st, state_out=st)
    torch.cuda.synchronize()
    assert s.data_ptr() == st.data_ptr()
    check(x, "bf16", y.cpu(), st.cpu(), "in-place")


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_decode_step_equals_single_step_forward(cuda_device, dt):
    x = synth.custom(4, 1, 96, dt, seed=21, random_state=True)
    g = to_dev(x, cuda_device)
    y_f, s_f = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"])
    st = g["state_in"].clone()
    y_d = wkv4.decode_step(g["k"][:, 0].contiguous(), g["v"][:, 0].contiguous(), g["w"], g["u"], st)
    torch.cuda.synchronize()
    assert torch.equal(y_d, y_f[:, 0]) and torch.equal(st, s_f)
    check(x, dt, y_f.cpu(), s_f.cpu(), "T=1")


@pytest.mark.parametrize("split", [1, 255, 256, 700])
def test_chained_calls_match_single_call(cuda_device, split):
    x = synth.custom(2, 1500, 160, "f32", seed=31, random_state=True, k_var=4.0,
                     td_range=(-8.0, 2.0), spike_frac=0.001)
    g = to_dev(x, cuda_device)
    y, s = wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"])
    y1, s1 = wkv4.forward(g["k"][:, :split].contiguous(), g["v"][:, :split].contiguous(), g["w"],
                          g["u"], g["state_in"])
    y2, s2 = wkv4.forward(g["k"][:, split:].contiguous(), g["v"][:, split:].contiguous(), g["w"],
                          g["u"], s1)
    torch.cuda.synchronize()
    yc = torch.cat([y1, y2], dim=1).cpu()
    check(x, "f32", yc, s2.cpu(), f"chained@{split}", calls=2)
    parity.check_y(yc, y.cpu().double().numpy(), x["v"], "f32", "chained vs single")


def test_forward_under_cuda_graph(cuda_device):
    """A forward call captured in a CUDA graph replays correctly."""
    x = synth.custom(2, 1024, 256, "f16", seed=41, random_state=True)
    g = to_dev(x, cuda_device)
    y = torch.empty_like(g["k"])
    s = torch.empty_like(g["state_in"])
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], y=y, state_out=s)  # warm-up
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        wkv4.forward(g["k"], g["v"], g["w"], g["u"], g["state_in"], y=y, state_out=s)
    y.zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    check(x, "f16", y.cpu(), s.cpu(), "graph")


@pytest.mark.parametrize("shape", [(128, 100, 2048, "f16"), (48, 600, 1000, "bf16"), (40, 300, 512, "f32")],
                         ids=lambda s: "B%dT%dC%d_%s" % s)
def test_persistent_clusters_walk_many_tiles(cuda_device, shape):
    """Far more channel tiles than clusters that fit at once (one round per
    tile): every cluster walks many tiles, alternating its parameter and
    aggregate slots, with the carried state and partial last tiles."""
    B, T, C, dt = shape
    x = synth.custom(B, T, C, dt, seed=B + T + C, random_state=True, k_var=2.0)
    y, s = gpu_forward(x, cuda_device, wkv4.KERNEL_SCAN)
    check(x, dt, y, s, f"persistent {shape}")
