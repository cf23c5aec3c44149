"""GPU parity of the state combine (wkv4_state_combine) and of a sequence
split over T run segment by segment on one GPU with the split's steps
(summaries from the empty state, prefixes by the device combine, recompute
from the prefix), against one fp64 oracle call over the whole sequence."""

import os

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, tsplit, wkv4
from tests import parity

pytestmark = pytest.mark.gpu

NT = os.cpu_count() or 1


@pytest.fixture(autouse=True)
def no_device_errors(cuda_device):
    yield
    assert wkv4.device_error(reset=True) == 0


def _state(B, C, seed, lift=0.0):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randn(B, C, generator=g), torch.rand(B, C, generator=g) * 1.5 + 0.5,
                        torch.rand(B, C, generator=g) * 4 - 2 + lift]).float()


@pytest.mark.parametrize("n_steps", [0, 1, 37, 100000])
def test_state_combine_matches_oracle(cuda_device, n_steps):
    B, C = 3, 1000
    x = synth.custom(1, 1, C, "f32", seed=4, td_range=(-8.0, 2.0))
    w = x["w"]
    sx, sy = _state(B, C, 1), _state(B, C, 2, lift=5.0)
    sx[:, 0, :8] = synth.zero_state(1, 8)[:, 0]      # an empty first state
    sy[:, 1, 8:16] = synth.zero_state(1, 8)[:, 0]    # an empty second segment
    out = wkv4.state_combine(sx.to(cuda_device), sy.to(cuda_device), n_steps, w.to(cuda_device))
    ref = oracle.combine_states(sx.double().numpy(), sy.double().numpy(), n_steps, w)
    parity.check_state(out.cpu(), ref, np.array([1.0]), sx, what=f"combine n={n_steps}")
    # x = None is the empty state; in place over y
    yd = sy.to(cuda_device)
    wkv4.state_combine(None, yd, n_steps, w.to(cuda_device), out=yd)
    torch.cuda.synchronize()
    assert torch.equal(yd.cpu(), sy)  # the empty state contributes exactly nothing


@pytest.mark.parametrize("shape", [(2, 3000, 256, "f32", 3), (1, 4100, 128, "bf16", 2),
                                   (4, 1024, 768, "f16", 4)],
                         ids=lambda s: "B%dT%dC%d_%s_x%d" % s)
def test_tsplit_segments_on_one_gpu(cuda_device, shape):
    B, T, C, dt, parts = shape
    wl = synth.Workload("custom", B=B, T=T, C=C, dtype=dt, seed=T + C, random_state=True,
                        k_var=2.0, spike_frac=0.001)
    x = synth.forward_inputs(wl)
    g = {k_: (t.to(cuda_device) if t is not None else None) for k_, t in x.items()}
    cuts = [0] + [int(T * (q + 0.7) / parts) for q in range(parts - 1)] + [T]
    segs = [(cuts[q], cuts[q + 1]) for q in range(parts)]
    ops = tsplit.DeviceOps()
    kk = [g["k"][:, a:b].contiguous() for a, b in segs]
    vv = [g["v"][:, a:b].contiguous() for a, b in segs]
    sums = [ops.forward(kk[q], vv[q], g["w"], g["u"], None)[1] for q in range(parts)]
    pre = tsplit.segment_prefixes(sums, [b - a for a, b in segs], g["w"], g["state_in"], ops)
    outs = [ops.forward(kk[q], vv[q], g["w"], g["u"], pre[q]) for q in range(parts)]
    torch.cuda.synchronize()
    y = torch.cat([o[0] for o in outs], dim=1).cpu()
    s_last = outs[-1][1].cpu()
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"], nthreads=NT)
    # the state entering the last segment went through `parts` combines of
    # fp32 states (each summary, each prefix): the 16-bit gate's calls term
    calls = 2 * parts
    ya = None if dt == "f32" else parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"], NT)
    parity.check_y(y, y_ref, x["v"], dt, f"split {shape} y", y_abs=ya, calls=calls)
    parity.check_state(s_last, s_ref, x["v"], x["state_in"], calls=calls + 1,
                       what=f"split {shape} state")
