"""The seeded generator draws what its recipe says and nothing else."""

import numpy as np
import torch

from rwkv_wkv_linear_b200 import synth


def test_deterministic_and_typed():
    a = synth.forward_inputs(synth.workload("rwkv4_169m_prefill", T=8))
    b = synth.forward_inputs(synth.workload("rwkv4_169m_prefill", T=8))
    for key in ("w", "u", "k", "v", "state_in"):
        assert torch.equal(a[key], b[key])
    assert a["k"].dtype == torch.float16 and a["k"].shape == (8, 8, 768)
    assert a["w"].dtype == torch.float32 and a["state_in"].shape == (3, 8, 768)
    assert torch.all(a["w"] < 0)
    assert torch.all(a["state_in"][1] >= 0.5) and torch.all(a["state_in"][1] <= 2.0)


def test_decay_and_bonus_ranges():
    x = synth.forward_inputs(synth.workload("long_t65536", T=4, C=4096))
    td = torch.log(-x["w"].double())
    assert td.min() >= -8.0 - 1e-6 and td.max() <= 2.0 + 1e-6
    assert x["u"].min() >= -3.0 and x["u"].max() <= 3.0


def test_spike_count_is_exact():
    wl = synth.workload("long_t65536", T=1000, C=512)
    x = synth.forward_inputs(wl)
    n = int((x["k"] == 30.0).sum())
    assert n == round(0.001 * 1000 * 512)


def test_variance_convention():
    x = synth.forward_inputs(synth.workload("rwkv4_14b_prefill", T=256))
    # N(0, 2) is variance 2: std sqrt(2)
    assert abs(float(x["k"].float().std()) - np.sqrt(2.0)) < 0.01
    assert abs(float(x["v"].float().std()) - 1.0) < 0.01
    assert x["state_in"] is None


def test_decode_steps_are_independently_seeded():
    wl = synth.workload("decode_b256", B=4, C=64)
    k0, v0 = synth.decode_step_inputs(wl, 0)
    k1, _ = synth.decode_step_inputs(wl, 1)
    k0b, _ = synth.decode_step_inputs(wl, 0)
    assert torch.equal(k0, k0b) and not torch.equal(k0, k1)
    assert k0.dtype == torch.bfloat16 and k0.shape == (4, 64)
