"""The parity gates can fail: broken implementations, run on the CPU against
the oracle, must be rejected (the kill-WKV negative control of "RWKV in a
self-built engine: a second non-attention paradigm (WKV/RNN)", Ablations /
Negative controls; and a recurrence without the max-trick)."""

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth
from tests import parity


def test_gate_accepts_the_oracle_rounded_to_io_dtype():
    for name, dt in (("tiny", "f32"), ("rwkv4_169m_prefill", "f16")):
        wl = synth.workload(name, B=1, T=64, C=256)
        x = synth.forward_inputs(wl)
        y, s = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
        y_io = torch.from_numpy(y).to(wl.torch_dtype)
        ya = parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"])
        parity.check_y(y_io, y, x["v"], dt, y_abs=ya)
        parity.check_state(s.astype(np.float32), s, x["v"], x["state_in"])


def test_gate_rejects_kill_wkv():
    x = synth.forward_inputs(synth.workload("tiny"))
    y, _ = oracle.forward(x["k"], x["v"], x["w"], x["u"], None)
    with pytest.raises(AssertionError):
        parity.check_y(x["v"], y, x["v"], "f32")


def test_gate_rejects_recurrence_without_max_trick():
    # +30 spikes (e^30 ~ 1e13) stay inside fp32 range; +100 ones do not
    wl = synth.workload("long_t65536", T=4096, C=64, spike_value=100.0)
    x = synth.forward_inputs(wl)
    k = x["k"].numpy().astype(np.float32)
    v = x["v"].numpy().astype(np.float32)
    w, u = x["w"].numpy(), x["u"].numpy()
    y_ref, _ = oracle.forward(k, v, w, u, None)
    # fp32 without rescaling: e^{100} overflows to inf and the output to NaN
    A = np.zeros((1, 64), np.float32)
    D = np.zeros((1, 64), np.float32)
    y = np.empty_like(k)
    with np.errstate(over="ignore", invalid="ignore"):
        for t in range(k.shape[1]):
            eb = np.exp(u + k[:, t]).astype(np.float32)
            y[:, t] = (A + eb * v[:, t]) / (D + eb)
            ek = np.exp(k[:, t]).astype(np.float32)
            A = (np.exp(w) * A + ek * v[:, t]).astype(np.float32)
            D = (np.exp(w) * D + ek).astype(np.float32)
    with pytest.raises(AssertionError):
        parity.check_y(y, y_ref, v, "f32")


def test_gate_rejects_wrong_state():
    x = synth.forward_inputs(synth.workload("rwkv4_169m_prefill", B=2, T=32, C=64))
    _, s = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    bad = s.copy()
    bad[2] += 1e-3  # a max that is off shifts the whole state
    with pytest.raises(AssertionError):
        parity.check_state(bad, s, x["v"], x["state_in"])


def test_ulp_grid():
    assert parity.ulp(np.array([1.0]), "f16")[0] == 2.0 ** -10
    assert parity.ulp(np.array([1.0]), "bf16")[0] == 2.0 ** -7
    assert parity.ulp(np.array([3.0]), "f16")[0] == 2.0 ** -9
    assert parity.ulp(np.array([0.0]), "f16")[0] == 2.0 ** -24
    assert parity.ulp(np.array([1e-6]), "f16")[0] == 2.0 ** -24


def test_y_abs_bounds_the_output_and_equals_it_for_positive_terms():
    x = synth.forward_inputs(synth.workload("rwkv4_169m_prefill", B=2, T=64, C=32))
    y, _ = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    ya = parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    assert np.all(ya >= np.abs(y) * (1 - 1e-12))
    s = x["state_in"].clone()
    s[0] = s[0].abs()
    yp, _ = oracle.forward(x["k"], x["v"].abs(), x["w"], x["u"], s)
    np.testing.assert_array_equal(parity.y_abs(x["k"], x["v"].abs(), x["w"], x["u"], s), yp)


def test_16_bit_gate_rejects_outputs_that_lose_bits_near_zero():
    """An fp16 output whose fp32 computation lost its low half (a 2^-12
    relative error against the terms) fails where the terms cancel, while
    the exact output rounded once to fp16 passes."""
    wl = synth.workload("rwkv4_169m_prefill", B=2, T=256, C=64)
    x = synth.forward_inputs(wl)
    y, _ = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    ya = parity.y_abs(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    parity.check_y(torch.from_numpy(y).half(), y, x["v"], "f16", y_abs=ya)
    rng = np.random.default_rng(0)
    noisy = y + rng.choice([-1.0, 1.0], size=y.shape) * 2.0 ** -12 * ya
    with pytest.raises(AssertionError):
        parity.check_y(torch.from_numpy(noisy).half(), y, x["v"], "f16", y_abs=ya)


def test_16_bit_gate_needs_y_abs():
    y = np.zeros((1, 2, 2))
    with pytest.raises(ValueError):
        parity.check_y(y, y, y, "bf16")
