"""Seeded synthetic inputs for the RWKV-4 WKV forward and decode workloads.

This module draws numbers and nothing else: it holds none of the WKV arithmetic,
so both the CUDA path and the CPU oracle can take their inputs from it without
sharing any of the method's code.

Workloads (sizes of the RWKV-4 models the pages discuss):

* ``tiny``                 B=1,  T=16,    C=768,  fp32 I/O, zero state.
* ``rwkv4_169m_prefill``   B=8,  T=1024,  C=768,  fp16 I/O, random state
  (RWKV-4-169m width; "RWKV in a self-built engine: a second non-attention
  paradigm (WKV/RNN)", Methods table, "Model" and "Precision" rows).
* ``rwkv4_14b_prefill``    B=4,  T=1024,  C=5120, bf16 I/O, zero state
  (d_model 5120 and 1K context of "RWKV-4 14B", "Every architecture field").
* ``rwkv4_14b_prefill_gated``  the same with the receptance gate (r ~ N(0, 4)).
* ``decode_b256``          B=256, C=5120, T=1 per call for 1024 calls, bf16.
* ``decode_slots_b256``    the same calls, each serving 256 of a pool of 1024
  conversation states (slot-indexed decode; ids drawn per call).
* ``long_t65536``          B=1,  T=65536, C=2048, fp32 I/O, 0.1% of k set to +30.
* ``token_shift_14b``      B=4,  T=1024,  C=5120, bf16: the token shift feeding k, v
  and r (x, the carried token and three mix vectors).

Recipe (the same for every workload; knobs per workload below):

* ``rng = numpy.random.default_rng(seed)``; draw order: time_decay[C], u[C],
  initial state (num[B,C], den[B,C], max[B,C]) when it is random, k[B,T,C],
  v[B,T,C], then the spike positions.
* ``N(0, s)`` names a normal of *variance* s (standard deviation sqrt(s)).
* ``w = -exp(time_decay)`` is evaluated in fp64 and rounded to fp32; u is fp32.
* k and v are drawn in fp64 and rounded to nearest-even into the I/O dtype
  (bf16 through torch's CPU cast).
* Spikes: exactly ``round(frac * B*T*C)`` distinct flat positions of k, drawn
  without replacement, are *set* to the spike value.
* Decode draws w, u from ``default_rng(seed)`` and each call's k, v from
  ``default_rng([seed, step])``; a slot-indexed decode call's ids are the first
  B of a permutation of the pool drawn from ``default_rng([seed, step, 1])``.
* The receptance r of the gated forward (y = sigmoid(r) wkv) is drawn from a
  stream of its own, ``default_rng([seed, 7])`` (a decode call's from
  ``default_rng([seed, step, 2])``), as N(0, 4) rounded to the I/O dtype, so
  that k, v and the state are the same draws with or without it.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

_TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    C: int
    dtype: str                     # "f32" | "f16" | "bf16": dtype of k, v and y
    seed: int
    k_var: float = 1.0
    v_var: float = 1.0
    td_range: tuple = (-6.0, 1.0)  # time_decay ~ U(lo, hi)
    u_range: tuple = (-1.0, 1.0)   # u ~ U(lo, hi)
    random_state: bool = False     # num ~ N(0,1), den ~ U(0.5,2), max ~ U(-2,2)
    spike_frac: float = 0.0
    spike_value: float = 30.0
    steps: int = 1                 # decode workloads: number of T=1 calls
    slots: int = 0                 # slot-indexed decode: states in the pool (0: one per row)
    op: str = "wkv"                # "wkv" or "token_shift"
    gated: bool = False            # the gated forward (y = sigmoid(r) wkv; r from receptance())

    @property
    def channel_steps(self) -> int:
        return self.B * self.T * self.C * self.steps

    @property
    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPES[self.dtype]

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, T=16, C=768, dtype="f32", seed=0),
    "rwkv4_169m_prefill": Workload("rwkv4_169m_prefill", B=8, T=1024, C=768, dtype="f16",
                                   seed=1, random_state=True),
    "rwkv4_14b_prefill": Workload("rwkv4_14b_prefill", B=4, T=1024, C=5120, dtype="bf16",
                                  seed=2, k_var=2.0),
    "rwkv4_14b_prefill_gated": Workload("rwkv4_14b_prefill_gated", B=4, T=1024, C=5120,
                                        dtype="bf16", seed=2, k_var=2.0, gated=True),
    "decode_b256": Workload("decode_b256", B=256, T=1, C=5120, dtype="bf16", seed=3,
                            steps=1024),
    "decode_slots_b256": Workload("decode_slots_b256", B=256, T=1, C=5120, dtype="bf16", seed=3,
                                  steps=1024, slots=1024),
    "token_shift_14b": Workload("token_shift_14b", B=4, T=1024, C=5120, dtype="bf16", seed=5,
                                op="token_shift"),
    "long_t65536": Workload("long_t65536", B=1, T=65536, C=2048, dtype="f32", seed=4,
                            k_var=4.0, td_range=(-8.0, 2.0), u_range=(-3.0, 3.0),
                            spike_frac=0.001, spike_value=30.0),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def _to_io(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round fp64 samples to nearest-even in the I/O dtype."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return t.to(_TORCH_DTYPES[dtype]).contiguous()


def _draw_params(rng: np.random.Generator, wl: Workload):
    td = rng.uniform(wl.td_range[0], wl.td_range[1], size=wl.C)
    u = rng.uniform(wl.u_range[0], wl.u_range[1], size=wl.C)
    w = torch.from_numpy((-np.exp(td)).astype(np.float32))
    return w, torch.from_numpy(u.astype(np.float32))


def forward_inputs(wl: Workload) -> dict:
    """Inputs of one forward call: w[C], u[C] fp32; k, v [B,T,C] in the I/O
    dtype; state_in [3,B,C] fp32 (planes num, den, max) or None for the zero
    state."""
    rng = np.random.default_rng(wl.seed)
    w, u = _draw_params(rng, wl)
    state = None
    if wl.random_state:
        num = rng.standard_normal((wl.B, wl.C))
        den = rng.uniform(0.5, 2.0, size=(wl.B, wl.C))
        mx = rng.uniform(-2.0, 2.0, size=(wl.B, wl.C))
        state = torch.from_numpy(np.stack([num, den, mx]).astype(np.float32)).contiguous()
    shape = (wl.B, wl.T, wl.C)
    k = rng.standard_normal(shape) * math.sqrt(wl.k_var)
    v = rng.standard_normal(shape) * math.sqrt(wl.v_var)
    if wl.spike_frac > 0.0:
        n = int(round(wl.spike_frac * k.size))
        idx = rng.choice(k.size, size=n, replace=False)
        k.reshape(-1)[idx] = wl.spike_value
    return {"w": w, "u": u, "k": _to_io(k, wl.dtype), "v": _to_io(v, wl.dtype),
            "state_in": state}


def receptance(wl: Workload, var: float = 4.0) -> torch.Tensor:
    """r [B, T, C] ~ N(0, var) in the I/O dtype for the gated forward."""
    rng = np.random.default_rng([wl.seed, 7])
    return _to_io(rng.standard_normal((wl.B, wl.T, wl.C)) * math.sqrt(var), wl.dtype)


def decode_receptance(wl: Workload, step: int, var: float = 4.0) -> torch.Tensor:
    """r [B, C] of gated decode call number ``step``."""
    rng = np.random.default_rng([wl.seed, step, 2])
    return _to_io(rng.standard_normal((wl.B, wl.C)) * math.sqrt(var), wl.dtype)


def decode_params(wl: Workload):
    """w[C], u[C] of a decode workload."""
    rng = np.random.default_rng(wl.seed)
    return _draw_params(rng, wl)


def decode_step_inputs(wl: Workload, step: int):
    """k, v [B,C] of decode call number ``step`` (freshly seeded per call)."""
    rng = np.random.default_rng([wl.seed, step])
    shape = (wl.B, wl.C)
    k = rng.standard_normal(shape) * math.sqrt(wl.k_var)
    v = rng.standard_normal(shape) * math.sqrt(wl.v_var)
    return _to_io(k, wl.dtype), _to_io(v, wl.dtype)


def shift_inputs(wl: Workload) -> dict:
    """Token-shift inputs: x [B,T,C] ~ N(0,1) and x_prev [B,C] ~ N(0,1) in the
    I/O dtype, mix_k, mix_v, mix_r [C] ~ U(0,1) fp32 (drawn in that order from
    default_rng(seed))."""
    rng = np.random.default_rng(wl.seed)
    x = rng.standard_normal((wl.B, wl.T, wl.C))
    x_prev = rng.standard_normal((wl.B, wl.C))
    mixes = [torch.from_numpy(rng.uniform(0.0, 1.0, size=wl.C).astype(np.float32)) for _ in range(3)]
    return {"x": _to_io(x, wl.dtype), "x_prev": _to_io(x_prev, wl.dtype), "mix": mixes}


def decode_slot_ids(wl: Workload, step: int) -> torch.Tensor:
    """int32 [B]: the distinct pool slots that decode call ``step`` serves."""
    rng = np.random.default_rng([wl.seed, step, 1])
    return torch.from_numpy(rng.permutation(wl.slots)[:wl.B].astype(np.int32))


def custom(B: int, T: int, C: int, dtype: str = "f32", seed: int = 0, **kw) -> dict:
    """Inputs of an arbitrary shape drawn with the same recipe."""
    return forward_inputs(Workload("custom", B=B, T=T, C=C, dtype=dtype, seed=seed, **kw))


def zero_state(B: int, C: int) -> torch.Tensor:
    """The empty state: num = den = 0 and max = -1e38 (fp32)."""
    s = torch.zeros((3, B, C), dtype=torch.float32)
    s[2].fill_(-1e38)
    return s
