"""The T split's rank logic (rwkv_wkv_linear_b200.tsplit) on CPU processes:
gloo ranks, each holding one consecutive segment of a sequence, with the
arithmetic steps done by the fp64 oracle (forward, combine_states); the
segments' outputs joined in rank order and the last rank's state must equal
one oracle call over the whole sequence."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from rwkv_wkv_linear_b200 import synth, tsplit


class OracleOps:
    """The split's arithmetic by the fp64 oracle, on CPU torch tensors."""

    def forward(self, k, v, w, u, state_in):
        y, s = oracle.forward(k, v, w, u, None if state_in is None else state_in.numpy())
        return torch.from_numpy(y), torch.from_numpy(s)

    def combine(self, x, y, n_steps, w):
        xs = oracle.empty_state(y.shape[1], y.shape[2]) if x is None else x.numpy()
        return torch.from_numpy(oracle.combine_states(xs, y.numpy(), n_steps, w))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    wl = synth.Workload("custom", B=2, T=97, C=24, dtype="f32", seed=3, random_state=True,
                        k_var=4.0, td_range=(-8.0, 2.0), u_range=(-3.0, 3.0),
                        spike_frac=0.01)
    return synth.forward_inputs(wl)


def _bounds(world):
    # uneven segments, the first shorter than the rest
    T = 97
    cuts = [0] + [int(T * (q + 0.6) / world) for q in range(world - 1)] + [T]
    return [(cuts[q], cuts[q + 1]) for q in range(world)]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _inputs()
        lo, hi = _bounds(world)[rank]
        k = x["k"][:, lo:hi].double()
        v = x["v"][:, lo:hi].double()
        y, s = tsplit.forward_tsplit(k, v, x["w"], x["u"], x["state_in"].double(),
                                     ops=OracleOps())
        out[rank] = (y.numpy(), s.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_tsplit_ranks_match_one_call(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    x = _inputs()
    y_ref, s_ref = oracle.forward(x["k"], x["v"], x["w"], x["u"], x["state_in"])
    y = np.concatenate([res[q][0] for q in range(world)], axis=1)
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)
    s = res[world - 1][1]
    m = np.maximum(s[2], s_ref[2])
    for i in (0, 1):
        np.testing.assert_allclose(s[i] * np.exp(s[2] - m), s_ref[i] * np.exp(s_ref[2] - m),
                                   rtol=1e-11, atol=1e-300)


def test_segment_prefixes_order_and_lengths():
    """The prefix entering segment r joins the segments before it in order,
    each decayed by the steps after it."""
    x = _inputs()
    ops = OracleOps()
    parts = _bounds(3)
    sums = [ops.forward(x["k"][:, a:b].double(), x["v"][:, a:b].double(), x["w"], x["u"], None)[1]
            for a, b in parts]
    pre = tsplit.segment_prefixes(sums, [b - a for a, b in parts], x["w"], x["state_in"].double(),
                                  ops)
    for r, (a, _) in enumerate(parts):
        _, want = oracle.forward(x["k"][:, :a], x["v"][:, :a], x["w"], x["u"], x["state_in"])
        got = pre[r].numpy()
        m = np.maximum(got[2], want[2])
        np.testing.assert_allclose(got[1] * np.exp(got[2] - m), want[1] * np.exp(want[2] - m),
                                   rtol=1e-12)
