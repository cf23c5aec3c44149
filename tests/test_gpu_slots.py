"""GPU parity of the slot-indexed batched decode (wkv4_decode_step_slots): a
pool of S states, B rows each stepping the slot it names, against the oracle's
gather / step / scatter; bit-exact against the plain decode step on the
gathered states; ids outside the pool."""

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import synth, wkv4
from tests import parity

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(autouse=True)
def clear_device_errors(cuda_device):
    wkv4.device_error(reset=True)
    yield


def _pool(S, C, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.stack([torch.randn(S, C, generator=g), torch.rand(S, C, generator=g) * 1.5 + 0.5,
                        torch.rand(S, C, generator=g) * 4 - 2]).float()


def _params(C, seed):
    x = synth.custom(1, 1, C, "f32", seed=seed)
    return x["w"], x["u"]


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("C", [640, 130])  # vector path; C % 4 != 0: one channel a thread
def test_slot_decode_matches_oracle_over_steps(cuda_device, dt, C):
    S, B, steps = 200, 64, 3
    w, u = _params(C, seed=C)
    pool = _pool(S, C, seed=3)
    pool_dev = pool.to(cuda_device)
    pool_ref = pool.double().numpy()
    g = torch.Generator().manual_seed(11)
    for step in range(steps):
        ids = torch.randperm(S, generator=g)[:B].to(torch.int32)
        k = (torch.randn(B, C, generator=g) * 2).to(TORCH_DT[dt])
        v = torch.randn(B, C, generator=g).to(TORCH_DT[dt])
        y = wkv4.decode_step_slots(k.to(cuda_device), v.to(cuda_device), w.to(cuda_device),
                                   u.to(cuda_device), pool_dev, ids.to(cuda_device))
        torch.cuda.synchronize()
        state_before = pool_ref[:, ids.numpy(), :]
        abs_pool = pool_ref.copy()
        abs_pool[0] = np.abs(abs_pool[0])
        ya, _, _ = oracle.decode_slots(k, v.abs(), w, u, abs_pool, ids)
        y_ref, pool_ref, skipped = oracle.decode_slots(k, v, w, u, pool_ref, ids)
        assert skipped == 0
        parity.check_y(y.cpu(), y_ref, v, dt, f"slots {dt} C={C} y step {step}", y_abs=ya)
        got = pool_dev.cpu().double().numpy()
        idx = ids.numpy()
        parity.check_state(got[:, idx, :], pool_ref[:, idx, :], v, state_before,
                           what=f"slots {dt} C={C} state step {step}")
        # the next step starts from the device's stepped rows (each step is checked on its own)
        pool_ref[:, idx, :] = got[:, idx, :]
    assert wkv4.device_error(reset=True) == 0


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_slot_decode_bit_exact_against_plain_decode(cuda_device, dt):
    S, B, C = 97, 40, 512
    w, u = (t.to(cuda_device) for t in _params(C, seed=5))
    pool = _pool(S, C, seed=8).to(cuda_device)
    g = torch.Generator().manual_seed(2)
    ids = torch.randperm(S, generator=g)[:B].to(torch.int32).to(cuda_device)
    k = torch.randn(B, C, generator=g).to(TORCH_DT[dt]).to(cuda_device)
    v = torch.randn(B, C, generator=g).to(TORCH_DT[dt]).to(cuda_device)
    gathered = pool[:, ids.long(), :].contiguous()
    y_plain = wkv4.decode_step(k, v, w, u, gathered)
    before = pool.clone()
    y_slots = wkv4.decode_step_slots(k, v, w, u, pool, ids)
    torch.cuda.synchronize()
    assert torch.equal(y_slots, y_plain)
    assert torch.equal(pool[:, ids.long(), :], gathered)
    others = torch.ones(S, dtype=torch.bool, device=cuda_device)
    others[ids.long()] = False
    assert torch.equal(pool[:, others, :], before[:, others, :])


def test_slot_ids_outside_the_pool_are_reported_and_skipped(cuda_device):
    S, C = 16, 256
    w, u = (t.to(cuda_device) for t in _params(C, seed=6))
    pool = _pool(S, C, seed=9).to(cuda_device)
    before = pool.clone()
    ids = torch.tensor([3, -1, S, 7], dtype=torch.int32, device=cuda_device)
    k = torch.randn(4, C, device=cuda_device)
    v = torch.randn(4, C, device=cuda_device)
    y = torch.full((4, C), 12345.0, device=cuda_device)
    wkv4.decode_step_slots(k, v, w, u, pool, ids, y=y)
    torch.cuda.synchronize()
    assert wkv4.device_error(reset=True) == -8  # WKV4_ERR_SLOT
    assert torch.all(y[1] == 12345.0) and torch.all(y[2] == 12345.0)
    assert not torch.any(y[0] == 12345.0) and not torch.any(y[3] == 12345.0)
    keep = [i for i in range(S) if i not in (3, 7)]
    assert torch.equal(pool[:, keep, :], before[:, keep, :])
    assert wkv4.device_error(reset=True) == 0
