"""GPU parity of the token shift (wkv4_token_shift) against the oracle's fp64
mix, element by element: three I/O types, aligned (16-byte vectors) and
unaligned (one channel a thread) shapes, runs that end mid-way, with and
without the carried token and the third output; chained calls against one
call (bitwise); T = 0."""

import numpy as np
import pytest
import torch

import oracle
from rwkv_wkv_linear_b200 import wkv4
from tests import parity

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _inputs(B, T, C, dt, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C, generator=g).to(TORCH_DT[dt])
    xp = torch.randn(B, C, generator=g).to(TORCH_DT[dt])
    mixes = [torch.rand(C, generator=g) for _ in range(3)]
    mixes[0][:3] = torch.tensor([0.0, 1.0, 0.5])
    return x, xp, mixes


def _bound(ref, x, xp, dt):
    """One unit in the last place of the output type at the reference, plus
    fp32 rounding of x_prev + mix (x - x_prev): 2^-21 (|x_t| + |x_{t-1}|)."""
    x = parity.to_f64(x)
    sh = np.concatenate([parity.to_f64(xp)[:, None], x[:, :-1]], axis=1)
    return parity.ulp(ref, dt) + 2.0 ** -21 * (np.abs(x) + np.abs(sh))


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", [(2, 37, 512), (3, 50, 130), (1, 16, 8)],
                         ids=lambda s: "B%dT%dC%d" % s)
@pytest.mark.parametrize("with_prev", [True, False])
def test_token_shift_matches_oracle(cuda_device, dt, shape, with_prev):
    B, T, C = shape
    x, xp, mixes = _inputs(B, T, C, dt, seed=B * 100 + T + C)
    xp_used = xp if with_prev else None
    dev = lambda t: None if t is None else t.to(cuda_device)
    xl = torch.empty(B, C, dtype=x.dtype, device=cuda_device)
    outs = wkv4.token_shift(dev(x), *[dev(m) for m in mixes], x_prev=dev(xp_used), x_last=xl)
    torch.cuda.synchronize()
    refs, last = oracle.token_shift(x, xp_used, mixes)
    xp64 = xp if with_prev else torch.zeros(B, C)
    for i, (o, r) in enumerate(zip(outs, refs)):
        err = np.abs(parity.to_f64(o.cpu()) - r)
        bound = _bound(r, x, xp64, dt)
        assert np.all(err <= bound), (i, float(np.max(err - bound)))
    assert torch.equal(xl.cpu(), x[:, -1])


def test_token_shift_two_outputs_and_chaining(cuda_device):
    B, T, C = 2, 70, 256
    x, xp, mixes = _inputs(B, T, C, "bf16", seed=4)
    x, xp = x.to(cuda_device), xp.to(cuda_device)
    mk, mv = mixes[0].to(cuda_device), mixes[1].to(cuda_device)
    whole_k, whole_v, none = wkv4.token_shift(x, mk, mv, x_prev=xp)
    assert none is None
    mid = torch.empty_like(xp)
    a_k, a_v, _ = wkv4.token_shift(x[:, :23].contiguous(), mk, mv, x_prev=xp, x_last=mid)
    b_k, b_v, _ = wkv4.token_shift(x[:, 23:].contiguous(), mk, mv, x_prev=mid)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([a_k, b_k], dim=1), whole_k)
    assert torch.equal(torch.cat([a_v, b_v], dim=1), whole_v)


def test_token_shift_zero_steps_copies_the_carried_token(cuda_device):
    B, C = 3, 64
    xp = torch.randn(B, C, device=cuda_device)
    xl = torch.full((B, C), 7.0, device=cuda_device)
    x = torch.empty(B, 0, C, device=cuda_device)
    m = torch.rand(C, device=cuda_device)
    wkv4.token_shift(x, m, m, x_prev=xp, x_last=xl)
    torch.cuda.synchronize()
    assert torch.equal(xl, xp)
    wkv4.token_shift(x, m, m, x_last=xl)
    torch.cuda.synchronize()
    assert torch.all(xl == 0)
