"""GPU parity of the adapter optimiser step (qlora_adam_step) against the
binary64 oracle (Adam with bias correction and decoupled weight decay; the
pages fix fp32 state at 12 bytes per adapter parameter).

Each check runs one GPU step from an fp32 state and the oracle step from the
same state upcast to binary64, with the scalars rounded to fp32 as the
kernel receives them.  Bar: m within 1e-6 of the magnitude of its two
terms, v within 1e-6 relative (a few fp32 roundings); master within 1e-6 of
the old value plus 1e-5 of the learning rate (the update carries fp32
rounding); the bf16 copy is bit-exact
against the round-to-nearest-even of the kernel's own fp32 master (the same
precision takes the same decision on both sides).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
import bit_nf4_quantized_21_b200 as q

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _state(n, seed, steps=3, lr=1e-3):
    """An fp32 state that has taken a few steps (non-zero moments)."""
    g = torch.Generator().manual_seed(seed)
    theta = (torch.randn(n, generator=g) * 0.02).double().numpy()
    m, v = np.zeros(n), np.zeros(n)
    for t in range(1, steps + 1):
        grad = (torch.randn(n, generator=g) * 1e-2).double().numpy()
        theta, m, v = O.adam_step(theta, m, v, grad, t, lr, 0.9, 0.999, 1e-8)
    f32 = lambda a: torch.tensor(a, dtype=torch.float32)
    return f32(theta), f32(m), f32(v), (torch.randn(n, generator=g) * 1e-2).float()


def _check(n, seed, grad_dtype=torch.float32, t=4, lr=1e-3, betas=(0.9, 0.999), eps=1e-8, wd=0.0, gscale=1.0):
    theta, m, v, grad = _state(n, seed, steps=t - 1, lr=lr)
    grad = grad.to(grad_dtype)
    dm, dmm, dv, dg = (x.to(DEV) for x in (theta, m, v, grad))
    param = torch.empty(n, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlora_adam_step(dm, dmm, dv, dg, t, lr, betas, eps, wd, param=param, grad_scale=gscale, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    # the oracle takes the scalars as the kernel receives them (fp32): a
    # bias correction 1 - beta^t amplifies a beta's own rounding ~t/(1-beta^t)-fold
    f = lambda x: float(np.float32(x))
    ot, om, ov = O.adam_step(theta.double().numpy(), m.double().numpy(), v.double().numpy(),
                             grad.double().numpy(), t, f(lr), f(betas[0]), f(betas[1]), f(eps),
                             weight_decay=f(wd), grad_scale=f(gscale))
    gt, gm, gv = (x.cpu().double().numpy() for x in (dm, dmm, dv))
    # bars relative to the terms (m and master can cancel; v cannot)
    g64 = grad.double().numpy() * gscale
    m_scale = betas[0] * np.abs(m.double().numpy()) + (1 - betas[0]) * np.abs(g64)
    assert np.all(np.abs(gm - om) <= 1e-6 * m_scale + 1e-37), "m"
    assert np.all(np.abs(gv - ov) <= 1e-6 * np.abs(ov) + 1e-37), "v"
    assert np.all(np.abs(gt - ot) <= 1e-6 * np.abs(theta.double().numpy()) + 1e-5 * lr), "master"
    assert torch.equal(param.cpu(), dm.cpu().to(torch.bfloat16)), "bf16 copy is not RNE of the master"
    # and against the oracle's own master: the bf16 copy is within one bf16
    # step of it (the two masters differ by fp32 rounding, which may flip the
    # rounding of a value next to a bf16 midpoint, never by more)
    pb = param.cpu().double().numpy()
    ulp = np.abs(ot) * 2.0 ** -7 + 1e-37
    assert np.all(np.abs(pb - ot) <= ulp), "bf16 copy vs the oracle's master"
    return dm, dmm, dv, param


@pytest.mark.parametrize("n", [1, 3, 4, 1001, (1 << 20) + 7])
def test_adam_step_matches_oracle(n):
    _check(n, seed=n)


def test_adam_step_bf16_gradients_decay_and_scale():
    _check(4099, seed=5, grad_dtype=torch.bfloat16, t=7, lr=2e-3, betas=(0.8, 0.95), eps=1e-6, wd=0.01,
           gscale=0.5)


def test_adam_first_step_from_zero_state():
    n = 2048
    g = torch.randn(n, generator=torch.Generator().manual_seed(9)) * 1e-3
    theta = torch.randn(n, generator=torch.Generator().manual_seed(10))
    dm, z1, z2, dg = theta.to(DEV), torch.zeros(n, device=DEV), torch.zeros(n, device=DEV), g.to(DEV)
    q.qlora_adam_step(dm, z1, z2, dg, 1, 1e-3, eps=1e-8)
    torch.cuda.synchronize()
    want = theta.double() - 1e-3 * g.double() / (g.double().abs() + 1e-8)
    assert torch.allclose(dm.cpu().double(), want, rtol=1e-6, atol=1e-8)


def test_adam_step_is_deterministic_and_flags_nonfinite():
    a = _check(5000, seed=11)
    b = _check(5000, seed=11)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    n = 100
    grad = torch.zeros(n, device=DEV)
    grad[37] = float("inf")
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    q.qlora_adam_step(torch.zeros(n, device=DEV), torch.zeros(n, device=DEV), torch.zeros(n, device=DEV), grad, 1,
                      1e-3, d_status=st)
    torch.cuda.synchronize()
    assert st.item() & 1
