"""The gradient check that smoke() applies to the GPU backward (__graft_entry__.check_backward),
exercised on the CPU: it accepts the oracle's own gradients and gradients perturbed within the
bf16 rounding it allows for, and rejects planted mistakes (a flipped dS sign, a wrong dK scale,
dV from unmasked weights)."""

import math

import numpy as np
import pytest
import torch

import __graft_entry__ as G
import oracle
from ring_blockwise_softmax_b200 import inputs as I


def _case(N=96, d=32, seed=77):
    q, k, v = I.make_small(1, 2, N, d, "bf16", seed=seed)
    do = I.draw((1, 2, N, d), seed, 3, "normal", 1.0, "bf16")
    pos = np.arange(N)
    allowed = oracle.allowed_mask(pos, pos, True)
    scale = 1 / math.sqrt(d)
    o = np.zeros((1, 2, N, d))
    lse = np.zeros((1, 2, N))
    for h in range(2):
        o[0, h], lse[0, h] = oracle.attention(q[0, h].double().numpy(), k[0, h].double().numpy(),
                                              v[0, h].double().numpy(), scale, allowed)
    o_t = torch.from_numpy(o).to(torch.bfloat16).float()
    lse_t = torch.from_numpy(lse).float()
    grads = [np.zeros((1, 2, N, d)) for _ in range(3)]
    for h in range(2):
        g = oracle.attention_backward(q[0, h].double().numpy(), k[0, h].double().numpy(), v[0, h].double().numpy(),
                                      o_t[0, h].double().numpy(), lse_t[0, h].double().numpy(),
                                      do[0, h].double().numpy(), scale, allowed)
        for a, x in zip(grads, g):
            a[0, h] = x
    return (q, k, v, o_t, lse_t, do, allowed), grads


def _run(args, grads):
    q, k, v, o, lse, do, allowed = args
    G.check_backward(q, k, v, o, lse, do, *(torch.from_numpy(x) for x in grads), allowed)


def test_accepts_the_oracle_gradients():
    args, grads = _case()
    _run(args, grads)


def test_accepts_bf16_sized_perturbations():
    args, grads = _case()
    rng = np.random.default_rng(5)
    # Relative 2^-9 noise per element stays well inside the 2^-7 * |.|-sum allowance.
    _run(args, [g * (1 + 2.0 ** -9 * rng.uniform(-1, 1, g.shape)) for g in grads])


@pytest.mark.parametrize("mistake", ["dq_sign", "dk_scale", "dv_unmasked"])
def test_rejects_planted_mistakes(mistake):
    args, grads = _case()
    dq, dk, dv = (g.copy() for g in grads)
    if mistake == "dq_sign":
        dq = -dq
    elif mistake == "dk_scale":
        dk = dk * 1.2
    else:
        q, k, v, o, lse, do, allowed = args
        d = q.shape[-1]
        for h in range(2):
            p = np.exp(q[0, h].double().numpy() @ k[0, h].double().numpy().T / math.sqrt(d)
                       - lse[0, h].double().numpy()[:, None])
            dv[0, h] = p.T @ do[0, h].double().numpy()
    with pytest.raises(AssertionError):
        _run(args, (dq, dk, dv))
