"""Pins of the oracle's AdamW step (the adapters' update): against torch.optim.AdamW run in
fp64 on the CPU (a library routine) over several steps, and two special cases with a closed
form."""

import numpy as np
import torch

from oracle import nf4_oracle as O


def test_adamw_matches_torch_over_steps():
    rng = np.random.default_rng(0)
    p0 = rng.standard_normal(1000)
    grads = [rng.standard_normal(1000) for _ in range(5)]
    kw = dict(lr=1e-3, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)
    tp = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([tp], **kw)
    p, m, v = p0.copy(), np.zeros(1000), np.zeros(1000)
    for t, g in enumerate(grads, start=1):
        tp.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v = O.adamw_step(p, g, m, v, t, 1e-3, 0.9, 0.999, 1e-8, 0.01)
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-13, atol=1e-15)


def test_first_step_moves_by_lr_times_sign():
    """At t = 1 without decay, m_hat = g and v_hat = g^2, so each weight moves by
    lr * g / (|g| + eps): lr * sign(g) up to eps."""
    g = np.array([3.0, -0.5, 1e-3])
    p, _, _ = O.adamw_step(np.zeros(3), g, np.zeros(3), np.zeros(3), 1, 0.01, 0.9, 0.999, 1e-12, 0.0)
    np.testing.assert_allclose(p, -0.01 * np.sign(g), rtol=1e-8)


def test_zero_gradient_only_decays():
    p0 = np.array([1.0, -2.0])
    p, m, v = O.adamw_step(p0, np.zeros(2), np.zeros(2), np.zeros(2), 1, 0.1, 0.9, 0.999, 1e-8, 0.5)
    np.testing.assert_allclose(p, p0 * (1 - 0.05))
    assert not m.any() and not v.any()
