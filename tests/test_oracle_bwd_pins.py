"""Pins for the backward oracle (oracle.bwd, oracle.rho_proj_bwd): facts fixed by
the mathematics and by library routines, not by the oracle's own formulas."""
from __future__ import annotations

import inspect
import textwrap

import numpy as np
import pytest
import torch

import oracle


def _case(seed, B=1, H=2, T=6, d=4, rho_scale=0.6):
    rng = np.random.default_rng(seed)
    q, k, v, dy = (rng.standard_normal((B, H, T, d)) for _ in range(4))
    rho = rho_scale * rng.standard_normal((B, H, T, d))
    return q, k, v, rho, dy


def pin_finite_differences(bwd):
    """<grad, delta> equals the central difference of L = <dY, Y> along delta, Y from
    the (separately pinned) forward oracle, for each input, causal and not."""
    for causal in (True, False):
        q, k, v, rho, dy = _case(61 if causal else 62)
        grads = bwd(q, k, v, rho, dy, causal=causal)
        rng = np.random.default_rng(63)
        for which, g in enumerate(grads):
            delta = rng.standard_normal(q.shape)
            eps = 1e-6

            def loss(sign):
                args = [q, k, v, rho]
                args[which] = args[which] + sign * eps * delta
                y, _ = oracle.fwd(*args, causal=causal)
                return float(np.sum(dy * y))

            fd = (loss(1.0) - loss(-1.0)) / (2 * eps)
            an = float(np.sum(g * delta))
            assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (causal, which, fd, an)


def pin_softmax_special_case(bwd):
    """rho = 0: dq, dk, dv are the gradients of softmax attention (autograd of the
    library SDPA)."""
    q, k, v, _, dy = _case(64, T=9, d=8)
    rho = np.zeros_like(q)
    dq, dk, dv, _ = bwd(q, k, v, rho, dy, causal=True)
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    y = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    y.backward(torch.tensor(dy))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(mine - ref.numpy())) < 1e-12


def pin_single_key_rows(bwd):
    """Row 0 of a causal head sees one key: y_0 = v_0, so dq_0 = 0, drho_0 = 0 and the
    row's dy flows entirely into dv_0."""
    q, k, v, rho, dy = _case(65, T=5)
    dy2 = np.zeros_like(dy)
    dy2[:, :, 0] = dy[:, :, 0]
    dq, dk, dv, dr = bwd(q, k, v, rho, dy2, causal=True)
    assert np.max(np.abs(dq[:, :, 0])) < 1e-14 and np.max(np.abs(dr[:, :, 0])) < 1e-14
    assert np.max(np.abs(dv[:, :, 0] - dy[:, :, 0])) < 1e-14
    assert np.max(np.abs(dv[:, :, 1:])) < 1e-14 and np.max(np.abs(dk)) < 1e-14


def pin_rho_projection_backward(_bwd=None):
    """dx and dW_R of rho = x W_R (per-head slices) equal autograd of the library matmul."""
    B, T, dm, H, d = 2, 3, 10, 2, 4
    rng = np.random.default_rng(66)
    x, W = rng.standard_normal((B, T, dm)), rng.standard_normal((dm, H * d))
    g = rng.standard_normal((B, H, T, d))
    dx, dW = oracle.rho_proj_bwd(x, W, g, H, d)
    tx, tW = (torch.tensor(a, requires_grad=True) for a in (x, W))
    rho = (tx @ tW).reshape(B, T, H, d).permute(0, 2, 1, 3)
    rho.backward(torch.tensor(g))
    assert np.max(np.abs(dx - tx.grad.numpy())) < 1e-12
    assert np.max(np.abs(dW - tW.grad.numpy())) < 1e-12


PINS = [pin_finite_differences, pin_softmax_special_case, pin_single_key_rows]


@pytest.mark.parametrize("pin", PINS + [pin_rho_projection_backward], ids=lambda p: p.__name__)
def test_bwd_pin(pin):
    pin(oracle.bwd)


BWD_MUTANTS = {
    "missing_one_plus_abar": ("dO = dY * (1.0 + abar)", "dO = dY"),
    "sign_of_dM": ("\n            dM = -dY\n", "\n            dM = dY\n"),
    "dS_without_abar": ("dS = G * (1.0 + abar - A) + dabar * A", "dS = G * (1.0 - A) + dabar * A"),
    "dS_without_dabar_term": ("dS = G * (1.0 + abar - A) + dabar * A", "dS = G * (1.0 + abar - A)"),
    "softmax_backward_without_centering": ("dZ = S * (dS - (S * dS).sum(axis=1, keepdims=True))", "dZ = S * dS"),
    "dk_probe_term_transposed": ("dZ.T @ Q * sc + dA.T @ R", "dZ.T @ Q * sc + dA @ R"),
    "drho_transposed": ("out[3][b, h] = dA @ K", "out[3][b, h] = dA.T @ K"),
    "dq_unscaled": ("out[0][b, h] = dZ @ K * sc", "out[0][b, h] = dZ @ K"),
}


def test_planted_backward_mistakes_are_caught():
    src = textwrap.dedent(inspect.getsource(oracle.bwd))
    survivors = []
    for name, (old, new) in BWD_MUTANTS.items():
        assert src.count(old) == 1, f"mutation {name}: pattern not found"
        ns = {"np": np}
        exec(compile(src.replace(old, new), f"<{name}>", "exec"), ns)
        caught = False
        for pin in PINS:
            try:
                pin(ns["bwd"])
            except AssertionError:
                caught = True
                break
        if not caught:
            survivors.append(name)
    assert not survivors, f"planted backward mistakes no pin detects: {survivors}"
