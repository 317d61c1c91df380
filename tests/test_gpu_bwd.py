"""Backward parity: parallax_fwd_train + parallax_bwd (through the C ABI)
against the fp64 oracle's gradients (oracle.bwd, the chain rule through the
definitions, itself pinned by finite differences in test_oracle_bwd_pins.py)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import softmax_learned_covariance_b200 as plx
from softmax_learned_covariance_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(B, H, T, d, seed, rho_scale=0.905):
    q, k, v, rho = inputs.fwd_bf16_inputs(B, H, T, d, rho_scale=rho_scale, seed=seed)
    dy = inputs.Tensor16(inputs.bf16_bits(np.random.default_rng(seed + 99).standard_normal((B, H, T, d))))
    return q, k, v, rho, dy


def _run(q, k, v, rho, dy, causal):
    t = [x.torch().to(DEV) for x in (q, k, v, rho, dy)]
    y, lse, o, abar = plx.parallax_fwd_train(*t[:4], causal=causal)
    grads = plx.parallax_bwd(*t[:4], y, o, abar, lse, t[4], causal=causal)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    return (y, lse, o, abar), [g.cpu().numpy() for g in grads]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 37, 64, 130, 300])
@pytest.mark.parametrize("causal", [True, False])
def test_bwd_small_shapes(T, causal, d):
    q, k, v, rho, dy = _case(1, 2, T, d, seed=400 + T + d)
    (y, lse, o, abar), g = _run(q, k, v, rho, dy, causal)
    ref = oracle.bwd(q.f64, k.f64, v.f64, rho.f64, dy.f64, causal=causal)
    cs = max(np.abs(r).max() for r in ref)
    for name, mine, r in zip(("dq", "dk", "dv", "drho"), g, ref):
        parity.assert_grad_parity(mine, r, 2, f"{name} T={T} causal={causal} d={d}", case_scale=cs)


def test_fwd_train_outputs():
    """y and lse as parallax_fwd gives them (bitwise); o against the oracle's softmax attention."""
    q, k, v, rho, _ = _case(2, 2, 333, 128, seed=7)
    t = [x.torch().to(DEV) for x in (q, k, v, rho)]
    y, lse, o, abar = plx.parallax_fwd_train(*t)
    y2, l2 = plx.parallax_fwd(*t)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(lse, l2)
    o_ref, _ = oracle.fwd(q.f64, k.f64, v.f64, None)
    parity.assert_bf16_parity(o.cpu().numpy(), o_ref, 2, "o")


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_t2048_two_heads(causal):
    """Several key and query blocks with ragged ends: B=1 H=2 T=2000 d=128."""
    q, k, v, rho, dy = _case(1, 2, 2000, 128, seed=51)
    _, g = _run(q, k, v, rho, dy, causal)
    ref = oracle.bwd(q.f64, k.f64, v.f64, rho.f64, dy.f64, causal=causal)
    cs = max(np.abs(r).max() for r in ref)
    for name, mine, r in zip(("dq", "dk", "dv", "drho"), g, ref):
        parity.assert_grad_parity(mine, r, 2, f"{name} T=2000 causal={causal}", case_scale=cs)


def test_bwd_zero_probe_matches_softmax_attention_gradients():
    """rho = 0: drho = dA K with dA = s (g.o - G), and dq, dk, dv are softmax
    attention's; checked against the oracle at rho = 0."""
    q, k, v, _, dy = _case(1, 2, 260, 128, seed=61)
    zero = inputs.Tensor16(np.zeros_like(q.bits))
    _, g = _run(q, k, v, zero, dy, True)
    ref = oracle.bwd(q.f64, k.f64, v.f64, zero.f64, dy.f64, causal=True)
    cs = max(np.abs(r).max() for r in ref)
    for name, mine, r in zip(("dq", "dk", "dv", "drho"), g, ref):
        parity.assert_grad_parity(mine, r, 2, f"{name} rho=0", case_scale=cs)


def test_bwd_b8_t4096_h16_two_heads_vs_oracle():
    """The timed backward shape, B=8 H=16 T=4096 d=128 causal, in one call: the
    gradients of the first and the last head against the oracle computed on
    those heads alone (each head's gradients depend on that head only)."""
    B, H, T, d = 8, 16, 4096, 128
    q, k, v, rho, dy = _case(B, H, T, d, seed=71)
    _, g = _run(q, k, v, rho, dy, True)
    for b, h in ((0, 0), (B - 1, H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.bwd(q.f64[sl], k.f64[sl], v.f64[sl], rho.f64[sl], dy.f64[sl], causal=True)
        cs = max(np.abs(r).max() for r in ref)
        for name, mine, r in zip(("dq", "dk", "dv", "drho"), g, ref):
            parity.assert_grad_parity(mine[sl], r, 2, f"{name} B=8 T=4096 head ({b},{h})", case_scale=cs)
