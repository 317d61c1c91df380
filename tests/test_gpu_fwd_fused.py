"""Prefill with the probe computed inside the kernel (parallax_fwd_fused):
rho = x W_R per query tile on the tensor cores, never written to HBM.

The oracle computes rho with its own projection (fp64) and the kernel keeps
rho in bf16, as parallax_rho_proj stores it; so the oracle's rho rows are
rounded to bf16 before its forward, which is the plainest reading of "rho
rounded as the kernel rounds it" (the fp32 accumulation order of the two
roundings can differ in the last bit of rho for a few elements, far inside the
gates).
"""
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


def _inputs(B, H, T, d_model, seed, w_scale=0.02):
    q, k, v, _ = inputs.fwd_bf16_inputs(B, H, T, 128, seed=seed)
    x, w = inputs.rho_proj_inputs(B, T, d_model, H, 128, w_scale=w_scale, seed=seed)
    return q, k, v, x, w


def _dev(t16):
    return t16.torch().to(DEV)


@pytest.mark.parametrize("T", [1, 129, 300, 700])
@pytest.mark.parametrize("causal", [True, False])
def test_fused_small_shapes(T, causal):
    B, H, dm = 2, 2, 256
    q, k, v, x, w = _inputs(B, H, T, dm, seed=200 + T)
    y, lse = plx.parallax_fwd_fused(_dev(q), _dev(k), _dev(v), _dev(x), _dev(w), causal=causal)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    rho = inputs.round_bf16(oracle.rho_proj(x.f64, w.f64, H, 128))
    yr, lr = oracle.fwd(q.f64, k.f64, v.f64, rho, causal=causal)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"fused T={T} causal={causal}")
    parity.assert_lse(lse.cpu().numpy(), lr, f"fused T={T}")


def test_fused_matches_two_launch_pipeline():
    """The same inputs through parallax_rho_proj + parallax_fwd: within the gates of each other."""
    B, H, T, dm = 2, 4, 1000, 512
    q, k, v, x, w = _inputs(B, H, T, dm, seed=321)
    dq, dk, dv, dx, dw = (_dev(t) for t in (q, k, v, x, w))
    y1, l1 = plx.parallax_fwd_fused(dq, dk, dv, dx, dw)
    rho = plx.parallax_rho_proj(dx, dw, H, 128)
    y2, l2 = plx.parallax_fwd(dq, dk, dv, rho)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    parity.assert_bf16_parity(y1.cpu().numpy(), y2.cpu().numpy().astype(np.float64), 2, "fused vs two launches")
    parity.assert_lse(l1.cpu().numpy(), l2.cpu().numpy().astype(np.float64), "fused vs two launches lse")


def test_fused_zero_projection_is_softmax_bitwise():
    """W_R = 0: rho = 0 in the kernel, so y equals the softmax-only instantiation bit for bit."""
    B, H, T, dm = 1, 3, 650, 128
    q, k, v, x, w = _inputs(B, H, T, dm, seed=77)
    zw = inputs.Tensor16(np.zeros_like(w.bits))
    yf, lf = plx.parallax_fwd_fused(_dev(q), _dev(k), _dev(v), _dev(x), _dev(zw))
    ys, ls = plx.parallax_fwd(_dev(q), _dev(k), _dev(v), None)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    assert torch.equal(yf, ys) and torch.equal(lf, ls)


def test_fused_long_prefill_t32768_sampled_rows():
    """B=1 T=32768 H=16 d=128 d_model=2048 (the long-prefill shape): sampled rows
    of three heads against the oracle (rho of those rows from the oracle's
    projection, rounded to bf16), and W_R = 0 bitwise equal to softmax only."""
    B, H, T, d, dm = 1, 16, 32768, 128, 2048
    q, k, v, x, w = _inputs(B, H, T, dm, seed=5)
    dq, dk, dv, dx, dw = (_dev(t) for t in (q, k, v, x, w))
    y, lse = plx.parallax_fwd_fused(dq, dk, dv, dx, dw)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    tok = np.array(sorted(set(range(6)) | set(range(T - 6, T)) | set(range(0, T, 4099))), np.int64)
    rho_rows = inputs.round_bf16(oracle.rho_proj(x.f64, w.f64, H, d, bt_list=tok))   # [n, H, d]
    heads = np.array([0, 7, 15])
    rho = np.zeros((B, H, T, d))
    rho[0][:, tok, :] = rho_rows.transpose(1, 0, 2)
    rows = (heads[:, None] * T + tok[None, :]).reshape(-1)
    yr, lr = oracle.fwd_rows(q.f64, k.f64, v.f64, rho, rows)
    yg = y.cpu().numpy().reshape(B * H * T, d)[rows]
    parity.assert_bf16_parity(yg.reshape(len(heads), -1, d), yr.reshape(len(heads), -1, d), 1, "fused t32768 rows")
    parity.assert_lse(lse.cpu().numpy().reshape(-1)[rows], lr, "fused t32768 lse")
    del y, lse
    zw = torch.zeros_like(dw)
    yf, lf = plx.parallax_fwd_fused(dq, dk, dv, dx, zw)
    ys, ls = plx.parallax_fwd(dq, dk, dv, None)
    torch.cuda.synchronize()
    assert torch.equal(yf, ys) and torch.equal(lf, ls)
