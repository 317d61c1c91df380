"""Prefill/forward parity: CUDA path (through the C ABI) vs the fp64 oracle."""
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


def _dev(t16):
    return t16.torch().to(DEV)


def _run_bf16(q, k, v, rho, causal=True, out_dtype=torch.float32):
    y, lse = plx.parallax_fwd(_dev(q), _dev(k), _dev(v), None if rho is None else _dev(rho), causal=causal,
                              out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    return y, lse


def test_fp32_tiny_causal_b1_h2_t128_d64():
    """fp32 path, B=1 H=2 T=128 d=64, rho ~ N(0, 0.1^2); plus the rho = 0 identity."""
    q, k, v, rho = inputs.fwd_f32_inputs()
    t = lambda a: torch.from_numpy(a).to(DEV)
    y, lse = plx.parallax_fwd(t(q), t(k), t(v), t(rho), causal=True)
    yr, lr = oracle.fwd(q, k, v, rho, causal=True)
    parity.assert_f32_parity(y.cpu().numpy(), yr, "fp32 tiny")
    parity.assert_lse(lse.cpu().numpy(), lr, "fp32 tiny lse")
    y0, _ = plx.parallax_fwd(t(q), t(k), t(v), t(np.zeros_like(rho)), causal=True)
    yn, _ = plx.parallax_fwd(t(q), t(k), t(v), None, causal=True)
    assert torch.equal(y0, yn), "rho = 0 must equal the softmax-only instantiation bitwise"
    ys, _ = oracle.fwd(q, k, v, None, causal=True)
    parity.assert_f32_parity(y0.cpu().numpy(), ys, "fp32 tiny rho=0")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 5, 64, 128, 129, 300, 512])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_small_shapes(T, causal, d):
    """Several query/key tiles, ragged tails, both masks, both head dims; rho at the 1.7B-layer scale."""
    q, k, v, rho = inputs.fwd_bf16_inputs(2, 3, T, d, seed=100 + T + d)
    y, lse = _run_bf16(q, k, v, rho, causal)
    yr, lr = oracle.fwd(q.f64, k.f64, v.f64, rho.f64, causal=causal)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"T={T} causal={causal} d={d}")
    parity.assert_lse(lse.cpu().numpy(), lr, f"T={T} d={d}")


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_softmax_identity_bitwise(d):
    """W_R = 0: the full kernel with rho = 0 equals its softmax-only instantiation bit for bit."""
    q, k, v, _ = inputs.fwd_bf16_inputs(2, 2, 700, d, seed=7)
    zero = inputs.Tensor16(np.zeros_like(q.bits))
    y0, l0 = _run_bf16(q, k, v, zero)
    yn, ln = _run_bf16(q, k, v, None)
    assert torch.equal(y0, yn) and torch.equal(l0, ln)
    yr, _ = oracle.fwd(q.f64, k.f64, v.f64, None)
    parity.assert_bf16_parity(yn.cpu().numpy(), yr, 2, "softmax only")


def test_bf16_output_dtype():
    """bf16 y is the rounded fp32 result: within the bf16 gate plus one bf16 ulp of the reference."""
    q, k, v, rho = inputs.fwd_bf16_inputs(1, 2, 256, 128, seed=9)
    y32, _ = _run_bf16(q, k, v, rho)
    y16, _ = _run_bf16(q, k, v, rho, out_dtype=torch.bfloat16)
    yr, _ = oracle.fwd(q.f64, k.f64, v.f64, rho.f64)
    ulp = np.abs(inputs.round_bf16(yr)) * 2.0 ** -7
    err = np.abs(y16.float().cpu().numpy() - yr)
    assert np.all(err <= parity.BF16_MAX_ABS + ulp)
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_prefill_b8_t4096_h16_sampled_rows():
    """B=8 T=4096 H=16 d=128 (the timed prefill shape): sampled rows of every head vs the oracle."""
    B, H, T, d = 8, 16, 4096, 128
    q, k, v, rho = inputs.fwd_bf16_inputs(B, H, T, d, seed=3)
    y, lse = _run_bf16(q, k, v, rho)
    y = y.cpu().numpy().reshape(B * H * T, d)
    lse = lse.cpu().numpy().reshape(-1)
    base = parity.sample_rows(T, n_head_rows=16, stride=509)
    heads = np.arange(B * H)
    rows = (heads[:, None] * T + base[None, :]).reshape(-1)
    yr, lr = oracle.fwd_rows(q.f64, k.f64, v.f64, rho.f64, rows)
    parity.assert_bf16_parity(y[rows].reshape(B * H, -1, d), yr.reshape(B * H, -1, d), 1, "prefill b8 t4096 rows")
    parity.assert_lse(lse[rows], lr, "prefill b8 t4096 lse")


def test_long_prefill_t32768_and_softmax_identity():
    """B=1 T=32768 H=16: sampled rows vs the oracle, and rho = 0 bitwise equal to softmax only."""
    B, H, T, d = 1, 16, 32768, 128
    q, k, v, rho = inputs.fwd_bf16_inputs(B, H, T, d, seed=5)
    y, lse = _run_bf16(q, k, v, rho)
    base = np.array(sorted(set(range(8)) | set(range(T - 8, T)) | set(range(0, T, 4099))), np.int64)
    heads = np.array([0, 7, 15])
    rows = (heads[:, None] * T + base[None, :]).reshape(-1)
    yr, lr = oracle.fwd_rows(q.f64, k.f64, v.f64, rho.f64, rows)
    yg = y.cpu().numpy().reshape(B * H * T, d)[rows]
    parity.assert_bf16_parity(yg.reshape(len(heads), -1, d), yr.reshape(len(heads), -1, d), 1, "t32768 rows")
    parity.assert_lse(lse.cpu().numpy().reshape(-1)[rows], lr, "t32768 lse")
    del y, lse
    zero = inputs.Tensor16(np.zeros_like(q.bits))
    y0, l0 = _run_bf16(q, k, v, zero)
    yn, ln = _run_bf16(q, k, v, None)
    assert torch.equal(y0, yn) and torch.equal(l0, ln)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [300, 4096])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_row_max_rises_after_the_first_tile(T, causal, d):
    """Planted keys lift rows' running max by > 8 log2 units in later key tiles
    (once or twice), so the kernel rescales O and M in TMEM while earlier tiles
    still carry much of the weight; y and lse against the oracle, and rho = 0
    bitwise equal to the softmax-only instantiation on the same inputs."""
    q, k, v, rho, spikes = inputs.fwd_rescale_inputs(1, 2, T, d, seed=11 + T)
    assert spikes
    y, lse = _run_bf16(q, k, v, rho, causal)
    yr, lr = oracle.fwd(q.f64, k.f64, v.f64, rho.f64, causal=causal)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"rescale T={T} causal={causal}")
    parity.assert_lse(lse.cpu().numpy(), lr, f"rescale T={T} lse")
    zero = inputs.Tensor16(np.zeros_like(q.bits))
    y0, l0 = _run_bf16(q, k, v, zero, causal)
    yn, ln = _run_bf16(q, k, v, None, causal)
    assert torch.equal(y0, yn) and torch.equal(l0, ln)
    ys, _ = oracle.fwd(q.f64, k.f64, v.f64, None, causal=causal)
    parity.assert_bf16_parity(yn.cpu().numpy(), ys, 2, f"rescale softmax-only T={T}")


def _scaled(t16, factor):
    """bf16 values times an exact power of two (bits re-rounded, exact in range)."""
    return inputs.Tensor16(inputs.bf16_bits(t16.f64 * factor))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("vexp", [-17, 14])
def test_bf16_v_far_from_unit_scale(vexp, d):
    """V scaled by 2^-17 (std 7.6e-6, below fp16's normal range) and by 2^14
    (std 16384, values past fp16's maximum 65504): the kernel's per-stage
    power-of-two scaling keeps fp16 precision; gates scaled with V."""
    T = 700
    q, k, v, rho = inputs.fwd_bf16_inputs(2, 2, T, d, seed=31 + d)
    vs = _scaled(v, 2.0 ** vexp)
    assert vexp < 0 or np.abs(vs.f64).max() > 65504
    for causal in (True, False):
        y, lse = _run_bf16(q, k, vs, rho, causal)
        yr, lr = oracle.fwd(q.f64, k.f64, vs.f64, rho.f64, causal=causal)
        parity.assert_bf16_parity_scaled(y.cpu().numpy(), yr, 2, 2.0 ** vexp, f"V x 2^{vexp} causal={causal}")
        parity.assert_lse(lse.cpu().numpy(), lr, f"V x 2^{vexp} lse")


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_large_probe(d):
    """rho with standard deviation 17 (|a| = |k . rho| around 190 at d = 128):
    the fp16 correction weights P o A/256 stay finite; gates scaled with rho."""
    q, k, v, _ = inputs.fwd_bf16_inputs(2, 2, 600, d, seed=41 + d)
    rho = inputs.fwd_bf16_inputs(2, 2, 600, d, rho_scale=17.0, seed=42 + d)[3]
    for causal in (True, False):
        y, lse = _run_bf16(q, k, v, rho, causal)
        yr, lr = oracle.fwd(q.f64, k.f64, v.f64, rho.f64, causal=causal)
        parity.assert_bf16_parity_scaled(y.cpu().numpy(), yr, 2, 17.0 / 0.905, f"rho std 17 causal={causal}")
        parity.assert_lse(lse.cpu().numpy(), lr, "rho std 17 lse")


def test_bf16_out_of_range_v_is_reported():
    """|v| >= 2^23 cannot be staged in fp16 even with the largest stage scale:
    the output is not finite and the device error word says so."""
    q, k, v, rho = inputs.fwd_bf16_inputs(1, 2, 200, 128, seed=51)
    bits = v.bits.copy()
    bits[0, 1, 150, 7] = inputs.bf16_bits(np.array([2.0 ** 30]))[0]
    y, _ = plx.parallax_fwd(_dev(q), _dev(k), _dev(inputs.Tensor16(bits)), _dev(rho))
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 9          # PARALLAX_ERR_DEVICE_RANGE
    assert plx.parallax_last_device_error() == 0          # cleared by the read
    yr, _ = oracle.fwd(q.f64, k.f64, v.f64, rho.f64)
    parity.assert_bf16_parity(y[0, :1].cpu().numpy(), yr[0, :1], 1, "the other head is unaffected")
