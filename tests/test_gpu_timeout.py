"""Failure detection without a GPU fault: a bounded device wait that nothing
will satisfy must give up, record PARALLAX_ERR_DEVICE_TIMEOUT and leave the
context usable for the next call."""
from __future__ import annotations

import pytest
import torch

import softmax_learned_covariance_b200 as plx
from softmax_learned_covariance_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
PARALLAX_ERR_DEVICE_TIMEOUT = 7


def test_forced_wait_timeout_is_reported_and_recoverable(monkeypatch):
    q, k, v, rho = inputs.fwd_bf16_inputs(1, 2, 256, 128, seed=77)
    dq, dk, dv, dr = (t.torch().to(DEV) for t in (q, k, v, rho))
    y_ok, _ = plx.parallax_fwd(dq, dk, dv, dr)
    assert plx.parallax_last_device_error() == 0
    # Test hook: the producer never issues the first K tile, so the UMMA issuer's
    # bounded wait on it expires; every other wait then sees the abort flag.
    monkeypatch.setenv("PARALLAX_DEBUG_FLAGS", "1")
    monkeypatch.setenv("PARALLAX_WAIT_TIMEOUT_MS", "50")
    plx.parallax_fwd(dq, dk, dv, dr)
    assert plx.parallax_last_device_error() == PARALLAX_ERR_DEVICE_TIMEOUT
    monkeypatch.delenv("PARALLAX_DEBUG_FLAGS")
    monkeypatch.delenv("PARALLAX_WAIT_TIMEOUT_MS")
    assert plx.parallax_last_device_error() == 0          # the word was cleared by the read
    y2, _ = plx.parallax_fwd(dq, dk, dv, dr)
    assert plx.parallax_last_device_error() == 0
    assert torch.equal(y2, y_ok)


def test_wait_budget_is_per_wait_not_per_kernel(monkeypatch):
    """A prefill that runs far longer than the wait budget (B=4 H=16 T=32768,
    ~30 ms, under a 10 ms budget) must not time out: the budget bounds each wait
    on its own.  Sampled rows of two heads are checked against the oracle."""
    import numpy as np

    import oracle
    from tests import parity

    B, H, T, d = 4, 16, 32768, 128
    g = torch.Generator(device=DEV)
    g.manual_seed(1234)

    def draw(scale=1.0):
        return (torch.randn((B, H, T, d), generator=g, device=DEV) * scale).to(torch.bfloat16)

    q, k, v, r = draw(), draw(), draw(), draw(0.905)
    monkeypatch.setenv("PARALLAX_WAIT_TIMEOUT_MS", "10")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    y, lse = plx.parallax_fwd(q, k, v, r)
    end.record()
    assert plx.parallax_last_device_error() == 0
    monkeypatch.delenv("PARALLAX_WAIT_TIMEOUT_MS")
    assert start.elapsed_time(end) > 10.0 * 2, "the run must outlast the wait budget"
    heads = [(0, 0), (3, 11)]
    rows = np.array(sorted(set(range(4)) | set(range(T - 4, T)) | set(range(0, T, 8191))), np.int64)

    def host(t, b, h):
        return inputs.Tensor16(t[b:b + 1, h:h + 1].contiguous().cpu().view(torch.int16).numpy().view(np.uint16))

    for b, h in heads:
        hq, hk, hv, hr = (host(t, b, h) for t in (q, k, v, r))
        yr, lr = oracle.fwd_rows(hq.f64, hk.f64, hv.f64, hr.f64, rows)
        yg = y[b, h].cpu().numpy()[rows]
        parity.assert_bf16_parity(yg[None], yr.reshape(1, len(rows), d), 1, f"long run head {b},{h}")
        parity.assert_lse(lse[b, h].cpu().numpy()[rows], lr, "long run lse")
