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
