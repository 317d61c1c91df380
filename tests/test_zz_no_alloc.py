"""parallax_decode_noalloc: the decode entry point for callers that cannot let the
library allocate (engines with a fixed, pre-reserved memory budget, latency-critical
decode loops that must not hit a cudaMalloc or a synchronizing cudaFree, plugin
callbacks that forbid allocation).  It keeps its split partials in a static device
array instead of scratch taken from the library's memory pool.  That every shape
fits the array on devices of up to 252 SMs is checked on the host by
tests/test_decode_plan_cpu.py.

Called through the C ABI directly and compared with parallax_decode on the same
inputs, on two calls in a row with different lengths, so stale contents of the
shared array would show.  Collected last so a failure here cannot hide another test.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest
import torch

import softmax_learned_covariance_b200 as plx
from softmax_learned_covariance_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _scratch_limit():
    src = open(os.path.join(ROOT, "include", "parallax.h")).read()
    m = re.search(r"#define PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", src)
    return int(m.group(1)) << int(m.group(2))


def _noalloc():
    f = plx.lib().parallax_decode_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P]
    f.restype = I
    return f


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(f, q, rho, kc, vc, sl, y, lse):
    B, H, Tcap, d = kc.shape
    return f(_p(q), _p(rho), _p(kc), _p(vc), _p(sl), _p(y), _p(lse), B, H, Tcap, d, plx.BF16, plx.F32,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_decode_matches_decode_on_two_calls():
    f = _noalloc()
    B, H, Tcap, d = 64, 16, 4096, 128
    assert 0 < plx.parallax_decode_workspace_bytes(B, H, Tcap, d) <= _scratch_limit()
    for call, seed in enumerate((501, 502)):
        sl = inputs.ragged_seqlens(B, Tcap, seed) if call else np.full((B,), Tcap, np.int32)
        q, rho, kc, vc, _ = inputs.decode_inputs(B, H, Tcap, d, seqlens=sl, seed=seed)
        dq, dr, dk, dv = (t.torch().to(DEV) for t in (q, rho, kc, vc))
        ds = torch.from_numpy(sl).to(DEV)
        y_ref, l_ref = plx.parallax_decode(dq, dr, dk, dv, ds)
        y = torch.full((B, H, d), float("nan"), device=DEV)
        lse = torch.full((B, H), float("nan"), device=DEV)
        assert _call_noalloc(f, dq, dr, dk, dv, ds, y, lse) == 0
        torch.cuda.synchronize()
        parity.assert_bf16_parity(y.cpu().numpy(), y_ref.cpu().numpy(), 2, f"noalloc call {call}")
        assert np.max(np.abs(lse.cpu().numpy() - l_ref.cpu().numpy())) <= parity.LSE_MAX_ABS
