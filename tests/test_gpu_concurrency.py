"""Calls on different streams and from different host threads at once.

Each call takes its scratch (the prefill's work counter and fp16 V copy, the
decodes' split partials) from the library's stream-ordered pool for itself, so
overlapping calls must not disturb one another.  Every result is checked
against the oracle."""
from __future__ import annotations

import threading

import numpy as np
import pytest
import torch

import oracle
import softmax_learned_covariance_b200 as plx
from softmax_learned_covariance_b200 import inputs
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _fwd_case(T, seed):
    q, k, v, r = inputs.fwd_bf16_inputs(1, 4, T, 128, seed=seed)
    yr, _ = oracle.fwd(q.f64, k.f64, v.f64, r.f64)
    return [t.torch().to(DEV) for t in (q, k, v, r)], yr


def _decode_case(B, Tcap, seed):
    sl = inputs.ragged_seqlens(B, Tcap, seed)
    q, r, kc, vc, sl = inputs.decode_inputs(B, 8, Tcap, 128, seqlens=sl, seed=seed)
    yr, _ = oracle.decode(q.f64, r.f64, kc.f64, vc.f64, sl)
    dev = [t.torch().to(DEV) for t in (q, r, kc, vc)] + [torch.from_numpy(sl).to(DEV)]
    return dev, yr


def test_fwd_and_decode_overlap_on_two_streams():
    (fq, fk, fv, fr), fref = _fwd_case(900, 41)
    dargs, dref = _decode_case(24, 3000, 42)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs_f, outs_d = [], []
    for _ in range(4):   # no synchronisation between the calls: the streams overlap
        with torch.cuda.stream(s1):
            outs_f.append(plx.parallax_fwd(fq, fk, fv, fr, stream=s1)[0])
        with torch.cuda.stream(s2):
            outs_d.append(plx.parallax_decode(*dargs, stream=s2)[0])
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    for y in outs_f:
        parity.assert_bf16_parity(y.cpu().numpy(), fref, 2, "fwd beside decode")
    for y in outs_d:
        parity.assert_bf16_parity(y.cpu().numpy(), dref, 2, "decode beside fwd")


def test_decodes_of_different_sizes_from_two_host_threads():
    cases = [_decode_case(8, 5000, 43), _decode_case(48, 2048, 44)]
    results = [[], []]
    errors = []

    def worker(i):
        try:
            torch.cuda.set_device(0)
            st = torch.cuda.Stream()
            args, _ = cases[i]
            with torch.cuda.stream(st):
                for _ in range(12):
                    results[i].append(plx.parallax_decode(*args, stream=st)[0])
            st.synchronize()
        except Exception as e:  # surfaced by the main thread
            errors.append(e)

    th = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    for i in range(2):
        assert len(results[i]) == 12
        for y in results[i]:
            parity.assert_bf16_parity(y.cpu().numpy(), cases[i][1], 2, f"thread {i}")
