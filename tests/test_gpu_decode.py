"""Decode parity: split-KV CUDA kernels (through the C ABI) vs the fp64 oracle."""
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


def _run(q, rho, kc, vc, sl, out_dtype=torch.float32):
    y, lse = plx.parallax_decode(q.torch().to(DEV), rho.torch().to(DEV), kc.torch().to(DEV), vc.torch().to(DEV),
                                 torch.from_numpy(sl).to(DEV), out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    return y, lse


def test_decode_b64_h16_ctx4096_all_heads():
    """B=64 H=16 d=128, contiguous cache of 4096 tokens: every head vs the oracle."""
    q, rho, kc, vc, sl = inputs.decode_inputs(64, 16, 4096, 128, seed=2)
    y, lse = _run(q, rho, kc, vc, sl)
    yr, lr = oracle.decode(q.f64, rho.f64, kc.f64, vc.f64, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, "decode b64 ctx4096")
    parity.assert_lse(lse.cpu().numpy(), lr, "decode b64 ctx4096 lse")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Tcap", [1, 7, 64, 300, 1000, 5000])
def test_ragged_lengths(Tcap, d):
    B, H = 5, 3
    rng = np.random.default_rng(Tcap + d)
    sl = rng.integers(1, Tcap + 1, size=B).astype(np.int32)
    sl[0] = 1
    sl[-1] = Tcap
    q, rho, kc, vc, _ = inputs.decode_inputs(B, H, Tcap, d, seqlens=sl, seed=Tcap)
    y, lse = _run(q, rho, kc, vc, sl)
    yr, lr = oracle.decode(q.f64, rho.f64, kc.f64, vc.f64, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"Tcap={Tcap} d={d}")
    parity.assert_lse(lse.cpu().numpy(), lr)


def test_empty_sequence_and_bf16_output():
    B, H, Tcap, d = 4, 2, 600, 128
    sl = np.array([0, 1, 599, 600], np.int32)
    q, rho, kc, vc, _ = inputs.decode_inputs(B, H, Tcap, d, seqlens=sl, seed=44)
    y, lse = _run(q, rho, kc, vc, sl)
    yr, lr = oracle.decode(q.f64, rho.f64, kc.f64, vc.f64, sl)
    yg = y.cpu().numpy()
    assert np.all(yg[0] == 0.0) and np.all(np.isneginf(lse.cpu().numpy()[0]))
    parity.assert_bf16_parity(yg[1:], yr[1:], 2, "nonempty")
    y16, _ = _run(q, rho, kc, vc, sl, out_dtype=torch.bfloat16)
    assert torch.equal(y16, y.to(torch.bfloat16))


def test_decode_ex_caller_workspace_matches():
    q, rho, kc, vc, sl = inputs.decode_inputs(8, 16, 8192, 128, seed=21)
    dq, dr, dk, dv, ds = (t.to(DEV) for t in (q.torch(), rho.torch(), kc.torch(), vc.torch(), torch.from_numpy(sl)))
    nbytes = plx.parallax_decode_workspace_bytes(8, 16, 8192, 128)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV)
    y1, l1 = plx.parallax_decode(dq, dr, dk, dv, ds)
    y2, l2 = plx.parallax_decode_ex(dq, dr, dk, dv, ds, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(l1, l2)
    if nbytes > 0:
        with pytest.raises(plx.ParallaxError):
            plx.parallax_decode_ex(dq, dr, dk, dv, ds, ws[: nbytes // 2])


def test_sweep_cell_sampled_heads():
    """One mid-size cell of the decode sweep (B=64, context 8192, ragged), sampled heads."""
    B, H, ctx, d = 64, 16, 8192, 128
    sl = inputs.ragged_seqlens(B, ctx, seed=4 + 13)
    q, rho, kc, vc, _ = inputs.decode_inputs(B, H, ctx, d, seqlens=sl, seed=4 + 13)
    y, lse = _run(q, rho, kc, vc, sl)
    bh = np.arange(0, B * H, 37)
    yr, lr = oracle.decode(q.f64, rho.f64, kc.f64, vc.f64, sl, bh_list=bh)
    parity.assert_bf16_parity(y.cpu().numpy().reshape(B * H, d)[bh], yr, 1, "sweep cell")
    parity.assert_lse(lse.cpu().numpy().reshape(-1)[bh], lr)


@pytest.mark.parametrize("B,ctx", [(1, 32768), (8, 8192)])
def test_long_context_cells_sampled_heads(B, ctx):
    """Long-context cells of the decode sweep with ragged lengths in [ctx/2, ctx]:
    B=1 ctx 32768 (one head is split into up to 256 chunks, merged by the
    16-warp combine) and B=8 ctx 8192.  Inputs drawn on the device with a
    seeded generator; sampled heads read back and checked against the oracle."""
    H, d = 16, 128
    sl = inputs.ragged_seqlens(B, ctx, 4 + 100 + B)
    q, r, kc, vc, ds = inputs.decode_inputs_device(B, H, ctx, d, sl, seed=4 + 100 + B, device=DEV)
    y, lse = plx.parallax_decode(q, r, kc, vc, ds)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    heads = [(b, h) for b in range(B) for h in (0, 7, 15)]

    def host(t):
        return inputs.Tensor16(t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16))

    for b, h in heads:
        hq, hr = host(q[b:b + 1, h:h + 1]), host(r[b:b + 1, h:h + 1])
        hk, hv = host(kc[b:b + 1, h:h + 1]), host(vc[b:b + 1, h:h + 1])
        yr, lr = oracle.decode(hq.f64, hr.f64, hk.f64, hv.f64, sl[b:b + 1])
        parity.assert_bf16_parity(y[b:b + 1, h:h + 1].cpu().numpy(), yr, 2, f"B={B} ctx={ctx} head {b},{h}")
        parity.assert_lse(lse[b:b + 1, h:h + 1].cpu().numpy(), lr)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_softmax_decode_reference(d):
    """parallax_softmax_decode (the pages' comparison baseline) against the oracle
    at rho = 0 (softmax attention), ragged lengths including 1 and Tcap; at
    d 64 / 128 it is bitwise parallax_decode with rho = 0 (same split, same sums)."""
    B, H, Tcap = 6, 4, 3000
    sl = np.array([1, 17, 1500, 2999, 3000, 256], np.int32)
    q, rho, kc, vc, _ = inputs.decode_inputs(B, H, Tcap, d, seqlens=sl, seed=700 + d)
    dq, dk, dv = q.torch().to(DEV), kc.torch().to(DEV), vc.torch().to(DEV)
    ds = torch.from_numpy(sl).to(DEV)
    y, lse = plx.parallax_softmax_decode(dq, dk, dv, ds)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == 0
    zero = np.zeros_like(rho.f64)
    yr, lr = oracle.decode(q.f64, zero, kc.f64, vc.f64, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"softmax decode d={d}")
    parity.assert_lse(lse.cpu().numpy(), lr)
    if d != 256:
        y0, l0 = plx.parallax_decode(dq, torch.zeros_like(rho.torch().to(DEV)), dk, dv, ds)
        torch.cuda.synchronize()
        assert torch.equal(y0, y) and torch.equal(l0, lse)
