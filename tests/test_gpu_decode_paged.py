"""Paged, grouped-head decode (through the C ABI) vs the fp64 oracle."""
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


def _dev(q, rho, kp, vp, table, sl):
    return (q.torch().to(DEV), rho.torch().to(DEV), kp.torch().to(DEV), vp.torch().to(DEV),
            torch.from_numpy(table).to(DEV), torch.from_numpy(sl).to(DEV))


def _run(args, out_dtype=torch.float32, expect_err=0):
    y, lse = plx.parallax_decode_paged(*args, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert plx.parallax_last_device_error() == expect_err
    return y, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("group", [1, 2, 4])
def test_paged_grouped_small(group, page_size, d):
    B, Hkv = 4, 2
    Hq = Hkv * group
    max_pages = max(2, 1100 // page_size)
    tcap = max_pages * page_size
    sl = np.array([0, 1, min(page_size + 1, tcap), tcap], np.int32)
    q, rho, kp, vp, table, sl = inputs.paged_decode_inputs(B, Hq, Hkv, page_size, max_pages, d, sl,
                                                           seed=group * 100 + page_size + d)
    y, lse = _run(_dev(q, rho, kp, vp, table, sl))
    yr, lr = oracle.decode_paged(q.f64, rho.f64, kp.f64, vp.f64, table, sl)
    yg, lg = y.cpu().numpy(), lse.cpu().numpy()
    assert np.all(yg[0] == 0.0) and np.all(np.isneginf(lg[0]))
    parity.assert_bf16_parity(yg[1:], yr[1:], 2, f"paged G={group} ps={page_size} d={d}")
    parity.assert_lse(lg[1:], lr[1:])


def test_paged_identity_table_matches_contiguous_decode():
    """A contiguous cache cut into pages in order, one query head per KV head:
    the paged call (tensor-core kernel) agrees with parallax_decode (CUDA-core
    split kernel) within the bf16 gate, and both with the oracle."""
    B, H, ps, max_pages, d = 6, 4, 64, 40, 128
    tcap = ps * max_pages
    sl = inputs.ragged_seqlens(B, tcap, 9)
    q, rho, kc, vc, sl = inputs.decode_inputs(B, H, tcap, d, seqlens=sl, seed=9)
    y_ref, l_ref = plx.parallax_decode(q.torch().to(DEV), rho.torch().to(DEV), kc.torch().to(DEV),
                                       vc.torch().to(DEV), torch.from_numpy(sl).to(DEV))

    def pages(t):
        return t.reshape(B, H, max_pages, ps, d).permute(0, 2, 1, 3, 4).reshape(B * max_pages, H, ps, d).contiguous()

    kp, vp = pages(kc.torch().to(DEV)), pages(vc.torch().to(DEV))
    table = torch.arange(B * max_pages, dtype=torch.int32, device=DEV).reshape(B, max_pages)
    y, lse = _run((q.torch().to(DEV), rho.torch().to(DEV), kp, vp, table, torch.from_numpy(sl).to(DEV)))
    parity.assert_bf16_parity(y.cpu().numpy(), y_ref.cpu().numpy(), 2, "paged vs contiguous")
    parity.assert_lse(lse.cpu().numpy(), l_ref.cpu().numpy())
    yr, _ = oracle.decode(q.f64, rho.f64, kc.f64, vc.f64, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, "paged vs oracle")


def test_bad_page_id_is_reported_and_unreached_entries_are_ignored():
    B, Hq, Hkv, ps, max_pages, d = 3, 4, 2, 32, 8, 128
    sl = np.array([100, 256, 33], np.int32)
    q, rho, kp, vp, table, sl = inputs.paged_decode_inputs(B, Hq, Hkv, ps, max_pages, d, sl, seed=77)
    num_pages = kp.bits.shape[0]
    # entries past each sequence's last page are never read: garbage is fine there
    table = table.copy()
    table[0, 4:] = -7
    table[2, 2:] = num_pages + 1000
    args = _dev(q, rho, kp, vp, table, sl)
    y, lse = _run(args)
    yr, lr = oracle.decode_paged(q.f64, rho.f64, kp.f64, vp.f64, np.where(table < 0, 0, table) % num_pages, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, "unreached garbage entries")
    # a reached entry out of range: no read through it, the device error word says so
    bad = table.copy()
    bad[1, 3] = num_pages + 5
    y2, _ = _run(_dev(q, rho, kp, vp, bad, sl), expect_err=8)   # PARALLAX_ERR_DEVICE_INDEX
    assert torch.all(torch.isfinite(y2))
    # the error word was cleared by reading it; the next good call is clean
    _run(args)


def test_paged_gqa_b8_hq16_hkv4_ctx2048_all_heads():
    B, Hq, Hkv, ps, max_pages, d = 8, 16, 4, 64, 32, 128
    sl = inputs.ragged_seqlens(B, ps * max_pages, 12)
    q, rho, kp, vp, table, sl = inputs.paged_decode_inputs(B, Hq, Hkv, ps, max_pages, d, sl, seed=12)
    y, lse = _run(_dev(q, rho, kp, vp, table, sl))
    yr, lr = oracle.decode_paged(q.f64, rho.f64, kp.f64, vp.f64, table, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, "paged gqa b8")
    parity.assert_lse(lse.cpu().numpy(), lr)
    y16, _ = _run(_dev(q, rho, kp, vp, table, sl), out_dtype=torch.bfloat16)
    assert torch.equal(y16, y.to(torch.bfloat16))


@pytest.mark.parametrize("group", [3, 8, 12])
def test_paged_group_sizes_beyond_one_tile(group):
    """Groups that fill a tensor-core tile exactly (8), partly (3) or span two tiles (12)."""
    B, Hkv, ps, max_pages, d = 3, 2, 32, 24, 128
    Hq = Hkv * group
    sl = np.array([ps * max_pages, 5, 400], np.int32)
    q, rho, kp, vp, table, sl = inputs.paged_decode_inputs(B, Hq, Hkv, ps, max_pages, d, sl, seed=300 + group)
    y, lse = _run(_dev(q, rho, kp, vp, table, sl))
    yr, lr = oracle.decode_paged(q.f64, rho.f64, kp.f64, vp.f64, table, sl)
    parity.assert_bf16_parity(y.cpu().numpy(), yr, 2, f"group {group}")
    parity.assert_lse(lse.cpu().numpy(), lr)
