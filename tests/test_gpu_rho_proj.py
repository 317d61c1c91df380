"""rho projection parity (tcgen05 GEMM through the C ABI) and the rho_proj -> fwd pipeline."""
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


def _check_rho(rho_gpu, ref, what):
    """bf16 output of an fp32-accumulated product: within one bf16 rounding of the fp64 value."""
    g = np.asarray(rho_gpu, np.float64)
    tol = np.abs(ref) * 2.0 ** -8 + 1e-4
    bad = np.abs(g - ref) > tol
    assert not bad.any(), f"{what}: {bad.sum()} elements off; worst {np.max(np.abs(g - ref)):.3e}"


@pytest.mark.parametrize("B,T,dm,H,d", [(1, 128, 64, 2, 128), (2, 200, 256, 4, 64), (1, 333, 512, 4, 128)])
def test_small_shapes_full(B, T, dm, H, d):
    x, w = inputs.rho_proj_inputs(B, T, dm, H, d, seed=B * T + dm)
    rho = plx.parallax_rho_proj(x.torch().to(DEV), w.torch().to(DEV), H, d)
    torch.cuda.synchronize()
    ref = oracle.rho_proj(x.f64, w.f64, H, d)
    _check_rho(rho.float().cpu().numpy(), ref, f"{(B, T, dm, H, d)}")


def test_projection_b8_t4096_dm2048_and_pipeline():
    """x [8,4096,2048], W_R [2048, 16*128]: sampled token rows vs the oracle; then rho_proj -> fwd
    on sampled rows vs the oracle run on the bf16-stored probe."""
    B, T, dm, H, d = 8, 4096, 2048, 16, 128
    x, w = inputs.rho_proj_inputs(B, T, dm, H, d, seed=3)
    rho = plx.parallax_rho_proj(x.torch().to(DEV), w.torch().to(DEV), H, d)
    torch.cuda.synchronize()
    bt = np.array(sorted(set(range(0, B * T, 613)) | {0, B * T - 1, T - 1, T}), np.int64)
    ref = oracle.rho_proj(x.f64, w.f64, H, d, bt_list=bt)          # [n, H, d]
    g = rho.float().cpu().numpy()                                     # [B, H, T, d]
    gs = g[bt // T, :, bt % T, :]
    _check_rho(gs, ref, "rho b8 t4096")

    q, k, v, _ = inputs.fwd_bf16_inputs(B, H, T, d, seed=33)
    y, _ = plx.parallax_fwd(q.torch().to(DEV), k.torch().to(DEV), v.torch().to(DEV), rho)
    torch.cuda.synchronize()
    # oracle probe rows for the sampled query rows, stored in bf16 as the library stores rho
    tok = np.array(sorted(set(range(0, T, 257)) | {1, 2, T - 1}), np.int64)
    bsel = np.array([0, 5], np.int64)
    bt2 = (bsel[:, None] * T + tok[None, :]).reshape(-1)
    rho_rows = inputs.round_bf16(oracle.rho_proj(x.f64, w.f64, H, d, bt_list=bt2))   # [n, H, d]
    rho_full = np.zeros((B, H, T, d))
    rho_full[bt2 // T, :, bt2 % T, :] = rho_rows
    rows = np.array([(b * H + h) * T + t for b in bsel for h in range(H) for t in tok], np.int64)
    yr, _ = oracle.fwd_rows(q.f64, k.f64, v.f64, rho_full, rows)
    yg = y.cpu().numpy().reshape(-1, d)[rows]
    parity.assert_bf16_parity(yg.reshape(len(bsel) * H, -1, d), yr.reshape(len(bsel) * H, -1, d), 1, "pipeline")


def test_zero_projection_gives_exact_zero_probe():
    x, w = inputs.rho_proj_inputs(1, 256, 256, 2, 128, seed=1)
    wz = torch.zeros(w.shape, dtype=torch.bfloat16, device=DEV)
    rho = plx.parallax_rho_proj(x.torch().to(DEV), wz, 2, 128)
    torch.cuda.synchronize()
    assert torch.count_nonzero(rho).item() == 0
