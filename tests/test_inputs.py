"""The seeded input generators: bf16 rounding matches a library conversion and
the same seed always gives the same bits."""
import numpy as np
import torch

from softmax_learned_covariance_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * s for s in (1e-3, 1.0, 1e3)]).astype(np.float32)
    # exact ties and near-ties
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ours = inputs.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = inputs.bf16_to_f64(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy())


def test_seeded_and_deterministic():
    a = inputs.fwd_bf16_inputs(1, 2, 40, 128, seed=11)
    b = inputs.fwd_bf16_inputs(1, 2, 40, 128, seed=11)
    c = inputs.fwd_bf16_inputs(1, 2, 40, 128, seed=12)
    assert all(np.array_equal(x.bits, y.bits) for x, y in zip(a, b))
    assert not np.array_equal(a[0].bits, c[0].bits)
    sl = inputs.ragged_seqlens(64, 4096, 4)
    assert sl.min() >= 2048 and sl.max() <= 4096


def test_sweep_grid_skips_cells_over_120GB():
    cells = inputs.sweep_cells()
    assert len(cells) == 30
    skipped = [(b, c) for _, b, c, _, s in cells if s]
    assert sorted(skipped) == [(1024, 32768), (2048, 8192), (2048, 32768)]


def test_paged_decode_inputs_shapes_and_table():
    sl = np.array([100, 0, 64], np.int32)
    q, rho, kp, vp, table, sl2 = inputs.paged_decode_inputs(3, 8, 2, 32, 5, 64, sl, seed=1, spare_pages=4)
    assert q.bits.shape == (3, 8, 64) and rho.bits.shape == (3, 8, 64)
    assert kp.bits.shape == vp.bits.shape == (3 * 5 + 4, 2, 32, 64)
    assert table.shape == (3, 5) and table.dtype == np.int32
    # distinct page ids drawn from the pool: every sequence's pages are its own
    flat = table.reshape(-1)
    assert len(set(flat.tolist())) == flat.size and flat.min() >= 0 and flat.max() < 3 * 5 + 4
    assert np.array_equal(sl2, sl)
    # deterministic in the seed
    again = inputs.paged_decode_inputs(3, 8, 2, 32, 5, 64, sl, seed=1, spare_pages=4)
    assert np.array_equal(again[4], table) and np.array_equal(again[2].bits, kp.bits)
