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


def test_rescale_inputs_raise_the_row_max_after_the_first_tile():
    """The planted keys lift a row's max score by > 8 in log2 units in a later
    128-key tile (one or two rises), while the keys before the rise still hold
    a sizeable share of the softmax weight, for causal and full rows alike."""
    T, d = 4096, 128
    q, k, v, rho, spikes = inputs.fwd_rescale_inputs(1, 1, T, d, seed=11)
    z = (q.f64[0, 0] @ k.f64[0, 0].T) / np.sqrt(d) * np.log2(np.e)
    assert len(spikes) >= 8
    for causal in (True, False):
        zc = np.where(np.tril(np.ones((T, T), bool)), z, -np.inf) if causal else z
        tmax = np.maximum.accumulate(zc.reshape(T, T // 128, 128).max(axis=2), axis=1)
        rises = (np.diff(tmax, axis=1) > 8).sum(axis=1)
        assert np.mean(rises >= 1) > 0.4 and np.any(rises >= 2)
        # weight share of the keys before a row's first rise: the part of O and
        # M that the rescale multiplies; it must be large for many rows
        w = np.exp2(zc - zc.max(axis=1, keepdims=True))
        first = np.argmax(np.diff(tmax, axis=1) > 8, axis=1) + 1
        rows = np.nonzero(rises >= 1)[0]
        before = np.array([w[i, :first[i] * 128].sum() / w[i].sum() for i in rows[::7]])
        assert np.quantile(before, 0.9) > 0.2 and before.max() > 0.3
