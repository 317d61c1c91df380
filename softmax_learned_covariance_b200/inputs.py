"""Seeded synthetic inputs for the Parallax operator, shared by tests, bench and smoke.

This module holds random-number generation, bf16 rounding and shape recipes
only -- none of the operator's arithmetic.  Both the CUDA path and the fp64
oracle read the values it produces: the device gets the bf16 bits, the oracle
gets the same bits widened exactly to fp64.

Recipe (host side): numpy ``default_rng(seed)`` (PCG64) draws ``standard_normal``
in fp64, the draw is scaled, narrowed to fp32, then rounded to bf16 with
round-to-nearest-even.  Arrays are drawn in a fixed order per workload so the
same seed always yields the same bits.

Workloads follow the shapes the pages' models use (Qwen-3 style 1.7B layer:
d_model 2048, 16 heads of 128, context 4096) and the decode sweep range
(batch 1..2048 x context 128..32768); values are N(0,1) for q, k, v and x,
N(0, 0.02^2) for W_R, so rho = x W_R has standard deviation about 0.905.
"""
from __future__ import annotations

import dataclasses

import numpy as np

# --------------------------------------------------------------------------- #
# bf16 helpers (bit manipulation only)
# --------------------------------------------------------------------------- #


def bf16_bits(a) -> np.ndarray:
    """Round to bf16 (round-to-nearest-even from the fp32 value); return uint16 bits."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to fp64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def round_bf16(a) -> np.ndarray:
    """fp64 array holding the bf16-rounded values of ``a`` (storage precision model)."""
    return bf16_to_f64(bf16_bits(a))


def to_torch_bf16(bits: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


# --------------------------------------------------------------------------- #
# workloads
# --------------------------------------------------------------------------- #


@dataclasses.dataclass
class Tensor16:
    """A bf16 input: its bits (for the device) and exact fp64 values (for the oracle)."""

    bits: np.ndarray

    @property
    def f64(self) -> np.ndarray:
        return bf16_to_f64(self.bits)

    def torch(self):
        return to_torch_bf16(self.bits)

    @property
    def shape(self):
        return self.bits.shape


def _normal(rng, shape, scale=1.0):
    return rng.standard_normal(size=shape) * scale


def _bf(rng, shape, scale=1.0) -> Tensor16:
    return Tensor16(bf16_bits(_normal(rng, shape, scale)))


def fwd_f32_inputs(B=1, H=2, T=128, d=64, rho_scale=0.1, seed=1):
    """fp32 forward inputs (tiny causal case): q,k,v ~ N(0,1), rho ~ N(0, rho_scale^2).

    Returns fp32 numpy arrays; the oracle reads them widened to fp64.
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, T, d)
    q = _normal(rng, shape).astype(np.float32)
    k = _normal(rng, shape).astype(np.float32)
    v = _normal(rng, shape).astype(np.float32)
    rho = _normal(rng, shape, rho_scale).astype(np.float32)
    return q, k, v, rho


def fwd_bf16_inputs(B, H, T, d, rho_scale=0.905, seed=3):
    """bf16 forward inputs: q,k,v ~ N(0,1); rho ~ N(0, rho_scale^2) drawn directly.

    rho_scale 0.905 matches rho = x W_R with x ~ N(0,1) over d_model 2048 and
    W_R ~ N(0, 0.02^2).
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, T, d)
    q = _bf(rng, shape)
    k = _bf(rng, shape)
    v = _bf(rng, shape)
    rho = _bf(rng, shape, rho_scale)
    return q, k, v, rho


def fwd_rescale_inputs(B, H, T, d, rho_scale=0.905, groups=8, spike=6.0, seed=11):
    """bf16 forward inputs whose running row max rises after the first key tile.

    Query row i belongs to group g = i % groups and is q_i = sqrt(d) e_g + 0.3 n
    (e_g the g-th unit vector, n ~ N(0,1)^d).  Keys are small, k ~ N(0, 0.05^2),
    so background scores are ~0 and every visible key keeps a weight near 1.
    For each group, one planted key k = spike * e_g in key tile 1 + 4g mod (tiles - 1)
    (128-key tiles) gives that group's rows a score of ~spike (6 nats = 8.7 in
    log2 units); for odd groups a second planted key one tile later scores
    ~2 * spike.  Rows of other groups score those keys at ~0.  v ~ N(0,1);
    rho ~ N(0, rho_scale^2).  Returns (q, k, v, rho, spikes) where spikes lists
    (group, key index, score) for each planted key.
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, T, d)
    grp = np.arange(T) % groups
    q = rng.standard_normal(size=shape) * 0.3
    q[..., np.arange(T), grp] += np.sqrt(d)
    k = rng.standard_normal(size=shape) * 0.05
    v = rng.standard_normal(size=shape)
    rho = rng.standard_normal(size=shape) * rho_scale
    spikes = []
    ntiles = (T + 127) // 128
    if ntiles >= 2:
        for g in range(groups):
            t1 = 1 + (4 * g) % (ntiles - 1)
            j1 = min(T - 1, t1 * 128 + (17 * g) % 128)
            k[..., j1, :] = 0.0
            k[..., j1, g] = spike
            spikes.append((g, j1, spike))
            if g % 2 == 1 and t1 + 1 < ntiles:
                j2 = min(T - 1, (t1 + 1) * 128 + (29 * g) % 128)
                k[..., j2, :] = 0.0
                k[..., j2, g] = 2 * spike
                spikes.append((g, j2, 2 * spike))
    return (Tensor16(bf16_bits(q)), Tensor16(bf16_bits(k)), Tensor16(bf16_bits(v)), Tensor16(bf16_bits(rho)),
            spikes)


def rho_proj_inputs(B, T, d_model=2048, H=16, d=128, w_scale=0.02, seed=3):
    """x ~ N(0,1) [B,T,d_model] and W_R ~ N(0, w_scale^2) [d_model, H*d], both bf16."""
    rng = np.random.default_rng(seed + 1000)
    x = _bf(rng, (B, T, d_model))
    w = _bf(rng, (d_model, H * d), w_scale)
    return x, w


def decode_inputs(B, H, Tcap, d, seqlens=None, rho_scale=0.05, seed=2):
    """Decode inputs: q, rho [B,H,d]; kcache, vcache [B,H,Tcap,d]; seqlens int32 [B].

    seqlens defaults to Tcap for every sequence (a full contiguous cache).
    """
    rng = np.random.default_rng(seed)
    q = _bf(rng, (B, H, d))
    rho = _bf(rng, (B, H, d), rho_scale)
    kc = _bf(rng, (B, H, Tcap, d))
    vc = _bf(rng, (B, H, Tcap, d))
    if seqlens is None:
        seqlens = np.full((B,), Tcap, np.int32)
    return q, rho, kc, vc, np.ascontiguousarray(seqlens, dtype=np.int32)


def paged_decode_inputs(B, Hq, Hkv, page_size, max_pages, d, seqlens, rho_scale=0.05, seed=6, spare_pages=3):
    """Paged, grouped-head decode inputs.

    q, rho [B, Hq, d]; kpages, vpages [num_pages, Hkv, page_size, d] with
    num_pages = B * max_pages + spare_pages; block_table int32 [B, max_pages]
    holding a random permutation of the page ids (so a sequence's pages are
    scattered through the pool and some pages belong to no sequence);
    seqlens int32 [B].
    """
    rng = np.random.default_rng(seed)
    num_pages = B * max_pages + spare_pages
    q = _bf(rng, (B, Hq, d))
    rho = _bf(rng, (B, Hq, d), rho_scale)
    kp = _bf(rng, (num_pages, Hkv, page_size, d))
    vp = _bf(rng, (num_pages, Hkv, page_size, d))
    table = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    return q, rho, kp, vp, np.ascontiguousarray(table), np.ascontiguousarray(seqlens, dtype=np.int32)


def ragged_seqlens(B, ctx, seed):
    """Integer lengths uniform in [ctx/2, ctx] (the decode sweep's ragged mix)."""
    rng = np.random.default_rng(seed + 7919)
    lo = max(1, ctx // 2)
    return rng.integers(lo, ctx + 1, size=B, dtype=np.int64).astype(np.int32)


def decode_inputs_device(B, H, Tcap, d, seqlens, rho_scale=0.05, seed=4, device="cuda"):
    """Large decode cells generated on the device with torch's seeded generator.

    Used where the cache does not fit comfortably in host memory.  Returns torch
    tensors (bf16 on ``device``) q, rho, kcache, vcache and int32 seqlens.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))

    def draw(shape, scale=1.0):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        # draw in slabs to bound the fp32 temporary
        flat = t.view(-1)
        step = 1 << 27
        for s in range(0, flat.numel(), step):
            n = min(step, flat.numel() - s)
            flat[s:s + n] = (torch.randn(n, generator=g, device=device, dtype=torch.float32) * scale).to(torch.bfloat16)
        return t

    q = draw((B, H, d))
    rho = draw((B, H, d), rho_scale)
    kc = draw((B, H, Tcap, d))
    vc = draw((B, H, Tcap, d))
    sl = torch.as_tensor(np.ascontiguousarray(seqlens, dtype=np.int32), device=device)
    return q, rho, kc, vc, sl


# Decode sweep grid (batch x context), heads 16, head dim 128.
SWEEP_BATCHES = (1, 8, 64, 256, 1024, 2048)
SWEEP_CONTEXTS = (128, 512, 2048, 8192, 32768)
SWEEP_CACHE_LIMIT_BYTES = 120 * 10**9


def sweep_cells(H=16, d=128):
    """(index, batch, ctx, cache_bytes, skipped) for each cell of the decode sweep."""
    cells = []
    idx = 0
    for b in SWEEP_BATCHES:
        for c in SWEEP_CONTEXTS:
            nbytes = 2 * b * H * c * d * 2
            cells.append((idx, b, c, nbytes, nbytes > SWEEP_CACHE_LIMIT_BYTES))
            idx += 1
    return cells
