"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, not by the oracle.

Each ``pin_*`` function checks one such fact against an oracle build.  The
``test_pin_*`` tests run them on the real oracle; ``test_planted_mistakes_are_caught``
compiles copies of the oracle source with one plausible mistake planted in each
(on the CPU) and requires that at least one pin fails for every copy.

Sources of the facts:
  * zubnet.ai news item on Parallax, paragraph 2: the output is softmax attention
    minus the KV covariance projected by the probe rho_i = W_R x_i, and W_R = 0
    recovers standard softmax exactly.
  * encorp.ai blog "Integraciones de IA personalizadas tras la atencion Parallax",
    section "Parallax conserva softmax..." and its FAQ: a zero projection reduces
    the layer exactly to softmax attention.
  * Mathematics of the definition: the covariance of a single point is zero;
    for two keys C rho = s0 s1 (a1 - a0)(v1 - v0); the covariance term is the
    derivative of softmax attention along a logit perturbation a_j = k_j . rho;
    invariances under value shifts, key shifts and linearity in rho.
"""
from __future__ import annotations

import json
import math
import os
import shutil
import tempfile

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, *shape, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _sdpa(q, k, v, causal=True):
    """Library softmax attention in fp64 (torch CPU), scale 1/sqrt(d)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal).numpy()


def _logsumexp(q, k, causal=True):
    d = q.shape[-1]
    z = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / math.sqrt(d)
    if causal:
        T = q.shape[-2]
        mask = torch.ones(T, T, dtype=torch.bool).triu(1)
        z = z.masked_fill(mask, float("-inf"))
    return torch.logsumexp(z, dim=-1).numpy()


# --------------------------------------------------------------------------- #
# pins (each takes an oracle build)
# --------------------------------------------------------------------------- #


def pin_softmax_special_case(orc):
    """rho = 0 reduces the layer to softmax attention: equal to library SDPA, and
    bitwise equal to the oracle's softmax-only call."""
    for causal in (True, False):
        q, k, v = (_rand(s, 2, 3, 37, 16) for s in (1, 2, 3))
        y0, lse0 = orc.fwd(q, k, v, np.zeros_like(q), causal=causal)
        yn, lsen = orc.fwd(q, k, v, None, causal=causal)
        assert np.array_equal(y0, yn), "rho = 0 must equal the softmax-only result bitwise"
        ref = _sdpa(q, k, v, causal)
        assert np.max(np.abs(y0 - ref)) < 1e-12
        assert np.max(np.abs(lse0 - _logsumexp(q, k, causal))) < 1e-12


def pin_single_key(orc):
    """A single key has zero covariance: causal row 0 returns v_0 exactly, whatever rho."""
    q, k, v = (_rand(s, 1, 2, 5, 8) for s in (4, 5, 6))
    rho = _rand(7, 1, 2, 5, 8, scale=3.0)
    y, lse = orc.fwd(q, k, v, rho, causal=True)
    assert np.array_equal(y[:, :, 0], v[:, :, 0])
    z0 = np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]) / math.sqrt(8)
    assert np.max(np.abs(lse[:, :, 0] - z0)) < 1e-14


def pin_two_key_closed_form(orc):
    """Row 1 (two keys): C rho = s0 s1 (a1 - a0)(v1 - v0), with s the two-way softmax."""
    d = 8
    q, k, v = (_rand(s, 1, 1, 2, d) for s in (8, 9, 10))
    rho = _rand(11, 1, 1, 2, d)
    y, _ = orc.fwd(q, k, v, rho, causal=True)
    z0 = q[0, 0, 1] @ k[0, 0, 0] / math.sqrt(d)
    z1 = q[0, 0, 1] @ k[0, 0, 1] / math.sqrt(d)
    s1 = 1.0 / (1.0 + math.exp(z0 - z1))
    s0 = 1.0 - s1
    a0 = k[0, 0, 0] @ rho[0, 0, 1]
    a1 = k[0, 0, 1] @ rho[0, 0, 1]
    o = s0 * v[0, 0, 0] + s1 * v[0, 0, 1]
    expect = o - s0 * s1 * (a1 - a0) * (v[0, 0, 1] - v[0, 0, 0])
    assert np.max(np.abs(y[0, 0, 1] - expect)) < 1e-13


def pin_golden_worked_example(orc):
    """The hand-derived example in tests/golden/two_key_worked_example.json."""
    with open(os.path.join(GOLDEN, "two_key_worked_example.json")) as f:
        g = json.load(f)
    arr = lambda key: np.array(g[key], dtype=np.float64)
    y, lse = orc.fwd(arr("q"), arr("k"), arr("v"), arr("rho"), causal=g["causal"])
    tol = g["tolerance_abs"]
    assert np.max(np.abs(y - arr("y"))) < tol
    assert np.max(np.abs(lse - arr("lse"))) < tol


def pin_derivative_of_softmax_attention(orc):
    """C_i rho_i is the derivative of softmax attention along the logit shift
    eps * (k_j . rho_i): with q' = q + eps sqrt(d) rho the scores become z + eps a.
    Checked against central differences of the library SDPA."""
    d = 16
    q, k, v = (_rand(s, 1, 2, 24, d) for s in (12, 13, 14))
    rho = _rand(15, 1, 2, 24, d, scale=0.3)
    for causal in (True, False):
        y, _ = orc.fwd(q, k, v, rho, causal=causal)
        eps = 1e-5
        fp = _sdpa(q + eps * math.sqrt(d) * rho, k, v, causal)
        fm = _sdpa(q - eps * math.sqrt(d) * rho, k, v, causal)
        deriv = (fp - fm) / (2 * eps)
        o = _sdpa(q, k, v, causal)
        assert np.max(np.abs(y - (o - deriv))) < 1e-7


def pin_explicit_covariance(orc):
    """Brute force on a tiny head: build C_i = sum_j s_j (v_j - o)(k_j - kbar)^T as a
    d x d matrix, then y_i = o - C_i rho_i (matrix form, not the oracle's vector form)."""
    T, d = 9, 5
    q, k, v = (_rand(s, T, d) for s in (16, 17, 18))
    rho = _rand(19, T, d)
    y, _ = orc.fwd(q[None, None], k[None, None], v[None, None], rho[None, None], causal=True)
    for i in range(T):
        z = k[: i + 1] @ q[i] / math.sqrt(d)
        s = np.exp(z - z.max())
        s /= s.sum()
        o = s @ v[: i + 1]
        kbar = s @ k[: i + 1]
        C = np.zeros((d, d))
        for j in range(i + 1):
            C += s[j] * np.outer(v[j] - o, k[j] - kbar)
        assert np.max(np.abs(y[0, 0, i] - (o - C @ rho[i]))) < 1e-13


def pin_one_pass_and_third_form(orc):
    """The one-pass expansion y = o - (m - o abar) and y = sum_j s_j (1 + abar - a_j) v_j."""
    T, d = 40, 12
    q, k, v = (_rand(s, T, d) for s in (20, 21, 22))
    rho = _rand(23, T, d, scale=2.0)
    y, _ = orc.fwd(q[None, None], k[None, None], v[None, None], rho[None, None], causal=False)
    z = q @ k.T / math.sqrt(d)
    s = np.exp(z - z.max(axis=1, keepdims=True))
    s /= s.sum(axis=1, keepdims=True)
    a = rho @ k.T                                   # a_ij = k_j . rho_i
    o = s @ v
    abar = (s * a).sum(axis=1, keepdims=True)
    m = (s * a) @ v
    y1 = o - (m - o * abar)
    y3 = (s * (1.0 + abar - a)) @ v
    scale = np.max(np.abs(y1))
    assert np.max(np.abs(y[0, 0] - y1)) < 1e-12 * max(1.0, scale)
    assert np.max(np.abs(y[0, 0] - y3)) < 1e-12 * max(1.0, scale)


def pin_invariants(orc):
    """Constant V gives y = c; shifting V shifts y; a common key shift leaves y unchanged;
    y is affine in rho."""
    B, H, T, d = 1, 2, 17, 8
    q, k, v = (_rand(s, B, H, T, d) for s in (24, 25, 26))
    rho = _rand(27, B, H, T, d)
    y, _ = orc.fwd(q, k, v, rho)
    c = _rand(28, d)
    yc, _ = orc.fwd(q, k, np.broadcast_to(c, v.shape), rho)
    assert np.max(np.abs(yc - c)) < 1e-12
    ys, _ = orc.fwd(q, k, v + c, rho)
    assert np.max(np.abs(ys - (y + c))) < 1e-12
    # Shifting every key by u adds q.u/sqrt(d) to all of a row's scores (softmax-invariant)
    # and rho.u to all of its a_j (absorbed by the centering).
    u = _rand(29, d)
    yk, _ = orc.fwd(q, k + u, v, rho)
    assert np.max(np.abs(yk - y)) < 1e-11
    y2, _ = orc.fwd(q, k, v, 2 * rho)
    y0, _ = orc.fwd(q, k, v, 0 * rho)
    assert np.max(np.abs((y2 - y) - (y - y0))) < 1e-11


def pin_rows_and_decode_agree_with_fwd(orc):
    """Row subsets equal the full call; a decode query over the first n cache rows equals
    causal row n-1 of the forward; an empty cache row gives y = 0, lse = -inf."""
    B, H, T, d = 2, 3, 21, 8
    q, k, v = (_rand(s, B, H, T, d) for s in (30, 31, 32))
    rho = _rand(33, B, H, T, d)
    y, lse = orc.fwd(q, k, v, rho)
    rows = np.array([0, 5, 20, 21, 63, 125])
    yr, lr = orc.fwd_rows(q, k, v, rho, rows)
    assert np.array_equal(yr, y.reshape(-1, d)[rows])
    assert np.array_equal(lr, lse.reshape(-1)[rows])
    seqlens = np.array([7, 21], np.int32)
    qd = np.stack([q[0, :, 6], q[1, :, 20]])
    rd = np.stack([rho[0, :, 6], rho[1, :, 20]])
    yd, ld = orc.decode(qd, rd, k, v, seqlens)
    assert np.max(np.abs(yd[0] - y[0, :, 6])) < 1e-14
    assert np.max(np.abs(yd[1] - y[1, :, 20])) < 1e-14
    assert np.max(np.abs(ld[0] - lse[0, :, 6])) < 1e-14
    ye, le = orc.decode(qd, rd, k, v, np.array([0, 3], np.int32))
    assert np.all(ye[0] == 0.0) and np.all(np.isneginf(le[0]))
    ys, ls = orc.decode(qd, rd, k, v, np.array([0, 3], np.int32), bh_list=np.array([4, 1]))
    assert np.array_equal(ys[0], ye[1, 1]) and np.array_equal(ys[1], ye[0, 1])


def pin_rho_projection(orc):
    """rho = per-head slices of x W_R: equal to the library matmul, and a one-hot x row
    selects one row of W_R."""
    B, T, dm, H, d = 2, 5, 24, 3, 4
    x = _rand(34, B, T, dm)
    W = _rand(35, dm, H * d)
    rho = orc.rho_proj(x, W, H, d)
    ref = (x @ W).reshape(B, T, H, d).transpose(0, 2, 1, 3)
    assert np.max(np.abs(rho - ref)) < 1e-12
    e = np.zeros((1, 1, dm))
    e[0, 0, 7] = 1.0
    r1 = orc.rho_proj(e, W, H, d)
    assert np.array_equal(r1[0, :, 0, :], W[7].reshape(H, d))
    rs = orc.rho_proj(x, W, H, d, bt_list=np.array([6, 0]))
    assert np.array_equal(rs[0], rho[1, :, 1, :]) and np.array_equal(rs[1], rho[0, :, 0, :])


def _paged_case(seed, B=3, Hq=4, Hkv=2, ps=4, max_pages=3, d=5):
    rng = np.random.default_rng(seed)
    num_pages = B * max_pages + 2
    q = rng.standard_normal((B, Hq, d))
    rho = 0.3 * rng.standard_normal((B, Hq, d))
    kp = rng.standard_normal((num_pages, Hkv, ps, d))
    vp = rng.standard_normal((num_pages, Hkv, ps, d))
    table = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages)
    seqlens = np.array([max_pages * ps, 1, ps + 1][:B], np.int32)
    return q, rho, kp, vp, table, seqlens


def pin_paged_layout(orc):
    """The paged, grouped-head decode is decode on the cache the pages describe:
    row t of sequence b is row t % page_size of page table[b, t // page_size], and
    query head h reads key/value head h // (Hq / Hkv).  The contiguous cache is
    built here row by row, independently of the oracle's gather."""
    q, rho, kp, vp, table, seqlens = _paged_case(41)
    B, Hq, d = q.shape
    _, Hkv, ps, _ = kp.shape
    group = Hq // Hkv
    tcap = table.shape[1] * ps
    kc = np.zeros((B, Hq, tcap, d))
    vc = np.zeros((B, Hq, tcap, d))
    for b in range(B):
        for h in range(Hq):
            for t in range(int(seqlens[b])):
                kc[b, h, t] = kp[table[b, t // ps], h // group, t % ps]
                vc[b, h, t] = vp[table[b, t // ps], h // group, t % ps]
    y, lse = orc.decode_paged(q, rho, kp, vp, table, seqlens)
    yr, lr = orc.decode(q, rho, kc, vc, seqlens)
    assert np.array_equal(y, yr) and np.array_equal(lse, lr)
    # renaming the physical pages (and the table with them) changes nothing
    perm = np.random.default_rng(42).permutation(kp.shape[0])
    inv = np.argsort(perm)
    y2, _ = orc.decode_paged(q, rho, kp[perm], vp[perm], inv[table], seqlens)
    assert np.array_equal(y2, y)
    # grouped heads = the same pool with every key/value head repeated group times
    y3, _ = orc.decode_paged(q, rho, np.repeat(kp, group, axis=1), np.repeat(vp, group, axis=1), table, seqlens)
    assert np.array_equal(y3, y)
    # a page the table does not reach is never read
    kp4 = kp.copy()
    unused = sorted(set(range(kp.shape[0])) - set(table.reshape(-1).tolist()))
    kp4[unused] = np.nan
    y4, _ = orc.decode_paged(q, rho, kp4, vp, table, seqlens)
    assert np.array_equal(y4, y)


PINS = [pin_softmax_special_case, pin_single_key, pin_two_key_closed_form,
        pin_golden_worked_example, pin_derivative_of_softmax_attention, pin_explicit_covariance,
        pin_one_pass_and_third_form, pin_invariants, pin_rows_and_decode_agree_with_fwd,
        pin_rho_projection, pin_paged_layout]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(oracle.default())


# --------------------------------------------------------------------------- #
# planted mistakes: every one must make at least one pin fail
# --------------------------------------------------------------------------- #

# Not listed, because they are not mistakes: centering k by any constant vector
# (e.g. an unweighted key mean) or dropping only one of the two centerings leaves
# C rho unchanged, since sum_j s_j (v_j - o) = 0 and sum_j s_j (a_j - abar) = 0.
MUTANTS = {
    "sign_of_correction": ("y_i[e] = o[e] - c[e];", "y_i[e] = o[e] + c[e];"),
    "no_centering_at_all": ("proj += (k_j[e] - kbar[e]) * rho_i[e];", "proj += k_j[e] * rho_i[e];",
                            "c[e] += w * (v_j[e] - o[e]);", "c[e] += w * v_j[e];"),
    "transposed_covariance": ("proj += (k_j[e] - kbar[e]) * rho_i[e];", "proj += (v_j[e] - o[e]) * rho_i[e];",
                              "c[e] += w * (v_j[e] - o[e]);", "c[e] += w * (k_j[e] - kbar[e]);"),
    "score_scale_1_over_d": ("1.0 / sqrt((double)d)", "1.0 / (double)d"),
    "causal_off_by_one": ("const long n = causal ? i + 1 : T;\n        double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));\n        row_parallax(q + head + (size_t)i * d, k + head, v + head,\n                     rho ? rho + head + (size_t)i * d : NULL, n, d,\n                     y + head",
                          "const long n = causal ? (i > 0 ? i : 1) : T;\n        double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));\n        row_parallax(q + head + (size_t)i * d, k + head, v + head,\n                     rho ? rho + head + (size_t)i * d : NULL, n, d,\n                     y + head"),
    "probe_of_wrong_row": ("rho ? rho + head + (size_t)i * d : NULL, n, d,\n                     y + head",
                           "rho ? rho + head : NULL, n, d,\n                     y + head"),
    "unweighted_covariance": ("const double w = z[j] * proj;", "const double w = proj / (double)n;"),
    "lse_base_2": ("*lse_i = mu + log(l);", "*lse_i = mu + log2(l);"),
    "missing_max_subtraction_in_lse": ("*lse_i = mu + log(l);", "*lse_i = log(l);"),
    "scale_from_key_count": ("1.0 / sqrt((double)d)", "1.0 / sqrt((double)n)"),
    "softmax_weights_unnormalised": ("for (j = 0; j < n; ++j) z[j] = z[j] / l;", "for (j = 0; j < n; ++j) z[j] = z[j];"),
    "rho_proj_transposed_w": ("acc += x_row[c] * W[(size_t)c * N + h * d + e];",
                              "acc += x_row[c] * W[(size_t)(h * d + e) * dm + c];"),
}


def _make_mutant(tmpdir, name, subs):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "parallax_oracle.c")).read()
    for old, new in zip(subs[0::2], subs[1::2]):
        assert src.count(old) >= 1, f"mutation {name}: pattern not found"
        src = src.replace(old, new)
    cpath = os.path.join(tmpdir, f"{name}.c")
    with open(cpath, "w") as f:
        f.write(src)
    return oracle.Oracle(oracle.compile_source(cpath, os.path.join(tmpdir, f"lib{name}.so")))


def test_planted_mistakes_are_caught():
    tmpdir = tempfile.mkdtemp(prefix="oracle_mutants_")
    survivors = []
    try:
        for name, subs in MUTANTS.items():
            orc = _make_mutant(tmpdir, name, subs)
            caught = []
            for pin in PINS:
                try:
                    pin(orc)
                except (AssertionError, ValueError):
                    caught.append(pin.__name__)
            if not caught:
                survivors.append(name)
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)
    assert not survivors, f"planted mistakes no pin detects: {survivors}"


# The paged decode's gather is Python (oracle/__init__.py); plant mistakes in a
# copy of that method and require pin_paged_layout to catch each.
GATHER_MUTANTS = {
    "page_and_row_swapped": ("pages, rows = bt[b, t // ps], t % ps", "pages, rows = bt[b, t % ps], t // ps"),
    "heads_interleaved": ("np.repeat(kp[pages, :, rows].transpose(1, 0, 2), group, axis=0)",
                          "np.tile(kp[pages, :, rows].transpose(1, 0, 2), (group, 1, 1))"),
    "table_row_of_wrong_sequence": ("pages, rows = bt[b, t // ps], t % ps", "pages, rows = bt[0, t // ps], t % ps"),
    "v_rows_from_k": ("vc[b, :, :t.size] = np.repeat(vp[pages", "vc[b, :, :t.size] = np.repeat(kp[pages"),
}


def test_planted_gather_mistakes_are_caught():
    import inspect
    import textwrap

    src = textwrap.dedent(inspect.getsource(oracle.Oracle.decode_paged))
    survivors = []
    for name, (old, new) in GATHER_MUTANTS.items():
        assert src.count(old) == 1, f"mutation {name}: pattern not found"
        ns = {"np": np, "_f64": oracle._f64}
        exec(compile(src.replace(old, new), f"<{name}>", "exec"), ns)
        orc = oracle.default()
        mutant = type("MutantOracle", (oracle.Oracle,), {"decode_paged": ns["decode_paged"]})
        m = mutant.__new__(mutant)
        m.__dict__.update(orc.__dict__)
        try:
            pin_paged_layout(m)
            survivors.append(name)
        except (AssertionError, ValueError, IndexError):
            pass
    assert not survivors, f"planted gather mistakes pin_paged_layout misses: {survivors}"
