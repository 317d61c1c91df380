"""fp64 CPU oracle for the Parallax attention operator.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  The
CUDA library never imports, links or calls anything here, and nothing here
imports the CUDA library.

The arithmetic lives in ``parallax_oracle.c`` (plain fp64 C, one row at a time,
in the order of the definition; see that file's header for the definition and
the passages it follows).  This module only builds that file with gcc and
marshals numpy arrays to it.

Parity status of each function (how it is pinned, see ``tests/test_oracle_pins.py``):
  fwd / fwd_rows / decode : pinned (softmax special case = library SDPA, closed
                            two-key form, hand-worked golden example, finite-
                            difference derivative of library SDPA, explicit
                            covariance matrix, invariants)
  rho_proj                : pinned (library matmul, one-hot rows)
  decode_paged            : pinned to decode, a layout change only (identity page
                            table on a contiguous cache, permuted pages, grouped
                            heads equal to replicated key/value heads)
  bwd / rho_proj_bwd      : pinned (central finite differences of the forward
                            oracle; at rho = 0, autograd of library SDPA; autograd
                            of a library matmul); no CUDA counterpart yet
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "parallax_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def compile_source(src: str, out: str) -> str:
    """Compile an oracle C source file into a shared library at ``out``."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile parallax_oracle.c into liboracle.so (gcc, no fast-math, no FMA contraction)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        compile_source(_SRC, _LIB)
    return _LIB


class Oracle:
    """ctypes binding of one build of parallax_oracle.c (the default build or a test's copy)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        lib.oracle_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I]
        lib.oracle_fwd_rows.argtypes = [P, P, P, P, I, I, I, I, I, P, L, P, P]
        lib.oracle_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, L]
        lib.oracle_rho_proj.argtypes = [P, P, P, I, I, I, I, I, P, L]
        lib.oracle_set_threads.argtypes = [I]
        for f in (lib.oracle_fwd, lib.oracle_fwd_rows, lib.oracle_decode,
                  lib.oracle_rho_proj, lib.oracle_max_threads):
            f.restype = I
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def set_threads(self, n: int) -> None:
        self.lib.oracle_set_threads(int(n))

    def fwd(self, q, k, v, rho=None, causal: bool = True):
        """y, lse for every row.  q,k,v,rho: [B,H,T,d] (rho None = softmax only)."""
        q, k, v, rho = _f64(q), _f64(k), _f64(v), _f64(rho)
        B, H, T, d = q.shape
        assert k.shape == v.shape == q.shape and (rho is None or rho.shape == q.shape)
        y = np.empty_like(q)
        lse = np.empty((B, H, T), np.float64)
        rc = self.lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(rho), _ptr(y), _ptr(lse),
                                 B, H, T, d, int(bool(causal)))
        if rc:
            raise ValueError(f"oracle_fwd rejected its arguments (code {rc})")
        return y, lse

    def fwd_rows(self, q, k, v, rho, rows, causal: bool = True):
        """y[n, d], lse[n] for flat row ids rows[n] = (b*H + h)*T + i."""
        q, k, v, rho = _f64(q), _f64(k), _f64(v), _f64(rho)
        B, H, T, d = q.shape
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        y = np.empty((rows.size, d), np.float64)
        lse = np.empty((rows.size,), np.float64)
        rc = self.lib.oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(rho), B, H, T, d,
                                      int(bool(causal)), _ptr(rows), rows.size, _ptr(y), _ptr(lse))
        if rc:
            raise ValueError(f"oracle_fwd_rows rejected its arguments (code {rc})")
        return y, lse

    def decode(self, q, rho, kcache, vcache, seqlens, bh_list=None):
        """Decode outputs.  q,rho: [B,H,d]; caches [B,H,Tcap,d]; seqlens [B].

        Returns y [B,H,d], lse [B,H] -- or, with bh_list (flat b*H+h ids),
        y [n,d], lse [n] for just those heads.
        """
        q, rho, kcache, vcache = _f64(q), _f64(rho), _f64(kcache), _f64(vcache)
        B, H, Tcap, d = kcache.shape
        sl = np.ascontiguousarray(seqlens, dtype=np.int32)
        if bh_list is None:
            y = np.empty((B, H, d), np.float64)
            lse = np.empty((B, H), np.float64)
            lst, n = None, 0
        else:
            lst = np.ascontiguousarray(bh_list, dtype=np.int64)
            n = lst.size
            y = np.empty((n, d), np.float64)
            lse = np.empty((n,), np.float64)
        rc = self.lib.oracle_decode(_ptr(q), _ptr(rho), _ptr(kcache), _ptr(vcache), _ptr(sl),
                                    _ptr(y), _ptr(lse), B, H, Tcap, d, _ptr(lst), n)
        if rc:
            raise ValueError(f"oracle_decode rejected its arguments (code {rc})")
        return y, lse

    def decode_paged(self, q, rho, kpages, vpages, block_table, seqlens, bh_list=None):
        """Decode over a paged cache with grouped query heads.

        q, rho: [B, Hq, d]; kpages, vpages: [num_pages, Hkv, page_size, d];
        block_table: [B, max_pages]; seqlens: [B].  Token t of sequence b is
        row t % page_size of page block_table[b, t // page_size], and query
        head h reads key/value head h // (Hq // Hkv).  The layout is undone
        here -- each head's rows are gathered into the contiguous [B, Hq, Tcap, d]
        cache of ``decode`` -- and the operator is ``decode``'s.
        """
        q, rho = _f64(q), _f64(rho)
        kp, vp = np.asarray(kpages), np.asarray(vpages)
        B, Hq, d = q.shape
        num_pages, Hkv, ps, _ = kp.shape
        bt = np.asarray(block_table, dtype=np.int64)
        sl = np.ascontiguousarray(seqlens, dtype=np.int32)
        max_pages = bt.shape[1]
        group = Hq // Hkv
        tcap = max_pages * ps
        kc = np.zeros((B, Hq, tcap, d), np.float64)
        vc = np.zeros((B, Hq, tcap, d), np.float64)
        for b in range(B):
            t = np.arange(int(sl[b]))
            pages, rows = bt[b, t // ps], t % ps
            # [L, Hkv, d] -> [Hkv, L, d] -> query heads h = kv head * group + g
            kc[b, :, :t.size] = np.repeat(kp[pages, :, rows].transpose(1, 0, 2), group, axis=0)
            vc[b, :, :t.size] = np.repeat(vp[pages, :, rows].transpose(1, 0, 2), group, axis=0)
        return self.decode(q, rho, kc, vc, sl, bh_list)

    def rho_proj(self, x, W_R, H: int, d: int, bt_list=None):
        """rho [B,H,T,d] = per-head slices of x @ W_R; or rho[n,H,d] for token rows bt_list."""
        x, W_R = _f64(x), _f64(W_R)
        B, T, dm = x.shape
        assert W_R.shape == (dm, H * d)
        if bt_list is None:
            out = np.empty((B, H, T, d), np.float64)
            lst, n = None, 0
        else:
            lst = np.ascontiguousarray(bt_list, dtype=np.int64)
            n = lst.size
            out = np.empty((n, H, d), np.float64)
        rc = self.lib.oracle_rho_proj(_ptr(x), _ptr(W_R), _ptr(out), B, T, dm, H, d, _ptr(lst), n)
        if rc:
            raise ValueError(f"oracle_rho_proj rejected its arguments (code {rc})")
        return out


def bwd(q, k, v, rho, dy, causal: bool = True):
    """Gradients of the Parallax forward: (dq, dk, dv, drho) for an upstream dy.

    The operator per head (zubnet.ai news item on Parallax, paragraph 2; the
    forward this module computes): Z = Q K^T / sqrt(d) (keys past the query
    masked when causal), S = softmax over keys, A = R K^T, abar = rowsum(S o A),
    O = S V, M = (S o A) V, Y = O - M + abar * O.  The pages train with this
    operator but print no backward; what follows is the chain rule through
    those definitions, in that order, for L = <dY, Y>:
        dO    = dY (1 + abar)            dabar = rowsum(dY o O)      dM = -dY
        dV    = S^T dO + (S o A)^T dM
        dS    = (dY V^T) o (1 + abar - A) + dabar o A
        dA    = S o (dabar - dY V^T)
        dZ    = S o (dS - rowsum(S o dS))           (softmax backward)
        dQ    = dZ K / sqrt(d)    dK = dZ^T Q / sqrt(d) + dA^T R    dR = dA K
    Plain fp64 numpy, one head at a time, no blocking.  q, k, v, rho, dy: [B, H, T, d].
    """
    q, k, v, rho, dy = (np.asarray(t, np.float64) for t in (q, k, v, rho, dy))
    B, H, T, d = q.shape
    out = [np.zeros_like(q) for _ in range(4)]
    mask = np.tril(np.ones((T, T), bool)) if causal else np.ones((T, T), bool)
    sc = 1.0 / np.sqrt(d)
    for b in range(B):
        for h in range(H):
            Q, K, V, R, dY = q[b, h], k[b, h], v[b, h], rho[b, h], dy[b, h]
            Z = np.where(mask, (Q @ K.T) * sc, -np.inf)
            S = np.exp(Z - Z.max(axis=1, keepdims=True))
            S = S / S.sum(axis=1, keepdims=True)
            A = R @ K.T
            abar = (S * A).sum(axis=1, keepdims=True)
            O = S @ V
            dO = dY * (1.0 + abar)
            dabar = (dY * O).sum(axis=1, keepdims=True)
            dM = -dY
            dV = S.T @ dO + (S * A).T @ dM
            G = dY @ V.T
            dS = G * (1.0 + abar - A) + dabar * A
            dA = S * (dabar - G)
            dZ = S * (dS - (S * dS).sum(axis=1, keepdims=True))
            out[0][b, h] = dZ @ K * sc
            out[1][b, h] = dZ.T @ Q * sc + dA.T @ R
            out[2][b, h] = dV
            out[3][b, h] = dA @ K
    return tuple(out)


def rho_proj_bwd(x, W_R, drho, H: int, d: int):
    """Gradients of rho[b, h, t, :] = x[b, t, :] W_R[:, h d:(h+1) d] for an upstream drho:
    dx = drho' W_R^T and dW_R = sum over (b, t) of x^T drho', with drho' the
    [B, T, H d] regrouping of drho.  fp64."""
    x, W, g = np.asarray(x, np.float64), np.asarray(W_R, np.float64), np.asarray(drho, np.float64)
    B, T, dm = x.shape
    g2 = g.transpose(0, 2, 1, 3).reshape(B, T, H * d)
    dx = g2 @ W.T
    dW = np.einsum("btc,btn->cn", x, g2)
    return dx, dW


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default() -> Oracle:
    """The oracle built from this directory's source (built on first use)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def max_threads() -> int:
    return default().max_threads()


def set_threads(n: int) -> None:
    default().set_threads(n)


def fwd(q, k, v, rho=None, causal: bool = True):
    return default().fwd(q, k, v, rho, causal)


def fwd_rows(q, k, v, rho, rows, causal: bool = True):
    return default().fwd_rows(q, k, v, rho, rows, causal)


def decode(q, rho, kcache, vcache, seqlens, bh_list=None):
    return default().decode(q, rho, kcache, vcache, seqlens, bh_list)


def decode_paged(q, rho, kpages, vpages, block_table, seqlens, bh_list=None):
    return default().decode_paged(q, rho, kpages, vpages, block_table, seqlens, bh_list)


def rho_proj(x, W_R, H: int, d: int, bt_list=None):
    return default().rho_proj(x, W_R, H, d, bt_list)
