"""C-ABI checks that need no GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before touching the device."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import softmax_learned_covariance_b200 as plx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"PARALLAX_API\s+[\w\s\*]+?\b(parallax_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    from softmax_learned_covariance_b200 import build

    build.build()
    return plx.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_strerror_covers_all_codes(L):
    for code in range(10):
        s = plx.parallax_strerror(code)
        assert s and s != "unknown status"
    assert plx.parallax_strerror(99) == "unknown status"


P = ctypes.c_void_p
A16 = P(0x10000)      # fake, 16-byte aligned (never dereferenced: validation fails first)
MIS = P(0x10008)      # fake, misaligned


def fwd(L, q=A16, k=A16, v=A16, rho=A16, y=A16, lse=None, B=1, H=1, T=8, d=128, causal=1, i=1, o=0):
    return L.parallax_fwd(q, k, v, rho, y, lse, B, H, T, d, causal, i, o, None)


def test_fwd_host_validation(L):
    assert fwd(L, q=None) == 1
    assert fwd(L, y=None) == 1
    assert fwd(L, T=0) == 2
    assert fwd(L, d=96) == 2
    assert fwd(L, B=-1) == 2
    assert fwd(L, k=MIS) == 3
    assert fwd(L, rho=MIS) == 3
    assert fwd(L, lse=P(0x10002)) == 3
    assert fwd(L, i=1, o=5) == 4
    assert fwd(L, i=0, o=1) == 4
    assert fwd(L, d=32, i=1, o=0) == 2      # head dims 64 and 128 only


def test_fwd_fused_host_validation(L):
    def ff(q=A16, k=A16, v=A16, x=A16, w=A16, y=A16, B=1, H=1, T=8, d=128, dm=128, i=1, o=0):
        return L.parallax_fwd_fused(q, k, v, x, w, y, None, B, H, T, d, dm, 1, i, o, None)
    assert ff(x=None) == 1
    assert ff(w=None) == 1
    assert ff(dm=100) == 2           # d_model must be a multiple of 64
    assert ff(T=0) == 2
    assert ff(w=MIS) == 3
    assert ff(i=0) == 4              # bf16 inputs only
    assert ff(d=64) == 5             # the fused probe is built for d = 128


def test_decode_host_validation(L):
    def dec(q=A16, rho=A16, kc=A16, vc=A16, sl=A16, y=A16, B=2, H=2, Tcap=16, d=128, i=1, o=0):
        return L.parallax_decode(q, rho, kc, vc, sl, y, None, B, H, Tcap, d, i, o, None)
    assert dec(rho=None) == 1
    assert dec(sl=None) == 1
    assert dec(Tcap=0) == 2
    assert dec(d=32) == 2
    assert dec(kc=MIS) == 3
    assert dec(i=0) == 4
    assert dec(o=7) == 4


def test_softmax_decode_host_validation(L):
    def sd(q=A16, kc=A16, vc=A16, sl=A16, y=A16, Tcap=16, d=256, i=1, o=0):
        return L.parallax_softmax_decode(q, kc, vc, sl, y, None, 2, 2, Tcap, d, i, o, None)
    assert sd(kc=None) == 1
    assert sd(d=96) == 2
    assert sd(Tcap=0) == 2
    assert sd(vc=MIS) == 3
    assert sd(i=0) == 4


def test_decode_paged_host_validation(L):
    def dec(q=A16, rho=A16, kp=A16, vp=A16, bt=A16, sl=A16, y=A16, B=2, Hq=4, Hkv=2, ps=64, mp=4, npg=8, d=128,
            i=1, o=0):
        return L.parallax_decode_paged(q, rho, kp, vp, bt, sl, y, None, B, Hq, Hkv, ps, mp, npg, d, i, o, None)
    assert dec(bt=None) == 1
    assert dec(vp=None) == 1
    assert dec(Hq=3) == 2          # not a multiple of Hkv
    assert dec(Hq=1) == 2          # fewer query heads than KV heads
    assert dec(ps=48) == 2         # not a power of two
    assert dec(ps=8) == 2          # below the minimum page size
    assert dec(ps=8192) == 2
    assert dec(mp=0) == 2
    assert dec(npg=0) == 2
    assert dec(d=96) == 2
    assert dec(kp=MIS) == 3
    assert dec(i=0) == 4
    assert dec(o=5) == 4


def test_rho_proj_host_validation(L):
    def rp(x=A16, w=A16, r=A16, B=1, T=4, dm=128, H=2, d=128, dt=1):
        return L.parallax_rho_proj(x, w, r, B, T, dm, H, d, dt, None)
    assert rp(x=None) == 1
    assert rp(dm=100) == 2
    assert rp(H=1, d=128) == 2           # H*d must be a multiple of 256
    assert rp(w=MIS) == 3
    assert rp(dt=0) == 4
