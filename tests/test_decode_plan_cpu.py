"""The decode split plan on the host (no GPU): sanity of the chunking, and the
bound on its split partials that the no-allocation decode's static array of
PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES relies on.

The plan is header-only C++ (csrc/decode_plan.h); this test compiles a small
sweep over it with the host C++ compiler and runs it.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "softmax_learned_covariance_b200", "csrc")

SWEEP = r"""
#include <cstdio>
#include "decode_plan.h"
int main() {
    const int Bs[] = {1, 2, 3, 7, 8, 16, 33, 64, 100, 256, 1000, 1024, 2048, 4096, 65536};
    const int Hs[] = {1, 2, 8, 16, 32, 40, 64, 128};
    const int Ts[] = {1, 2, 100, 127, 128, 129, 500, 1000, 4096, 5000, 8192, 32768, 65537, 131072, 1048576};
    const int Ss[] = {1, 2, 16, 100, 132, 148, 160, 200, 252};
    long checked = 0;
    for (int sms : Ss) for (int B : Bs) for (int H : Hs) for (int T : Ts) for (int d = 64; d <= 128; d += 64) {
        const plx::DecodePlan p = plx::plan_decode(B, H, T, d, sms);
        // chunking covers the cache exactly once
        if (p.nsplit < 1 || p.chunk < 1) { printf("bad plan %d %d %d %d\n", B, H, T, sms); return 1; }
        if ((long)p.nsplit * p.chunk < T || (long)(p.nsplit - 1) * p.chunk >= T) { printf("cover %d %d %d\n", B, H, T); return 1; }
        if (p.nsplit > 1 && p.chunk % 128 != 0) { printf("chunk %d\n", p.chunk); return 1; }
        const size_t need = plx::decode_partials_bytes(B, H, d, p);
        if (need > plx::decode_partials_bound(sms, 128)) { printf("bound %d %d %d %d %zu\n", B, H, T, sms, need); return 1; }
        if (need > LIMIT) { printf("limit %d %d %d %d %zu\n", B, H, T, sms, need); return 1; }
        const plx::DecodePlan pg = plx::plan_decode_paged(B, H, (H % 4 == 0) ? H / 4 : H, T, d, sms);
        if (plx::decode_partials_bytes(B, H, d, pg) > plx::decode_partials_bound(sms, 128) * 2) { printf("paged\n"); return 1; }
        ++checked;
    }
    printf("%ld\n", checked);
    return 0;
}
"""


def _limit():
    src = open(os.path.join(ROOT, "include", "parallax.h")).read()
    m = re.search(r"#define PARALLAX_DECODE_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", src)
    return int(m.group(1)) << int(m.group(2))


def test_plan_partials_fit_the_static_scratch_up_to_252_sms(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    src = tmp_path / "sweep.cpp"
    src.write_text(SWEEP)
    exe = tmp_path / "sweep"
    subprocess.check_call([cxx, "-std=c++17", "-O1", f"-DLIMIT={_limit()}ul", "-I", CSRC, str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
    assert int(out.stdout.strip()) == 9 * 15 * 8 * 15 * 2   # every (sms, B, H, Tcap, d) cell checked
