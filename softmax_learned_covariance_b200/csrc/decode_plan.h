// decode_plan.h -- split plan of the decode kernels (host code, no CUDA types).
//
// Kept free of CUDA headers so the plan, and the bound on its scratch that the
// no-allocation decode relies on, can be compiled and swept by a plain C++
// compiler on a machine without a GPU.
#pragma once
#include <cstddef>

namespace plx {

struct DecodePlan {
    int nsplit;      // chunks per sequence (units per head)
    int chunk;       // tokens per chunk: a multiple of 128, or the whole cache
};

// Units of (b, h, chunk): about 64 per SM (4 waves of resident CTAs) so the
// block scheduler can balance ragged lengths; chunks are multiples of 128
// tokens (a unit's partial state is 2d + 3 floats, ~1% of a 128-token chunk's
// K/V bytes).  B * H * nsplit never exceeds 64 * sm_count when nsplit > 1.
inline DecodePlan plan_decode(int B, int H, int Tcap, int d, int sm_count) {
    (void)d;
    DecodePlan p;
    const long bh = (long)B * H;
    const long want_units = 64L * sm_count;
    long nsplit = want_units / bh;
    if (nsplit < 1) nsplit = 1;
    long chunk = ((long)Tcap + nsplit - 1) / nsplit;
    chunk = ((chunk + 127) / 128) * 128;
    if (chunk >= Tcap) chunk = Tcap;                 // one unit per sequence
    p.chunk = (int)chunk;
    p.nsplit = (int)(((long)Tcap + chunk - 1) / chunk);
    return p;
}

// Bytes of split partials (mu, l, abar, O[d], M[d] per unit); 0 with one unit per head.
inline size_t decode_partials_bytes(int B, int H, int d, const DecodePlan &p) {
    if (p.nsplit <= 1) return 0;
    return (size_t)B * H * p.nsplit * (2 * d + 3) * sizeof(float);
}

// Largest partials any shape can need on a device with `sm_count` SMs.
constexpr size_t decode_partials_bound(int sm_count, int d_max) {
    return (size_t)64 * sm_count * (2 * d_max + 3) * sizeof(float);
}

// The paged decode's tensor-core units serve up to 8 query heads of a KV head
// and are sized like four split-kernel units, so that each warp streams enough
// tiles to amortise its pipeline fill and the final merge.
inline DecodePlan plan_decode_paged(int B, int Hq, int Hkv, int Tcap, int d, int sm_count) {
    const int group = Hq / Hkv;
    return plan_decode(B, Hkv * ((group + 7) / 8) * 4, Tcap, d, sm_count);
}

}  // namespace plx
