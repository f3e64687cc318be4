// prefill_common.cuh -- work-item geometry shared by the prefill kernels.
#pragma once

#include "fia_plan.h"

namespace fia {

// kModeAlibiMma: the ALiBi bias inside a key tile added by one extra K-step
// of the QK^T MMA (16-bit cache, positive qkScale); kModeAlibi adds it in
// the softmax (int8 cache, or any scale).  kModePlainGqa: kModePlain for GQA
// (g >= 2) over a 16-bit cache, whose pairs end both tiles on the same key
// tile.
enum { kModePlain = 0, kModeAlibi = 1, kModePse = 2, kModeAlibiMma = 3, kModePlainGqa = 4 };

struct SubGeom {
    bool valid;
    int q0, h, rows, n;
};
struct PairGeom {
    int b, kvh, cu_q, qlen, kvlen;
    SubGeom t[2];
    int nA, nB;   // key tiles of tile 0 (0 if absent) and tile 1; nA <= nB
    int j0;       // first key tile (past 0 only under a band mask; both tiles share it)
};

template <bool BAND>
__device__ __forceinline__ PairGeom pair_geom(const PrefillArgs &a, const PrefillItem *items,
                                              const SeqInfo *seqs, int idx) {
    const PrefillItem it = items[idx];
    const SeqInfo si = seqs[it.b];
    const bool causal = (a.c.mask_type == 9 || a.c.mask_type == 3);
    PairGeom g;
    g.b = it.b; g.kvh = it.kvh; g.cu_q = si.cu_q; g.qlen = si.qlen; g.kvlen = si.kvlen;
    g.j0 = 0;
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        SubGeom &s = g.t[x];
        s.valid = it.h[x] >= 0;
        s.q0 = it.q0[x];
        s.h = it.h[x];
        s.rows = s.valid ? min(kPrefillBM, si.qlen - it.q0[x]) : 0;
        // keys the tile's rows can see: [lo, hi) (same rule as the host plan)
        const int qmin = si.kvlen - si.qlen + it.q0[x], qmax = qmin + s.rows - 1;
        int lo = 0, hi = causal ? min(si.kvlen, qmax + 1) : si.kvlen;
        if constexpr (BAND) {
            lo = max(0, qmin - a.c.pre);
            hi = min(si.kvlen, qmax + a.c.next + 1);
        }
        s.n = (s.valid && hi > lo) ? (hi + kPrefillBN - 1) / kPrefillBN - lo / kPrefillBN : 0;
        if (BAND && s.valid && hi > lo) g.j0 = lo / kPrefillBN;
    }
    g.nA = g.t[0].n;
    g.nB = g.t[1].n;
    return g;
}

}  // namespace fia
