// Geometry of the packed sign layout and of the kernel's tiling, shared by
// the host packer and the CUDA kernels of libfluxbin.  The layout itself is
// defined in include/fluxbin.h ("Packed sign layout").
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define FB_HD __host__ __device__ constexpr
#else
#define FB_HD constexpr
#endif

namespace fluxbin {

constexpr int kLanes = 32;          // rows per slab = lanes per warp = shared-memory banks
constexpr int kWarps = 8;           // warps per CTA
constexpr int kThreads = kWarps * kLanes;
constexpr int kSlabsPerWarp = 2;    // row slabs a warp keeps accumulators for
constexpr int kSlabsPerCta = kWarps * kSlabsPerWarp;
constexpr int kRowsPerCta = kSlabsPerCta * kLanes;  // 512
constexpr int kMaxCluster = 16;     // CTAs that reduce their split-K partials through DSMEM
// partial sums a CTA receives in a cluster reduction: C slices of ceil(512/C) rows
constexpr int kRedRows = kRowsPerCta + kMaxCluster;
constexpr int kMaxBatch = 16;

// Sub-vectors of one base inside a unit.
FB_HD int subvecs_per_unit(int nb) { return kLanes / nb; }
// Columns covered by one unit.
FB_HD int unit_cols(int nb, int mu) { return subvecs_per_unit(nb) * mu; }
// Units of a branch with ncols columns.
FB_HD int64_t branch_units(int64_t ncols, int nb, int mu) {
    const int w = unit_cols(nb, mu);
    return ncols > 0 ? (ncols + w - 1) / w : 0;
}
FB_HD int64_t row_slabs(int64_t M) { return M > 0 ? (M + kLanes - 1) / kLanes : 0; }
// uint32 words of one (row slab, unit) chunk.
FB_HD int chunk_words(int mu) { return kLanes * mu; }
FB_HD int64_t branch_words(int64_t M, int64_t ncols, int nb, int mu) {
    return row_slabs(M) * branch_units(ncols, nb, mu) * chunk_words(mu);
}

// Sub-vectors per row-scale group inside a unit (gsv).  A branch whose scales
// change every gsv < P sub-vectors uses the grouped visit order below; every
// other branch uses the plain diagonal order (gsv == P).
FB_HD int group_subvecs(int nb, int mu, int scale_group) {
    const int P = subvecs_per_unit(nb);
    return (scale_group > 0 && scale_group < P * mu) ? scale_group / mu : P;
}

// Step at which lane L visits (base k, sub-vector j of the unit).
//   diagonal (gsv == P): k = (q/P + L/P) mod nb, j = (L + q) mod P
//   grouped  (gsv <  P): lane L = gsv*m + s, step q = gsv*a + e;
//                        kg = (a + m) mod (32/gsv), k = kg / (P/gsv),
//                        j = gsv*(kg mod (P/gsv)) + (e xor s)
FB_HD int visit_step(int L, int k, int j, int nb, int gsv) {
    const int P = subvecs_per_unit(nb);
    if (gsv >= P) {
        const int a = ((k - L / P) % nb + nb) % nb;
        const int d = ((j - L) % P + P) % P;
        return a * P + d;
    }
    const int KG = kLanes / gsv, NG = P / gsv;
    const int m = L / gsv, sg = L % gsv;
    const int e = (j % gsv) ^ sg;
    const int kg = k * NG + j / gsv;
    const int a = ((kg - m) % KG + KG) % KG;
    return a * gsv + e;
}
// Bank (table slot k*P + j) that lane L reads at step q.
FB_HD int visit_bank(int L, int q, int nb, int gsv) {
    const int P = subvecs_per_unit(nb);
    if (gsv >= P) {
        const int k = (q / P + L / P) % nb;
        const int j = (L + q) % P;
        return k * P + j;
    }
    const int KG = kLanes / gsv, NG = P / gsv;
    const int m = L / gsv, sg = L % gsv;
    const int a = q / gsv, e = q % gsv;
    const int kg = (a + m) % KG;
    return (kg / NG) * P + gsv * (kg % NG) + (e ^ sg);
}
// Group (base k, scale group g of the unit) whose sum lane L completes at
// slot a = q / gsv of the grouped order: returned as kg = k*(P/gsv) + g.
FB_HD int visit_group(int L, int a, int gsv) {
    const int KG = kLanes / gsv;
    return (a + L / gsv) % KG;
}

}  // namespace fluxbin
