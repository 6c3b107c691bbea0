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

// Step at which lane L visits (base k, sub-vector j of the unit).
FB_HD int visit_step(int L, int k, int j, int nb) {
    const int P = subvecs_per_unit(nb);
    const int a = ((k - L / P) % nb + nb) % nb;
    const int d = ((j - L) % P + P) % P;
    return a * P + d;
}
// Bank (table slot) that lane L reads at step q: base k = (q/P + L/P) mod nb,
// sub-vector j = (L + q) mod P, slot k*P + j.
FB_HD int visit_bank(int L, int q, int nb) {
    const int P = subvecs_per_unit(nb);
    const int k = (q / P + L / P) % nb;
    const int j = (L + q) % P;
    return k * P + j;
}

}  // namespace fluxbin
