// Instantiations of the table precompute kernel and of the batch-1 lookup
// kernel on precomputed tables (mu = 8, per-row scales): 16 lookup warps with
// 4 row slabs each (2048 rows per CTA) or 2 (1024 rows).
#include "fluxbin_lut1h.cuh"

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);
using TabKernelFn = void (*)(KernelArgs, float*, NormArgs);
using HKernelFn = void (*)(KernelArgs, const float*);

namespace {
template <int SPW>
HKernelFn pick_h(int nb0, int nb1) {
#define FB_H_NB1(NB0)                                               \
    switch (nb1) {                                                  \
        case 0: return &fluxbin_lut1h_kernel<NB0, 0, 16, SPW>;     \
        case 1: return &fluxbin_lut1h_kernel<NB0, 1, 16, SPW>;     \
        case 2: return &fluxbin_lut1h_kernel<NB0, 2, 16, SPW>;     \
        case 4: return &fluxbin_lut1h_kernel<NB0, 4, 16, SPW>;     \
        default: return nullptr;                                    \
    }
    switch (nb0) {
        case 1: FB_H_NB1(1)
        case 2: FB_H_NB1(2)
        case 4: FB_H_NB1(4)
        default: return nullptr;
    }
#undef FB_H_NB1
}
}  // namespace

namespace {
template <bool NORM>
TabKernelFn pick_t(int nb0, int nb1) {
#define FB_T_NB1(NB0)                                                \
    switch (nb1) {                                                   \
        case 0: return &fluxbin_tables_kernel<NB0, 0, NORM>;        \
        case 1: return &fluxbin_tables_kernel<NB0, 1, NORM>;        \
        case 2: return &fluxbin_tables_kernel<NB0, 2, NORM>;        \
        case 4: return &fluxbin_tables_kernel<NB0, 4, NORM>;        \
        default: return nullptr;                                     \
    }
    switch (nb0) {
        case 1: FB_T_NB1(1)
        case 2: FB_T_NB1(2)
        case 4: FB_T_NB1(4)
        default: return nullptr;
    }
#undef FB_T_NB1
}
}  // namespace

// norm: the variant fused with the preceding RMS normalisation
TabKernelFn select_tables_kernel(int nb0, int nb1, bool norm) {
    return norm ? pick_t<true>(nb0, nb1) : pick_t<false>(nb0, nb1);
}

HKernelFn select_kernel_lut1h(int spw, int nb0, int nb1) {
    if (spw == 4) return pick_h<4>(nb0, nb1);
    if (spw == 2) return pick_h<2>(nb0, nb1);
    return nullptr;
}

int lut1h_threads(int spw) { return spw == 4 ? L1hGeom<16, 4>::kThreads : L1hGeom<16, 2>::kThreads; }
int lut1h_smem_bytes(int spw) { return spw == 4 ? L1hGeom<16, 4>::kSmemBytes : L1hGeom<16, 2>::kSmemBytes; }
int lut1h_slabs(int spw) { return spw == 4 ? L1hGeom<16, 4>::kSlabs : L1hGeom<16, 2>::kSlabs; }

}  // namespace fluxbin
