// Kernel instantiations for sub-vector length mu = 8.
#include "fluxbin_kernel.cuh"

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);

namespace {
template <int BT, int GS1>
KernelFn pick(int nb0, int nb1) {
#define FB_NB1(NB0)                                                        \
    switch (nb1) {                                                         \
        case 0: return GS1 ? nullptr : &fluxbin_lut_kernel<8, NB0, 0, BT, 0>; \
        case 1: return &fluxbin_lut_kernel<8, NB0, 1, BT, GS1>;          \
        case 2: return &fluxbin_lut_kernel<8, NB0, 2, BT, GS1>;          \
        case 4: return &fluxbin_lut_kernel<8, NB0, 4, BT, GS1>;          \
        default: return nullptr;                                           \
    }
    switch (nb0) {
        case 1: FB_NB1(1)
        case 2: FB_NB1(2)
        case 4: FB_NB1(4)
        default: return nullptr;
    }
#undef FB_NB1
}
// Three CTAs per SM (batch 1, per-row or block-wise salient scales).
KernelFn pick3(int nb0, int nb1) {
#define FB_NB1(NB0)                                                  \
    switch (nb1) {                                                   \
        case 0: return &fluxbin_lut_kernel<8, NB0, 0, 1, 0, 3>;     \
        case 1: return &fluxbin_lut_kernel<8, NB0, 1, 1, 0, 3>;     \
        case 2: return &fluxbin_lut_kernel<8, NB0, 2, 1, 0, 3>;     \
        case 4: return &fluxbin_lut_kernel<8, NB0, 4, 1, 0, 3>;     \
        default: return nullptr;                                     \
    }
    switch (nb0) {
        case 1: FB_NB1(1)
        case 2: FB_NB1(2)
        case 4: FB_NB1(4)
        default: return nullptr;
    }
#undef FB_NB1
}
}  // namespace

// Batch-1 build with three CTAs per SM (no grouped salient scales), for large
// layers; nullptr otherwise.
KernelFn select_kernel_mu8_3(int nb0, int nb1, int bt, int gs1) {
    return (bt == 1 && gs1 == 0) ? pick3(nb0, nb1) : nullptr;
}

// Tables of one batch row take 64 KiB (two 32 KiB halves); one batch row per
// CTA.  gs1 > 0: the salient branch has row scales per group of gs1
// sub-vectors.
KernelFn select_kernel_mu8(int nb0, int nb1, int bt, int gs1) {
    if (gs1 > 0) {
        if (bt != 1) return nullptr;
        if (gs1 == 1) return pick<1, 1>(nb0, nb1);
        if (gs1 == 2) return pick<1, 2>(nb0, nb1);
        if (gs1 == 4) return pick<1, 4>(nb0, nb1);
        return nullptr;
    }
    if (bt == 1) return pick<1, 0>(nb0, nb1);
    return nullptr;
}

}  // namespace fluxbin
