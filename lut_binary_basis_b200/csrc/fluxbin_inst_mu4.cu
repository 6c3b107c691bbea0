// Kernel instantiations for sub-vector length mu = 4.
#include "fluxbin_kernel.cuh"

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);

namespace {
template <int BT>
KernelFn pick(int nb0, int nb1) {
#define FB_NB1(NB0)                                             \
    switch (nb1) {                                              \
        case 0: return &fluxbin_lut_kernel<4, NB0, 0, BT>;  \
        case 1: return &fluxbin_lut_kernel<4, NB0, 1, BT>;  \
        case 2: return &fluxbin_lut_kernel<4, NB0, 2, BT>;  \
        case 4: return &fluxbin_lut_kernel<4, NB0, 4, BT>;  \
        default: return nullptr;                                \
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

// Tables of one batch row take 4 KiB; the batch tile is bounded by registers.
KernelFn select_kernel_mu4(int nb0, int nb1, int bt) {
    if (bt == 1) return pick<1>(nb0, nb1);
    if (bt == 2) return pick<2>(nb0, nb1);
    if (bt == 4) return pick<4>(nb0, nb1);
    return nullptr;
}

}  // namespace fluxbin
