// Tensor-core kernel instantiations (sub-vector length 4 or 8, per-row scales).
#include "fluxbin_tc.cuh"

namespace fluxbin {

using TcKernelFn = void (*)(TcArgs);

namespace {
template <int MU>
TcKernelFn pick_tc(int nb0, int nb1) {
#define FB_TC_NB1(NB0)                                          \
    switch (nb1) {                                              \
        case 0: return &fluxbin_tc_kernel<MU, NB0, 0>;         \
        case 1: return &fluxbin_tc_kernel<MU, NB0, 1>;         \
        case 2: return &fluxbin_tc_kernel<MU, NB0, 2>;         \
        case 4: return &fluxbin_tc_kernel<MU, NB0, 4>;         \
        default: return nullptr;                                \
    }
    switch (nb0) {
        case 1: FB_TC_NB1(1)
        case 2: FB_TC_NB1(2)
        case 4: FB_TC_NB1(4)
        default: return nullptr;
    }
#undef FB_TC_NB1
}
}  // namespace

TcKernelFn select_tc_kernel(int mu, int nb0, int nb1) {
    if (mu == 8) return pick_tc<8>(nb0, nb1);
    if (mu == 4) return pick_tc<4>(nb0, nb1);
    return nullptr;
}

}  // namespace fluxbin
