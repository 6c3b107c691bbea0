// Instantiations of the warp-specialised batch-1 LUT kernel (mu = 8, per-row
// scales): 16 lookup warps (1024 rows, one CTA per SM) or 8 (512 rows, two
// CTAs per SM).
#include "fluxbin_lut1.cuh"
#include "fluxbin_lut2.cuh"

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);

namespace {
template <int LW>
KernelFn pick_l1(int nb0, int nb1) {
#define FB_L1_NB1(NB0)                                         \
    switch (nb1) {                                             \
        case 0: return &fluxbin_lut1_kernel<NB0, 0, LW, 2>;   \
        case 1: return &fluxbin_lut1_kernel<NB0, 1, LW, 2>;   \
        case 2: return &fluxbin_lut1_kernel<NB0, 2, LW, 2>;   \
        case 4: return &fluxbin_lut1_kernel<NB0, 4, LW, 2>;   \
        default: return nullptr;                               \
    }
    switch (nb0) {
        case 1: FB_L1_NB1(1)
        case 2: FB_L1_NB1(2)
        case 4: FB_L1_NB1(4)
        default: return nullptr;
    }
#undef FB_L1_NB1
}
}  // namespace

KernelFn select_kernel_lut1(int lw, int nb0, int nb1) {
    if (lw == 16) return pick_l1<16>(nb0, nb1);
    if (lw == 8) return pick_l1<8>(nb0, nb1);
    return nullptr;
}

int lut1_threads(int lw) { return lw == 16 ? L1Geom<16>::kThreads : L1Geom<8>::kThreads; }
int lut1_smem_bytes(int lw) { return lw == 16 ? L1Geom<16>::kSmemBytes : L1Geom<8>::kSmemBytes; }
int lut1_slabs(int lw) { return lw == 16 ? L1Geom<16>::kSlabs : L1Geom<8>::kSlabs; }

// Batch pairs on fp16-pair tables (fluxbin_lut2.cuh), 16 lookup warps.

KernelFn select_kernel_lut2(int nb0, int nb1) {
#define FB_L2_NB1(NB0)                                         \
    switch (nb1) {                                             \
        case 0: return &fluxbin_lut2_kernel<NB0, 0, 16>;      \
        case 1: return &fluxbin_lut2_kernel<NB0, 1, 16>;      \
        case 2: return &fluxbin_lut2_kernel<NB0, 2, 16>;      \
        case 4: return &fluxbin_lut2_kernel<NB0, 4, 16>;      \
        default: return nullptr;                               \
    }
    switch (nb0) {
        case 1: FB_L2_NB1(1)
        case 2: FB_L2_NB1(2)
        case 4: FB_L2_NB1(4)
        default: return nullptr;
    }
#undef FB_L2_NB1
}
int lut2_threads() { return L2Geom<16>::kThreads; }
int lut2_smem_bytes() { return L2Geom<16>::kSmemBytes; }
int lut2_slabs() { return L2Geom<16>::kSlabs; }

}  // namespace fluxbin
