// FluxBin LUT GEMV kernel for sm_100a (B200).
//
// Computes, for one layer, y[b] (+)= W x[b] with
//   W = sum_k diag(r_k) B_k diag(c_k)  (+ the salient branch through its column map),
// never forming a floating-point W (FluxBin summary, Section 3 "LUT-Based GEMV
// Kernel" and "Virtual Columnar Mapping"; Appendix C.1).
//
// Work decomposition.  The packed signs of a branch are cut into units of
// P = 32/nb sub-vectors per base (32 tables per unit) and into row slabs of 32
// rows (include/fluxbin.h, "Packed sign layout").  A CTA of 8 warps owns 1024
// rows (each warp 4 slabs, each lane one row per slab), one batch chunk of BT
// rows and a contiguous range of units (a split of the reduction dimension).
// For every unit it
//   1. builds the unit's 32 tables per batch row in shared memory: the column
//      scale is fused into the activation (v = c (.) x, the salient branch
//      gathering x through its column map) and the 2^mu signed partial sums of
//      each sub-vector are enumerated in Gray-code order, one fp32 add per entry
//      (LUT building with scale fusion, Section 3; Appendix C.1);
//   2. has every lane stream its rows' packed words with 128-bit loads
//      (prefetched one unit ahead into registers) and, at each of 32 steps,
//      turn the next mu-bit pattern into a shared-memory address and add the
//      table entry into an fp32 register accumulator.  The layout's visit
//      order puts the 32 lanes of a warp on 32 different tables, each in its
//      own bank, so the random-looking lookups never conflict;
//   3. after its last unit, multiplies each accumulator by its row scale (per
//      row, or per row and column block after every unit), and either stores
//      y or adds its partial into an fp32 workspace, the last CTA of a row group
//      to arrive writing y and re-zeroing the workspace (split-K reduction; the
//      pages use global atomics across K tiles, Appendix E.3).
//
// Tables live in rows of 256 bytes: entry e of the tables for batch row b and
// unit parity h sits at b*2^mu*256 + e*256 + h*128 + bank*4, so consecutive
// units alternate between the two 128-byte halves (double buffering with one
// barrier per unit) and, for mu = 8, a byte-permute of the packed word with a
// per-lane offset register yields the whole address in one instruction.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "fluxbin_layout.h"

namespace fluxbin {

struct BranchArgs {
    const uint4* words;     // packed signs (16-byte aligned)
    const __half* r;        // row scales
    const __half* c;        // column scales [nb][ncols]
    const int32_t* gather;  // column map (null: identity)
    int32_t ncols;          // dense columns of this branch
    int32_t units;          // units of this branch
    int32_t rgroup;         // 0: per-row scales; G: per-row per-G-column scales
    int32_t ngroups;        // ceil(ncols / G)
};

struct KernelArgs {
    BranchArgs br[2];       // 0: global, 1: salient (units == 0 when absent)
    const __half* x;        // [B][N]
    void* y;                // [B][M]
    int32_t M, N, B;
    int32_t Ms;             // row slabs
    int32_t Mp;             // Ms * 32
    int32_t n_rg, n_ks, n_bc;
    uint32_t flags;
    float* ws_acc;          // [B][Mp] split-K partial sums (zero between calls)
    unsigned int* ws_cnt;   // [n_rg * n_bc] arrival counters (zero between calls)
};

constexpr uint32_t kFlagAccumulate = 1u;
constexpr uint32_t kFlagYFp32 = 2u;
constexpr uint32_t kFlagEarlyWeights = 4u;

template <int MU>
struct Geom {
    static constexpr int kEntries = 1 << MU;
    static constexpr int kPairBytes = kEntries * 256;  // both halves of one batch row
    static constexpr int kVecs = MU / 4;                // uint4 per lane per unit
};

extern __shared__ __align__(1024) unsigned char fb_smem[];

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t byte_off) {
    return *reinterpret_cast<const float*>(fb_smem + byte_off);
}

__device__ __forceinline__ void sts_f32(uint32_t byte_off, float v) {
    *reinterpret_cast<float*>(fb_smem + byte_off) = v;
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Per-lane byte offsets of the 32 tables visited at steps q = 0..31, packed
// three per register with a zero top byte (for mu = 8 address generation).
template <int NB>
__device__ __forceinline__ void make_offsets_packed(int lane, uint32_t (&offp)[11]) {
#pragma unroll
    for (int r = 0; r < 11; ++r) {
        uint32_t v = 0;
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            const int q = 3 * r + m;
            if (q < 32) v |= (uint32_t)(visit_bank(lane, q, NB) * 4) << (8 * m);
        }
        offp[r] = v;
    }
}

template <int NB>
__device__ __forceinline__ void make_offsets_full(int lane, uint32_t (&offr)[32]) {
#pragma unroll
    for (int q = 0; q < 32; ++q) offr[q] = (uint32_t)(visit_bank(lane, q, NB) * 4);
}

template <int MU>
struct Offsets;
template <>
struct Offsets<8> {
    uint32_t o[11];
    template <int NB>
    __device__ __forceinline__ void make(int lane) { make_offsets_packed<NB>(lane, o); }
    // (pattern byte q%4 of w) << 8 | offset of step q
    __device__ __forceinline__ uint32_t addr(uint32_t w, int q) const {
        return __byte_perm(w, o[q / 3], (uint32_t)(4 + q % 3) | ((uint32_t)(q % 4) << 4) | 0x7700u);
    }
};
template <>
struct Offsets<4> {
    uint32_t o[32];
    template <int NB>
    __device__ __forceinline__ void make(int lane) { make_offsets_full<NB>(lane, o); }
    // (nibble q%8 of w) << 8 | offset of step q
    __device__ __forceinline__ uint32_t addr(uint32_t w, int q) const {
        const int n = q % 8;
        const uint32_t e8 = (n >= 2) ? ((w >> (4 * n - 8)) & 0xF00u) : ((w << (8 - 4 * n)) & 0xF00u);
        return e8 | o[q];
    }
};

// Index of the lowest set bit of i > 0 (the bit that flips between Gray codes i-1 and i).
__host__ __device__ __forceinline__ constexpr int lowest_bit(int i) {
    int t = 0;
    while (!((i >> t) & 1)) ++t;
    return t;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// 32 lookup-accumulate steps of one lane for one row slab and unit.
template <int MU, int NB, int HALF, int BT>
__device__ __forceinline__ void lookup_unit(const uint4 (&w)[Geom<MU>::kVecs], const Offsets<MU>& off,
                                            float (&acc)[BT][NB]) {
    constexpr int P = 32 / NB;
    constexpr int kStepsPerWord = 32 / MU;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const int wi = q / kStepsPerWord;
        const uint32_t word = word_of(w[wi / 4], wi % 4);
        const uint32_t a = off.addr(word, q);
#pragma unroll
        for (int b = 0; b < BT; ++b)
            acc[b][q / P] += lds_f32(a + (uint32_t)(b * Geom<MU>::kPairBytes + HALF * 128));
    }
}

// Tables of one unit for BT batch rows.  Lane = bank = (base k, sub-vector j).
template <int MU, int NB, int HALF, int BT>
__device__ __forceinline__ void build_unit(const KernelArgs& a, const BranchArgs& br, int ul, int b0,
                                           int warp, int lane) {
    constexpr int P = 32 / NB;
    constexpr int LO = MU < 5 ? MU : 5;        // bits enumerated in Gray-code order
    constexpr int NBLK = 1 << (MU - LO);       // entry blocks per batch row
    const int k = lane / P, j = lane % P;
    const int64_t n0 = ((int64_t)ul * P + j) * MU;
    float cv[MU];
    int col[MU];
#pragma unroll
    for (int t = 0; t < MU; ++t) {
        const int64_t n = n0 + t;
        cv[t] = 0.f;
        col[t] = 0;
        if (n < br.ncols) {
            const int cc = br.gather ? __ldg(br.gather + n) : (int)n;
            if (cc >= 0 && cc < a.N) {
                cv[t] = __half2float(br.c[(int64_t)k * br.ncols + n]);
                col[t] = cc;
            }
        }
    }
    for (int z = warp; z < BT * NBLK; z += kWarps) {
        const int bl = z / NBLK, hi = z % NBLK;
        const int bb = b0 + bl;
        float v[MU];
#pragma unroll
        for (int t = 0; t < MU; ++t)
            v[t] = (bb < a.B && cv[t] != 0.f) ? cv[t] * __half2float(a.x[(int64_t)bb * a.N + col[t]]) : 0.f;
        float T = 0.f;
#pragma unroll
        for (int t = LO; t < MU; ++t) T += ((hi >> (t - LO)) & 1) ? v[t] : -v[t];
#pragma unroll
        for (int t = 0; t < LO; ++t) T -= v[t];
        const uint32_t base = (uint32_t)(bl * Geom<MU>::kPairBytes + HALF * 128 + lane * 4);
        sts_f32(base + (uint32_t)(hi << LO) * 256u, T);
#pragma unroll
        for (int i = 1; i < (1 << LO); ++i) {
            const int t = lowest_bit(i);
            const int g = i ^ (i >> 1);
            T += ((g >> t) & 1) ? 2.f * v[t] : -2.f * v[t];
            sts_f32(base + (uint32_t)((hi << LO) | g) * 256u, T);
        }
    }
}

template <int MU>
__device__ __forceinline__ void load_unit_slab(const KernelArgs& a, int u, int sl, int lane,
                                               uint4 (&w)[Geom<MU>::kVecs]) {
    const bool br1 = u >= a.br[0].units;
    const int ul = br1 ? u - a.br[0].units : u;
    const uint4* base = br1 ? a.br[1].words : a.br[0].words;
    const int U = br1 ? a.br[1].units : a.br[0].units;
    if (sl < a.Ms) {
        const uint4* p = base + ((int64_t)sl * U + ul) * (8 * MU) + lane;
#pragma unroll
        for (int h = 0; h < Geom<MU>::kVecs; ++h) w[h] = ld_stream(p + h * 32);
    } else {
#pragma unroll
        for (int h = 0; h < Geom<MU>::kVecs; ++h) w[h] = make_uint4(0, 0, 0, 0);
    }
}

// One unit of branch BR: build its tables, then every slab's lookups, with
// the next unit's packed words requested as soon as a slab's registers free up.
template <int MU, int BR, int NB, int HALF, int BT>
__device__ __forceinline__ void unit_step(const KernelArgs& a, int u, int u_end, int ul, int b0, int slab0,
                                          int warp, int lane, const Offsets<MU>& off,
                                          uint4 (&wb)[kSlabsPerWarp][Geom<MU>::kVecs],
                                          float (&acc)[kSlabsPerWarp][BT][NB],
                                          float (&tot)[kSlabsPerWarp][BT]) {
    const BranchArgs& br = a.br[BR];
    build_unit<MU, NB, HALF, BT>(a, br, ul, b0, warp, lane);
    __syncthreads();
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        uint4 cur[Geom<MU>::kVecs];
#pragma unroll
        for (int h = 0; h < Geom<MU>::kVecs; ++h) cur[h] = wb[rs][h];
        if (u + 1 < u_end) load_unit_slab<MU>(a, u + 1, slab0 + rs, lane, wb[rs]);
        lookup_unit<MU, NB, HALF, BT>(cur, off, acc[rs]);
    }
    if (br.rgroup > 0) {
        // block-wise row scales: the unit lies in one column block
        constexpr int P = 32 / NB;
        const int g = (int)(((int64_t)ul * P * MU) / br.rgroup);
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
            for (int ai = 0; ai < NB; ++ai) {
                const int k = (ai + lane / P) % NB;
                const float sc = i < a.M ? __half2float(br.r[((int64_t)k * br.ngroups + g) * a.M + i]) : 0.f;
#pragma unroll
                for (int b = 0; b < BT; ++b) {
                    tot[rs][b] = fmaf(sc, acc[rs][b][ai], tot[rs][b]);
                    acc[rs][b][ai] = 0.f;
                }
            }
        }
    }
}

template <int MU, int BR, int NB, int BT>
__device__ __forceinline__ void run_branch(const KernelArgs& a, int u_lo, int u_hi, int u_end, int& v, int b0,
                                           int slab0, int warp, int lane,
                                           uint4 (&wb)[kSlabsPerWarp][Geom<MU>::kVecs],
                                           float (&acc)[kSlabsPerWarp][BT][NB],
                                           float (&tot)[kSlabsPerWarp][BT]) {
    if (u_lo >= u_hi) return;
    Offsets<MU> off;
    off.template make<NB>(lane);
    const int ubase = BR ? a.br[0].units : 0;
    for (int u = u_lo; u < u_hi; ++u, ++v) {
        if (v & 1)
            unit_step<MU, BR, NB, 1, BT>(a, u, u_end, u - ubase, b0, slab0, warp, lane, off, wb, acc, tot);
        else
            unit_step<MU, BR, NB, 0, BT>(a, u, u_end, u - ubase, b0, slab0, warp, lane, off, wb, acc, tot);
    }
}

// Row-scale epilogue of one branch with per-row scales.
template <int NB, int BT>
__device__ __forceinline__ void apply_row_scales(const KernelArgs& a, const BranchArgs& br, int slab0, int lane,
                                                 const float (&acc)[kSlabsPerWarp][BT][NB],
                                                 float (&tot)[kSlabsPerWarp][BT]) {
    constexpr int P = 32 / NB;
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
        if (i >= a.M) continue;
#pragma unroll
        for (int ai = 0; ai < NB; ++ai) {
            const int k = (ai + lane / P) % NB;
            const float sc = __half2float(br.r[(int64_t)k * a.M + i]);
#pragma unroll
            for (int b = 0; b < BT; ++b) tot[rs][b] = fmaf(sc, acc[rs][b][ai], tot[rs][b]);
        }
    }
}

__device__ __forceinline__ void store_y(const KernelArgs& a, int b, int i, float v) {
    const int64_t o = (int64_t)b * a.M + i;
    if (a.flags & kFlagYFp32) {
        float* y = static_cast<float*>(a.y);
        y[o] = (a.flags & kFlagAccumulate) ? y[o] + v : v;
    } else {
        __half* y = static_cast<__half*>(a.y);
        y[o] = __float2half_rn((a.flags & kFlagAccumulate) ? __half2float(y[o]) + v : v);
    }
}

template <int MU, int NB0, int NB1, int BT, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) fluxbin_lut_kernel(const KernelArgs a) {
    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
    const int tid = threadIdx.x, warp = tid / kLanes, lane = tid % kLanes;
    const int bc = blockIdx.x % a.n_bc;
    const int ks = (blockIdx.x / a.n_bc) % a.n_ks;
    const int rg = blockIdx.x / (a.n_bc * a.n_ks);
    const int b0 = bc * BT;
    const int slab0 = rg * kSlabsPerCta + warp * kSlabsPerWarp;
    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);
    const int u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    const int u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);

    // Let the next kernel on the stream start its own prologue.
    asm volatile("griddepcontrol.launch_dependents;");

    uint4 wb[kSlabsPerWarp][Geom<MU>::kVecs];
    const bool early = (a.flags & kFlagEarlyWeights) != 0;
    if (early && u_begin < u_end) {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) load_unit_slab<MU>(a, u_begin, slab0 + rs, lane, wb[rs]);
    }
    // Everything below may read what the preceding kernel wrote.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!early && u_begin < u_end) {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) load_unit_slab<MU>(a, u_begin, slab0 + rs, lane, wb[rs]);
    }

    float acc0[kSlabsPerWarp][BT][NB0];
    float acc1[kSlabsPerWarp][BT][NB1E];
    float tot[kSlabsPerWarp][BT];
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs)
#pragma unroll
        for (int b = 0; b < BT; ++b) {
            tot[rs][b] = 0.f;
#pragma unroll
            for (int q = 0; q < NB0; ++q) acc0[rs][b][q] = 0.f;
#pragma unroll
            for (int q = 0; q < NB1E; ++q) acc1[rs][b][q] = 0.f;
        }

    int v = 0;
    run_branch<MU, 0, NB0, BT>(a, u_begin, min(u_end, U0), u_end, v, b0, slab0, warp, lane, wb, acc0, tot);
    if constexpr (NB1 > 0)
        run_branch<MU, 1, NB1, BT>(a, max(u_begin, U0), u_end, u_end, v, b0, slab0, warp, lane, wb, acc1, tot);

    // Row scales (per-row case; the block-wise case was applied per unit).
    if (a.br[0].rgroup == 0 && u_begin < min(u_end, U0))
        apply_row_scales<NB0, BT>(a, a.br[0], slab0, lane, acc0, tot);
    if constexpr (NB1 > 0) {
        if (a.br[1].rgroup == 0 && max(u_begin, U0) < u_end)
            apply_row_scales<NB1, BT>(a, a.br[1], slab0, lane, acc1, tot);
    }

    if (a.n_ks == 1) {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
            if (i >= a.M) continue;
#pragma unroll
            for (int b = 0; b < BT; ++b)
                if (b0 + b < a.B) store_y(a, b0 + b, i, tot[rs][b]);
        }
        return;
    }

    // Split-K: add this CTA's partial sums; the last CTA of the group finishes.
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
        if (i >= a.M) continue;
#pragma unroll
        for (int b = 0; b < BT; ++b)
            if (b0 + b < a.B) red_add_f32(a.ws_acc + (int64_t)(b0 + b) * a.Mp + i, tot[rs][b]);
    }
    __threadfence();
    __syncthreads();
    __shared__ unsigned int s_last;
    unsigned int* cnt = a.ws_cnt + (rg * a.n_bc + bc);
    if (tid == 0) s_last = (atomicAdd(cnt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int row0 = rg * kRowsPerCta;
    for (int e = tid; e < kRowsPerCta * BT; e += kThreads) {
        const int b = e / kRowsPerCta, i = row0 + e % kRowsPerCta;
        if (i >= a.M || b0 + b >= a.B) continue;
        float* p = a.ws_acc + (int64_t)(b0 + b) * a.Mp + i;
        const float val = __ldcg(p);
        __stcg(p, 0.f);
        store_y(a, b0 + b, i, val);
    }
    if (tid == 0) *cnt = 0u;
}

}  // namespace fluxbin
