// FluxBin LUT GEMV kernel for sm_100a (B200).
//
// Computes, for one layer, y[b] (+)= W x[b] with
//   W = sum_k diag(r_k) B_k diag(c_k)  (+ the salient branch through its column map),
// never forming a floating-point W (FluxBin summary, Section 3 "LUT-Based GEMV
// Kernel" and "Virtual Columnar Mapping"; Appendix C.1).
//
// Work decomposition.  The packed signs of a branch are cut into units of
// P = 32/nb sub-vectors per base (32 tables per unit) and into row slabs of 32
// rows (include/fluxbin.h, "Packed sign layout").  A CTA of 8 warps owns 512
// rows (each warp two slabs, each lane one row per slab), one batch chunk of
// BT rows and a contiguous range of units (a split of the reduction
// dimension).  For every unit it
//   1. forms the unit's 32*mu activation products v = c (.) x once, one slot
//      per thread, two units ahead of their use (column scale fused into the
//      activation; the salient branch gathers x through its column map),
//      parked in a small double-buffered shared array;
//   2. builds the unit's 32 tables per batch row from them: the 2^mu signed
//      partial sums of every sub-vector, enumerated in Gray-code order, one
//      fp32 add per entry (LUT building with scale fusion, Section 3;
//      Appendix C.1);
//   3. has every lane stream its rows' packed words with 128-bit loads,
//      requested two units ahead into registers, and at each of 32 steps turn
//      the next mu-bit pattern into a shared-memory address (one byte-permute
//      with a per-lane offset word) and add the table entry into an fp32
//      register.  The layout's visit order puts the 32 lanes of a warp on 32
//      different tables, each in its own bank: the lookups never conflict;
//   4. after its last unit multiplies each accumulator by its row scale (per
//      row, or per row and column block after every unit) and reduces the
//      split-K partials: inside a thread-block cluster through distributed
//      shared memory (fixed order, no global traffic), or, when the reduction
//      is wider than a cluster, through an fp32 workspace where the last CTA to
//      arrive writes y (the pages reduce across K tiles with global atomics,
//      Appendix E.3).
// Everything that belongs to the layer (packed words, scales, column map) is
// requested before the kernel waits for its predecessor on the stream
// (programmatic dependent launch); only activations, outputs and workspace
// are touched after that wait.
//
// Shared memory (byte offsets from the start of the dynamic allocation):
//   tables  BT * 2^mu * 256: entry e of the tables of batch row b for unit
//           parity h at b*2^mu*256 + e*256 + h*128 + bank*4 (consecutive units
//           alternate halves: double buffering with one barrier per unit)
//   vbuf    2 * BT * 32*mu floats: [parity][b][t][bank] activation products
//   red     BT * 528 floats: [b][source rank][row of this CTA's slice], the
//           split-K partials the cluster's CTAs push to the slice owner
//   scales  (grouped salient branch only) 2 * (32/gsv) * 512 fp16: the row
//           scales of each (base, group) of the unit, [parity][group][row]
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

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
    int32_t cluster;        // 1: the n_ks CTAs of a row group form a cluster and reduce in DSMEM
    uint32_t flags;
    float* ws_acc;          // [B][Mp] split-K partial sums (zero between calls)
    unsigned int* ws_cnt;   // [n_rg * n_bc] arrival counters (zero between calls)
    unsigned int* err;      // device error word (kernels with bounded waits set a bit when one gives up)
};

// The element-wise operator preceding a layer, fused into its table
// precompute (fluxbin_tables.cuh, NORM): RMS normalisation.
struct NormArgs {
    const __half* gamma;    // [N] RMSNorm weight
    float eps;              // added to mean(h^2)
    __half* x_out;          // [N] normalised activation (fp16), or null
};

constexpr uint32_t kFlagAccumulate = 1u;
constexpr uint32_t kFlagYFp32 = 2u;
constexpr uint32_t kFlagEarlyWeights = 4u;
constexpr uint32_t kFlagPathLut = 8u;
constexpr uint32_t kFlagPathTc = 16u;
constexpr uint32_t kFlagTestWaitTimeout = 32u;
constexpr uint32_t kFlagSeparateTables = 64u;

template <int MU, int BT>
struct Geom {
    static constexpr int kEntries = 1 << MU;
    static constexpr int kPairBytes = kEntries * 256;      // both halves of one batch row
    static constexpr int kVecs = MU / 4;                    // uint4 per lane per unit
    static constexpr int kLo = MU == 8 ? 4 : 2;             // entry bits enumerated per build block
    static constexpr int kBlocks = 1 << (MU - kLo);         // build blocks per batch row
    static constexpr int kSlots = 32 * MU;                  // activation products per unit and batch row
    static constexpr int kTableBytes = BT * kPairBytes;
    static constexpr int kVbufOff = kTableBytes;
    static constexpr int kVbufBytes = 2 * BT * kSlots * 4;
    static constexpr int kRedOff = kVbufOff + kVbufBytes;
    static constexpr int kRedBytes = BT * kRedRows * 4;
    static constexpr int kScaleOff = kRedOff + kRedBytes;  // grouped salient branch: staged scales
};

// Byte offsets (bank * 4) of the tables lane L visits at steps 3r, 3r+1, 3r+2,
// packed into bytes 0..2 of word [nb index][order][r][L]; byte 3 is zero.
// Order 0 is the diagonal visit order, orders 1..3 the grouped order with
// 1, 2 or 4 sub-vectors per row-scale group.
struct OffsetTable {
    uint32_t w[3][4][11][32];
};
constexpr OffsetTable make_offset_table() {
    OffsetTable t{};
    for (int nbi = 0; nbi < 3; ++nbi)
        for (int o = 0; o < 4; ++o)
            for (int r = 0; r < 11; ++r)
                for (int L = 0; L < 32; ++L) {
                    const int nb = 1 << nbi;
                    const int gsv = o == 0 ? subvecs_per_unit(nb) : (1 << (o - 1));
                    uint32_t v = 0;
                    for (int m = 0; m < 3; ++m) {
                        const int q = 3 * r + m;
                        if (q < 32) v |= (uint32_t)(visit_bank(L, q, nb, gsv) * 4) << (8 * m);
                    }
                    t.w[nbi][o][r][L] = v;
                }
    return t;
}
__device__ const OffsetTable kOffsetTable = make_offset_table();

template <int GSV>
constexpr int order_index() { return GSV == 0 ? 0 : (GSV == 1 ? 1 : (GSV == 2 ? 2 : 3)); }

template <int NB>
constexpr int nb_index() { return NB == 1 ? 0 : (NB == 2 ? 1 : 2); }

extern __shared__ __align__(1024) unsigned char fb_smem[];

__device__ __forceinline__ uint32_t smem_base() { return (uint32_t)__cvta_generic_to_shared(fb_smem); }

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Plain (compiler-scheduled) shared-memory access by byte offset from the
// start of the dynamic allocation.
template <typename T>
__device__ __forceinline__ T& smem_at(uint32_t byte_off) {
    return *reinterpret_cast<T*>(fb_smem + byte_off);
}

// Table entry at a byte offset from the start of the dynamic allocation (the
// tables sit at offset 0).  An ordinary load through the shared array lets
// the compiler fold the array's address into the load's immediate offset,
// so a lookup costs one byte-permute and one load.
template <int OFF>
__device__ __forceinline__ float table_entry(uint32_t byte_off) {
    return *reinterpret_cast<const float*>(fb_smem + OFF + byte_off);
}

// The dynamic shared memory of a kernel without static shared variables
// starts right after the 1 KiB the system reserves per CTA (in a cluster
// launch the CTA's rank sits in bits 24 and up of its shared addresses).
// Kernels that address tables absolutely check this at entry and otherwise
// take their add-based loop.
constexpr uint32_t kDynSmemBase = 0x400u;

// Table entry / entry word at an absolute shared address (+ a constant).
template <int IMM>
__device__ __forceinline__ float lds_f32_abs(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(IMM));
    return v;
}
template <int IMM>
__device__ __forceinline__ uint32_t lds_u32_abs(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(IMM));
    return v;
}

// Shared-memory access by 32-bit shared address (+ a constant byte offset).
__device__ __forceinline__ uint64_t lds_b64(uint32_t addr) {
    uint64_t v;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
    return v;
}
template <int OFF>
__device__ __forceinline__ void sts_b64_at(uint32_t addr, uint64_t v) {
    asm volatile("st.shared.b64 [%0+%1], %2;" ::"r"(addr), "n"(OFF), "l"(v) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Two fp32 values in one 64-bit register, added pairwise by one instruction.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t x;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(lo), "f"(hi));
    return x;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t x, uint64_t y) {
    uint64_t z;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
    return z;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t x, uint64_t y) {
    uint64_t z;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
    return z;
}
__device__ __forceinline__ float sum_f32x2(uint64_t x) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
    return lo + hi;
}

__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Store a float at a shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ void st_dsmem_f32(uint32_t local_smem_addr, uint32_t rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_smem_addr), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

template <int MU>
struct Offsets {
    uint32_t o[11];
    template <int NB, int GSV>
    __device__ __forceinline__ void load(int lane) {
#pragma unroll
        for (int r = 0; r < 11; ++r) o[r] = __ldg(&kOffsetTable.w[nb_index<NB>()][order_index<GSV>()][r][lane]);
    }
    // Absolute addressing (mu = 8): with the CTA's rank byte in byte 3 of every
    // offset word, (rank << 24) | (pattern << 8) | bank*4, byte 2 zero (the
    // sign of a bank offset byte, below 128, replicated by the permute's
    // sign mode); the shared base goes into the load's immediate.
    __device__ __forceinline__ void set_rank_byte(uint32_t hi_byte) {
#pragma unroll
        for (int r = 0; r < 11; ++r) o[r] = (o[r] & 0x00FFFFFFu) | hi_byte;
    }
    __device__ __forceinline__ uint32_t addr_abs(uint32_t w, int q) const {
        uint32_t d;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(o[q / 3]),
            "r"((uint32_t)((4 + q % 3) | ((q % 4) << 4) | (0xC << 8) | (0x7 << 12))));
        return d;
    }
    // table byte offset of the entry step q selects: (pattern << 8) | bank*4
    __device__ __forceinline__ uint32_t addr(uint32_t w, int q) const {
        if constexpr (MU == 8) {
            return __byte_perm(w, o[q / 3], (uint32_t)(4 + q % 3) | ((uint32_t)(q % 4) << 4) | 0x7700u);
        } else {
            const int n = q % 8;
            const uint32_t e8 = (n >= 2) ? ((w >> (4 * n - 8)) & 0xF00u) : ((w << (8 - 4 * n)) & 0xF00u);
            return __byte_perm(e8, o[q / 3], (uint32_t)(4 + q % 3) | 0x7710u);
        }
    }
};

// Calls f(std::integral_constant<int, I>) for I = 0 .. N-1 (compile-time indices).
template <int I, int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for<I + 1, N>(f);
    }
}

__host__ __device__ __forceinline__ constexpr int lowest_bit(int i) {
    int t = 0;
    while (!((i >> t) & 1)) ++t;
    return t;
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// 32 lookup-accumulate steps of one lane for one row slab and unit.  Steps
// q and q+1 always feed the same accumulator; their entries are added as a
// pair (one paired fp32 add per two lookups) and folded into acc at the end.
template <int MU, int NB, int HALF, int BT>
__device__ __forceinline__ void lookup_unit(const uint4 (&w)[Geom<MU, BT>::kVecs], const Offsets<MU>& off,
                                            float (&acc)[BT][NB]) {
    constexpr int P = 32 / NB;
    constexpr int kStepsPerWord = 32 / MU;
    uint64_t pair[BT][NB];
#pragma unroll
    for (int b = 0; b < BT; ++b)
#pragma unroll
        for (int i = 0; i < NB; ++i) pair[b][i] = 0ull;
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        const int wi0 = q / kStepsPerWord, wi1 = (q + 1) / kStepsPerWord;
        const uint32_t a0 = off.addr(word_of(w[wi0 / 4], wi0 % 4), q);
        const uint32_t a1 = off.addr(word_of(w[wi1 / 4], wi1 % 4), q + 1);
        static_for<0, BT>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            constexpr int OFF = b * Geom<MU, BT>::kPairBytes + HALF * 128;
            const float f0 = table_entry<OFF>(a0);
            const float f1 = table_entry<OFF>(a1);
            pair[b][q / P] = add_f32x2(pair[b][q / P], pack_f32x2(f0, f1));
        });
    }
#pragma unroll
    for (int b = 0; b < BT; ++b)
#pragma unroll
        for (int i = 0; i < NB; ++i) acc[b][i] += sum_f32x2(pair[b][i]);
}

// Salient branch with row scales per group of GSV sub-vectors (grouped visit
// order): after the GSV steps of slot a the lane has the whole contribution of
// one (base, group) kg = (a + lane/GSV) mod KG to its row and multiplies it by
// that group's row scale, staged in shared memory as [kg][row of the CTA].
// One batch row (BT == 1).
template <int MU, int NB, int GSV, int HALF>
__device__ __forceinline__ void lookup_unit_grouped(const uint4 (&w)[kSlabsPerWarp][Geom<MU, 1>::kVecs],
                                                    const Offsets<MU>& off, uint32_t scale_row_off,
                                                    int lane, float (&tot)[kSlabsPerWarp][1]) {
    constexpr int kStepsPerWord = 32 / MU;
    constexpr int KG = 32 / GSV;
    const int m = lane / GSV;
#pragma unroll
    for (int a = 0; a < KG; ++a) {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            float g = 0.f;
#pragma unroll
            for (int e = 0; e < GSV; ++e) {
                const int q = a * GSV + e;
                const int wi = q / kStepsPerWord;
                g += table_entry<HALF * 128>(off.addr(word_of(w[rs][wi / 4], wi % 4), q));
            }
            const uint32_t kg = (uint32_t)((a + m) & (KG - 1));
            const float sc = __half2float(
                smem_at<const __half>(scale_row_off + (kg * kRowsPerCta + (uint32_t)(rs * kLanes)) * 2u));
            tot[rs][0] = fmaf(sc, g, tot[rs][0]);
        }
    }
}

// The activation-product slot a thread owns: bit t = s / 32, bank c = s % 32.
// Its layer data (column scale, activation column) are requested a unit
// before they are needed and kept as loaded: nothing at the request waits for
// the loads.  The column is checked and the scale converted when the slot is
// consumed.
struct SlotRaw {
    __half c;  // column scale (0 for padding)
    int col;   // activation column as the column map holds it (-1 for padding)
};

template <int MU, int NB0, int NB1>
__device__ __forceinline__ SlotRaw slot_raw(const KernelArgs& a, int u, int s) {
    SlotRaw r{__float2half(0.f), -1};
    const bool br1 = NB1 > 0 && u >= a.br[0].units;
    // select fields one by one (a reference chosen at run time would force a
    // local copy of the kernel parameters)
    const __half* cptr = br1 ? a.br[1].c : a.br[0].c;
    const int32_t* gptr = br1 ? a.br[1].gather : a.br[0].gather;
    const int ncols = br1 ? a.br[1].ncols : a.br[0].ncols;
    // sub-vectors per base and unit of each branch (compile-time divisors)
    constexpr int P0 = 32 / NB0, P1 = NB1 > 0 ? 32 / NB1 : 32;
    const int ul = br1 ? u - a.br[0].units : u;
    const int cb = s % 32, t = s / 32;
    const int k = br1 ? cb / P1 : cb / P0;
    const int j = br1 ? cb % P1 : cb % P0;
    const int64_t n = (int64_t)ul * (br1 ? P1 * MU : P0 * MU) + j * MU + t;
    if (n < ncols) {
        r.col = gptr ? __ldg(gptr + n) : (int)n;
        r.c = cptr[(int64_t)k * ncols + n];
    }
    return r;
}

// A consumed slot: its fp32 column scale (0 for padding and out-of-range
// columns) and its activation column (-1 for those).
struct SlotStatic {
    float c;
    int col;
};

__device__ __forceinline__ SlotStatic resolve_slot(const KernelArgs& a, const SlotRaw& r) {
    const bool ok = r.col >= 0 && r.col < a.N;
    return SlotStatic{ok ? __half2float(r.c) : 0.f, ok ? r.col : -1};
}

template <int BT>
__device__ __forceinline__ void slot_x(const KernelArgs& a, int b0, int col, __half (&xv)[BT]) {
#pragma unroll
    for (int b = 0; b < BT; ++b)
        xv[b] = (col >= 0 && b0 + b < a.B) ? a.x[(int64_t)(b0 + b) * a.N + col] : __float2half(0.f);
}

template <int MU, int BT>
__device__ __forceinline__ void store_products(uint32_t sbase, int parity, int s, float c, const __half (&xv)[BT]) {
#pragma unroll
    for (int b = 0; b < BT; ++b)
        sts_f32(sbase + Geom<MU, BT>::kVbufOff + ((parity * BT + b) * Geom<MU, BT>::kSlots + s) * 4,
                c * __half2float(xv[b]));
}

// Tables of one unit for BT batch rows.  A thread builds the entries of one
// block of 2^lo consecutive patterns for two adjacent banks (tables) at once:
// both tables' values travel as one fp32 pair, so every Gray-code step is one
// paired add and one 64-bit store.  Item (b, block, bank pair) = thread index
// strided by the CTA size; the 16 bank pairs of a block are 16 consecutive
// threads, so a half-warp stores 128 contiguous bytes.
template <int MU, int HALF, int BT>
__device__ __forceinline__ void build_unit(uint32_t sbase, int tid) {
    using G = Geom<MU, BT>;
    constexpr int LO = G::kLo;
    constexpr int NBLK = G::kBlocks;
    constexpr int kItems = BT * NBLK * 16;
    constexpr uint64_t kSign2 = 0x8000000080000000ull;
#pragma unroll
    for (int it0 = 0; it0 < kItems; it0 += kThreads) {
        const int it = it0 + tid;
        if (kItems % kThreads != 0 && it >= kItems) break;
        const int bl = it / (NBLK * 16), hi = (it / 16) % NBLK, pj = it % 16;
        const uint32_t va = sbase + G::kVbufOff + (uint32_t)(((HALF * BT + bl) * G::kSlots + 2 * pj) * 4);
        // entry of pattern hi << lo: +v_t for the set high bits, -v_t otherwise
        uint64_t T = 0;
#pragma unroll
        for (int t = LO; t < MU; ++t) {
            const uint64_t flip = ((hi >> (t - LO)) & 1) ? 0ull : kSign2;
            const uint64_t vt = lds_b64(va + t * 128) ^ flip;
            T = t == LO ? vt : add_f32x2(T, vt);
        }
        uint64_t d[LO];
#pragma unroll
        for (int t = 0; t < LO; ++t) {
            const uint64_t vt = lds_b64(va + t * 128);
            T = sub_f32x2(T, vt);
            d[t] = add_f32x2(vt, vt);
        }
        const uint32_t base = sbase + (uint32_t)(bl * G::kPairBytes + pj * 8) + (uint32_t)(hi << LO) * 256u;
        sts_b64_at<HALF * 128>(base, T);
        static_for<1, (1 << LO)>([&](auto ic) {
            constexpr int i = decltype(ic)::value;
            constexpr int t = lowest_bit(i);
            constexpr int g = i ^ (i >> 1);
            T = ((g >> t) & 1) ? add_f32x2(T, d[t]) : sub_f32x2(T, d[t]);
            sts_b64_at<g * 256 + HALF * 128>(base, T);
        });
    }
}

template <int MU, int BT>
__device__ __forceinline__ void load_unit_slab(const KernelArgs& a, int u, int sl, int lane,
                                               uint4 (&w)[Geom<MU, BT>::kVecs]) {
    const bool br1 = u >= a.br[0].units;
    const int ul = br1 ? u - a.br[0].units : u;
    const uint4* base = br1 ? a.br[1].words : a.br[0].words;
    const int U = br1 ? a.br[1].units : a.br[0].units;
    if (sl < a.Ms) {
        const uint4* p = base + ((int64_t)sl * U + ul) * (8 * MU) + lane;
#pragma unroll
        for (int h = 0; h < Geom<MU, BT>::kVecs; ++h) w[h] = ld_stream(p + h * 32);
    } else {
#pragma unroll
        for (int h = 0; h < Geom<MU, BT>::kVecs; ++h) w[h] = make_uint4(0, 0, 0, 0);
    }
}

// Per-thread state of the activation-product pipeline: the next unit's
// products (column scale and activations loaded) and the layer data of the
// unit after it (requested, not yet consumed).
template <int BT>
struct ProductPipe {
    float c1;
    __half x1[BT];
    SlotRaw s2;
};

template <int MU, int BT>
struct WeightRegs {
    uint4 w[2][kSlabsPerWarp][Geom<MU, BT>::kVecs];
};

// Row scales of the grouped salient branch for unit u (a salient unit),
// staged for parity `par` as [kg][row of the CTA]: the KG (base, group)
// pairs of the unit each hold 512 contiguous fp16 row scales, copied 8 rows
// at a time by asynchronous 16-byte copies when M is a multiple of 8 and the
// array is 16-byte aligned (element by element otherwise).  The caller waits
// for the copies before the barrier that publishes them.
template <int MU, int NB1, int GS1>
__device__ __forceinline__ void stage_group_scales(const KernelArgs& a, int u, int rg, int tid, int par) {
    if constexpr (GS1 > 0) {
        constexpr int P = 32 / NB1, NG = P / GS1, KG = 32 / GS1;
        constexpr int kChunks = kRowsPerCta / 8;
        const int ul = u - a.br[0].units;
        const __half* r = a.br[1].r;
        const int ng = a.br[1].ngroups;
        const int row0 = rg * kRowsPerCta;
        const bool vec = (a.M % 8) == 0 && (reinterpret_cast<uintptr_t>(r) % 16) == 0;
        const uint32_t dst0 = smem_base() + Geom<MU, 1>::kScaleOff + (uint32_t)(par * KG * kRowsPerCta) * 2u;
#pragma unroll 2
        for (int e = tid; e < KG * kChunks; e += kThreads) {
            const int kg = e / kChunks, c = e % kChunks;
            const int k = kg / NG, gg = ul * NG + kg % NG;
            const int row = row0 + c * 8;
            const uint32_t dst = dst0 + (uint32_t)(kg * kRowsPerCta + c * 8) * 2u;
            const __half* src = r + ((int64_t)k * ng + gg) * a.M + row;
            if (vec && gg < ng && row + 8 <= a.M) {
                cp_async16(dst, src);
            } else {
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    const __half v = (gg < ng && row + t < a.M) ? src[t] : __float2half(0.f);
                    asm volatile("st.shared.b16 [%0], %1;" ::"r"(dst + 2u * t), "h"(*reinterpret_cast<const unsigned short*>(&v)) : "memory");
                }
            }
        }
        cp_async_commit();
    }
}

// Per-unit (block-wise) row scales of the lane's rows, kept as fp16 pairs in
// a two-entry ring by unit parity like the packed words: the scales of unit u
// are consumed at the end of its step and the entry is refilled with those of
// unit u+2.  Units whose branch has per-row scales (or grouped salient scales)
// leave the entry untouched.
struct ScaleRing {
    __half2 r[2][kSlabsPerWarp][2];
};

template <int MU, int NB0, int NB1, int GS1>
__device__ __forceinline__ void load_block_scales(const KernelArgs& a, int u, int slab0, int lane,
                                                  __half2 (&dst)[kSlabsPerWarp][2]) {
    const bool br1 = NB1 > 0 && u >= a.br[0].units;
    if (br1 && GS1 > 0) return;
    const int rgroup = br1 ? a.br[1].rgroup : a.br[0].rgroup;
    if (rgroup <= 0) return;
    const __half* r = br1 ? a.br[1].r : a.br[0].r;
    const int ng = br1 ? a.br[1].ngroups : a.br[0].ngroups;
    const int nb = br1 ? (NB1 > 0 ? NB1 : 1) : NB0;
    const int P = 32 / nb;
    const int ul = br1 ? u - a.br[0].units : u;
    const int g = (int)(((int64_t)ul * P * MU) / rgroup);
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
        __half v[4];
#pragma unroll
        for (int ai = 0; ai < 4; ++ai) {
            const int k = (ai + lane / P) % nb;
            v[ai] = (ai < nb && i < a.M) ? r[((int64_t)k * ng + g) * a.M + i] : __float2half(0.f);
        }
        dst[rs][0] = __halves2half2(v[0], v[1]);
        dst[rs][1] = __halves2half2(v[2], v[3]);
    }
}

__device__ __forceinline__ float ring_scale(const __half2 (&e)[kSlabsPerWarp][2], int rs, int ai) {
    const __half2 p = e[rs][ai / 2];
    return __half2float((ai & 1) ? __high2half(p) : __low2half(p));
}

// One unit of branch BR: build its tables, form the next unit's products and
// request the inputs two units ahead, then every slab's lookups, refilling
// each slab's registers with the unit two ahead as soon as they are consumed.
template <int MU, int BR, int NB, int HALF, int BT, int NB0, int NB1, int GS1>
__device__ __forceinline__ void unit_step(const KernelArgs& a, int u, int u_end, int ul, int b0, int rg, int slab0,
                                          int warp, int lane, int tid, uint32_t sbase, const Offsets<MU>& off,
                                          ProductPipe<BT>& pp, WeightRegs<MU, BT>& wb, ScaleRing& sr,
                                          float (&acc)[kSlabsPerWarp][BT][NB],
                                          float (&tot)[kSlabsPerWarp][BT]) {
    const BranchArgs& br = a.br[BR];
    constexpr int P = 32 / NB;
    constexpr bool kGrouped = BR == 1 && GS1 > 0;
    build_unit<MU, HALF, BT>(sbase, tid);
    if (tid < Geom<MU, BT>::kSlots && u + 1 < u_end) {
        store_products<MU, BT>(sbase, HALF ^ 1, tid, pp.c1, pp.x1);
        const SlotStatic st = resolve_slot(a, pp.s2);
        pp.c1 = st.c;
        slot_x<BT>(a, b0, st.col, pp.x1);
        if (u + 3 < u_end) pp.s2 = slot_raw<MU, NB0, NB1>(a, u + 3, tid);
    }
    if constexpr (GS1 > 0) cp_async_wait_all();  // this unit's staged salient scales
    __syncthreads();
    if constexpr (GS1 > 0) {
        // every warp is past the lookups of unit u-1, whose scale buffer this
        // reuses; the next barrier publishes it for unit u+1
        if (u + 1 < u_end && u + 1 >= a.br[0].units) stage_group_scales<MU, NB1, GS1>(a, u + 1, rg, tid, HALF ^ 1);
    }
    if constexpr (kGrouped) {
        static_assert(BT == 1, "grouped salient scales are built for one batch row per CTA");
        uint4 cur[kSlabsPerWarp][Geom<MU, BT>::kVecs];
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
#pragma unroll
            for (int h = 0; h < Geom<MU, BT>::kVecs; ++h) cur[rs][h] = wb.w[HALF][rs][h];
            if (u + 2 < u_end) load_unit_slab<MU, BT>(a, u + 2, slab0 + rs, lane, wb.w[HALF][rs]);
        }
        const uint32_t scale_row_off = Geom<MU, 1>::kScaleOff +
            (uint32_t)((HALF * (32 / GS1)) * kRowsPerCta + (slab0 % kSlabsPerCta) * kLanes + lane) * 2u;
        (void)P;
        lookup_unit_grouped<MU, NB, GS1, HALF>(cur, off, scale_row_off, lane, tot);
    } else {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            uint4 cur[Geom<MU, BT>::kVecs];
#pragma unroll
            for (int h = 0; h < Geom<MU, BT>::kVecs; ++h) cur[h] = wb.w[HALF][rs][h];
            if (u + 2 < u_end) load_unit_slab<MU, BT>(a, u + 2, slab0 + rs, lane, wb.w[HALF][rs]);
            lookup_unit<MU, NB, HALF, BT>(cur, off, acc[rs]);
        }
    }
    if (!kGrouped && br.rgroup > 0) {
        // block-wise row scales: the unit lies in one column block
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs)
#pragma unroll
            for (int ai = 0; ai < NB; ++ai)
#pragma unroll
                for (int b = 0; b < BT; ++b) {
                    tot[rs][b] = fmaf(ring_scale(sr.r[HALF], rs, ai), acc[rs][b][ai], tot[rs][b]);
                    acc[rs][b][ai] = 0.f;
                }
    }
    if (u + 2 < u_end) load_block_scales<MU, NB0, NB1, GS1>(a, u + 2, slab0, lane, sr.r[HALF]);
}

template <int MU, int BR, int NB, int BT, int NB0, int NB1, int GS1>
__device__ __forceinline__ void run_branch(const KernelArgs& a, int u_lo, int u_hi, int u_end, int& v, int b0, int rg,
                                           int slab0, int warp, int lane, int tid, uint32_t sbase,
                                           ProductPipe<BT>& pp, WeightRegs<MU, BT>& wb, ScaleRing& sr,
                                           const Offsets<MU>& off, float (&acc)[kSlabsPerWarp][BT][NB],
                                           float (&tot)[kSlabsPerWarp][BT]) {
    if (u_lo >= u_hi) return;
    const int ubase = BR ? a.br[0].units : 0;
    for (int u = u_lo; u < u_hi; ++u, ++v) {
        if (v & 1)
            unit_step<MU, BR, NB, 1, BT, NB0, NB1, GS1>(a, u, u_end, u - ubase, b0, rg, slab0, warp, lane, tid, sbase,
                                                        off, pp, wb, sr, acc, tot);
        else
            unit_step<MU, BR, NB, 0, BT, NB0, NB1, GS1>(a, u, u_end, u - ubase, b0, rg, slab0, warp, lane, tid, sbase,
                                                        off, pp, wb, sr, acc, tot);
    }
}

// Per-row scales of the lane's rows for one branch: sc[rs][a] = r_{k(a)}[row],
// kept in fp16 as loaded (converted where they are applied, after the last
// unit, so that nothing waits for these loads).
template <int NB>
__device__ __forceinline__ void fetch_row_scales(const KernelArgs& a, const BranchArgs& br, int slab0, int lane,
                                                 __half (&sc)[kSlabsPerWarp][NB]) {
    constexpr int P = 32 / NB;
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
        for (int ai = 0; ai < NB; ++ai) {
            const int k = (ai + lane / P) % NB;
            sc[rs][ai] = __float2half(0.f);
            if (i < a.M && br.rgroup == 0 && br.units > 0) sc[rs][ai] = br.r[(int64_t)k * a.M + i];
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

// Up to two CTAs per SM when one batch row is resident (their table builds
// then overlap each other's lookups); larger batch tiles run one CTA per SM
// with up to 255 registers a thread.  Large layers at batch 1 may run a
// build with three CTAs per SM (MB = 3, 80 registers a thread, a few bytes
// spilled) whose extra warps hide more of the lookup latency.
template <int BT>
constexpr int min_blocks() { return BT == 1 ? 2 : 1; }

template <int MU, int NB0, int NB1, int BT, int GS1, int MB = min_blocks<BT>()>
__global__ void __launch_bounds__(kThreads, MB) fluxbin_lut_kernel(const KernelArgs a) {
    using G = Geom<MU, BT>;
    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
    const int tid = threadIdx.x, warp = tid / kLanes, lane = tid % kLanes;
    const int ks = blockIdx.x % a.n_ks;
    const int bc = (blockIdx.x / a.n_ks) % a.n_bc;
    const int rg = blockIdx.x / (a.n_ks * a.n_bc);
    const int b0 = bc * BT;
    const int slab0 = rg * kSlabsPerCta + warp * kSlabsPerWarp;
    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);
    const int u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    const int u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);
    const uint32_t sbase = smem_base();

    // Let the next kernel on the stream start its own prologue.
    asm volatile("griddepcontrol.launch_dependents;");

    WeightRegs<MU, BT> wb;
    ScaleRing sr;
    __half sc0[kSlabsPerWarp][NB0], sc1[kSlabsPerWarp][NB1E];
    // visit offsets of the first branch (a constant table): requested before
    // the dependency wait
    Offsets<MU> off0;
    off0.template load<NB0, 0>(lane);
    SlotRaw st0{__float2half(0.f), -1}, st1 = st0, st2 = st0;
    const bool slot_owner = tid < G::kSlots;
    const bool early = (a.flags & kFlagEarlyWeights) != 0;
    auto fetch_layer = [&]() {
#pragma unroll
        for (int d = 0; d < 2; ++d)
            if (u_begin + d < u_end) {
#pragma unroll
                for (int rs = 0; rs < kSlabsPerWarp; ++rs)
                    load_unit_slab<MU, BT>(a, u_begin + d, slab0 + rs, lane, wb.w[d][rs]);
            }
        if (u_begin < u_end) load_block_scales<MU, NB0, NB1, GS1>(a, u_begin, slab0, lane, sr.r[0]);
        if (u_begin + 1 < u_end) load_block_scales<MU, NB0, NB1, GS1>(a, u_begin + 1, slab0, lane, sr.r[1]);
        fetch_row_scales<NB0>(a, a.br[0], slab0, lane, sc0);
        if constexpr (NB1 > 0) fetch_row_scales<NB1>(a, a.br[1], slab0, lane, sc1);
        if (slot_owner) {
            if (u_begin < u_end) st0 = slot_raw<MU, NB0, NB1>(a, u_begin, tid);
            if (u_begin + 1 < u_end) st1 = slot_raw<MU, NB0, NB1>(a, u_begin + 1, tid);
            if (u_begin + 2 < u_end) st2 = slot_raw<MU, NB0, NB1>(a, u_begin + 2, tid);
        }
    };
    if (early) fetch_layer();
    // Everything below may read what the preceding kernel wrote.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!early) fetch_layer();

    ProductPipe<BT> pp;
    if (slot_owner) {
        __half x0[BT];
        const SlotStatic s0 = resolve_slot(a, st0), s1 = resolve_slot(a, st1);
        slot_x<BT>(a, b0, s0.col, x0);
        slot_x<BT>(a, b0, s1.col, pp.x1);
        if (u_begin < u_end) store_products<MU, BT>(sbase, 0, tid, s0.c, x0);
        pp.c1 = s1.c;
    }
    if constexpr (GS1 > 0) {
        if (u_begin < u_end && u_begin >= U0) stage_group_scales<MU, NB1, GS1>(a, u_begin, rg, tid, 0);
        cp_async_wait_all();
    }
    if (slot_owner) {
        pp.s2 = st2;
    }
    __syncthreads();

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
    run_branch<MU, 0, NB0, BT, NB0, NB1, GS1>(a, u_begin, min(u_end, U0), u_end, v, b0, rg, slab0, warp, lane, tid,
                                              sbase, pp, wb, sr, off0, acc0, tot);
    if constexpr (NB1 > 0) {
        if (max(u_begin, U0) < u_end) {
            Offsets<MU> off1;
            off1.template load<NB1, GS1>(lane);
            run_branch<MU, 1, NB1, BT, NB0, NB1, GS1>(a, max(u_begin, U0), u_end, u_end, v, b0, rg, slab0, warp, lane,
                                                      tid, sbase, pp, wb, sr, off1, acc1, tot);
        }
    }

    // Row scales (per-row case; the block-wise case was applied per unit).
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs)
#pragma unroll
        for (int b = 0; b < BT; ++b) {
#pragma unroll
            for (int q = 0; q < NB0; ++q) tot[rs][b] = fmaf(__half2float(sc0[rs][q]), acc0[rs][b][q], tot[rs][b]);
            if constexpr (NB1 > 0) {
#pragma unroll
                for (int q = 0; q < NB1; ++q) tot[rs][b] = fmaf(__half2float(sc1[rs][q]), acc1[rs][b][q], tot[rs][b]);
            }
        }

    const int row0 = rg * kRowsPerCta;
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

    if (a.cluster) {
        // Split-K reduction inside the cluster: CTA r owns rows [r*chunk,
        // (r+1)*chunk) of the row group.  Every CTA pushes each partial to the
        // owner's shared memory, slot [b][own rank][row - r*chunk]; one cluster
        // barrier publishes the stores; each owner then sums its slots in rank
        // order from local memory (deterministic) and writes y.
        const int C = a.n_ks;
        const int rank = (int)cluster_rank();
        const int chunk = (kRowsPerCta + C - 1) / C;
        const uint32_t red = sbase + G::kRedOff;
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int lr = (warp * kSlabsPerWarp + rs) * kLanes + lane;
            const int owner = lr / chunk, j = lr % chunk;
#pragma unroll
            for (int b = 0; b < BT; ++b)
                st_dsmem_f32(red + (uint32_t)((b * C + rank) * chunk + j) * 4u, (uint32_t)owner, tot[rs][b]);
        }
        cluster_sync_all();
        for (int e = tid; e < BT * chunk; e += kThreads) {
            const int b = e / chunk, j = e % chunk, lr = rank * chunk + j;
            const int i = row0 + lr;
            if (lr >= kRowsPerCta || i >= a.M || b0 + b >= a.B) continue;
            const float* slot = &smem_at<const float>(G::kRedOff + (uint32_t)(b * C * chunk + j) * 4u);
            float s = 0.f;
#pragma unroll 16
            for (int c = 0; c < C; ++c) s += slot[c * chunk];
            store_y(a, b0 + b, i, s);
        }
        return;
    }

    // Split-K through the workspace: add this CTA's partials; the last CTA of
    // the row group to arrive finishes the sum, writes y and re-zeroes it.
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
        if (i >= a.M) continue;
#pragma unroll
        for (int b = 0; b < BT; ++b)
            if (b0 + b < a.B) red_add_f32(a.ws_acc + (int64_t)(b0 + b) * a.Mp + i, tot[rs][b]);
    }
    __syncthreads();
    __shared__ unsigned int s_last;
    unsigned int* cnt = a.ws_cnt + (rg * a.n_bc + bc);
    if (tid == 0) {
        __threadfence();   // cumulative: orders the CTA's adds (barrier above) before the count
        s_last = (atomicAdd(cnt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
        __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    // each lane finishes its own rows, all loads before the first store
    float val[kSlabsPerWarp][BT];
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
        for (int b = 0; b < BT; ++b)
            val[rs][b] = (i < a.M && b0 + b < a.B) ? __ldcg(a.ws_acc + (int64_t)(b0 + b) * a.Mp + i) : 0.f;
    }
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
        for (int b = 0; b < BT; ++b)
            if (i < a.M && b0 + b < a.B) {
                __stcg(a.ws_acc + (int64_t)(b0 + b) * a.Mp + i, 0.f);
                store_y(a, b0 + b, i, val[rs][b]);
            }
    }
    if (tid == 0) *cnt = 0u;
}

}  // namespace fluxbin
