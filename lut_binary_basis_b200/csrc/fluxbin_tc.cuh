// FluxBin layer on the fifth-generation tensor cores (sm_100a), for batches
// large enough that the LUT path stops being a table lookup and becomes a
// dense contraction (the pages' LUT kernels degrade as the batch grows;
// LUT-TC §2.2 reads LUT mpGEMM as a GEMM whose one operand is 1-bit).
//
//   y[b][i] (+)= sum_k r_k[i] * sum_n B_k[i][n] * v_k[b][n],   v_k = c_k (.) x
//
// The +-1 signs of every base are expanded to fp16 (exactly +-1) in shared
// memory only, unit by unit, and contracted with the fp16 activation products
// v_k by tcgen05.mma (M = 128 rows, N = 16 batch rows, K = 16), one fp32
// accumulator per base in tensor memory; the row scales are applied to the
// accumulators in the epilogue.  No floating-point weight matrix exists
// anywhere: the signs stream from HBM in the same packed layout the LUT path
// reads (include/fluxbin.h, "Packed sign layout"), and a unit's expanded
// tile lives in shared memory only while its MMAs run.
//
// Work: items (128-row tile, range of units) are spread over a persistent
// grid of one CTA per SM.  Per unit the 16 worker warps of a CTA (four
// threads per row)
//   1. wait until the MMAs that last read the unit's buffer have finished,
//   2. expand their rows' packed bytes into the A buffer and form the unit's
//      fp16 products v into the B buffer, then signal the buffer full;
// and a seventeenth warp waits for the buffer, issues the unit's 16 MMAs and
// commits them to the buffer's "empty" mbarrier (two buffers: the tensor
// cores work on unit u while the workers prepare unit u+1).
// Partial sums of items that split the units of a tile are added into the
// fp32 workspace; the last item of a tile to arrive writes y.
//
// Shared memory (dynamic, byte offsets):
//   A    2 x 64 KiB, K-major with the 128-byte swizzle: per buffer, base k,
//        64-column block a = j/8 and 8-row group g, one 1 KiB atom at
//        ((k*P/8 + a)*16 + g) KiB; row r%8 of the group at +128*(r%8); the
//        16-byte chunk of sub-vector j at +16*((j%8) xor (r%8))
//   B    2 x 8 KiB, the same for the 16 batch rows (2 row groups per block)
//   lut  128 B: the four fp16 +-1 values of every 4-bit sign pattern (one
//        8-byte entry per bank pair, so 32 lanes never conflict)
//   bar  per buffer a "full" mbarrier (the 16 worker warps have prepared a
//        unit) and an "empty" one (its MMAs have finished), then the
//        tensor-memory address and the issuer's drain flag
//
// Every mbarrier wait is bounded (spin_limit polls).  A wait that gives up
// sets bit 0 of the device error word and the affected outputs become NaN;
// the issuing thread then still waits (with the full limit) for the last
// commit it made on each buffer, and the tensor memory is freed only once
// those MMAs are known to have finished (bit 1 of the error word when not).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "fluxbin_kernel.cuh"

namespace fluxbin {

constexpr int kTcRows = 128;
constexpr int kTcThreads = 512;            // four threads per row: each expands a quarter of the row's bytes
constexpr int kTcN = 16;                   // batch rows per MMA (padded with zeros)
constexpr int kTcTmemCols = 128;           // up to 8 accumulators of 16 fp32 columns
constexpr int kTcABytes = 32 * kTcRows * 16;   // one buffer: 32 (base, sub-vector) x 128 rows x 16 B
constexpr int kTcBBytes = 32 * kTcN * 16;
constexpr int kTcAOff = 0;
constexpr int kTcBOff = 2 * kTcABytes;
constexpr int kTcLutOff = kTcBOff + 2 * kTcBBytes;   // 16 x 8 B: fp16 +-1 of the 4 bits of a nibble
constexpr int kTcBarOff = kTcLutOff + 128;
constexpr int kTcSmemBytes = kTcBarOff + 48;
constexpr uint32_t kTcSpinLimit = 1u << 26;   // mbarrier polls before a wait is declared failed
constexpr uint32_t kTcTestSpinLimit = 64u;    // the same under the wait-timeout test hook

struct TcArgs {
    BranchArgs br[2];       // 0: global, 1: salient (units == 0 when absent); per-row scales only
    const __half* x;        // [B][N]
    void* y;                // [B][M]
    int32_t M, N, B;
    int32_t Ms;             // row slabs of 32
    int32_t Mp;             // Ms * 32 (workspace row pitch)
    int32_t n_rt;           // 128-row tiles
    int32_t n_ks;           // unit ranges per tile
    int32_t n_items;        // n_rt * n_ks
    uint32_t flags;
    float* ws_acc;          // [B][Mp], zero between calls
    unsigned int* ws_cnt;   // [n_rt], zero between calls
    unsigned int* err;      // bit 0: a wait gave up; bit 1: tensor memory kept (MMAs not drained)
    int32_t vec_x;          // 1: x rows and the global column scales allow 16-byte loads (N % 8 == 0, aligned)
    uint32_t spin_limit;    // mbarrier polls before a wait gives up
    int32_t test_stall;     // test hook: the workers never signal a buffer full
};

// ---------------------------------------------------------------------------
// tcgen05 / mbarrier primitives (PTX ISA 8.6+, sm_100a)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tc_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Polls the mbarrier until the phase with the given parity has completed;
// false when the poll limit is reached.
__device__ __forceinline__ bool tc_mbar_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done) : "r"(bar), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: start
// address, leading byte offset 1 (unused by swizzled K-major layouts), stride
// byte offset 1024 (between 8-row atoms), descriptor version 1, layout
// SWIZZLE_128B.  Atoms are 1024-byte aligned (base offset 0).
__device__ __forceinline__ uint64_t tc_smem_desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major,
// N = 16, M = 128.
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcN >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

// A unit's K axis concatenates its bases: sub-vector j of base k covers
// K = (k*P + j)*MU .. +MU-1.  Byte offset of element block (k, j) of row r in
// an operand buffer with `groups` 8-row groups per 64-column atom: atom
// ck/8, 16-byte chunk ck%8 (xor-swizzled with r%8), ck = (k*P + j)*MU/8, and
// for MU = 4 the half (k*P + j)%2 of that chunk.
template <int MU, int NB>
__device__ __forceinline__ uint32_t sw128_block(int k, int j, int r, int groups) {
    constexpr int P = 32 / NB;
    const int kj = k * P + j;
    const int ck = MU == 8 ? kj : (kj >> 1);
    const int half = MU == 8 ? 0 : (kj & 1);
    return (uint32_t)((((ck >> 3) * groups + (r >> 3)) << 10) + ((r & 7) << 7) + (((ck & 7) ^ (r & 7)) << 4) +
                      (half << 3));
}

// The MMAs of one unit (nb bases x P*MU/16 K steps of 16; 16 for MU = 8, 8
// for MU = 4): the descriptors of the unit's A and B buffers are built once;
// each MMA adds its operands' offsets (in 16-byte units) to the start-address
// field.  Accumulator k of the branch lives at TMEM column (acc0 + k) * 16.
template <int MU, int NB>
__device__ __forceinline__ void tc_issue_unit(uint32_t tmem, int acc0, uint32_t abuf, uint32_t bbuf, bool first) {
    constexpr int P = 32 / NB;
    const uint64_t da = tc_smem_desc_sw128(abuf);
    const uint64_t db = tc_smem_desc_sw128(bbuf);
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        const uint32_t d = tmem + (uint32_t)((acc0 + k) * kTcN);
#pragma unroll
        for (int s = 0; s < P * MU / 16; ++s) {
            // K step s starts at chunk ck0 = (k*P*MU + 16 s)/8: atom ck0/8, then
            // 16 bytes per chunk inside it (offsets in 16-byte units)
            const int ck0 = (k * P * MU) / 8 + 2 * s;
            const uint64_t a_off = (uint64_t)((ck0 >> 3) * (kTcRows / 8) * 64 + (ck0 & 7));
            const uint64_t b_off = (uint64_t)((ck0 >> 3) * (kTcN / 8) * 64 + (ck0 & 7));
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                ::"r"(d), "l"(da + a_off), "l"(db + b_off), "r"(kTcIdesc), "r"((first && s == 0) ? 0u : 1u));
        }
    }
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 4 fp32 columns of this warp's 32 TMEM lanes (a warp reaches the lane
// quarter warp % 4).
__device__ __forceinline__ void tc_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Entry n of the nibble table: fp16 +1 for a set bit, -1 for a clear one,
// bit t of n in fp16 slot t.
__device__ __forceinline__ uint2 nibble_signs(uint32_t n) {
    uint32_t w[2];
#pragma unroll
    for (int i = 0; i < 2; ++i)
        w[i] = (((n >> (2 * i)) & 1u) ? 0x3C00u : 0xBC00u) | ((((n >> (2 * i + 1)) & 1u) ? 0x3C00u : 0xBC00u) << 16);
    return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------------------
// Per-unit preparation
// ---------------------------------------------------------------------------

// Branch-dependent fields of unit u, selected field by field.
struct TcUnit {
    const uint4* words;
    const __half* c;
    const int32_t* gather;
    int ncols, U, ul, nb, br;
};
template <int NB0, int NB1>
__device__ __forceinline__ TcUnit tc_unit(const TcArgs& a, int u) {
    const bool br1 = NB1 > 0 && u >= a.br[0].units;
    TcUnit t;
    t.br = br1 ? 1 : 0;
    t.words = br1 ? a.br[1].words : a.br[0].words;
    t.c = br1 ? a.br[1].c : a.br[0].c;
    t.gather = br1 ? a.br[1].gather : a.br[0].gather;
    t.ncols = br1 ? a.br[1].ncols : a.br[0].ncols;
    t.U = br1 ? a.br[1].units : a.br[0].units;
    t.ul = br1 ? u - a.br[0].units : u;
    t.nb = br1 ? (NB1 > 0 ? NB1 : 1) : NB0;
    return t;
}

__device__ __forceinline__ uint2 ld_stream64(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Bytes 8*quarter .. 8*quarter+7 of row `slab*32 + lane` in unit u (zeros
// past the last slab): half (quarter % 2) of the lane's (quarter / 2)-th
// 128-bit word of the unit's chunk.
__device__ __forceinline__ uint32_t ld_stream32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// MU = 8: bytes 8*quarter .. +7 of row `slab*32 + lane` in unit u (half
// quarter%2 of the lane's (quarter/2)-th 128-bit word of the unit's chunk);
// MU = 4: word `quarter` of the lane's one 128-bit word.  Zeros past the last
// slab.
template <int MU, int NB0, int NB1>
__device__ __forceinline__ void tc_load_words(const TcArgs& a, int u, int slab, int lane, int quarter, uint2& w) {
    const TcUnit t = tc_unit<NB0, NB1>(a, u);
    const uint4* chunk = t.words + ((int64_t)slab * t.U + t.ul) * (8 * MU);
    if (slab >= a.Ms) {
        w = make_uint2(0, 0);
    } else if (MU == 8) {
        w = ld_stream64(reinterpret_cast<const char*>(chunk + (quarter >> 1) * 32 + lane) + 8 * (quarter & 1));
    } else {
        w = make_uint2(ld_stream32(reinterpret_cast<const char*>(chunk + lane) + 4 * quarter), 0u);
    }
}

// Writes the fp16 +-1 expansion of a quarter of one row's sign bytes (steps
// 8*quarter .. 8*quarter+7, held in w) into the A buffer: step q of lane L is
// sub-vector j = (L+q) mod P of base k = (q/P + L/P) mod nb (diagonal visit
// order).  At iteration it the lane takes the step whose chunk lands in
// swizzled slot (it + L) mod 8, so the 8 rows of an atom store to 8 distinct
// bank groups.
template <int MU, int NB>
__device__ __forceinline__ void tc_expand_quarter(uint32_t abuf, uint32_t lut, int row, int lane, int quarter,
                                                  const uint2& w) {
    constexpr int P = 32 / NB;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        if constexpr (MU == 8) {
            const int qq = ((((it + lane) & 7) ^ (lane & 7)) - lane) & 7;
            const int q = 8 * quarter + qq;
            const uint32_t p = (qq < 4 ? w.x : w.y) >> (8 * (qq & 3));
            const int k = ((q / P) + (lane / P)) % NB;
            const int j = (lane + q) & (P - 1);
            const uint2 lo = lds64(lut + ((p << 3) & 0x78u));
            const uint2 hi = lds64(lut + ((p >> 1) & 0x78u));
            sts128(abuf + sw128_block<MU, NB>(k, j, row, kTcRows / 8), lo.x, lo.y, hi.x, hi.y);
        } else {
            const int q = 8 * quarter + it;
            const uint32_t p = w.x >> (4 * it);
            const int k = ((q / P) + (lane / P)) % NB;
            const int j = (lane + q) & (P - 1);
            const uint2 v = lds64(lut + ((p << 3) & 0x78u));
            asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(abuf + sw128_block<MU, NB>(k, j, row, kTcRows / 8)),
                         "r"(v.x), "r"(v.y) : "memory");
        }
    }
}

// Operands of the fp16 products v_k[b][n] = c_k[n] * x[b][col(n)] of one
// unit, requested a step or two before they are used: thread t forms the 8
// columns of (base, sub-vector) kj = t/16 for batch row t%16, so that
// consecutive lanes store consecutive 16-byte slots.  A unit of
// the global branch reads 16-byte slices (of c and of the batch row of x)
// when vec_x allows; otherwise, and for the gathered salient branch, element
// by element.
struct TcProd {
    uint4 c;          // 8 fp16 column scales (zero past the branch's columns)
    uint4 x;          // 8 fp16 activations of the batch row
};

template <int MU, int NB0, int NB1>
__device__ __forceinline__ void tc_prod_load(const TcArgs& a, int u, int tid, TcProd& o) {
    const TcUnit t = tc_unit<NB0, NB1>(a, u);
    const int P = 32 / t.nb;
    const int b = tid & 15;
    if ((tid >> 4) >= 4 * MU) return;   // the unit has 4*MU chunks of 8 columns
    {
        // chunk tid/16 of the unit's K axis: base k, columns n0 .. n0+7 of the branch
        const int kk0 = (tid >> 4) * 8, k = kk0 / (P * MU);
        const int n0 = t.ul * P * MU + kk0 % (P * MU);
        if (!t.br && !t.gather && a.vec_x && n0 + 8 <= t.ncols) {
            o.c = __ldg(reinterpret_cast<const uint4*>(t.c + (int64_t)k * t.ncols + n0));
            o.x = b < a.B ? __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)b * a.N + n0))
                          : make_uint4(0, 0, 0, 0);
            return;
        }
        uint32_t c[4] = {0u, 0u, 0u, 0u}, x[4] = {0u, 0u, 0u, 0u};
        const unsigned short* cs = reinterpret_cast<const unsigned short*>(t.c);
        const unsigned short* xs = reinterpret_cast<const unsigned short*>(a.x);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int n = n0 + i;
            int cc = n < t.ncols ? (t.gather ? __ldg(t.gather + n) : n) : -1;
            if (cc >= a.N) cc = -1;
            const uint32_t sh = 16u * (i & 1);
            if (cc >= 0) {
                c[i / 2] |= (uint32_t)cs[(int64_t)k * t.ncols + n] << sh;
                if (b < a.B) x[i / 2] |= (uint32_t)xs[(int64_t)b * a.N + cc] << sh;
            }
        }
        o.c = make_uint4(c[0], c[1], c[2], c[3]);
        o.x = make_uint4(x[0], x[1], x[2], x[3]);
    }
}

__device__ __forceinline__ uint32_t mul_h2(uint32_t c, uint32_t x) {
    const float2 cf = __half22float2(*reinterpret_cast<const __half2*>(&c));
    const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&x));
    const __half2 hv = __floats2half2_rn(cf.x * xf.x, cf.y * xf.y);
    return *reinterpret_cast<const uint32_t*>(&hv);
}

template <int MU, int NB>
__device__ __forceinline__ void tc_prod_store(const TcProd& o, int tid, uint32_t bbuf) {
    constexpr int P = 32 / NB;
    const int b = tid & 15, ck = tid >> 4;
    if (ck >= 4 * MU) return;
    // chunk ck holds 8 consecutive K of the unit: block (k, j) with (k*P + j)*MU = 8*ck
    const int kj = ck * 8 / MU;
    sts128(bbuf + sw128_block<MU, NB>(kj / P, kj % P, b, kTcN / 8), mul_h2(o.c.x, o.x.x), mul_h2(o.c.y, o.x.y),
           mul_h2(o.c.z, o.x.z), mul_h2(o.c.w, o.x.w));
}

__device__ __forceinline__ void tc_store_y(const TcArgs& a, int b, int i, float v) {
    const int64_t o = (int64_t)b * a.M + i;
    if (a.flags & kFlagYFp32) {
        float* y = static_cast<float*>(a.y);
        y[o] = (a.flags & kFlagAccumulate) ? y[o] + v : v;
    } else {
        __half* y = static_cast<__half*>(a.y);
        y[o] = __float2half_rn((a.flags & kFlagAccumulate) ? __half2float(y[o]) + v : v);
    }
}

// ---------------------------------------------------------------------------
// Kernel
// ---------------------------------------------------------------------------

// Worker-only barrier (the issuer warp does not take part).
__device__ __forceinline__ void tc_worker_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kTcThreads) : "memory");
}

__device__ __forceinline__ void tc_mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Item bounds, shared by the workers and the issuer.
struct TcItem {
    int rt, u_begin, u_end;
};
__device__ __forceinline__ TcItem tc_item(const TcArgs& a, int item, int U) {
    TcItem it;
    it.rt = item / a.n_ks;
    const int ks = item % a.n_ks;
    it.u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    it.u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);
    return it;
}

template <int MU, int NB0, int NB1>
__global__ void __launch_bounds__(kTcThreads + 32, 1) fluxbin_tc_kernel(const TcArgs a) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sb = smem_base();
    const uint32_t full0 = sb + kTcBarOff;        // buffer b holds a prepared unit: full0 + 8*b
    const uint32_t empty0 = sb + kTcBarOff + 16;  // buffer b's MMAs have finished: empty0 + 8*b
    const uint32_t tslot = sb + kTcBarOff + 32;
    constexpr int kWorkerWarps = kTcThreads / 32;

    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tslot),
                     "r"(kTcTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid < 16) {
        const uint2 e = nibble_signs((uint32_t)tid);
        asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(sb + kTcLutOff + 8u * tid), "r"(e.x), "r"(e.y)
                     : "memory");
    }
    if (tid == 0) {
        tc_mbar_init(full0, kWorkerWarps);
        tc_mbar_init(full0 + 8, kWorkerWarps);
        tc_mbar_init(empty0, 1);
        tc_mbar_init(empty0 + 8, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = smem_at<const uint32_t>(kTcBarOff + 32);
    // the swizzled operand atoms need 1024-byte alignment (the dynamic shared
    // memory is declared so); anything else is reported, never computed on
    bool ok = (sb & 1023u) == 0;

    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);

    if (warp == kWorkerWarps) {
        // ---- issuer: one thread issues every unit's MMAs in order ----
        if (lane == 0) {
            uint32_t fills0 = 0u, fills1 = 0u;   // completed fills of each buffer seen so far
            uint32_t issued0 = 0u, issued1 = 0u; // commits issued on each buffer
            int g = 0;
            for (int item = blockIdx.x; item < a.n_items && ok; item += gridDim.x) {
                const TcItem it = tc_item(a, item, U);
                bool first0 = true, first1 = true;
                for (int u = it.u_begin; u < it.u_end && ok; ++u, ++g) {
                    const int bf = g & 1;
                    const bool br1 = NB1 > 0 && u >= U0;
                    const uint32_t f = bf ? fills1 : fills0;
                    ok = tc_mbar_wait(full0 + 8u * bf, f & 1, a.spin_limit);
                    if (bf) fills1 += 1;
                    else fills0 += 1;
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t abuf = sb + kTcAOff + (uint32_t)bf * kTcABytes;
                    const uint32_t bbuf = sb + kTcBOff + (uint32_t)bf * kTcBBytes;
                    if (NB1 > 0 && br1) {
                        constexpr int NB1E = NB1 > 0 ? NB1 : 1;
                        tc_issue_unit<MU, NB1E>(tmem, NB0, abuf, bbuf, first1);
                        first1 = false;
                    } else {
                        tc_issue_unit<MU, NB0>(tmem, 0, abuf, bbuf, first0);
                        first0 = false;
                    }
                    tc_commit(empty0 + 8u * bf);
                    if (bf) issued1 += 1;
                    else issued0 += 1;
                }
            }
            if (!ok) atomicOr(a.err, 1u);
            // Every MMA this thread issued must have finished before the
            // accumulators are released, whatever happened to the waits above:
            // wait (bounded, with the full limit) for the last commit on each
            // buffer.  Only a tensor core that stopped answering leaves this
            // undrained; the tensor memory is then kept rather than freed
            // under running MMAs.
            bool drained = true;
            if (issued0 > 0) drained = tc_mbar_wait(empty0, (issued0 - 1) & 1, kTcSpinLimit) && drained;
            if (issued1 > 0) drained = tc_mbar_wait(empty0 + 8, (issued1 - 1) & 1, kTcSpinLimit) && drained;
            smem_at<uint32_t>(kTcBarOff + 36) = drained ? 1u : 0u;
        }
        __syncwarp();
    } else {
        // ---- workers: 16 warps, four threads per row ----
        uint32_t commits0 = 0u, commits1 = 0u;   // commits made on each buffer so far
        int g = 0;                               // units processed by this CTA (buffer = g & 1)
        bool waited = false;
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            const TcItem it = tc_item(a, item, U);
            const int rt = it.rt, u_begin = it.u_begin, u_end = it.u_end;
            const int quarter = warp >> 2;          // which 8 bytes of the row this thread expands
            const int slab = rt * (kTcRows / kLanes) + (warp & 3);
            const int row = (warp & 3) * kLanes + lane;   // row within the tile
            const int grow = rt * kTcRows + row;

            uint2 wq[2];                         // this thread's 8 packed bytes of units u and u+1 (ring by parity)
            const bool early = (a.flags & kFlagEarlyWeights) != 0 || waited;
            if (early) {
                if (u_begin < u_end) tc_load_words<MU, NB0, NB1>(a, u_begin, slab, lane, quarter, wq[0]);
                if (u_begin + 1 < u_end) tc_load_words<MU, NB0, NB1>(a, u_begin + 1, slab, lane, quarter, wq[1]);
            }
            if (!waited) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
            }
            if (!early) {
                if (u_begin < u_end) tc_load_words<MU, NB0, NB1>(a, u_begin, slab, lane, quarter, wq[0]);
                if (u_begin + 1 < u_end) tc_load_words<MU, NB0, NB1>(a, u_begin + 1, slab, lane, quarter, wq[1]);
            }
            TcProd pq[2];                        // product operands of units u and u+1 (ring by parity)
            if (u_begin < u_end) tc_prod_load<MU, NB0, NB1>(a, u_begin, tid, pq[0]);
            if (u_begin + 1 < u_end) tc_prod_load<MU, NB0, NB1>(a, u_begin + 1, tid, pq[1]);
            // per-row scales of this thread's row
            float rsc[2][4];
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int nb = q ? NB1 : NB0;
                    rsc[q][k] = (k < nb && grow < a.M && a.br[q].units > 0)
                                    ? __half2float(a.br[q].r[(int64_t)k * a.M + grow]) : 0.f;
                }

            for (int u = u_begin; u < u_end; ++u, ++g) {
                const int bf = g & 1;
                const int par = (u - u_begin) & 1;
                const bool br1 = NB1 > 0 && u >= U0;
                const uint32_t cb = bf ? commits1 : commits0;
                if (cb > 0 && ok) ok = tc_mbar_wait(empty0 + 8u * bf, (cb - 1) & 1, a.spin_limit);
                const uint32_t abuf = sb + kTcAOff + (uint32_t)bf * kTcABytes;
                const uint32_t bbuf = sb + kTcBOff + (uint32_t)bf * kTcBBytes;
                const uint2 cur = par ? wq[1] : wq[0];
                const TcProd pc = par ? pq[1] : pq[0];
                if (u + 2 < u_end) {
                    if (par) {
                        tc_load_words<MU, NB0, NB1>(a, u + 2, slab, lane, quarter, wq[1]);
                        tc_prod_load<MU, NB0, NB1>(a, u + 2, tid, pq[1]);
                    } else {
                        tc_load_words<MU, NB0, NB1>(a, u + 2, slab, lane, quarter, wq[0]);
                        tc_prod_load<MU, NB0, NB1>(a, u + 2, tid, pq[0]);
                    }
                }
                if (NB1 > 0 && br1) {
                    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
                    tc_prod_store<MU, NB1E>(pc, tid, bbuf);
                    tc_expand_quarter<MU, NB1E>(abuf, sb + kTcLutOff, row, lane, quarter, cur);
                } else {
                    tc_prod_store<MU, NB0>(pc, tid, bbuf);
                    tc_expand_quarter<MU, NB0>(abuf, sb + kTcLutOff, row, lane, quarter, cur);
                }
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && !a.test_stall) tc_mbar_arrive(full0 + 8u * bf);
                if (bf) commits1 += 1;
                else commits0 += 1;
            }

            // epilogue: this thread's row, batch rows 4*quarter .. 4*quarter+3
            float part[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) part[b] = 0.f;
            if (u_end > u_begin) {
                const int lb = (g - 1) & 1;
                const uint32_t cl = lb ? commits1 : commits0;
                if (ok) ok = tc_mbar_wait(empty0 + 8u * lb, (cl - 1) & 1, a.spin_limit);
                tc_fence_after();
                const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * kLanes) << 16) + (uint32_t)(4 * quarter);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const bool used = q == 0 ? (u_begin < U0) : (NB1 > 0 && u_end > U0);
                    if (!used) continue;
                    const int nb = q ? NB1 : NB0;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (k >= nb) continue;
                        float d[4];
                        tc_ld4(lane_base + (uint32_t)(((q ? NB0 : 0) + k) * kTcN), d);
                        tc_wait_ld();
#pragma unroll
                        for (int b = 0; b < 4; ++b) part[b] = fmaf(rsc[q][k], d[b], part[b]);
                    }
                }
                tc_fence_before();
            }
            if (!ok) {
#pragma unroll
                for (int b = 0; b < 4; ++b) part[b] = __int_as_float(0x7fc00000);
            }
            const int bb = 4 * quarter;
            if (a.n_ks == 1) {
                if (grow < a.M) {
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (bb + b < a.B) tc_store_y(a, bb + b, grow, part[b]);
                }
            } else {
                if (grow < a.M) {
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        if (bb + b < a.B) red_add_f32(a.ws_acc + (int64_t)(bb + b) * a.Mp + grow, part[b]);
                }
                __threadfence();
                tc_worker_sync();
                __shared__ unsigned int s_last_tc;
                if (tid == 0) s_last_tc = (atomicAdd(a.ws_cnt + rt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
                tc_worker_sync();
                if (s_last_tc) {
                    __threadfence();
                    if (grow < a.M)
                        for (int b = bb; b < bb + 4 && b < a.B; ++b) {
                            float* p = a.ws_acc + (int64_t)b * a.Mp + grow;
                            const float val = __ldcg(p);
                            __stcg(p, 0.f);
                            tc_store_y(a, b, grow, val);
                        }
                    if (tid == 0) a.ws_cnt[rt] = 0u;
                }
                tc_worker_sync();   // s_last_tc is rewritten by the next item
            }
        }
        if (!ok && tid == 0) atomicOr(a.err, 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        // the issuer's drain result (written before the barrier above)
        if (smem_at<const uint32_t>(kTcBarOff + 36) != 0u) {
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols)
                         : "memory");
        } else if (lane == 0) {
            atomicOr(a.err, 2u);
        }
    }
}

}  // namespace fluxbin
