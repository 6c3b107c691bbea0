// FluxBin LUT GEMV for one activation row (batch 1), sub-vector length 8,
// on precomputed tables (sm_100a).
//
// The tables of every unit are built once per call by fluxbin_tables_kernel
// (the precompute as a separate operator, LUT Tensor Core notes, Section
// 3.1.1) into a global table buffer that stays in L2.  This kernel only looks
// them up (FluxBin summary, Section 3 "LUT-Based GEMV Kernel"; Appendix C.1):
//
//   * the tables of a unit pair (64 KiB, the shared-memory layout itself)
//     come from the table buffer into one of two shared-memory regions by a
//     1-D bulk copy that completes on the region's "full" mbarrier; one lane
//     of the last warp issues the copies, refilling a region once every warp
//     has released it on its "empty" mbarrier;
//   * LW warps, each owning SPW row slabs of 32 rows, stream their
//     rows' packed words with 128-bit loads two units ahead into registers
//     and run the 32 lookup-accumulate steps per slab and unit (a
//     byte-permute forms the entry address, a shared load fetches it, pairs of
//     entries are added by one paired fp32 add).
//
// No thread of this kernel builds a table or forms an activation product, so
// the lookup warps' issue slots go to lookups; the table bytes cross shared
// memory once per CTA and unit, as they would if built there.  A CTA owns
// LW*SPW*32 rows (2048 for LW = 16, SPW = 4).  Every wait is bounded; a wait
// that gives up sets bit 2 of the device error word and the CTA's outputs
// become NaN, and the producer waits for the copies it issued before the
// CTA exits.
//
// Shared memory (byte offsets from the start of the dynamic allocation):
//   region r (0, 1)  65536 bytes at r * 65536: entry e of the tables of the
//                    pair's unit h at e*256 + h*128 + bank*4
//   red              rows + 16 floats: split-K partials pushed by the cluster
//   bar              full[2], empty[2] mbarriers, then the last-arrival flag
#pragma once

#include "fluxbin_lut1.cuh"
#include "fluxbin_tables.cuh"

namespace fluxbin {

template <int LW, int SPW>
struct L1hGeom {
    static constexpr int kThreads = LW * kLanes;
    static constexpr int kSlabs = LW * SPW;
    static constexpr int kRows = kSlabs * kLanes;
    static constexpr int kRegionBytes = kTabPairBytes;
    static constexpr int kRedOff = 2 * kRegionBytes;
    static constexpr int kRedFloats = kRows + kMaxCluster;
    static constexpr int kBarOff = kRedOff + kRedFloats * 4;
    static constexpr int kSmemBytes = kBarOff + 64;
};

__device__ __forceinline__ void l1h_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void l1h_bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// 32 lookup-accumulate steps of one lane for one row slab and unit whose
// tables sit at byte offset OFF of the dynamic shared memory.
template <int NB, int OFF>
__device__ __forceinline__ void l1h_lookup_unit(const uint4 (&w)[2], const Offsets<8>& off, float (&acc)[NB]) {
    constexpr int P = 32 / NB;
    uint64_t pair[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) pair[i] = 0ull;
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        const uint32_t a0 = off.addr(word_of(w[q / 16], (q / 4) % 4), q);
        const uint32_t a1 = off.addr(word_of(w[(q + 1) / 16], ((q + 1) / 4) % 4), q + 1);
        const float f0 = table_entry<OFF>(a0);
        const float f1 = table_entry<OFF>(a1);
        pair[q / P] = add_f32x2(pair[q / P], pack_f32x2(f0, f1));
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) acc[i] += sum_f32x2(pair[i]);
}

// The lookups of one unit pair in region R: unit 2v + h for h = 0, 1 when it
// lies in [u_begin, u_end); weights of unit u + 2 requested as soon as unit u
// is consumed.
template <int NB0, int NB1, int SPW, int R>
__device__ __forceinline__ void l1h_pair(const KernelArgs& a, int v, int u_begin, int u_end, int U0, int slab0,
                                         int lane, Offsets<8>& off, bool& off_is_sal,
                                         uint4 (&wr)[2][SPW][2], float (&acc0)[SPW][NB0],
                                         float (&acc1)[SPW][NB1 > 0 ? NB1 : 1]) {
    static_for<0, 2>([&](auto hc) {
        constexpr int h = decltype(hc)::value;
        const int u = 2 * v + h;
        if (u >= u_begin && u < u_end) {
            if (NB1 > 0 && u >= U0) {
                if constexpr (NB1 > 0) {
                    if (!off_is_sal) {
                        off.template load<NB1, 0>(lane);
                        off_is_sal = true;
                    }
#pragma unroll
                    for (int rs = 0; rs < SPW; ++rs) {
                        l1h_lookup_unit<NB1, R * kTabPairBytes + h * 128>(wr[h][rs], off, acc1[rs]);
                        if (u + 2 < u_end) load_unit_slab<8, 1>(a, u + 2, slab0 + rs, lane, wr[h][rs]);
                    }
                }
            } else {
#pragma unroll
                for (int rs = 0; rs < SPW; ++rs) {
                    l1h_lookup_unit<NB0, R * kTabPairBytes + h * 128>(wr[h][rs], off, acc0[rs]);
                    if (u + 2 < u_end) load_unit_slab<8, 1>(a, u + 2, slab0 + rs, lane, wr[h][rs]);
                }
            }
        }
    });
}

template <int NB0, int NB1, int LW, int SPW>
__global__ void __launch_bounds__(L1hGeom<LW, SPW>::kThreads, 1)
    fluxbin_lut1h_kernel(const KernelArgs a, const float* tables) {
    using G = L1hGeom<LW, SPW>;
    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
    const int tid = threadIdx.x, warp = tid / kLanes, lane = tid % kLanes;
    const int ks = blockIdx.x % a.n_ks;
    const int rg = blockIdx.x / a.n_ks;
    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);
    const int u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    const int u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);
    const int v_begin = u_begin / 2, v_end = (u_end + 1) / 2;   // unit pairs touched: [v_begin, v_end)
    const uint32_t sbase = smem_base();
    const uint32_t full0 = sbase + G::kBarOff;        // region r: full0 + 8r
    const uint32_t empty0 = sbase + G::kBarOff + 16;  // region r: empty0 + 8r
    const bool early = (a.flags & kFlagEarlyWeights) != 0;

    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        l1_mbar_init(full0, 1);
        l1_mbar_init(full0 + 8, 1);
        l1_mbar_init(empty0, LW);
        l1_mbar_init(empty0 + 8, LW);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    bool ok = true;
    float tot[SPW];
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) tot[rs] = 0.f;
    const int slab0 = rg * G::kSlabs + warp * SPW;
    const bool producer = warp == LW - 1 && lane == 0;   // issues the table copies
    uint32_t issued[2] = {0u, 0u};
    auto copy_pair = [&](int v, int r) {
        l1h_expect_tx(full0 + 8u * r, (uint32_t)kTabPairBytes);
        l1h_bulk_copy(sbase + (uint32_t)(r * kTabPairBytes), tables + (int64_t)v * (kTabPairBytes / 4),
                      (uint32_t)kTabPairBytes, full0 + 8u * r);
        issued[r] += 1;
    };

    uint4 wr[2][SPW][2];
    Offsets<8> off;
    bool off_is_sal = NB1 > 0 && u_begin >= U0;
    if (off_is_sal) {
        if constexpr (NB1 > 0) off.template load<NB1, 0>(lane);
    } else {
        off.template load<NB0, 0>(lane);
    }
    auto fetch = [&]() {
        // unit u goes to ring entry u % 2 (register indices stay compile-time)
        static_for<0, 2>([&](auto ec) {
            constexpr int e = decltype(ec)::value;
            const int u = u_begin + ((u_begin & 1) ^ e);   // the unit of [u_begin, u_begin + 2) with u % 2 == e
            if (u < u_end) {
#pragma unroll
                for (int rs = 0; rs < SPW; ++rs) load_unit_slab<8, 1>(a, u, slab0 + rs, lane, wr[e][rs]);
            }
        });
    };
    if (early) fetch();
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the tables are the preceding kernel's output
    if (!early) fetch();
    if (producer) {
        if (v_begin < v_end) copy_pair(v_begin, 0);
        if (v_begin + 1 < v_end) copy_pair(v_begin + 1, 1);
    }

    float acc0[SPW][NB0], acc1[SPW][NB1E];
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
#pragma unroll
        for (int q = 0; q < NB0; ++q) acc0[rs][q] = 0.f;
#pragma unroll
        for (int q = 0; q < NB1E; ++q) acc1[rs][q] = 0.f;
    }
    // row scales of the lane's rows, requested with the last unit pair and
    // kept as loaded until they are applied
    __half sc0[SPW][NB0], sc1[SPW][NB1E];
    auto fetch_scales = [&]() {
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int row = (slab0 + rs) * kLanes + lane;
#pragma unroll
            for (int q = 0; q < NB0; ++q) {
                const int k = (q + lane / (32 / NB0)) % NB0;
                sc0[rs][q] = row < a.M ? a.br[0].r[(int64_t)k * a.M + row] : __float2half(0.f);
            }
#pragma unroll
            for (int q = 0; q < NB1E; ++q) {
                const int k = (q + lane / (32 / NB1E)) % NB1E;
                sc1[rs][q] = (NB1 > 0 && row < a.M && a.br[1].units > 0) ? a.br[1].r[(int64_t)k * a.M + row]
                                                                        : __float2half(0.f);
            }
        }
    };
    if (v_begin >= v_end) fetch_scales();
    int i = 0;
    for (int v = v_begin; v < v_end; ++v, ++i) {
        const int r = i & 1;
        if (v + 1 == v_end) fetch_scales();
        if (ok) ok = l1_mbar_wait(full0 + 8u * r, (uint32_t)((i >> 1) & 1));
        if (r)
            l1h_pair<NB0, NB1, SPW, 1>(a, v, u_begin, u_end, U0, slab0, lane, off, off_is_sal, wr, acc0, acc1);
        else
            l1h_pair<NB0, NB1, SPW, 0>(a, v, u_begin, u_end, U0, slab0, lane, off, off_is_sal, wr, acc0, acc1);
        __syncwarp();
        if (lane == 0) l1_mbar_arrive(empty0 + 8u * r);
        if (producer && v + 2 < v_end) {
            // refill region r with pair v + 2 once every warp has released it
            if (ok) ok = l1_mbar_wait(empty0 + 8u * r, (uint32_t)((i >> 1) & 1));
            if (ok) copy_pair(v + 2, r);
        }
        __syncwarp();
    }
    // every copy issued has landed before the CTA may exit
    if (producer) {
        for (int rr = 0; rr < 2; ++rr)
            if (issued[rr] > 0) (void)l1_mbar_wait(full0 + 8u * rr, (issued[rr] - 1) & 1);
    }
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
#pragma unroll
        for (int q = 0; q < NB0; ++q) tot[rs] = fmaf(__half2float(sc0[rs][q]), acc0[rs][q], tot[rs]);
        if constexpr (NB1 > 0) {
#pragma unroll
            for (int q = 0; q < NB1; ++q) tot[rs] = fmaf(__half2float(sc1[rs][q]), acc1[rs][q], tot[rs]);
        }
    }

    if (!ok) {
        atomicOr(a.err, 4u);
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) tot[rs] = __int_as_float(0x7fc00000);
    }
    const int row0 = rg * G::kRows;
    if (a.n_ks == 1) {
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int row = (slab0 + rs) * kLanes + lane;
            if (row < a.M) store_y(a, 0, row, tot[rs]);
        }
        return;
    }
    if (a.cluster) {
        // Split-K reduction inside the cluster (see fluxbin_lut1.cuh).
        const int C = a.n_ks;
        const int rank = (int)cluster_rank();
        const int chunk = (G::kRows + C - 1) / C;
        const uint32_t red = sbase + G::kRedOff;
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int lr = (warp * SPW + rs) * kLanes + lane;
            const int owner = lr / chunk, j = lr % chunk;
            st_dsmem_f32(red + (uint32_t)(rank * chunk + j) * 4u, (uint32_t)owner, tot[rs]);
        }
        cluster_sync_all();
        for (int j = tid; j < chunk; j += G::kThreads) {
            const int lr = rank * chunk + j;
            const int i = row0 + lr;
            if (lr >= G::kRows || i >= a.M) continue;
            const float* slot = &smem_at<const float>(G::kRedOff + (uint32_t)j * 4u);
            float s = 0.f;
#pragma unroll 16
            for (int c = 0; c < C; ++c) s += slot[c * chunk];
            store_y(a, 0, i, s);
        }
        return;
    }
    // Split-K through the workspace: add this CTA's partials; the last CTA of
    // the row group to arrive finishes the sum, writes y and re-zeroes it.
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
        const int row = (slab0 + rs) * kLanes + lane;
        if (row < a.M) red_add_f32(a.ws_acc + row, tot[rs]);
    }
    __syncthreads();
    unsigned int* cnt = a.ws_cnt + rg;
    uint32_t& s_last = smem_at<uint32_t>(G::kBarOff + 32);
    if (tid == 0) {
        __threadfence();   // cumulative: orders the CTA's adds (barrier above) before the count
        s_last = (atomicAdd(cnt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
        __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    // each lane finishes its own rows, all loads before the first store
    float val[SPW];
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
        const int row = (slab0 + rs) * kLanes + lane;
        val[rs] = row < a.M ? __ldcg(a.ws_acc + row) : 0.f;
    }
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
        const int row = (slab0 + rs) * kLanes + lane;
        if (row < a.M) {
            __stcg(a.ws_acc + row, 0.f);
            store_y(a, 0, row, val[rs]);
        }
    }
    if (tid == 0) *cnt = 0u;
}

}  // namespace fluxbin
