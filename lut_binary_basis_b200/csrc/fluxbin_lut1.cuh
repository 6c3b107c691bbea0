// FluxBin LUT GEMV for one activation row (batch 1), sub-vector length 8,
// warp-specialised (sm_100a).
//
// Computes y (+)= W x for one layer with per-row scales, like
// fluxbin_lut_kernel (FluxBin summary, Section 3 "LUT-Based GEMV Kernel" and
// "Virtual Columnar Mapping"; Appendix C.1), with the work of a CTA divided
// between two kinds of warps instead of every warp doing everything:
//
//   * builder warps (LW/4 of them) form each unit's activation products
//     v = c (.) x (the salient branch gathering x through its column map) and
//     build the unit's 32 tables of 2^8 signed partial sums into one stage of
//     a two-stage table ring in shared memory (Gray-code order, two paired
//     fp32 adds and one 128-bit store per four entries);
//   * lookup warps (LW of them, two row slabs of 32 rows each) stream their
//     rows' packed words with 128-bit loads two units ahead into registers and
//     run the 32 lookup-accumulate steps per slab and unit: one byte-permute
//     forms the entry address, one shared load fetches it, pairs of entries
//     are added by one paired fp32 add.
//
// The two kinds meet only at per-stage mbarriers: a stage is "full" when the
// builder warps have published its tables, "empty" when every lookup warp is
// done with it.  No CTA-wide barrier sits in the unit loop, so a slow lookup
// warp delays the builders by at most one stage and never the other lookup
// warps.  A CTA owns LW*64 rows (1024 for LW = 16): every table build is
// shared by twice the rows of the two-CTAs-per-SM kernel, which halves the
// shared-memory stores per lookup.  Every wait is bounded; a wait that gives
// up sets bit 2 of the device error word and the CTA's outputs become NaN
// (nothing asynchronous is in flight in this kernel, so it can then return).
//
// Shared memory (byte offsets from the start of the dynamic allocation):
//   tables  256 * 256: entry e of the tables of stage h at e*256 + h*128 + bank*4
//   vbuf    2 * 256 floats: [h][bit t][bank] activation products of a unit
//   red     LW*64 + 16 floats: split-K partials pushed by the cluster's CTAs
//   bar     full[2], empty[2] mbarriers, then the last-arrival flag
#pragma once

#include "fluxbin_kernel.cuh"

namespace fluxbin {

template <int LW, int SPW = kSlabsPerWarp>
struct L1Geom {
    static constexpr int kLookupWarps = LW;
    static constexpr int kBuildWarps = LW / 4;
    static constexpr int kBuildThreads = kBuildWarps * kLanes;
    static constexpr int kThreads = (LW + kBuildWarps) * kLanes;
    static constexpr int kSlabs = LW * SPW;
    static constexpr int kRows = kSlabs * kLanes;
    static constexpr int kSlots = 256;                          // products per unit (32 tables x 8 bits)
    static constexpr int kSlotsPerThread = kSlots / kBuildThreads;
    static constexpr int kVbufOff = 256 * 256;
    static constexpr int kRedOff = kVbufOff + 2 * kSlots * 4;
    static constexpr int kRedFloats = kRows + kMaxCluster;
    static constexpr int kBarOff = kRedOff + kRedFloats * 4;
    static constexpr int kSmemBytes = kBarOff + 64;
};

constexpr uint32_t kL1SpinLimit = 1u << 24;   // mbarrier polls before a wait gives up

__device__ __forceinline__ void l1_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void l1_mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Waits for the phase of the given parity to complete; false when the poll
// limit is reached.
__device__ __forceinline__ bool l1_mbar_wait(uint32_t bar, uint32_t parity) {
    for (uint32_t it = 0; it < kL1SpinLimit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done) : "r"(bar), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}
template <int NT>
__device__ __forceinline__ void l1_builder_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

__device__ __forceinline__ void lds_v4(uint32_t addr, uint64_t& lo, uint64_t& hi) {
    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(lo), "=l"(hi) : "r"(addr));
}
template <int OFF>
__device__ __forceinline__ void sts_v4_at(uint32_t addr, uint64_t lo, uint64_t hi) {
    asm volatile("st.shared.v2.b64 [%0+%1], {%2, %3};" ::"r"(addr), "n"(OFF), "l"(lo), "l"(hi) : "memory");
}

// Tables of one unit into stage H: item it (of 128) builds the 16 entries
// (hi << 4) .. (hi << 4) + 15 of the four tables in banks 4 qd .. 4 qd + 3
// (qd = it % 8), the four tables' values travelling as two fp32 pairs: every
// Gray-code step is two paired adds and one 128-bit store.  A warp's store
// covers four 128-byte runs of distinct entry rows (four wavefronts, no
// conflict).
template <int H, int NT>
__device__ __forceinline__ void l1_build_unit(uint32_t sbase, int bt) {
    constexpr int kVbuf = L1Geom<16>::kVbufOff;
    constexpr uint64_t kSign2 = 0x8000000080000000ull;
#pragma unroll
    for (int it0 = 0; it0 < 128; it0 += NT) {
        const int it = it0 + bt;
        const int hi = it / 8, qd = it % 8;
        const uint32_t va = sbase + kVbuf + (uint32_t)((H * 256 + 4 * qd) * 4);
        uint64_t T0 = 0, T1 = 0;
#pragma unroll
        for (int t = 4; t < 8; ++t) {
            const uint64_t flip = ((hi >> (t - 4)) & 1) ? 0ull : kSign2;
            uint64_t v0, v1;
            lds_v4(va + t * 128, v0, v1);
            T0 = t == 4 ? (v0 ^ flip) : add_f32x2(T0, v0 ^ flip);
            T1 = t == 4 ? (v1 ^ flip) : add_f32x2(T1, v1 ^ flip);
        }
        uint64_t d0[4], d1[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint64_t v0, v1;
            lds_v4(va + t * 128, v0, v1);
            T0 = sub_f32x2(T0, v0);
            T1 = sub_f32x2(T1, v1);
            d0[t] = add_f32x2(v0, v0);
            d1[t] = add_f32x2(v1, v1);
        }
        const uint32_t base = sbase + (uint32_t)(qd * 16) + (uint32_t)(hi << 4) * 256u;
        sts_v4_at<H * 128>(base, T0, T1);
        static_for<1, 16>([&](auto ic) {
            constexpr int i = decltype(ic)::value;
            constexpr int t = lowest_bit(i);
            constexpr int g = i ^ (i >> 1);
            if constexpr ((g >> t) & 1) {
                T0 = add_f32x2(T0, d0[t]);
                T1 = add_f32x2(T1, d1[t]);
            } else {
                T0 = sub_f32x2(T0, d0[t]);
                T1 = sub_f32x2(T1, d1[t]);
            }
            sts_v4_at<g * 256 + H * 128>(base, T0, T1);
        });
    }
}

// Per-thread geometry of the builder's product slots: slot s is bit t = s/32
// of bank cb = s%32, i.e. column j*8 + t of base k = cb/P, sub-vector
// j = cb%P of every unit of a branch with P sub-vectors per base.  Fixed for
// the whole launch: per unit only the unit's column offset changes.
template <int SPT>
struct L1Slots {
    int32_t noff[2][SPT];           // column of the slot inside a unit, per branch
    const __half* cptr[2][SPT];     // the slot's base row of the column scales, per branch
};

// 32 lookup-accumulate steps of one lane for one row slab and unit (stage H).
// ABS: the permute forms the absolute shared address and the base rides in
// the load's immediate (one instruction less per lookup); otherwise the
// table offset is added to the shared array's address.
template <int NB, int H, bool ABS>
__device__ __forceinline__ void l1_lookup_unit(const uint4 (&w)[2], const Offsets<8>& off, float (&acc)[NB]) {
    constexpr int P = 32 / NB;
    uint64_t pair[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) pair[i] = 0ull;
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        const uint32_t w0 = word_of(w[q / 16], (q / 4) % 4), w1 = word_of(w[(q + 1) / 16], ((q + 1) / 4) % 4);
        float f0, f1;
        if constexpr (ABS) {
            f0 = lds_f32_abs<kDynSmemBase + H * 128>(off.addr_abs(w0, q));
            f1 = lds_f32_abs<kDynSmemBase + H * 128>(off.addr_abs(w1, q + 1));
        } else {
            f0 = table_entry<H * 128>(off.addr(w0, q));
            f1 = table_entry<H * 128>(off.addr(w1, q + 1));
        }
        pair[q / P] = add_f32x2(pair[q / P], pack_f32x2(f0, f1));
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) acc[i] += sum_f32x2(pair[i]);
}

// Lookup warps: one unit of branch BR in stage H (the k-th unit of the CTA).
// The packed words travel in a ring of D register sets per slab: a slab's
// words for unit u + D are requested as soon as its unit-u lookups are done.
template <int BR, int NB, int H, bool ABS, int SPW, int D>
__device__ __forceinline__ void l1_lookup_step(const KernelArgs& a, int u, int u_end, int k, int slab0, int lane,
                                               uint32_t full_bar, uint32_t empty_bar, const Offsets<8>& off,
                                               uint4 (&wr)[D][SPW][2], float (&acc)[SPW][NB], bool& ok) {
    constexpr int RS = D == 2 ? H : 0;
    if (ok) ok = l1_mbar_wait(full_bar, (uint32_t)((k >> 1) & 1));
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) {
        l1_lookup_unit<NB, H, ABS>(wr[RS][rs], off, acc[rs]);
        if (u + D < u_end) load_unit_slab<8, 1>(a, u + D, slab0 + rs, lane, wr[RS][rs]);
    }
    __syncwarp();
    if (lane == 0) l1_mbar_arrive(empty_bar);
}

template <int NB0, int NB1, int LW, int SPW>
__global__ void __launch_bounds__(L1Geom<LW, SPW>::kThreads, LW == 16 ? 1 : 2)
    fluxbin_lut1_kernel(const KernelArgs a) {
    using G = L1Geom<LW, SPW>;
    constexpr int D = SPW >= 4 ? 1 : 2;   // units of packed words held ahead per slab
    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
    const int tid = threadIdx.x, warp = tid / kLanes, lane = tid % kLanes;
    const int ks = blockIdx.x % a.n_ks;
    const int rg = blockIdx.x / a.n_ks;
    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);
    const int u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    const int u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);
    const uint32_t sbase = smem_base();
    const uint32_t full0 = sbase + G::kBarOff;       // stage h: full0 + 8h
    const uint32_t empty0 = sbase + G::kBarOff + 16; // stage h: empty0 + 8h
    const bool early = (a.flags & kFlagEarlyWeights) != 0;

    asm volatile("griddepcontrol.launch_dependents;");
    if (tid == 0) {
        l1_mbar_init(full0, G::kBuildWarps);
        l1_mbar_init(full0 + 8, G::kBuildWarps);
        l1_mbar_init(empty0, LW);
        l1_mbar_init(empty0 + 8, LW);
    }
    __syncthreads();

    bool ok = true;
    float tot[SPW];
#pragma unroll
    for (int rs = 0; rs < SPW; ++rs) tot[rs] = 0.f;
    const int slab0 = rg * G::kSlabs + warp * SPW;

    if (warp < LW) {
        // ---------------- lookup warps ----------------
        uint4 wr[D][SPW][2];
        __half sc0[SPW][NB0], sc1[SPW][NB1E];
        Offsets<8> off;
        off.template load<NB0, 0>(lane);
        // Row scales of the lane's rows (kept as loaded, converted where
        // applied): requested before the wait with D = 2, with the last unit
        // otherwise (registers are tight with four slabs per warp).
        auto fetch_scales = [&]() {
#pragma unroll
            for (int rs = 0; rs < SPW; ++rs) {
                const int row = (slab0 + rs) * kLanes + lane;
#pragma unroll
                for (int q = 0; q < NB0; ++q) {
                    const int kb = (q + lane / (32 / NB0)) % NB0;
                    sc0[rs][q] = row < a.M ? a.br[0].r[(int64_t)kb * a.M + row] : __float2half(0.f);
                }
#pragma unroll
                for (int q = 0; q < NB1E; ++q) {
                    const int kb = (q + lane / (32 / NB1E)) % NB1E;
                    sc1[rs][q] = (NB1 > 0 && row < a.M && a.br[1].units > 0) ? a.br[1].r[(int64_t)kb * a.M + row]
                                                                            : __float2half(0.f);
                }
            }
        };
        auto fetch = [&]() {
#pragma unroll
            for (int d = 0; d < D; ++d)
                if (u_begin + d < u_end) {
#pragma unroll
                    for (int rs = 0; rs < SPW; ++rs)
                        load_unit_slab<8, 1>(a, u_begin + d, slab0 + rs, lane, wr[d][rs]);
                }
            if (D == 2 || u_end - u_begin <= 1) fetch_scales();
        };
        if (early) fetch();
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (!early) fetch();

        float acc0[SPW][NB0], acc1[SPW][NB1E];
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
#pragma unroll
            for (int q = 0; q < NB0; ++q) acc0[rs][q] = 0.f;
#pragma unroll
            for (int q = 0; q < NB1E; ++q) acc1[rs][q] = 0.f;
        }
        auto lookups = [&](auto abs_c) {
            constexpr bool ABS = decltype(abs_c)::value;
            if constexpr (ABS) off.set_rank_byte(sbase & 0xFF000000u);
            int k = 0;
            for (int u = u_begin; u < min(u_end, U0); ++u, ++k) {
                if (D == 1 && u + 1 == u_end && u > u_begin) fetch_scales();
                if (k & 1)
                    l1_lookup_step<0, NB0, 1, ABS, SPW, D>(a, u, u_end, k, slab0, lane, full0 + 8, empty0 + 8, off,
                                                           wr, acc0, ok);
                else
                    l1_lookup_step<0, NB0, 0, ABS, SPW, D>(a, u, u_end, k, slab0, lane, full0, empty0, off, wr, acc0,
                                                           ok);
            }
            if constexpr (NB1 > 0) {
                if (max(u_begin, U0) < u_end) {
                    Offsets<8> off1;
                    off1.template load<NB1, 0>(lane);
                    if constexpr (ABS) off1.set_rank_byte(sbase & 0xFF000000u);
                    for (int u = max(u_begin, U0); u < u_end; ++u, ++k) {
                        if (D == 1 && u + 1 == u_end && u > u_begin) fetch_scales();
                        if (k & 1)
                            l1_lookup_step<1, NB1, 1, ABS, SPW, D>(a, u, u_end, k, slab0, lane, full0 + 8, empty0 + 8,
                                                                   off1, wr, acc1, ok);
                        else
                            l1_lookup_step<1, NB1, 0, ABS, SPW, D>(a, u, u_end, k, slab0, lane, full0, empty0, off1,
                                                                   wr, acc1, ok);
                    }
                }
            }
        };
        if ((sbase & 0x00FFFFFFu) == kDynSmemBase)
            lookups(std::true_type{});
        else
            lookups(std::false_type{});
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
#pragma unroll
            for (int q = 0; q < NB0; ++q) tot[rs] = fmaf(__half2float(sc0[rs][q]), acc0[rs][q], tot[rs]);
            if constexpr (NB1 > 0) {
#pragma unroll
                for (int q = 0; q < NB1; ++q) tot[rs] = fmaf(__half2float(sc1[rs][q]), acc1[rs][q], tot[rs]);
            }
        }
    } else {
        // ---------------- builder warps ----------------
        constexpr int SPT = G::kSlotsPerThread;
        constexpr int NT = G::kBuildThreads;
        constexpr int P0 = 32 / NB0, P1 = 32 / NB1E;
        const int bt = tid - LW * kLanes;
        L1Slots<SPT> sl;
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
            const int sidx = bt + i * NT, cb = sidx % 32, t = sidx / 32;
            sl.noff[0][i] = (cb % P0) * 8 + t;
            sl.cptr[0][i] = a.br[0].c + (int64_t)(cb / P0) * a.br[0].ncols;
            sl.noff[1][i] = (cb % P1) * 8 + t;
            sl.cptr[1][i] = NB1 > 0 ? a.br[1].c + (int64_t)(cb / P1) * a.br[1].ncols : a.br[0].c;
        }
        // Layer data of the slots for unit u2 (column scale as loaded, activation
        // column or -1): requested two units before use.
        __half c_nx[SPT];
        int col_nx[SPT];
        auto request = [&](int u2) {
            const bool b1 = NB1 > 0 && u2 >= U0;
            const int ul = b1 ? u2 - U0 : u2;
            const int ncols = b1 ? a.br[1].ncols : a.br[0].ncols;
            const int32_t* gp = b1 ? a.br[1].gather : a.br[0].gather;
            const int n0 = ul * (b1 ? P1 * 8 : P0 * 8);
#pragma unroll
            for (int i = 0; i < SPT; ++i) {
                const int n = n0 + (b1 ? sl.noff[1][i] : sl.noff[0][i]);
                c_nx[i] = __float2half(0.f);
                col_nx[i] = -1;
                if (n < ncols) {
                    c_nx[i] = (b1 ? sl.cptr[1][i] : sl.cptr[0][i])[n];
                    col_nx[i] = gp ? __ldg(gp + n) : n;
                }
            }
        };
        // Operands of the next unit: column scale and activation (zero for
        // padding and for a column outside [0, N)).
        __half c_cu[SPT], x_cu[SPT];
        auto advance = [&]() {
#pragma unroll
            for (int i = 0; i < SPT; ++i) {
                const bool okc = col_nx[i] >= 0 && col_nx[i] < a.N;
                c_cu[i] = okc ? c_nx[i] : __float2half(0.f);
                x_cu[i] = okc ? a.x[col_nx[i]] : __float2half(0.f);
            }
        };
        if (early && u_begin < u_end) request(u_begin);
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (!early && u_begin < u_end) request(u_begin);
        advance();
        if (u_begin + 1 < u_end) request(u_begin + 1);
        int k = 0;
        for (int u = u_begin; u < u_end; ++u, ++k) {
            const int h = k & 1;
            if (k >= 2 && ok) ok = l1_mbar_wait(empty0 + 8u * h, (uint32_t)(((k >> 1) - 1) & 1));
#pragma unroll
            for (int i = 0; i < SPT; ++i)
                sts_f32(sbase + G::kVbufOff + (uint32_t)((h * G::kSlots + bt + i * NT) * 4),
                        __half2float(c_cu[i]) * __half2float(x_cu[i]));
            if (u + 1 < u_end) {
                advance();
                if (u + 2 < u_end) request(u + 2);
            }
            l1_builder_sync<NT>();
            if (h)
                l1_build_unit<1, NT>(sbase, bt);
            else
                l1_build_unit<0, NT>(sbase, bt);
            __syncwarp();
            if (lane == 0) l1_mbar_arrive(full0 + 8u * h);
        }
    }

    if (!ok) {
        atomicOr(a.err, 4u);
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) tot[rs] = __int_as_float(0x7fc00000);
    }
    const bool lookup_warp = warp < LW;
    const int row0 = rg * G::kRows;
    if (a.n_ks == 1) {
        if (lookup_warp) {
#pragma unroll
            for (int rs = 0; rs < SPW; ++rs) {
                const int i = (slab0 + rs) * kLanes + lane;
                if (i < a.M) store_y(a, 0, i, tot[rs]);
            }
        }
        return;
    }
    if (a.cluster) {
        // Split-K reduction inside the cluster: CTA r owns rows [r*chunk,
        // (r+1)*chunk) of the row group; every CTA pushes its partials to the
        // owner's shared memory, one cluster barrier publishes them, the owner
        // sums its C slots in rank order (deterministic) and writes y.
        const int C = a.n_ks;
        const int rank = (int)cluster_rank();
        const int chunk = (G::kRows + C - 1) / C;
        const uint32_t red = sbase + G::kRedOff;
        if (lookup_warp) {
#pragma unroll
            for (int rs = 0; rs < SPW; ++rs) {
                const int lr = (warp * SPW + rs) * kLanes + lane;
                const int owner = lr / chunk, j = lr % chunk;
                st_dsmem_f32(red + (uint32_t)(rank * chunk + j) * 4u, (uint32_t)owner, tot[rs]);
            }
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
    // The CTA barrier orders every thread's adds before thread 0's fence and
    // counter increment (the fence is cumulative), so one fence per CTA
    // publishes them.
    if (lookup_warp) {
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
            if (i < a.M) red_add_f32(a.ws_acc + i, tot[rs]);
        }
    }
    __syncthreads();
    unsigned int* cnt = a.ws_cnt + rg;
    uint32_t& s_last = smem_at<uint32_t>(G::kBarOff + 32);
    if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(cnt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
        __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    // Each lookup lane finishes its own rows: every load is issued before the
    // first store, so the sums take one round trip.
    if (lookup_warp) {
        float val[SPW];
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
            val[rs] = i < a.M ? __ldcg(a.ws_acc + i) : 0.f;
        }
#pragma unroll
        for (int rs = 0; rs < SPW; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
            if (i < a.M) {
                __stcg(a.ws_acc + i, 0.f);
                store_y(a, 0, i, val[rs]);
            }
        }
    }
    if (tid == 0) *cnt = 0u;
}

}  // namespace fluxbin
