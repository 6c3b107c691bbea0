// FluxBin LUT GEMM for batches of 2-16 on fp16-pair tables, sub-vector
// length 8, warp-specialised (sm_100a).
//
// Two batch rows share every table lookup: entry e of table (bank) b holds,
// in one 32-bit word, the fp16 partial sums of both rows (table quantisation
// to fp16, LUT Tensor Core notes, Section 3.1.3), so one shared load and one
// byte-permute address serve both rows, and the table of a unit for two rows
// takes the 32 KiB one row takes in fp32 (the LUT work per weight bit does not
// grow with the batch, FluxBin summary, Section 4).  A CTA owns 1024 rows of
// W, one pair of batch rows and a range of units, with the warp roles of the
// batch-1 kernel (fluxbin_lut1.cuh):
//
//   * builder warps form both rows' activation products v = c (.) x in fp32
//     and build each unit's tables in fp32 in Gray-code order, rounding every
//     entry pair to fp16 once (one paired convert per two entries) into a
//     stage of the two-stage ring;
//   * lookup warps fetch the entry words of two consecutive steps, add them
//     as fp16 pairs (one paired fp16 add), and add the pair's two halves into
//     the two rows' fp32 accumulators (mixed-precision adds).
//
// The stage protocol, bounded waits, error reporting and split-K reductions
// are those of the batch-1 kernel, per batch row.
//
// Shared memory (byte offsets from the start of the dynamic allocation):
//   tables  256 * 256: word of entry e, bank b, stage h at e*256 + h*128 + b*4
//           (low half: the pair's first row, high half: its second)
//   vbuf    2 * 2 * 256 floats: [h][row][bit t][bank] activation products
//   red     2 * (LW*64 + 16) floats: split-K partials, per row of the pair
//   bar     full[2], empty[2] mbarriers, then the last-arrival flag
#pragma once

#include "fluxbin_lut1.cuh"

namespace fluxbin {

template <int LW>
struct L2Geom {
    static constexpr int kBuildWarps = LW / 4;
    static constexpr int kBuildThreads = kBuildWarps * kLanes;
    static constexpr int kThreads = (LW + kBuildWarps) * kLanes;
    static constexpr int kSlabs = LW * kSlabsPerWarp;
    static constexpr int kRows = kSlabs * kLanes;
    static constexpr int kSlots = 256;
    static constexpr int kSlotsPerThread = kSlots / kBuildThreads;
    static constexpr int kVbufOff = 256 * 256;
    static constexpr int kRedOff = kVbufOff + 2 * 2 * kSlots * 4;
    static constexpr int kRedFloats = kRows + kMaxCluster;   // per row of the pair
    static constexpr int kBarOff = kRedOff + 2 * kRedFloats * 4;
    static constexpr int kSmemBytes = kBarOff + 64;
};

__device__ __forceinline__ uint32_t cvt_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ void split_f32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint32_t add_f16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// acc0 += low half of w, acc1 += high half (fp16 operands, fp32 sums)
__device__ __forceinline__ void acc_f16x2(uint32_t w, float& acc0, float& acc1) {
    unsigned short lo, hi;
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
    asm("add.rn.f32.f16 %0, %1, %0;" : "+f"(acc0) : "h"(lo));
    asm("add.rn.f32.f16 %0, %1, %0;" : "+f"(acc1) : "h"(hi));
}
template <int OFF>
__device__ __forceinline__ uint32_t table_word(uint32_t byte_off) {
    return *reinterpret_cast<const uint32_t*>(fb_smem + OFF + byte_off);
}

// Tables of one unit for both rows into stage H: item it (of 128) builds the
// 16 entries (hi << 4) .. (hi << 4) + 15 of the four banks 4 qd .. 4 qd + 3
// (qd = it % 8) for both rows; every Gray-code step is four paired fp32 adds,
// four paired converts to fp16 and one 128-bit store of four entry words.
template <int H, int NT>
__device__ __forceinline__ void l2_build_unit(uint32_t sbase, int bt) {
    constexpr int kVbuf = L2Geom<16>::kVbufOff;
    constexpr uint64_t kSign2 = 0x8000000080000000ull;
#pragma unroll
    for (int it0 = 0; it0 < 128; it0 += NT) {
        const int it = it0 + bt;
        const int hi = it / 8, qd = it % 8;
        uint64_t T[2][2], d[2][4][2];
#pragma unroll
        for (int row = 0; row < 2; ++row) {
            const uint32_t va = sbase + kVbuf + (uint32_t)(((H * 2 + row) * 256 + 4 * qd) * 4);
#pragma unroll
            for (int t = 4; t < 8; ++t) {
                const uint64_t flip = ((hi >> (t - 4)) & 1) ? 0ull : kSign2;
                uint64_t v0, v1;
                lds_v4(va + t * 128, v0, v1);
                T[row][0] = t == 4 ? (v0 ^ flip) : add_f32x2(T[row][0], v0 ^ flip);
                T[row][1] = t == 4 ? (v1 ^ flip) : add_f32x2(T[row][1], v1 ^ flip);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                uint64_t v0, v1;
                lds_v4(va + t * 128, v0, v1);
                T[row][0] = sub_f32x2(T[row][0], v0);
                T[row][1] = sub_f32x2(T[row][1], v1);
                d[row][t][0] = add_f32x2(v0, v0);
                d[row][t][1] = add_f32x2(v1, v1);
            }
        }
        const uint32_t base = sbase + (uint32_t)(qd * 16) + (uint32_t)(hi << 4) * 256u;
        auto store = [&](auto gc) {
            constexpr int g = decltype(gc)::value;
            float a[2][4];
#pragma unroll
            for (int row = 0; row < 2; ++row) {
                split_f32x2(T[row][0], a[row][0], a[row][1]);
                split_f32x2(T[row][1], a[row][2], a[row][3]);
            }
            const uint64_t lo = (uint64_t)cvt_f16x2(a[0][0], a[1][0]) | ((uint64_t)cvt_f16x2(a[0][1], a[1][1]) << 32);
            const uint64_t hw = (uint64_t)cvt_f16x2(a[0][2], a[1][2]) | ((uint64_t)cvt_f16x2(a[0][3], a[1][3]) << 32);
            sts_v4_at<g * 256 + H * 128>(base, lo, hw);
        };
        store(std::integral_constant<int, 0>{});
        static_for<1, 16>([&](auto ic) {
            constexpr int i = decltype(ic)::value;
            constexpr int t = lowest_bit(i);
            constexpr int g = i ^ (i >> 1);
#pragma unroll
            for (int row = 0; row < 2; ++row) {
                if constexpr ((g >> t) & 1) {
                    T[row][0] = add_f32x2(T[row][0], d[row][t][0]);
                    T[row][1] = add_f32x2(T[row][1], d[row][t][1]);
                } else {
                    T[row][0] = sub_f32x2(T[row][0], d[row][t][0]);
                    T[row][1] = sub_f32x2(T[row][1], d[row][t][1]);
                }
            }
            store(std::integral_constant<int, g>{});
        });
    }
}

// 32 lookup steps of one lane for one row slab and unit (stage H), both rows
// (ABS: absolute addressing as in the batch-1 kernel).
template <int NB, int H, bool ABS>
__device__ __forceinline__ void l2_lookup_unit(const uint4 (&w)[2], const Offsets<8>& off, float (&acc)[NB][2]) {
    constexpr int P = 32 / NB;
#pragma unroll
    for (int q = 0; q < 32; q += 2) {
        const uint32_t w0 = word_of(w[q / 16], (q / 4) % 4), w1 = word_of(w[(q + 1) / 16], ((q + 1) / 4) % 4);
        uint32_t e0, e1;
        if constexpr (ABS) {
            e0 = lds_u32_abs<kDynSmemBase + H * 128>(off.addr_abs(w0, q));
            e1 = lds_u32_abs<kDynSmemBase + H * 128>(off.addr_abs(w1, q + 1));
        } else {
            e0 = table_word<H * 128>(off.addr(w0, q));
            e1 = table_word<H * 128>(off.addr(w1, q + 1));
        }
        acc_f16x2(add_f16x2(e0, e1), acc[q / P][0], acc[q / P][1]);
    }
}

template <int BR, int NB, int H, bool ABS>
__device__ __forceinline__ void l2_lookup_step(const KernelArgs& a, int u, int u_end, int k, int slab0, int lane,
                                               uint32_t full_bar, uint32_t empty_bar, const Offsets<8>& off,
                                               uint4 (&wr)[2][kSlabsPerWarp][2], float (&acc)[kSlabsPerWarp][NB][2],
                                               bool& ok) {
    if (ok) ok = l1_mbar_wait(full_bar, (uint32_t)((k >> 1) & 1));
#pragma unroll
    for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
        l2_lookup_unit<NB, H, ABS>(wr[H][rs], off, acc[rs]);
        if (u + 2 < u_end) load_unit_slab<8, 1>(a, u + 2, slab0 + rs, lane, wr[H][rs]);
    }
    __syncwarp();
    if (lane == 0) l1_mbar_arrive(empty_bar);
}

template <int NB0, int NB1, int LW>
__global__ void __launch_bounds__(L2Geom<LW>::kThreads, 1) fluxbin_lut2_kernel(const KernelArgs a) {
    using G = L2Geom<LW>;
    constexpr int NB1E = NB1 > 0 ? NB1 : 1;
    const int tid = threadIdx.x, warp = tid / kLanes, lane = tid % kLanes;
    const int ks = blockIdx.x % a.n_ks;
    const int bp = (blockIdx.x / a.n_ks) % a.n_bc;   // batch pair
    const int rg = blockIdx.x / (a.n_ks * a.n_bc);
    const int b0 = 2 * bp;
    const int U0 = a.br[0].units;
    const int U = U0 + (NB1 > 0 ? a.br[1].units : 0);
    const int u_begin = (int)(((int64_t)ks * U) / a.n_ks);
    const int u_end = (int)(((int64_t)(ks + 1) * U) / a.n_ks);
    const uint32_t sbase = smem_base();
    const uint32_t full0 = sbase + G::kBarOff;
    const uint32_t empty0 = sbase + G::kBarOff + 16;
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
    float tot[kSlabsPerWarp][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const int slab0 = rg * G::kSlabs + warp * kSlabsPerWarp;

    if (warp < LW) {
        // ---------------- lookup warps ----------------
        uint4 wr[2][kSlabsPerWarp][2];
        __half sc0[kSlabsPerWarp][NB0], sc1[kSlabsPerWarp][NB1E];
        Offsets<8> off;
        off.template load<NB0, 0>(lane);
        auto fetch = [&]() {
#pragma unroll
            for (int d = 0; d < 2; ++d)
                if (u_begin + d < u_end) {
#pragma unroll
                    for (int rs = 0; rs < kSlabsPerWarp; ++rs)
                        load_unit_slab<8, 1>(a, u_begin + d, slab0 + rs, lane, wr[d][rs]);
                }
            fetch_row_scales<NB0>(a, a.br[0], slab0, lane, sc0);
            if constexpr (NB1 > 0) fetch_row_scales<NB1>(a, a.br[1], slab0, lane, sc1);
        };
        if (early) fetch();
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (!early) fetch();

        float acc0[kSlabsPerWarp][NB0][2], acc1[kSlabsPerWarp][NB1E][2];
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int q = 0; q < NB0; ++q) acc0[rs][q][r] = 0.f;
#pragma unroll
                for (int q = 0; q < NB1E; ++q) acc1[rs][q][r] = 0.f;
            }
        auto lookups = [&](auto abs_c) {
            constexpr bool ABS = decltype(abs_c)::value;
            if constexpr (ABS) off.set_rank_byte(sbase & 0xFF000000u);
            int k = 0;
            for (int u = u_begin; u < min(u_end, U0); ++u, ++k) {
                if (k & 1)
                    l2_lookup_step<0, NB0, 1, ABS>(a, u, u_end, k, slab0, lane, full0 + 8, empty0 + 8, off, wr, acc0,
                                                   ok);
                else
                    l2_lookup_step<0, NB0, 0, ABS>(a, u, u_end, k, slab0, lane, full0, empty0, off, wr, acc0, ok);
            }
            if constexpr (NB1 > 0) {
                if (max(u_begin, U0) < u_end) {
                    Offsets<8> off1;
                    off1.template load<NB1, 0>(lane);
                    if constexpr (ABS) off1.set_rank_byte(sbase & 0xFF000000u);
                    for (int u = max(u_begin, U0); u < u_end; ++u, ++k) {
                        if (k & 1)
                            l2_lookup_step<1, NB1, 1, ABS>(a, u, u_end, k, slab0, lane, full0 + 8, empty0 + 8, off1,
                                                           wr, acc1, ok);
                        else
                            l2_lookup_step<1, NB1, 0, ABS>(a, u, u_end, k, slab0, lane, full0, empty0, off1, wr,
                                                           acc1, ok);
                    }
                }
            }
        };
        if ((sbase & 0x00FFFFFFu) == kDynSmemBase)
            lookups(std::true_type{});
        else
            lookups(std::false_type{});
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int q = 0; q < NB0; ++q)
                    tot[rs][r] = fmaf(__half2float(sc0[rs][q]), acc0[rs][q][r], tot[rs][r]);
                if constexpr (NB1 > 0) {
#pragma unroll
                    for (int q = 0; q < NB1; ++q)
                        tot[rs][r] = fmaf(__half2float(sc1[rs][q]), acc1[rs][q][r], tot[rs][r]);
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
        const bool row1 = b0 + 1 < a.B;
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
        __half c_cu[SPT], x_cu[SPT][2];
        auto advance = [&]() {
#pragma unroll
            for (int i = 0; i < SPT; ++i) {
                const bool okc = col_nx[i] >= 0 && col_nx[i] < a.N;
                c_cu[i] = okc ? c_nx[i] : __float2half(0.f);
                x_cu[i][0] = okc ? a.x[(int64_t)b0 * a.N + col_nx[i]] : __float2half(0.f);
                x_cu[i][1] = (okc && row1) ? a.x[(int64_t)(b0 + 1) * a.N + col_nx[i]] : __float2half(0.f);
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
            for (int i = 0; i < SPT; ++i) {
                const float c = __half2float(c_cu[i]);
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    sts_f32(sbase + G::kVbufOff + (uint32_t)(((h * 2 + r) * G::kSlots + bt + i * NT) * 4),
                            c * __half2float(x_cu[i][r]));
            }
            if (u + 1 < u_end) {
                advance();
                if (u + 2 < u_end) request(u + 2);
            }
            l1_builder_sync<NT>();
            if (h)
                l2_build_unit<1, NT>(sbase, bt);
            else
                l2_build_unit<0, NT>(sbase, bt);
            __syncwarp();
            if (lane == 0) l1_mbar_arrive(full0 + 8u * h);
        }
    }

    if (!ok) {
        atomicOr(a.err, 4u);
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) tot[rs][0] = tot[rs][1] = __int_as_float(0x7fc00000);
    }
    const bool lookup_warp = warp < LW;
    const int row0 = rg * G::kRows;
    if (a.n_ks == 1) {
        if (lookup_warp) {
#pragma unroll
            for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
                const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    if (i < a.M && b0 + r < a.B) store_y(a, b0 + r, i, tot[rs][r]);
            }
        }
        return;
    }
    if (a.cluster) {
        const int C = a.n_ks;
        const int rank = (int)cluster_rank();
        const int chunk = (G::kRows + C - 1) / C;
        const uint32_t red = sbase + G::kRedOff;
        if (lookup_warp) {
#pragma unroll
            for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
                const int lr = (warp * kSlabsPerWarp + rs) * kLanes + lane;
                const int owner = lr / chunk, j = lr % chunk;
#pragma unroll
                for (int r = 0; r < 2; ++r)
                    st_dsmem_f32(red + (uint32_t)(r * G::kRedFloats + rank * chunk + j) * 4u, (uint32_t)owner,
                                 tot[rs][r]);
            }
        }
        cluster_sync_all();
        for (int e = tid; e < 2 * chunk; e += G::kThreads) {
            const int r = e / chunk, j = e % chunk;
            const int lr = rank * chunk + j;
            const int i = row0 + lr;
            if (lr >= G::kRows || i >= a.M || b0 + r >= a.B) continue;
            const float* slot = &smem_at<const float>(G::kRedOff + (uint32_t)(r * G::kRedFloats + j) * 4u);
            float s = 0.f;
#pragma unroll 16
            for (int c = 0; c < C; ++c) s += slot[c * chunk];
            store_y(a, b0 + r, i, s);
        }
        return;
    }
    if (lookup_warp) {
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
            for (int r = 0; r < 2; ++r)
                if (i < a.M && b0 + r < a.B) red_add_f32(a.ws_acc + (int64_t)(b0 + r) * a.Mp + i, tot[rs][r]);
        }
    }
    __syncthreads();
    unsigned int* cnt = a.ws_cnt + (rg * a.n_bc + bp);
    uint32_t& s_last = smem_at<uint32_t>(G::kBarOff + 32);
    if (tid == 0) {
        __threadfence();   // cumulative: orders the CTA's adds (barrier above) before the count
        s_last = (atomicAdd(cnt, 1u) == (unsigned)(a.n_ks - 1)) ? 1u : 0u;
        __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    // each lookup lane finishes its own rows, all loads before the first store
    if (lookup_warp) {
        float val[kSlabsPerWarp][2];
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
            for (int r = 0; r < 2; ++r)
                val[rs][r] = (i < a.M && b0 + r < a.B) ? __ldcg(a.ws_acc + (int64_t)(b0 + r) * a.Mp + i) : 0.f;
        }
#pragma unroll
        for (int rs = 0; rs < kSlabsPerWarp; ++rs) {
            const int i = (slab0 + rs) * kLanes + lane;
#pragma unroll
            for (int r = 0; r < 2; ++r)
                if (i < a.M && b0 + r < a.B) {
                    __stcg(a.ws_acc + (int64_t)(b0 + r) * a.Mp + i, 0.f);
                    store_y(a, b0 + r, i, val[rs][r]);
                }
        }
    }
    if (tid == 0) *cnt = 0u;
}

}  // namespace fluxbin
