// FluxBin table precompute as a separate operator (sm_100a).
//
// The LUT Tensor Core notes (Section 3.1.1) move the table precompute out of
// the lookup kernel into an operator of its own, run once and read by every
// lookup unit, instead of rebuilding the same tables in every CTA that needs
// them.  This kernel builds, for one layer and one activation row, every
// unit's 32 tables of 2^8 signed partial sums of v = c (.) x (scale fusion,
// FluxBin summary, Section 3 "LUT-Based GEMV Kernel"; the salient branch
// gathers x and its column scales through its column map, Section 3 "Virtual
// Columnar Mapping") into a global table buffer that the batch-1 lookup
// kernel (fluxbin_lut1h.cuh) copies into shared memory with bulk copies.
//
// Table buffer layout (fp32): units are paired, v = u / 2, h = u % 2; entry e
// of table (bank) b of unit u at byte
//     v * 65536 + e * 256 + h * 128 + b * 4,
// which is exactly the shared-memory layout the lookups address (one 64 KiB
// copy per unit pair).  The bank of table (base k, sub-vector j) is k*P + j.
//
// One CTA of 256 threads builds one unit: the 256 activation products (one
// per thread) go to shared memory, then thread t builds the 8 entries
// (hi << 4) | (half << 3) | 0..7 of the four tables in banks 4 qd .. 4 qd + 3
// (t/2 = 8 hi + qd, half = t % 2) in Gray-code order (two paired fp32 adds
// and one 16-byte store per step).
//
// NORM: the precompute fused with the element-wise operator that precedes
// the layer (LUT Tensor Core notes, Section 3.1.1, fusion of the precompute
// into the preceding operator), taken to be the RMS normalisation of a
// LLaMA-style block: the kernel reads the un-normalised activation h and
// forms x = h (.) gamma / sqrt(mean(h^2) + eps) itself (in fp32, never
// rounded to fp16 on the way to the tables).  Every CTA sums h^2 over the
// whole row in the same order, so all of them use the same 1/rms; CTA v also
// writes its slice of x (rounded to fp16) when asked to.
#pragma once

#include "fluxbin_kernel.cuh"

namespace fluxbin {

constexpr int kTabThreads = 256;
constexpr int kTabPairBytes = 65536;

__device__ __forceinline__ void stg_v4(float* p, uint64_t lo, uint64_t hi) {
    asm volatile("st.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(lo), "l"(hi) : "memory");
}

template <int NB0, int NB1, bool NORM>
__global__ void __launch_bounds__(kTabThreads) fluxbin_tables_kernel(const KernelArgs a, float* tables,
                                                                      const NormArgs nrm) {
    __shared__ __align__(16) float vbuf[8][32];   // [bit t][bank]
    __shared__ float wsum[kTabThreads / 32];
    const int tid = threadIdx.x;
    const int u = blockIdx.x;              // one unit per CTA
    const int v = u >> 1, h = u & 1;       // its pair and half in the table buffer
    asm volatile("griddepcontrol.launch_dependents;");
    // layer data of this thread's product slot (before the dependency wait)
    const SlotRaw raw = slot_raw<8, NB0, NB1>(a, u, tid);
    // x was written by the preceding kernel; the table buffer may still be
    // read by it
    asm volatile("griddepcontrol.wait;" ::: "memory");
    float r_inv = 1.f;
    if constexpr (NORM) {
        // 1/rms of the whole row: per-thread strided sums, then the warps'
        // sums in warp order (the same order in every CTA)
        float ss = 0.f;
        if ((a.N & 7) == 0 && (reinterpret_cast<uintptr_t>(a.x) & 15) == 0) {
            // 16-byte loads of 8 entries
            const uint4* h8 = reinterpret_cast<const uint4*>(a.x);
            for (int n = tid; n < a.N / 8; n += kTabThreads) {
                const uint4 w = __ldg(h8 + n);
                const uint32_t qw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&qw[e]));
                    ss = fmaf(f.x, f.x, ss);
                    ss = fmaf(f.y, f.y, ss);
                }
            }
        } else {
            for (int n = tid; n < a.N; n += kTabThreads) {
                const float hv = __half2float(a.x[n]);
                ss = fmaf(hv, hv, ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (tid % 32 == 0) wsum[tid / 32] = ss;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kTabThreads / 32; ++w) tot += wsum[w];
        r_inv = rsqrtf(tot / (float)a.N + nrm.eps);
        if (nrm.x_out) {
            const int chunk = (a.N + (int)gridDim.x - 1) / (int)gridDim.x;
            const int n1 = min(a.N, (u + 1) * chunk);
            for (int n = u * chunk + tid; n < n1; n += kTabThreads)
                nrm.x_out[n] = __float2half_rn(__half2float(a.x[n]) * __half2float(nrm.gamma[n]) * r_inv);
        }
    }
    {
        const SlotStatic sl = resolve_slot(a, raw);
        __half xv[1];
        slot_x<1>(a, 0, sl.col, xv);
        float xf = __half2float(xv[0]);
        if constexpr (NORM) xf = (sl.col >= 0 && sl.col < a.N) ? xf * __half2float(nrm.gamma[sl.col]) * r_inv : 0.f;
        vbuf[tid / 32][tid % 32] = sl.c * xf;
    }
    __syncthreads();
    // thread t: entries (hi << 4) | (half << 3) | 0..7 of the four tables in
    // banks 4 qd .. 4 qd + 3, with it = t/2 = 8 hi + qd and half = t % 2
    const int it = tid >> 1, half = tid & 1;
    const int hi = it / 8, qd = it % 8;
    constexpr uint64_t kSign2 = 0x8000000080000000ull;
    uint64_t T0 = 0, T1 = 0, d0[3], d1[3];
#pragma unroll
    for (int t = 3; t < 8; ++t) {
        const bool plus = t == 3 ? half != 0 : ((hi >> (t - 4)) & 1) != 0;
        const uint64_t flip = plus ? 0ull : kSign2;
        const uint64_t v0 = *reinterpret_cast<const uint64_t*>(&vbuf[t][4 * qd]) ^ flip;
        const uint64_t v1 = *reinterpret_cast<const uint64_t*>(&vbuf[t][4 * qd + 2]) ^ flip;
        T0 = t == 3 ? v0 : add_f32x2(T0, v0);
        T1 = t == 3 ? v1 : add_f32x2(T1, v1);
    }
#pragma unroll
    for (int t = 0; t < 3; ++t) {
        const uint64_t v0 = *reinterpret_cast<const uint64_t*>(&vbuf[t][4 * qd]);
        const uint64_t v1 = *reinterpret_cast<const uint64_t*>(&vbuf[t][4 * qd + 2]);
        T0 = sub_f32x2(T0, v0);
        T1 = sub_f32x2(T1, v1);
        d0[t] = add_f32x2(v0, v0);
        d1[t] = add_f32x2(v1, v1);
    }
    // entry e of bank 4 qd at float index v*16384 + e*64 + h*32 + 4 qd
    float* base = tables + (int64_t)v * (kTabPairBytes / 4) + ((hi << 4) | (half << 3)) * 64 + h * 32 + 4 * qd;
    stg_v4(base, T0, T1);
    static_for<1, 8>([&](auto ic) {
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
        stg_v4(base + g * 64, T0, T1);
    });
}

}  // namespace fluxbin
