// C-ABI device entry points of libfluxbin: argument validation, kernel
// selection, grid sizing and the launch.  Declarations and the full contract
// are in include/fluxbin.h.
#include <algorithm>
#include <cmath>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>
#include <unordered_map>

#include "fluxbin_host.h"
#include "fluxbin_kernel.cuh"
#include "fluxbin_tc.cuh"

// Set by the tensor-core kernel when one of its bounded waits gives up; read
// and cleared by fluxbin_device_status.  One copy per device.
static __device__ unsigned int g_fluxbin_device_error;

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);
KernelFn select_kernel_mu8(int nb0, int nb1, int bt, int gs1);
KernelFn select_kernel_mu4(int nb0, int nb1, int bt, int gs1);
KernelFn select_kernel_mu8_3(int nb0, int nb1, int bt, int gs1);
using TcKernelFn = void (*)(TcArgs);
TcKernelFn select_tc_kernel(int mu, int nb0, int nb1);
KernelFn select_kernel_lut1(int lw, int nb0, int nb1);
KernelFn select_kernel_lut2(int nb0, int nb1);
int lut2_threads();
int lut2_smem_bytes();
int lut2_slabs();
using TabKernelFn = void (*)(KernelArgs, float*, NormArgs);
using HKernelFn = void (*)(KernelArgs, const float*);
TabKernelFn select_tables_kernel(int nb0, int nb1, bool norm);
HKernelFn select_kernel_lut1h(int spw, int nb0, int nb1);
int lut1h_threads(int spw);
int lut1h_smem_bytes(int spw);
int lut1h_slabs(int spw);
int lut1_threads(int lw);
int lut1_smem_bytes(int lw);
int lut1_slabs(int lw);

// Automatic path choice for a layer both paths can run.  At mu = 8 the LUT
// path on fp16-pair tables (fluxbin_lut2.cuh) is faster than the tensor cores
// at every batch measured on B200 (us per call, LUT / tensor cores):
// 28672x8192 B=8 91.5/183, B=16 182/196; 8192x28672 B=16 161/208;
// 11008x4096 B=16 46.5/64.0; 4096x11008 B=16 34.0/65.9.  At mu = 4 (tables
// of one row, fluxbin_kernel.cuh): 4096x4096 B=16 31.0/38.1; 8192x28672 B=8
// 241/255, B=16 473/256; the tensor cores win from batch 16 on layers above
// 4096x4096 and from batch 8 on layers with at least 16384 rows.
static bool prefer_tensor_cores(int64_t M, int64_t N, int B, int mu) {
    if (mu == 8) return false;
    return (B >= 16 && M * N > (int64_t)4096 * 4096) || (B >= 8 && M >= 16384);
}

namespace {

thread_local char g_last_error[256] = "";

// Records a failed CUDA call for fluxbin_last_error() and clears the error state.
int cuda_fail(cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    (void)cudaGetLastError();
    return FLUXBIN_ERR_CUDA;
}

// Batch rows whose tables a CTA keeps resident (the rest go to other CTAs).
// At mu = 8 one row per CTA: two CTAs per SM, each streaming the weights
// for its own batch row (mostly from L2 after the first), beat one CTA per
// SM holding two rows' tables (B200, B = 2 / 4: 11008x4096 12.7 -> 11.4 /
// 21.4 -> 18.7 us, 4096x11008 17.5 -> 13.0 / 27.4 -> 19.7 us, 4096x4096
// 8.8 -> 6.6 / 12.1 -> 9.4 us).
int batch_tile(int mu, int B) {
    if (mu == 8) return 1;
    return B <= 1 ? 1 : (B <= 2 ? 2 : 4);
}

// Tables plus the double-buffered activation products (see fluxbin_kernel.cuh).
size_t table_smem_bytes(int mu, int bt) {
    return (size_t)bt * ((size_t)1 << mu) * 256u + 2u * (size_t)bt * 32u * (size_t)mu * sizeof(float);
}
// Staged row scales of a grouped salient branch: two parities of one fp16
// per slot (32/gs1 of them) and row of the CTA.
size_t scale_smem_bytes(int gs1) { return gs1 > 0 ? 2u * (32u / (size_t)gs1) * kRowsPerCta * 2u : 0u; }
// Cluster reduction buffer: one fp32 partial per row of the CTA and batch row.
size_t red_smem_bytes(int bt) { return (size_t)bt * kRedRows * sizeof(float); }

struct DeviceInfo {
    int sm_count = 0;
    int max_smem = 0;
};

struct FuncInfo {
    int blocks_per_sm = 0;  // with the reduction buffer
};

// CTA shape of a kernel for the planner: row slabs per CTA, threads, dynamic
// shared memory.
struct CtaShape {
    int slabs;
    int threads;
    size_t smem;
};


std::mutex g_mu;
std::unordered_map<int, DeviceInfo> g_dev;
std::unordered_map<uint64_t, FuncInfo> g_func;
std::unordered_map<uint64_t, int> g_clusters;

int device_info(int dev, DeviceInfo* out) {
    auto it = g_dev.find(dev);
    if (it != g_dev.end()) {
        *out = it->second;
        return FLUXBIN_OK;
    }
    DeviceInfo di;
    if (cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&di.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return FLUXBIN_ERR_CUDA;
    g_dev.emplace(dev, di);
    *out = di;
    return FLUXBIN_OK;
}

// Per-function, per-device set-up: opt in to the dynamic shared memory of the
// largest launch and to non-portable cluster sizes; occupancy.
int func_info_shape(KernelFn fn, int dev, size_t smem_max, int threads, const DeviceInfo& di, FuncInfo* out) {
    const uint64_t key = (reinterpret_cast<uint64_t>(fn) << 8) ^ (uint64_t)dev;
    auto it = g_func.find(key);
    if (it != g_func.end()) {
        *out = it->second;
        return FLUXBIN_OK;
    }
    FuncInfo fi;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return cuda_fail(e);
    // the dynamic allocation shares the per-block limit with the static one
    if ((size_t)di.max_smem < smem_max + fa.sharedSizeBytes) return FLUXBIN_ERR_SMEM_BUDGET;
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fi.blocks_per_sm, fn, threads, smem_max)) != cudaSuccess)
        return cuda_fail(e);
    if (fi.blocks_per_sm < 1) return FLUXBIN_ERR_SMEM_BUDGET;
    g_func.emplace(key, fi);
    *out = fi;
    return FLUXBIN_OK;
}

int func_info(KernelFn fn, int dev, int mu, int bt, int gs1, const DeviceInfo& di, FuncInfo* out) {
    return func_info_shape(fn, dev, table_smem_bytes(mu, bt) + red_smem_bytes(bt) + scale_smem_bytes(gs1), kThreads,
                           di, out);
}

CtaShape v1_shape(int mu, int bt, int gs1) {
    return CtaShape{kSlabsPerCta, kThreads, table_smem_bytes(mu, bt) + red_smem_bytes(bt) + scale_smem_bytes(gs1)};
}

// How many clusters of `csize` CTAs can be resident at once (0: none).
int max_active_clusters(KernelFn fn, int dev, int csize, size_t smem, int threads = kThreads) {
    const uint64_t key = (reinterpret_cast<uint64_t>(fn) << 12) ^ ((uint64_t)dev << 8) ^ (uint64_t)csize;
    auto it = g_clusters.find(key);
    if (it != g_clusters.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)csize);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    g_clusters.emplace(key, n);
    return n;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct BranchIn {
    const uint32_t* words;
    const uint16_t* r;
    const uint16_t* c;
    const int32_t* gather;
    int32_t ncols, nb, rgroup;
};

// Launch shape: the split of the units over CTAs and how it is reduced.
struct Plan {
    int n_rg = 1;
    int n_ks = 1;
    bool cluster = false;
};

// Row groups (of the CTA's rows) times batch chunks fix the number of CTA
// groups; the units of a group are split over several CTAs, either a cluster
// whose partials are reduced in DSMEM (the widest split for which every
// cluster is resident at once, up to one CTA per CTA slot of the GPU) or, with
// a workspace from the caller, a split reduced through the workspace.
//
// The workspace split is as wide as one CTA per slot allows, then narrowed to
// as few CTAs as give the same units per CTA; it is taken unless a resident
// cluster split leaves each CTA as few units.  A call's time is set by its
// slowest CTA, i.e. by the units per CTA and by how many CTAs share an SM:
// clusters must sit inside one GPU processing cluster, which caps their width
// and places them unevenly.  Measured on B200 at batch 1 (graph of calls):
// 4096x4096 5.37 -> 4.01 us (one cluster of 16 per row group against 17 CTAs
// through the workspace), 4096x4096 at 2.75 bits with block-wise scales 7.75
// -> 5.35 us, 4096x11008 at 2.75 bits 11.81 -> 9.89 us, 8192x28672 at mu = 4
// 55.8 -> 41.7 us; 4096x4096 at batch 2 6.52 -> 5.45 us.
Plan make_plan(KernelFn fn, int dev, const CtaShape& cs, int64_t Ms, int64_t U, int n_bc, const DeviceInfo& di,
               const FuncInfo& fi, bool have_ws, bool fill_gpu = false) {
    Plan p;
    p.n_rg = (int)((Ms + cs.slabs - 1) / cs.slabs);
    const int64_t groups = (int64_t)p.n_rg * n_bc;
    const int64_t slots = (int64_t)di.sm_count * fi.blocks_per_sm;
    const size_t smem = cs.smem;
    const int64_t ks_cap = std::min<int64_t>(U, slots / groups);
    const int64_t units_wide = ks_cap >= 1 ? (U + ks_cap - 1) / ks_cap : U;
    const int64_t ks_wide = (U + units_wide - 1) / units_wide;
    const bool wide_ok = have_ws && ks_wide >= 2;

    // One CTA per SM and more CTA groups than slots: without a split the last
    // wave runs partly empty.  A split through the workspace that evens the
    // waves out pays for its reduction; each further split costs ~4% of a
    // CTA's time (B200, 28672x8192 at batch 16 on the batch-pair kernel:
    // 224 CTAs 168.7 us, split 2 174.8, 3 154.6, 4 164.4, 6 167.7; the model
    // ceil(groups*ks/slots)/ks * (1 + 0.04 (ks-1)) ranks them the same way).
    if (fill_gpu && have_ws && groups > slots && U >= 2) {
        auto cost = [&](int64_t ks) {
            return (double)((groups * ks + slots - 1) / slots) / (double)ks * (1.0 + 0.04 * (double)(ks - 1));
        };
        const double base = cost(1);
        int64_t best = 1;
        double best_cost = base;
        for (int64_t ks = 2; ks <= std::min<int64_t>(U, 8); ++ks)
            if (cost(ks) < best_cost) {
                best = ks;
                best_cost = cost(ks);
            }
        if (best > 1 && best_cost < 0.98 * base) {
            p.n_ks = (int)best;
            p.cluster = false;
            return p;
        }
    }

    int64_t want = slots / groups;
    if (want > U) want = U;
    if (want > kMaxCluster) want = kMaxCluster;
    for (int64_t ks = want; ks >= 2; --ks) {
        if (have_ws && groups * ks * 2 < di.sm_count) break;  // too few CTAs: use the workspace instead
        if (max_active_clusters(fn, dev, (int)ks, smem, cs.threads) >= groups) {
            if (wide_ok && units_wide < (U + ks - 1) / ks) break;  // the workspace split is shorter
            p.n_ks = (int)ks;
            p.cluster = true;
            // One CTA per SM: a cluster size that fits fewer CTAs than the
            // GPU has slots leaves SMs idle; split one CTA per slot through
            // the workspace instead when that fills at least an eighth more.
            const int64_t ks_ws = std::min<int64_t>(U, slots / groups);
            if (fill_gpu && have_ws && ks_ws * 8 >= ks * 9) {
                p.n_ks = (int)ks_ws;
                p.cluster = false;
            }
            return p;
        }
    }
    if (wide_ok) {
        p.n_ks = (int)ks_wide;
        p.cluster = false;
        return p;
    }
    if (groups * 2 >= di.sm_count || U <= 1 || !have_ws) {
        p.n_ks = 1;  // enough row groups (or no workspace): no split at all
        return p;
    }
    int64_t ks = (slots + groups / 2) / groups;
    if (ks > U) ks = U;
    if (ks < 1) ks = 1;
    p.n_ks = (int)ks;
    p.cluster = false;
    return p;
}

constexpr int kMaxDevicesTc = 64;
std::mutex g_tc_mu;
std::unordered_map<uint64_t, bool> g_tc_func;
unsigned int* g_err_addr[kMaxDevicesTc] = {};

int device_error_address(int dev, unsigned int** out) {
    if (dev < 0 || dev >= kMaxDevicesTc) return FLUXBIN_ERR_CUDA;
    if (!g_err_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fluxbin_device_error) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return FLUXBIN_ERR_CUDA;
        }
        g_err_addr[dev] = static_cast<unsigned int*>(p);
    }
    *out = g_err_addr[dev];
    return FLUXBIN_OK;
}

// The layer on the tensor cores (fluxbin_tc.cuh): per-row scales, mu = 4 or 8,
// 1 <= B <= 16, a workspace always (the split of a tile's units is reduced
// through it).  Items (128-row tile, unit range) run on a persistent grid of
// one CTA per SM; the unit ranges are split so that there are about four
// items per SM.
int run_tc(int32_t M, int32_t N, int mu, const BranchIn& g, const BranchIn* s, int nb1, const uint16_t* d_x, int32_t B,
           void* d_y, uint32_t flags, void* ws, size_t ws_bytes, void* stream, int* uses_ws) {
    const size_t need = workspace_bytes_for(M, B);
    if (!ws || ws_bytes < need) return FLUXBIN_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return FLUXBIN_ERR_MISALIGNED;
    TcKernelFn fn = select_tc_kernel(mu, g.nb, nb1);
    if (!fn) return FLUXBIN_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    DeviceInfo di;
    unsigned int* err = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int st = device_info(dev, &di);
        if (st != FLUXBIN_OK) return st;
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        int st = device_error_address(dev, &err);
        if (st != FLUXBIN_OK) return st;
        const uint64_t key = (reinterpret_cast<uint64_t>(fn) << 8) ^ (uint64_t)dev;
        if (g_tc_func.find(key) == g_tc_func.end()) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) return cuda_fail(e);
            if ((size_t)di.max_smem < (size_t)kTcSmemBytes + fa.sharedSizeBytes) return FLUXBIN_ERR_SMEM_BUDGET;
            int blocks = 0;
            if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmemBytes)) !=
                    cudaSuccess ||
                (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, kTcThreads + 32, kTcSmemBytes)) !=
                    cudaSuccess)
                return cuda_fail(e);
            if (blocks < 1) return FLUXBIN_ERR_SMEM_BUDGET;
            g_tc_func.emplace(key, true);
        }
    }
    TcArgs a = {};
    const BranchIn* in[2] = {&g, nb1 ? s : nullptr};
    for (int q = 0; q < 2; ++q) {
        BranchArgs& o = a.br[q];
        if (!in[q] || in[q]->ncols == 0) continue;
        o.words = reinterpret_cast<const uint4*>(in[q]->words);
        o.r = reinterpret_cast<const __half*>(in[q]->r);
        o.c = reinterpret_cast<const __half*>(in[q]->c);
        o.gather = in[q]->gather;
        o.ncols = in[q]->ncols;
        o.units = (int32_t)branch_units(in[q]->ncols, in[q]->nb, mu);
    }
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = B;
    a.Ms = (int32_t)row_slabs(M);
    a.Mp = a.Ms * kLanes;
    a.n_rt = (M + kTcRows - 1) / kTcRows;
    int64_t ks = (4 * (int64_t)di.sm_count + a.n_rt - 1) / a.n_rt;
    if (ks > U) ks = U;
    if (ks < 1) ks = 1;
    a.n_ks = (int32_t)ks;
    a.n_items = a.n_rt * a.n_ks;
    if (uses_ws) {  // plan query only
        *uses_ws = a.n_ks > 1 ? 1 : 0;
        return FLUXBIN_OK;
    }
    a.test_stall = (flags & kFlagTestWaitTimeout) ? 1 : 0;
    a.spin_limit = a.test_stall ? kTcTestSpinLimit : kTcSpinLimit;
    a.flags = flags & ~kFlagTestWaitTimeout;
    const size_t acc = (((size_t)B * a.Mp * sizeof(float)) + 255) & ~(size_t)255;
    a.ws_acc = static_cast<float*>(ws);
    a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    a.err = err;
    a.vec_x = (N % 8 == 0 && aligned(d_x, 16) && aligned(g.c, 16)) ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.n_items < di.sm_count ? a.n_items : di.sm_count));
    cfg.blockDim = dim3(kTcThreads + 32);   // 16 worker warps and the MMA-issuing warp
    cfg.dynamicSmemBytes = kTcSmemBytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t le = cudaLaunchKernelEx(&cfg, fn, a);
    if (le != cudaSuccess) return cuda_fail(le);
    return FLUXBIN_OK;
}

// Branch arguments of a launch.
void fill_branches(KernelArgs& a, int mu, const BranchIn& g, const BranchIn* s, int nb1) {
    const BranchIn* in[2] = {&g, nb1 ? s : nullptr};
    for (int q = 0; q < 2; ++q) {
        BranchArgs& o = a.br[q];
        if (!in[q] || in[q]->ncols == 0) continue;
        o.words = reinterpret_cast<const uint4*>(in[q]->words);
        o.r = reinterpret_cast<const __half*>(in[q]->r);
        o.c = reinterpret_cast<const __half*>(in[q]->c);
        o.gather = in[q]->gather;
        o.ncols = in[q]->ncols;
        o.units = (int32_t)branch_units(in[q]->ncols, in[q]->nb, mu);
        o.rgroup = in[q]->rgroup;
        o.ngroups = in[q]->rgroup > 0 ? (in[q]->ncols + in[q]->rgroup - 1) / in[q]->rgroup : 0;
    }
}

// Batch 1, mu = 8, per-row scales: the warp-specialised kernel
// (fluxbin_lut1.cuh).  16 lookup warps per CTA (1024 rows, one CTA per SM)
// when that plan keeps most SMs busy, else 8 (512 rows, two CTAs per SM).
int run_lut1(int32_t M, int32_t N, const BranchIn& g, const BranchIn* s, int nb1, const uint16_t* d_x, void* d_y,
             uint32_t flags, void* ws, size_t ws_bytes, void* stream, int* uses_ws) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    KernelArgs a = {};
    fill_branches(a, 8, g, s, nb1);
    a.Ms = (int32_t)row_slabs(M);
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    const bool have_ws = ws && ws_bytes >= workspace_bytes_for(M, 1) && aligned(ws, 16);
    DeviceInfo di;
    unsigned int* err = nullptr;
    KernelFn fn = nullptr;
    Plan plan;
    int lw = 16;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int st = device_info(dev, &di);
        if (st != FLUXBIN_OK) return st;
        KernelFn f16 = select_kernel_lut1(16, g.nb, nb1), f8 = select_kernel_lut1(8, g.nb, nb1);
        if (!f16 || !f8) return FLUXBIN_ERR_UNSUPPORTED;
        FuncInfo i16, i8;
        const CtaShape c16{lut1_slabs(16), lut1_threads(16), (size_t)lut1_smem_bytes(16)};
        const CtaShape c8{lut1_slabs(8), lut1_threads(8), (size_t)lut1_smem_bytes(8)};
        if ((st = func_info_shape(f16, dev, c16.smem, c16.threads, di, &i16)) != FLUXBIN_OK) return st;
        if ((st = func_info_shape(f8, dev, c8.smem, c8.threads, di, &i8)) != FLUXBIN_OK) return st;
        const Plan p16 = make_plan(f16, dev, c16, a.Ms, U, 1, di, i16, have_ws, true);
        const Plan p8 = make_plan(f8, dev, c8, a.Ms, U, 1, di, i8, have_ws);
        const int64_t busy16 = (int64_t)p16.n_rg * p16.n_ks;   // CTAs = SMs in use
        if (busy16 * 4 >= (int64_t)di.sm_count * 3) {
            fn = f16;
            plan = p16;
        } else {
            fn = f8;
            plan = p8;
            lw = 8;
        }
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        const int st = device_error_address(dev, &err);
        if (st != FLUXBIN_OK) return st;
    }
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = 1;
    a.Mp = a.Ms * kLanes;
    a.n_rg = plan.n_rg;
    a.n_bc = 1;
    a.n_ks = plan.n_ks;
    a.cluster = plan.cluster ? 1 : 0;
    a.flags = flags;
    a.err = err;
    if (uses_ws) {  // plan query only
        *uses_ws = (a.n_ks > 1 && !plan.cluster) ? 1 : 0;
        return FLUXBIN_OK;
    }
    if (a.n_ks > 1 && !plan.cluster) {
        if (!have_ws) return ws ? (aligned(ws, 16) ? FLUXBIN_ERR_WORKSPACE : FLUXBIN_ERR_MISALIGNED)
                                : FLUXBIN_ERR_WORKSPACE;
        const size_t acc = (((size_t)a.Mp * sizeof(float)) + 255) & ~(size_t)255;
        a.ws_acc = static_cast<float*>(ws);
        a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.n_rg * a.n_ks));
    cfg.blockDim = dim3((unsigned)lut1_threads(lw));
    cfg.dynamicSmemBytes = (size_t)lut1_smem_bytes(lw);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (plan.cluster) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)a.n_ks;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    const cudaError_t le = cudaLaunchKernelEx(&cfg, fn, a);
    if (le != cudaSuccess) return cuda_fail(le);
    return FLUXBIN_OK;
}

// Batches of 2-16, mu = 8, per-row scales: pairs of batch rows on fp16-pair
// tables (fluxbin_lut2.cuh), one CTA per SM, 1024 rows x one batch pair x a
// range of units per CTA.
int run_lut2(int32_t M, int32_t N, const BranchIn& g, const BranchIn* s, int nb1, const uint16_t* d_x, int32_t B,
             void* d_y, uint32_t flags, void* ws, size_t ws_bytes, void* stream, int* uses_ws) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    KernelArgs a = {};
    fill_branches(a, 8, g, s, nb1);
    a.Ms = (int32_t)row_slabs(M);
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    const int n_bp = (B + 1) / 2;
    const bool have_ws = ws && ws_bytes >= workspace_bytes_for(M, B) && aligned(ws, 16);
    DeviceInfo di;
    unsigned int* err = nullptr;
    KernelFn fn = select_kernel_lut2(g.nb, nb1);
    if (!fn) return FLUXBIN_ERR_UNSUPPORTED;
    Plan plan;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int st = device_info(dev, &di);
        if (st != FLUXBIN_OK) return st;
        FuncInfo fi;
        const CtaShape cs{lut2_slabs(), lut2_threads(), (size_t)lut2_smem_bytes()};
        if ((st = func_info_shape(fn, dev, cs.smem, cs.threads, di, &fi)) != FLUXBIN_OK) return st;
        plan = make_plan(fn, dev, cs, a.Ms, U, n_bp, di, fi, have_ws, true);
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        const int st = device_error_address(dev, &err);
        if (st != FLUXBIN_OK) return st;
    }
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = B;
    a.Mp = a.Ms * kLanes;
    a.n_rg = plan.n_rg;
    a.n_bc = n_bp;
    a.n_ks = plan.n_ks;
    a.cluster = plan.cluster ? 1 : 0;
    a.flags = flags;
    a.err = err;
    if (uses_ws) {  // plan query only
        *uses_ws = (a.n_ks > 1 && !plan.cluster) ? 1 : 0;
        return FLUXBIN_OK;
    }
    if (a.n_ks > 1 && !plan.cluster) {
        if (!have_ws) return FLUXBIN_ERR_WORKSPACE;
        const size_t acc = (((size_t)B * a.Mp * sizeof(float)) + 255) & ~(size_t)255;
        a.ws_acc = static_cast<float*>(ws);
        a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.n_rg * a.n_bc * a.n_ks));
    cfg.blockDim = dim3((unsigned)lut2_threads());
    cfg.dynamicSmemBytes = (size_t)lut2_smem_bytes();
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (plan.cluster) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)a.n_ks;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    const cudaError_t le = cudaLaunchKernelEx(&cfg, fn, a);
    if (le != cudaSuccess) return cuda_fail(le);
    return FLUXBIN_OK;
}

// Batch 1, mu = 8, per-row scales, with room for the table buffer in the
// workspace: the table precompute as its own kernel (fluxbin_tables.cuh),
// then the lookups on the precomputed tables (fluxbin_lut1h.cuh), 1024 or
// 2048 rows per CTA.
int run_lut1h(int32_t M, int32_t N, const BranchIn& g, const BranchIn* s, int nb1, const uint16_t* d_x, void* d_y,
              uint32_t flags, void* ws, void* stream, int* uses_ws, const NormArgs* norm = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    KernelArgs a = {};
    fill_branches(a, 8, g, s, nb1);
    a.Ms = (int32_t)row_slabs(M);
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    DeviceInfo di;
    unsigned int* err = nullptr;
    HKernelFn fn = nullptr;
    TabKernelFn tfn = select_tables_kernel(g.nb, nb1, norm != nullptr);
    Plan plan;
    int spw = 4;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int st = device_info(dev, &di);
        if (st != FLUXBIN_OK) return st;
        HKernelFn f4 = select_kernel_lut1h(4, g.nb, nb1), f2 = select_kernel_lut1h(2, g.nb, nb1);
        if (!f4 || !f2 || !tfn) return FLUXBIN_ERR_UNSUPPORTED;
        FuncInfo i4, i2;
        const CtaShape c4{lut1h_slabs(4), lut1h_threads(4), (size_t)lut1h_smem_bytes(4)};
        const CtaShape c2{lut1h_slabs(2), lut1h_threads(2), (size_t)lut1h_smem_bytes(2)};
        KernelFn k4 = reinterpret_cast<KernelFn>(f4), k2 = reinterpret_cast<KernelFn>(f2);
        if ((st = func_info_shape(k4, dev, c4.smem, c4.threads, di, &i4)) != FLUXBIN_OK) return st;
        if ((st = func_info_shape(k2, dev, c2.smem, c2.threads, di, &i2)) != FLUXBIN_OK) return st;
        const Plan p4 = make_plan(k4, dev, c4, a.Ms, U, 1, di, i4, true, true);
        const Plan p2 = make_plan(k2, dev, c2, a.Ms, U, 1, di, i2, true, true);
        // 1024 rows per CTA whenever that plan keeps three quarters of the
        // SMs busy (the 2048-row build spills; B200, batch 1: 28672x8192
        // 28.5 -> 27.1 us, 8192x28672 30.9 -> 29.0 us), else 2048 if that
        // one does
        const auto fills = [&](const Plan& p) { return (int64_t)p.n_rg * p.n_ks * 4 >= (int64_t)di.sm_count * 3; };
        if (!fills(p2) && fills(p4)) {
            fn = f4;
            plan = p4;
        } else {
            fn = f2;
            plan = p2;
            spw = 2;
        }
    }
    if (uses_ws) {  // plan query only: the tables always live in the workspace
        *uses_ws = 1;
        return FLUXBIN_OK;
    }
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        const int st = device_error_address(dev, &err);
        if (st != FLUXBIN_OK) return st;
    }
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = 1;
    a.Mp = a.Ms * kLanes;
    a.n_rg = plan.n_rg;
    a.n_bc = 1;
    a.n_ks = plan.n_ks;
    a.cluster = plan.cluster ? 1 : 0;
    a.flags = flags;
    a.err = err;
    const size_t acc = (((size_t)a.Mp * sizeof(float)) + 255) & ~(size_t)255;
    a.ws_acc = static_cast<float*>(ws);
    a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    float* tables = reinterpret_cast<float*>(static_cast<char*>(ws) + workspace_bytes_for(M, 1));

    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t tc = {};
    tc.gridDim = dim3((unsigned)U);
    tc.blockDim = dim3(256);   // fluxbin_tables_kernel: one unit per CTA of 256 threads
    tc.stream = static_cast<cudaStream_t>(stream);
    tc.attrs = attr;
    tc.numAttrs = 1;
    cudaError_t le = cudaLaunchKernelEx(&tc, tfn, a, tables, norm ? *norm : NormArgs{nullptr, 0.f, nullptr});
    if (le != cudaSuccess) return cuda_fail(le);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.n_rg * a.n_ks));
    cfg.blockDim = dim3((unsigned)lut1h_threads(spw));
    cfg.dynamicSmemBytes = (size_t)lut1h_smem_bytes(spw);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (plan.cluster) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)a.n_ks;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    le = cudaLaunchKernelEx(&cfg, fn, a, static_cast<const float*>(tables));
    if (le != cudaSuccess) return cuda_fail(le);
    return FLUXBIN_OK;
}

// Validates the arguments, chooses the path and the launch plan and launches
// the layer.  With `uses_ws` non-null nothing is launched: it reports whether
// the chosen plan reduces through the workspace.
int run(int32_t M, int32_t N, int mu, const BranchIn& g, const BranchIn* s, const uint16_t* d_x, int32_t B,
        void* d_y, uint32_t flags, void* ws, size_t ws_bytes, void* stream, int* uses_ws = nullptr) {
    if (flags & ~(kFlagAccumulate | kFlagYFp32 | kFlagEarlyWeights | kFlagPathLut | kFlagPathTc |
                  kFlagTestWaitTimeout | kFlagSeparateTables))
        return FLUXBIN_ERR_INVALID_ARG;
    if ((flags & kFlagSeparateTables) && (flags & kFlagPathTc)) return FLUXBIN_ERR_INVALID_ARG;
    if ((flags & kFlagPathLut) && (flags & kFlagPathTc)) return FLUXBIN_ERR_INVALID_ARG;
    if ((flags & kFlagTestWaitTimeout) && !(flags & kFlagPathTc)) return FLUXBIN_ERR_INVALID_ARG;
    if (uses_ws) *uses_ws = 0;
    if (B < 0 || B > kMaxBatch) return B < 0 ? FLUXBIN_ERR_BAD_SHAPE : FLUXBIN_ERR_UNSUPPORTED;
    if (M == 0 || B == 0) return FLUXBIN_OK;
    if (!d_y || (N > 0 && !d_x)) return FLUXBIN_ERR_INVALID_ARG;
    const bool y32 = (flags & kFlagYFp32) != 0;
    if (!aligned(d_y, y32 ? 4 : 2) || !aligned(d_x, 2)) return FLUXBIN_ERR_MISALIGNED;
    const BranchIn* brs[2] = {&g, s};
    for (int q = 0; q < 2; ++q) {
        const BranchIn* b = brs[q];
        if (!b || b->ncols == 0) continue;
        if (!b->words || !b->r || !b->c) return FLUXBIN_ERR_INVALID_ARG;
        if (!aligned(b->words, 16)) return FLUXBIN_ERR_MISALIGNED;
        if (!aligned(b->r, 2) || !aligned(b->c, 2) || !aligned(b->gather, 4)) return FLUXBIN_ERR_MISALIGNED;
    }
    const int nb1 = (s && s->ncols > 0) ? s->nb : 0;
    // the tensor-core path: per-row scales, mu = 8, a batch large enough for
    // the contraction to pay (or asked for explicitly)
    const bool tc_fits = (mu == 8 || mu == 4) && g.rgroup == 0 && (!nb1 || s->rgroup == 0);
    if ((flags & kFlagPathTc) && !tc_fits) return FLUXBIN_ERR_UNSUPPORTED;
    if ((flags & kFlagPathTc) ||
        (!(flags & (kFlagPathLut | kFlagSeparateTables)) && tc_fits && prefer_tensor_cores(M, N, B, mu) && ws &&
         ws_bytes >= workspace_bytes_for(M, B)))
        return run_tc(M, N, mu, g, s, nb1, d_x, B, d_y, flags & ~(kFlagPathLut | kFlagPathTc), ws, ws_bytes, stream,
                      uses_ws);
    // batch 1, mu = 8, per-row scales: the table precompute as its own kernel
    // when asked for (and the workspace has room for the tables); otherwise,
    // for large layers, the warp-specialised kernel (B200, batch 1:
    // 28672x8192 25.3 -> 22.0 us, 8192x28672 29.1 -> 21.2 us).  From 2^25
    // weights with a workspace (11008x4096 and 4096x11008 7.0 -> 6.7 us with
    // the workspace split of both kernels), from 2^27 without; 4096x4096
    // stays on the kernel below (4.0 against 4.2 us).  With the precompute as
    // its own kernel the large layers measured 25.2 and 31.3 us: the lookups
    // alone took longer than the warp-specialised kernel with its in-CTA
    // build, and the precompute ran before them.
    if (B == 1 && mu == 8 && g.rgroup == 0 && (!nb1 || s->rgroup == 0)) {
        const int64_t U = branch_units(g.ncols, g.nb, mu) + (nb1 ? branch_units(s->ncols, nb1, mu) : 0);
        if (flags & kFlagSeparateTables) {
            if (!ws || ws_bytes < workspace_bytes_for(M, 1) + table_bytes_for(U)) return FLUXBIN_ERR_WORKSPACE;
            if (!aligned(ws, 16)) return FLUXBIN_ERR_MISALIGNED;
            return run_lut1h(M, N, g, s, nb1, d_x, d_y, flags & ~kFlagSeparateTables, ws, stream, uses_ws);
        }
        const bool ws_ok = ws && ws_bytes >= workspace_bytes_for(M, 1) && aligned(ws, 16);
        if ((int64_t)M * N >= ((int64_t)1 << (ws_ok ? 25 : 27)))
            return run_lut1(M, N, g, s, nb1, d_x, d_y, flags, ws, ws_bytes, stream, uses_ws);
    } else if (flags & kFlagSeparateTables) {
        return FLUXBIN_ERR_UNSUPPORTED;
    }
    // batches of 2-16, mu = 8, per-row scales: pairs of batch rows on
    // fp16-pair tables (B200, us per call against one-row fp32 tables below:
    // 28672x8192 B=2 26.4/49.0, B=4 47.0/104, B=16 182/346; 11008x4096 B=2
    // 10.8/11.4, B=8 17.9/37.3; 4096x4096 B=4 8.9/9.4, B=16 15.0/26.7; only
    // 4096x4096 at B=2 stays faster below, 6.5/7.1)
    if (B >= 2 && mu == 8 && g.rgroup == 0 && (!nb1 || s->rgroup == 0) &&
        (B >= 4 || (int64_t)M * N > (int64_t)4096 * 4096))
        return run_lut2(M, N, g, s, nb1, d_x, B, d_y, flags, ws, ws_bytes, stream, uses_ws);
    // salient row scales finer than a unit: grouped visit order, one batch row per CTA
    const int gs1 = (nb1 && s->rgroup > 0 && s->rgroup < unit_cols(nb1, mu)) ? s->rgroup / mu : 0;
    const int bt = gs1 ? 1 : batch_tile(mu, B);
    KernelFn fn = mu == 8 ? select_kernel_mu8(g.nb, nb1, bt, gs1) : select_kernel_mu4(g.nb, nb1, bt, gs1);
    if (!fn) return FLUXBIN_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    DeviceInfo di;
    FuncInfo fi;
    Plan plan;
    KernelArgs a = {};
    const BranchIn* in[2] = {&g, nb1 ? s : nullptr};
    for (int q = 0; q < 2; ++q) {
        BranchArgs& o = a.br[q];
        if (!in[q] || in[q]->ncols == 0) continue;
        o.words = reinterpret_cast<const uint4*>(in[q]->words);
        o.r = reinterpret_cast<const __half*>(in[q]->r);
        o.c = reinterpret_cast<const __half*>(in[q]->c);
        o.gather = in[q]->gather;
        o.ncols = in[q]->ncols;
        o.units = (int32_t)branch_units(in[q]->ncols, in[q]->nb, mu);
        o.rgroup = in[q]->rgroup;
        o.ngroups = in[q]->rgroup > 0 ? (in[q]->ncols + in[q]->rgroup - 1) / in[q]->rgroup : 0;
    }
    a.Ms = (int32_t)row_slabs(M);
    const int n_bc = (B + bt - 1) / bt;
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int st = device_info(dev, &di);
        if (st != FLUXBIN_OK) return st;
        st = func_info(fn, dev, mu, bt, gs1, di, &fi);
        if (st != FLUXBIN_OK) return st;
        const bool have_ws = ws && ws_bytes >= workspace_bytes_for(M, B) && aligned(ws, 16);
        plan = make_plan(fn, dev, v1_shape(mu, bt, gs1), a.Ms, U, n_bc, di, fi, have_ws);
        // The build with three CTAs per SM (80 registers, a few bytes spilled)
        // pays where its extra slots widen the split: large layers (B200,
        // batch 1: 28672x8192 27.3 -> 25.8 us, 8192x28672 32.7 -> 29.5 us;
        // batch 2 / 4: 54.7 -> 49.3 / 92.2 -> 84.9 us), and layers that two
        // CTAs per SM would not split at all (11008x4096 at batch 8: 50.8 ->
        // 37.3 us).  Otherwise it is slower (7B-sized layers at batch 1-4 by
        // 5-30%; 28672x8192 at batch 4, same split, 104.7 -> 136.1 us).
        if (mu == 8) {
            KernelFn f3 = select_kernel_mu8_3(g.nb, nb1, bt, gs1);
            FuncInfo fi3;
            if (f3 && func_info(f3, dev, mu, bt, gs1, di, &fi3) == FLUXBIN_OK) {
                const Plan p3 = make_plan(f3, dev, v1_shape(mu, bt, gs1), a.Ms, U, n_bc, di, fi3, have_ws);
                const bool large = (int64_t)M * N >= ((int64_t)1 << 27);
                if ((large && (B == 1 || p3.n_ks > plan.n_ks)) || (plan.n_ks == 1 && p3.n_ks >= 2)) {
                    fn = f3;
                    fi = fi3;
                    plan = p3;
                }
            }
        }
    }
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = B;
    a.Mp = a.Ms * kLanes;
    a.n_rg = plan.n_rg;
    a.n_bc = n_bc;
    a.n_ks = plan.n_ks;
    a.cluster = plan.cluster ? 1 : 0;
    a.flags = flags;
    if (uses_ws) {  // plan query only
        *uses_ws = (a.n_ks > 1 && !plan.cluster) ? 1 : 0;
        return FLUXBIN_OK;
    }
    if (a.n_ks > 1 && !plan.cluster) {
        const size_t need = workspace_bytes_for(M, B);
        if (!ws || ws_bytes < need) return FLUXBIN_ERR_WORKSPACE;
        if (!aligned(ws, 16)) return FLUXBIN_ERR_MISALIGNED;
        const size_t acc = (((size_t)B * a.Mp * sizeof(float)) + 255) & ~(size_t)255;
        a.ws_acc = static_cast<float*>(ws);
        a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((int64_t)a.n_rg * a.n_bc * a.n_ks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = table_smem_bytes(mu, bt) + red_smem_bytes(bt) + scale_smem_bytes(gs1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (plan.cluster) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)a.n_ks;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    const cudaError_t le = cudaLaunchKernelEx(&cfg, fn, a);
    if (le != cudaSuccess) return cuda_fail(le);
    return FLUXBIN_OK;
}

}  // namespace

int linear_impl(const fluxbin_layer_desc* desc, const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c,
                const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs, const int32_t* d_idx,
                const uint16_t* d_x, int32_t B, void* d_y, uint32_t flags, void* d_workspace,
                size_t workspace_bytes, void* stream, int* uses_ws) {
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    const fluxbin_layer_desc& d = *desc;
    BranchIn g{d_words, d_r, d_c, nullptr, d.N, d.Kb, d.row_scale_group};
    BranchIn s{d_swords, d_rs, d_cs, d_idx, has_salient(d) ? d.n_sal : 0, d.Ks ? d.Ks : 1, d.sal_scale_group};
    if (has_salient(d) && !d_idx) return FLUXBIN_ERR_INVALID_ARG;
    return run(d.M, d.N, d.mu, g, has_salient(d) ? &s : nullptr, d_x, B, d_y, flags, d_workspace,
               workspace_bytes, stream, uses_ws);
}

}  // namespace fluxbin

using namespace fluxbin;

extern "C" {

const char* fluxbin_last_error(void) { return g_last_error; }

int fluxbin_device_status(uint32_t* out_flags) {
    if (!out_flags) return FLUXBIN_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    unsigned int* err = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_tc_mu);
        const int st = device_error_address(dev, &err);
        if (st != FLUXBIN_OK) return st;
    }
    unsigned int v = 0;
    cudaError_t e = cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v) e = cudaMemset(err, 0, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e);
    *out_flags = v;
    return FLUXBIN_OK;
}

int fluxbin_layer_workspace_bytes(const fluxbin_layer_desc* desc, int32_t B, size_t* bytes) {
    if (!bytes) return FLUXBIN_ERR_INVALID_ARG;
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    if (B < 0) return FLUXBIN_ERR_BAD_SHAPE;
    size_t n = workspace_bytes_for(desc->M, B);
    if (desc->M > 0 && hoistable(*desc, B)) n += table_bytes_for(layer_units(*desc));
    *bytes = n;
    return FLUXBIN_OK;
}

int fluxbin_lut_gemv(int32_t M, int32_t N, int32_t ncols, int32_t nbases, int32_t mu, int32_t row_scale_group,
                     const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c, const int32_t* d_gather,
                     const uint16_t* d_x, int32_t B, void* d_y, uint32_t flags, void* d_workspace,
                     size_t workspace_bytes, void* stream) {
    if (M < 0 || N < 0 || ncols < 0 || row_scale_group < 0) return FLUXBIN_ERR_BAD_SHAPE;
    if (!valid_mu(mu) || !valid_nb(nbases)) return FLUXBIN_ERR_UNSUPPORTED;
    if (!d_gather && ncols > N) return FLUXBIN_ERR_BAD_SHAPE;
    if (row_scale_group > 0 && row_scale_group % unit_cols(nbases, mu)) return FLUXBIN_ERR_UNSUPPORTED;
    BranchIn g{d_words, d_r, d_c, d_gather, ncols, nbases, row_scale_group};
    return run(M, N, mu, g, nullptr, d_x, B, d_y, flags, d_workspace, workspace_bytes, stream);
}

int fluxbin_linear(const fluxbin_layer_desc* desc, const uint32_t* d_words, const uint16_t* d_r,
                   const uint16_t* d_c, const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs,
                   const int32_t* d_idx, const uint16_t* d_x, int32_t B, void* d_y, uint32_t flags,
                   void* d_workspace, size_t workspace_bytes, void* stream) {
    return linear_impl(desc, d_words, d_r, d_c, d_swords, d_rs, d_cs, d_idx, d_x, B, d_y, flags, d_workspace,
                       workspace_bytes, stream, nullptr);
}

int fluxbin_linear_rmsnorm(const fluxbin_layer_desc* desc, const uint32_t* d_words, const uint16_t* d_r,
                           const uint16_t* d_c, const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs,
                           const int32_t* d_idx, const uint16_t* d_h, const uint16_t* d_gamma, float eps,
                           uint16_t* d_x_out, void* d_y, uint32_t flags, void* d_workspace, size_t workspace_bytes,
                           void* stream) {
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    const fluxbin_layer_desc& d = *desc;
    if (flags & ~(kFlagAccumulate | kFlagYFp32 | kFlagEarlyWeights)) return FLUXBIN_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return FLUXBIN_ERR_INVALID_ARG;   // negative, NaN or infinite
    if (d.M == 0) return FLUXBIN_OK;
    if (d.N == 0) return FLUXBIN_ERR_BAD_SHAPE;   // no mean of h^2 to take
    if (!hoistable(d, 1)) return FLUXBIN_ERR_UNSUPPORTED;
    if (!d_h || !d_gamma || !d_y) return FLUXBIN_ERR_INVALID_ARG;
    if (has_salient(d) && !d_idx) return FLUXBIN_ERR_INVALID_ARG;
    const bool y32 = (flags & kFlagYFp32) != 0;
    if (!aligned(d_h, 2) || !aligned(d_gamma, 2) || !aligned(d_x_out, 2) || !aligned(d_y, y32 ? 4 : 2))
        return FLUXBIN_ERR_MISALIGNED;
    if (d_x_out) {
        // the kernel reads all of h while writing x: they must not overlap
        const uintptr_t h0 = reinterpret_cast<uintptr_t>(d_h), x0 = reinterpret_cast<uintptr_t>(d_x_out);
        const uintptr_t n = (uintptr_t)d.N * 2u;
        if (x0 < h0 + n && h0 < x0 + n) return FLUXBIN_ERR_INVALID_ARG;
    }
    BranchIn g{d_words, d_r, d_c, nullptr, d.N, d.Kb, d.row_scale_group};
    BranchIn s{d_swords, d_rs, d_cs, d_idx, has_salient(d) ? d.n_sal : 0, d.Ks ? d.Ks : 1, d.sal_scale_group};
    const BranchIn* brs[2] = {&g, has_salient(d) ? &s : nullptr};
    for (int q = 0; q < 2; ++q) {
        const BranchIn* b = brs[q];
        if (!b || b->ncols == 0) continue;
        if (!b->words || !b->r || !b->c) return FLUXBIN_ERR_INVALID_ARG;
        if (!aligned(b->words, 16)) return FLUXBIN_ERR_MISALIGNED;
        if (!aligned(b->r, 2) || !aligned(b->c, 2) || !aligned(b->gather, 4)) return FLUXBIN_ERR_MISALIGNED;
    }
    const int nb1 = has_salient(d) ? d.Ks : 0;
    if (!d_workspace || workspace_bytes < workspace_bytes_for(d.M, 1) + table_bytes_for(layer_units(d)))
        return FLUXBIN_ERR_WORKSPACE;
    if (!aligned(d_workspace, 16)) return FLUXBIN_ERR_MISALIGNED;
    const NormArgs norm{reinterpret_cast<const __half*>(d_gamma), eps, reinterpret_cast<__half*>(d_x_out)};
    return run_lut1h(d.M, d.N, g, has_salient(d) ? &s : nullptr, nb1, d_h, d_y, flags, d_workspace, stream, nullptr,
                     &norm);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point without a workspace argument, for callers that cannot allocate
// device memory (see fluxbin_linear_static_scratch in include/fluxbin.h).
// ---------------------------------------------------------------------------

// The scratch lives in the library's own device memory, one copy per device
// that loads the library.  In host code this name is only a stand-in for the
// symbol, not a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_fluxbin_static_scratch[FLUXBIN_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device, looked up once
// per device (with that device current) and cached.
int static_scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FLUXBIN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fluxbin_static_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return FLUXBIN_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FLUXBIN_OK;
}

}  // namespace

extern "C" int fluxbin_linear_static_scratch(const fluxbin_layer_desc* desc, const uint32_t* d_words,
                                             const uint16_t* d_r, const uint16_t* d_c, const uint32_t* d_swords,
                                             const uint16_t* d_rs, const uint16_t* d_cs, const int32_t* d_idx,
                                             const uint16_t* d_x, int32_t B, void* d_y, uint32_t flags,
                                             void* stream) {
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    if (B < 0) return FLUXBIN_ERR_BAD_SHAPE;
    if (B > kMaxBatch) return FLUXBIN_ERR_UNSUPPORTED;
    const size_t need = workspace_bytes_for(desc->M, B);
    if (need > (size_t)FLUXBIN_STATIC_SCRATCH_BYTES) return FLUXBIN_ERR_SCRATCH_LIMIT;
    if (need == 0)  // nothing to launch (M == 0 or B == 0): validate and return
        return fluxbin_linear(desc, d_words, d_r, d_c, d_swords, d_rs, d_cs, d_idx, d_x, B, d_y, flags, nullptr, 0,
                              stream);
    void* scratch = nullptr;
    const int sa = static_scratch_address(&scratch);
    if (sa != FLUXBIN_OK) return sa;
    // Plans that reduce inside a cluster or not at all never touch the
    // scratch: those calls launch the layer alone (and keep their overlap with
    // the previous kernel on the stream).  A plan that reduces through the
    // scratch first clears the part it uses, since the previous call on this
    // device may have left anything there.
    int uses = 0;
    int st2 = linear_impl(desc, d_words, d_r, d_c, d_swords, d_rs, d_cs, d_idx, d_x, B, d_y, flags, scratch,
                          (size_t)FLUXBIN_STATIC_SCRATCH_BYTES, stream, &uses);
    if (st2 != FLUXBIN_OK) return st2;
    if (uses && cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        (void)cudaGetLastError();
        return FLUXBIN_ERR_CUDA;
    }
    return linear_impl(desc, d_words, d_r, d_c, d_swords, d_rs, d_cs, d_idx, d_x, B, d_y, flags, scratch,
                       (size_t)FLUXBIN_STATIC_SCRATCH_BYTES, stream, nullptr);
}
