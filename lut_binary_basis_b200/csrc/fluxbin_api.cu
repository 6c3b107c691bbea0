// C-ABI device entry points of libfluxbin: argument validation, kernel
// selection, grid sizing and the launch.  Declarations and the full contract
// are in include/fluxbin.h.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "fluxbin_host.h"
#include "fluxbin_kernel.cuh"

namespace fluxbin {

using KernelFn = void (*)(KernelArgs);
KernelFn select_kernel_mu8(int nb0, int nb1, int bt);
KernelFn select_kernel_mu4(int nb0, int nb1, int bt);

namespace {

// Batch rows whose tables a CTA keeps resident (the rest go to other CTAs).
int batch_tile(int mu, int B) {
    if (mu == 8) return B <= 1 ? 1 : 2;
    return B <= 1 ? 1 : (B <= 2 ? 2 : 4);
}

size_t table_smem_bytes(int mu, int bt) { return (size_t)bt * ((size_t)1 << mu) * 256u; }

struct LaunchInfo {
    int blocks_per_sm = 0;
    int sm_count = 0;
    int max_smem = 0;
};

std::mutex g_mu;
std::unordered_map<uint64_t, LaunchInfo> g_info;

int launch_info(KernelFn fn, size_t smem, LaunchInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FLUXBIN_ERR_CUDA;
    const uint64_t key = (reinterpret_cast<uint64_t>(fn) << 8) ^ (uint64_t)dev;
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_info.find(key);
    if (it != g_info.end()) {
        *out = it->second;
        return FLUXBIN_OK;
    }
    LaunchInfo li;
    if (cudaDeviceGetAttribute(&li.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&li.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return FLUXBIN_ERR_CUDA;
    if ((size_t)li.max_smem < smem + 1024) return FLUXBIN_ERR_SMEM_BUDGET;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return FLUXBIN_ERR_CUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&li.blocks_per_sm, fn, kThreads, smem) != cudaSuccess)
        return FLUXBIN_ERR_CUDA;
    if (li.blocks_per_sm < 1) return FLUXBIN_ERR_SMEM_BUDGET;
    g_info.emplace(key, li);
    *out = li;
    return FLUXBIN_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct BranchIn {
    const uint32_t* words;
    const uint16_t* r;
    const uint16_t* c;
    const int32_t* gather;
    int32_t ncols, nb, rgroup;
};

int run(int32_t M, int32_t N, int mu, const BranchIn& g, const BranchIn* s, const uint16_t* d_x, int32_t B,
        void* d_y, uint32_t flags, void* ws, size_t ws_bytes, void* stream) {
    if (flags & ~(kFlagAccumulate | kFlagYFp32 | kFlagEarlyWeights)) return FLUXBIN_ERR_INVALID_ARG;
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
    const int bt = batch_tile(mu, B);
    KernelFn fn = mu == 8 ? select_kernel_mu8(g.nb, nb1, bt) : select_kernel_mu4(g.nb, nb1, bt);
    if (!fn) return FLUXBIN_ERR_UNSUPPORTED;
    const size_t smem = table_smem_bytes(mu, bt);
    LaunchInfo li;
    int st = launch_info(fn, smem, &li);
    if (st != FLUXBIN_OK) return st;

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
    a.x = reinterpret_cast<const __half*>(d_x);
    a.y = d_y;
    a.M = M;
    a.N = N;
    a.B = B;
    a.Ms = (int32_t)row_slabs(M);
    a.Mp = a.Ms * kLanes;
    a.n_rg = (a.Ms + kSlabsPerCta - 1) / kSlabsPerCta;
    a.n_bc = (B + bt - 1) / bt;
    a.flags = flags;
    const int64_t U = (int64_t)a.br[0].units + a.br[1].units;
    const int64_t groups = (int64_t)a.n_rg * a.n_bc;
    const int64_t target = (int64_t)li.sm_count * li.blocks_per_sm;
    int64_t ks = (target + groups / 2) / groups;
    if (ks > U) ks = U;
    if (ks < 1) ks = 1;
    a.n_ks = (int32_t)ks;
    if (a.n_ks > 1) {
        const size_t need = workspace_bytes_for(M, B);
        if (!ws || ws_bytes < need) return FLUXBIN_ERR_WORKSPACE;
        if (!aligned(ws, 16)) return FLUXBIN_ERR_MISALIGNED;
        const size_t acc = (((size_t)B * a.Mp * sizeof(float)) + 255) & ~(size_t)255;
        a.ws_acc = static_cast<float*>(ws);
        a.ws_cnt = reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + acc);
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(groups * a.n_ks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, a) != cudaSuccess) {
        (void)cudaGetLastError();
        return FLUXBIN_ERR_CUDA;
    }
    return FLUXBIN_OK;
}

}  // namespace
}  // namespace fluxbin

using namespace fluxbin;

extern "C" {

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
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    const fluxbin_layer_desc& d = *desc;
    BranchIn g{d_words, d_r, d_c, nullptr, d.N, d.Kb, d.row_scale_group};
    BranchIn s{d_swords, d_rs, d_cs, d_idx, has_salient(d) ? d.n_sal : 0, d.Ks ? d.Ks : 1, d.sal_scale_group};
    if (has_salient(d) && !d_idx) return FLUXBIN_ERR_INVALID_ARG;
    return run(d.M, d.N, d.mu, g, has_salient(d) ? &s : nullptr, d_x, B, d_y, flags, d_workspace,
               workspace_bytes, stream);
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
    // the previous call on this device may have left anything there
    if (cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        (void)cudaGetLastError();
        return FLUXBIN_ERR_CUDA;
    }
    return fluxbin_linear(desc, d_words, d_r, d_c, d_swords, d_rs, d_cs, d_idx, d_x, B, d_y, flags, scratch,
                          (size_t)FLUXBIN_STATIC_SCRATCH_BYTES, stream);
}
