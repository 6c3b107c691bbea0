// Host packer and host-only queries of libfluxbin (no CUDA calls).
//
// The packer writes the +-1 bases as sign bits in uint32 words in the
// device layout defined in include/fluxbin.h ("Packed sign layout"): the
// FluxBin summary's Section 3 "LUT-Based GEMV Kernel" reads compressed
// weights with bitwise operations, and the news article on FluxBin notes the
// weights are streamed as compressed uint32 words, never rebuilt as floats.
#include <string.h>

#include <algorithm>
#include <thread>
#include <vector>

#include "fluxbin_host.h"

using namespace fluxbin;

namespace {

// Packs rows [i0, i1) of one branch.  Every row writes only the words of its
// own lane (the layout interleaves the 32 rows of a slab word by word), so
// disjoint row ranges can be packed concurrently.
int pack_rows(const int8_t* signs, int64_t M, int64_t ncols, int nb, int mu, const uint8_t* qtab, int64_t i0,
              int64_t i1, uint32_t* words) {
    const int P = subvecs_per_unit(nb);
    const int64_t U = branch_units(ncols, nb, mu);
    const int64_t cw = chunk_words(mu);
    const int64_t nsub = (ncols + mu - 1) / mu;
    for (int k = 0; k < nb; ++k) {
        for (int64_t i = i0; i < i1; ++i) {
            const int8_t* row = signs + ((int64_t)k * M + i) * ncols;
            const int L = (int)(i % kLanes);
            const uint8_t* qrow = qtab + ((size_t)L * nb + k) * P;
            uint32_t* slab = words + (i / kLanes) * U * cw + (int64_t)L * 4;
            int bad = 0;
            for (int64_t jg = 0; jg < nsub; ++jg) {
                const int64_t n0 = jg * mu;
                const int len = (int)std::min<int64_t>(mu, ncols - n0);
                uint32_t pat = 0;
                for (int t = 0; t < len; ++t) {
                    const int8_t v = row[n0 + t];
                    pat |= (uint32_t)(v == 1) << t;
                    bad |= (v != 1) & (v != -1);
                }
                const int pos = qrow[jg % P] * mu;
                slab[(jg / P) * cw + (int64_t)(pos / 128) * kLanes * 4 + (pos / 32) % 4] |= pat << (pos % 32);
            }
            if (bad) return FLUXBIN_ERR_BAD_SHAPE;
        }
    }
    return FLUXBIN_OK;
}

// Packs one branch: signs [nb][M][ncols] (+-1) -> words (device layout);
// gsv selects the visit order (see fluxbin_layout.h).
int pack_branch(const int8_t* signs, int64_t M, int64_t ncols, int nb, int mu, int gsv, uint32_t* words) {
    const int P = subvecs_per_unit(nb);
    const int64_t total = branch_words(M, ncols, nb, mu);
    memset(words, 0, (size_t)total * sizeof(uint32_t));
    std::vector<uint8_t> qtab((size_t)kLanes * nb * P);
    for (int L = 0; L < kLanes; ++L)
        for (int k = 0; k < nb; ++k)
            for (int j = 0; j < P; ++j) qtab[((size_t)L * nb + k) * P + j] = (uint8_t)visit_step(L, k, j, nb, gsv);
    const int64_t slabs = (M + kLanes - 1) / kLanes;
    const int64_t work = M * ncols * nb;
    unsigned nt = std::max(1u, std::thread::hardware_concurrency());
    if (nt > 32) nt = 32;
    if (work < (int64_t)1 << 22 || slabs < 2) nt = 1;
    if ((int64_t)nt > slabs) nt = (unsigned)slabs;
    std::vector<int> status(nt, FLUXBIN_OK);
    auto job = [&](unsigned t) {
        const int64_t s0 = slabs * t / nt, s1 = slabs * (t + 1) / nt;
        status[t] = pack_rows(signs, M, ncols, nb, mu, qtab.data(), s0 * kLanes, std::min(M, s1 * kLanes), words);
    };
    if (nt == 1) {
        job(0);
    } else {
        std::vector<std::thread> th;
        for (unsigned t = 0; t < nt; ++t) th.emplace_back(job, t);
        for (auto& x : th) x.join();
    }
    for (int st : status)
        if (st != FLUXBIN_OK) return st;
    return FLUXBIN_OK;
}

}  // namespace

extern "C" {

const char* fluxbin_status_string(int status) {
    switch (status) {
        case FLUXBIN_OK: return "ok";
        case FLUXBIN_ERR_INVALID_ARG: return "invalid argument";
        case FLUXBIN_ERR_BAD_SHAPE: return "bad shape";
        case FLUXBIN_ERR_MISALIGNED: return "misaligned pointer";
        case FLUXBIN_ERR_UNSUPPORTED: return "unsupported configuration";
        case FLUXBIN_ERR_SMEM_BUDGET: return "shared-memory budget exceeded";
        case FLUXBIN_ERR_WORKSPACE: return "workspace missing or too small";
        case FLUXBIN_ERR_CUDA: return "CUDA error";
        case FLUXBIN_ERR_SCRATCH_LIMIT: return "layer too large for the static scratch";
        default: return "unknown status";
    }
}

int fluxbin_version(void) { return 1 * 10000 + 0 * 100 + 0; }

int fluxbin_packed_sizes(const fluxbin_layer_desc* desc, size_t* words_bytes, size_t* swords_bytes) {
    if (!words_bytes || !swords_bytes) return FLUXBIN_ERR_INVALID_ARG;
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    *words_bytes = (size_t)branch_words(desc->M, desc->N, desc->Kb, desc->mu) * sizeof(uint32_t);
    *swords_bytes = has_salient(*desc)
        ? (size_t)branch_words(desc->M, desc->n_sal, desc->Ks, desc->mu) * sizeof(uint32_t) : 0;
    return FLUXBIN_OK;
}

int fluxbin_pack(const fluxbin_layer_desc* desc, const int8_t* signs, const int8_t* sal_signs,
                 const int32_t* sal_idx, uint32_t* words_out, uint32_t* swords_out) {
    const int st = validate_desc(desc);
    if (st != FLUXBIN_OK) return st;
    const fluxbin_layer_desc& d = *desc;
    const int64_t nw = branch_words(d.M, d.N, d.Kb, d.mu);
    if (nw > 0 && (!signs || !words_out)) return FLUXBIN_ERR_INVALID_ARG;
    if (has_salient(d)) {
        if (!sal_signs || !sal_idx || !swords_out) return FLUXBIN_ERR_INVALID_ARG;
        for (int32_t t = 0; t < d.n_sal; ++t) {
            if (sal_idx[t] < 0 || sal_idx[t] >= d.N) return FLUXBIN_ERR_BAD_SHAPE;
            if (t > 0 && sal_idx[t] <= sal_idx[t - 1]) return FLUXBIN_ERR_BAD_SHAPE;
        }
    }
    if (nw > 0) {
        const int r = pack_branch(signs, d.M, d.N, d.Kb, d.mu, subvecs_per_unit(d.Kb), words_out);
        if (r != FLUXBIN_OK) return r;
    }
    if (has_salient(d) && branch_words(d.M, d.n_sal, d.Ks, d.mu) > 0) {
        const int r = pack_branch(sal_signs, d.M, d.n_sal, d.Ks, d.mu, group_subvecs(d.Ks, d.mu, d.sal_scale_group),
                                  swords_out);
        if (r != FLUXBIN_OK) return r;
    }
    return FLUXBIN_OK;
}

int fluxbin_workspace_bytes(int32_t M, int32_t B, size_t* bytes) {
    if (!bytes) return FLUXBIN_ERR_INVALID_ARG;
    if (M < 0 || B < 0) return FLUXBIN_ERR_BAD_SHAPE;
    *bytes = workspace_bytes_for(M, B);
    return FLUXBIN_OK;
}

}  // extern "C"
