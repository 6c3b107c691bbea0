// Host-side validation shared by the packer and the device entry points.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/fluxbin.h"
#include "fluxbin_layout.h"

namespace fluxbin {

inline bool valid_nb(int nb) { return nb == 1 || nb == 2 || nb == 4; }
inline bool valid_mu(int mu) { return mu == 4 || mu == 8; }

inline bool has_salient(const fluxbin_layer_desc& d) { return d.Ks > 0 && d.n_sal > 0; }

// Salient row-scale groups: whole units, or a power-of-two number of whole
// sub-vectors (1, 2 or 4) that divides a unit (grouped visit order).
inline bool valid_salient_group(int nb, int mu, int s) {
    const int w = unit_cols(nb, mu);
    if (s % w == 0) return true;
    if (s % mu) return false;
    const int g = s / mu;
    return (g == 1 || g == 2 || g == 4) && w % s == 0;
}

// Checks the shape fields of a layer description.
inline int validate_desc(const fluxbin_layer_desc* d) {
    if (!d) return FLUXBIN_ERR_INVALID_ARG;
    if (d->M < 0 || d->N < 0 || d->n_sal < 0 || d->row_scale_group < 0 || d->sal_scale_group < 0)
        return FLUXBIN_ERR_BAD_SHAPE;
    if (!valid_mu(d->mu) || !valid_nb(d->Kb)) return FLUXBIN_ERR_UNSUPPORTED;
    if (d->Ks != 0 && !valid_nb(d->Ks)) return FLUXBIN_ERR_UNSUPPORTED;
    if (d->n_sal > d->N) return FLUXBIN_ERR_BAD_SHAPE;
    if (d->Ks == 0 && d->n_sal != 0) return FLUXBIN_ERR_BAD_SHAPE;
    // block-wise row scales: a block must hold whole units, so that the scale
    // is constant across the unit a CTA accumulates before applying it
    if (d->row_scale_group > 0 && d->row_scale_group % unit_cols(d->Kb, d->mu)) return FLUXBIN_ERR_UNSUPPORTED;
    if (has_salient(*d) && d->sal_scale_group > 0 && !valid_salient_group(d->Ks, d->mu, d->sal_scale_group))
        return FLUXBIN_ERR_UNSUPPORTED;
    return FLUXBIN_OK;
}

inline size_t workspace_bytes_for(int64_t M, int64_t B) {
    if (M <= 0 || B <= 0) return 0;
    const int64_t Mp = row_slabs(M) * kLanes;
    const int64_t n_rg = (row_slabs(M) + kSlabsPerCta - 1) / kSlabsPerCta;
    size_t acc = (size_t)(B * Mp) * sizeof(float);
    acc = (acc + 255) & ~(size_t)255;
    // arrival counters: one per 512-row group and batch chunk (LUT path) or
    // one per 128-row tile (tensor-core path), whichever is more
    const int64_t n_rt = (row_slabs(M) + 3) / 4;
    size_t cnt = (size_t)(n_rg * B > n_rt ? n_rg * B : n_rt) * sizeof(unsigned int);
    return acc + ((cnt + 255) & ~(size_t)255);
}

// Table buffer of the batch-1 path with the precompute as its own kernel:
// one 64 KiB block per pair of units (fluxbin_tables.cuh).
inline size_t table_bytes_for(int64_t units) { return units > 0 ? (size_t)((units + 1) / 2) * 65536u : 0u; }

// Whether a layer at batch B can run its table precompute as a separate
// kernel (batch 1, mu = 8, per-row scales in both branches).
inline bool hoistable(const fluxbin_layer_desc& d, int64_t B) {
    return B == 1 && d.mu == 8 && d.row_scale_group == 0 && (!has_salient(d) || d.sal_scale_group == 0);
}

inline int64_t layer_units(const fluxbin_layer_desc& d) {
    return branch_units(d.N, d.Kb, d.mu) + (has_salient(d) ? branch_units(d.n_sal, d.Ks, d.mu) : 0);
}

}  // namespace fluxbin
