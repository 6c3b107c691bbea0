// Host-side FluxBin decomposition fitting: finds the +-1 bases and the row and
// column scales of W ~= sum_k diag(r_k) B_k diag(c_k) (plus the salient
// refinement on chosen columns) by alternating minimisation of the weighted
// reconstruction error.  Declarations and the full contract are in
// include/fluxbin.h ("Decomposition fitting").
//
// FluxBin summary, Section 3 "Parameter Optimization" (alternating
// minimisation, joint evaluation of all 2^Kb sign combinations), Appendix A.1
// (closed-form scales: with the bases and the other scale fixed, one scalar
// least-squares problem per row or column), Appendix A.2 (element-wise
// exhaustive sign search, globally optimal for fixed scales), Section 3
// "Salient-Aware Hybrid Bases" (the salient branch fits the global residual on
// the salient columns with its own bases), Appendix C.2 (block-wise row
// scales).
//
// Work is split over host threads by fixed blocks of rows; every reduction
// over rows adds the blocks' partial sums in block order, so the result does
// not depend on the number of threads.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "fluxbin_host.h"

namespace fluxbin {
namespace {

constexpr int kRowBlock = 64;   // rows per work block
constexpr int kMaxFitBases = 8;

// Runs f(block) for every block 0..n_blocks-1 on up to hardware_concurrency threads.
template <typename F>
void parallel_blocks(int64_t n_blocks, F&& f) {
    unsigned hw = std::thread::hardware_concurrency();
    int64_t nt = std::min<int64_t>(n_blocks, hw ? (int64_t)hw : 1);
    if (nt <= 1) {
        for (int64_t b = 0; b < n_blocks; ++b) f(b);
        return;
    }
    std::vector<std::thread> ts;
    ts.reserve((size_t)nt);
    for (int64_t t = 0; t < nt; ++t)
        ts.emplace_back([&, t]() {
            for (int64_t b = t; b < n_blocks; b += nt) f(b);
        });
    for (auto& th : ts) th.join();
}

// One branch being fitted: W [M][N] (row stride ldw), column weights h [N],
// bases B [nb][M][N] (+1/-1), row scales r [nb][M] (G == 0) or [nb][ng][M],
// column scales c [nb][N].
struct Branch {
    int64_t M, N;
    int nb, G;
    int64_t ng;
    const double* W;
    int64_t ldw;
    const double* h;
    int8_t* B;
    double* r;
    double* c;

    int64_t group(int64_t j) const { return G > 0 ? j / G : 0; }
    double rs(int k, int64_t i, int64_t j) const { return r[((int64_t)k * ng + group(j)) * M + i]; }
    double& rs_at(int k, int64_t g, int64_t i) { return r[((int64_t)k * ng + g) * M + i]; }
    int8_t b(int k, int64_t i, int64_t j) const { return B[((int64_t)k * M + i) * N + j]; }
    int8_t& b_at(int k, int64_t i, int64_t j) { return B[((int64_t)k * M + i) * N + j]; }
    // W_ij minus every base except `skip` (skip = -1: minus all bases)
    double residual(int64_t i, int64_t j, int skip) const {
        double v = W[i * ldw + j];
        for (int l = 0; l < nb; ++l)
            if (l != skip) v -= rs(l, i, j) * (double)b(l, i, j) * c[(int64_t)l * N + j];
        return v;
    }
};

// Appendix A.1, row scales of base k: per row (block) sum_j h_j R_ij B_ij c_j /
// sum_j h_j c_j^2 with R the residual of the other bases.
void update_rows(Branch& br, int k) {
    const int64_t N = br.N;
    std::vector<double> den((size_t)br.ng, 0.0);
    for (int64_t j = 0; j < N; ++j) den[(size_t)br.group(j)] += br.h[j] * br.c[(int64_t)k * N + j] * br.c[(int64_t)k * N + j];
    const int64_t nblk = (br.M + kRowBlock - 1) / kRowBlock;
    parallel_blocks(nblk, [&](int64_t blk) {
        std::vector<double> num((size_t)br.ng);
        for (int64_t i = blk * kRowBlock; i < std::min(br.M, (blk + 1) * kRowBlock); ++i) {
            std::fill(num.begin(), num.end(), 0.0);
            for (int64_t j = 0; j < N; ++j)
                num[(size_t)br.group(j)] += br.h[j] * br.residual(i, j, k) * (double)br.b(k, i, j) * br.c[(int64_t)k * N + j];
            for (int64_t g = 0; g < br.ng; ++g) br.rs_at(k, g, i) = den[(size_t)g] != 0.0 ? num[(size_t)g] / den[(size_t)g] : 0.0;
        }
    });
}

// The matching closed form for the column scales of base k:
// c_j = sum_i R_ij B_ij r_i(j) / sum_i r_i(j)^2 (h_j cancels within a column).
void update_cols(Branch& br, int k) {
    const int64_t N = br.N;
    const int64_t nblk = (br.M + kRowBlock - 1) / kRowBlock;
    std::vector<double> num((size_t)(nblk * N), 0.0), den((size_t)(nblk * N), 0.0);
    parallel_blocks(nblk, [&](int64_t blk) {
        double* pn = num.data() + blk * N;
        double* pd = den.data() + blk * N;
        for (int64_t i = blk * kRowBlock; i < std::min(br.M, (blk + 1) * kRowBlock); ++i)
            for (int64_t j = 0; j < N; ++j) {
                const double ri = br.rs(k, i, j);
                pn[j] += br.residual(i, j, k) * (double)br.b(k, i, j) * ri;
                pd[j] += ri * ri;
            }
    });
    for (int64_t j = 0; j < N; ++j) {
        double sn = 0.0, sd = 0.0;
        for (int64_t blk = 0; blk < nblk; ++blk) {
            sn += num[(size_t)(blk * N + j)];
            sd += den[(size_t)(blk * N + j)];
        }
        br.c[(int64_t)k * N + j] = sd != 0.0 ? sn / sd : 0.0;
    }
}

// Appendix A.2: every element takes the sign combination (first of equals in
// the order p = 0 .. 2^nb - 1, bit k of p set meaning +1) that minimises its
// squared error.
void search_signs(Branch& br) {
    const int64_t N = br.N;
    const int nb = br.nb;
    const int64_t nblk = (br.M + kRowBlock - 1) / kRowBlock;
    parallel_blocks(nblk, [&](int64_t blk) {
        double s[kMaxFitBases];
        for (int64_t i = blk * kRowBlock; i < std::min(br.M, (blk + 1) * kRowBlock); ++i)
            for (int64_t j = 0; j < N; ++j) {
                for (int k = 0; k < nb; ++k) s[k] = br.rs(k, i, j) * br.c[(int64_t)k * N + j];
                const double w = br.W[i * br.ldw + j];
                double best = INFINITY;
                int bp = 0;
                for (int p = 0; p < (1 << nb); ++p) {
                    double a = 0.0;
                    for (int k = 0; k < nb; ++k) a += ((p >> k) & 1) ? s[k] : -s[k];
                    const double e = (w - a) * (w - a);
                    if (e < best) {
                        best = e;
                        bp = p;
                    }
                }
                for (int k = 0; k < nb; ++k) br.b_at(k, i, j) = ((bp >> k) & 1) ? 1 : -1;
            }
    });
}

// Greedy residual start: B_k = sign(R) (sign(0) = +1), c_k = 1, r_k by the
// row closed form with c = 1, then the next base on what is left.
void init_greedy(Branch& br) {
    const int64_t N = br.N;
    for (int k = 0; k < br.nb; ++k) {
        for (int64_t j = 0; j < N; ++j) br.c[(int64_t)k * N + j] = 1.0;
        const int64_t nblk = (br.M + kRowBlock - 1) / kRowBlock;
        // signs of the residual of the bases already placed (k is not yet part of it)
        parallel_blocks(nblk, [&](int64_t blk) {
            for (int64_t i = blk * kRowBlock; i < std::min(br.M, (blk + 1) * kRowBlock); ++i)
                for (int64_t j = 0; j < N; ++j) {
                    double v = br.W[i * br.ldw + j];
                    for (int l = 0; l < k; ++l) v -= br.rs(l, i, j) * (double)br.b(l, i, j) * br.c[(int64_t)l * N + j];
                    br.b_at(k, i, j) = v >= 0.0 ? 1 : -1;
                }
        });
        // bases after k do not exist yet: zero their scales so residual(.., k) sees only 0..k-1
        for (int l = k + 1; l < br.nb; ++l) {
            for (int64_t q = 0; q < br.ng * br.M; ++q) br.r[(int64_t)l * br.ng * br.M + q] = 0.0;
            for (int64_t j = 0; j < N; ++j) br.c[(int64_t)l * N + j] = 0.0;
        }
        update_rows(br, k);
    }
}

double weighted_error(const Branch& br) {
    const int64_t nblk = (br.M + kRowBlock - 1) / kRowBlock;
    std::vector<double> part((size_t)nblk, 0.0);
    parallel_blocks(nblk, [&](int64_t blk) {
        double s = 0.0;
        for (int64_t i = blk * kRowBlock; i < std::min(br.M, (blk + 1) * kRowBlock); ++i)
            for (int64_t j = 0; j < br.N; ++j) {
                const double e = br.residual(i, j, -1);
                s += br.h[j] * e * e;
            }
        part[(size_t)blk] = s;
    });
    double t = 0.0;
    for (double v : part) t += v;
    return t;
}

void fit_branch(Branch& br, int iters) {
    init_greedy(br);
    for (int it = 0; it < iters; ++it) {
        for (int k = 0; k < br.nb; ++k) {
            update_rows(br, k);
            update_cols(br, k);
        }
        search_signs(br);
    }
}

int check_fit_args(int64_t M, int64_t N, int nb, int G, int iters) {
    if (M < 0 || N < 0 || G < 0 || iters < 0) return FLUXBIN_ERR_BAD_SHAPE;
    if (nb < 1 || nb > kMaxFitBases) return FLUXBIN_ERR_UNSUPPORTED;
    return FLUXBIN_OK;
}

}  // namespace
}  // namespace fluxbin

using namespace fluxbin;

extern "C" int fluxbin_fit(int32_t M, int32_t N, int32_t nbases, int32_t row_scale_group, int32_t iters,
                           const double* W, const double* col_weight, int8_t* signs_out, double* r_out,
                           double* c_out, double* objective_out) {
    int st = check_fit_args(M, N, nbases, row_scale_group, iters);
    if (st != FLUXBIN_OK) return st;
    if ((int64_t)M * N > 0 && (!W || !signs_out || !r_out || !c_out)) return FLUXBIN_ERR_INVALID_ARG;
    std::vector<double> ones;
    if (!col_weight) {
        ones.assign((size_t)N, 1.0);
        col_weight = ones.data();
    }
    for (int32_t j = 0; j < N; ++j)
        if (!(col_weight[j] >= 0.0)) return FLUXBIN_ERR_BAD_SHAPE;
    Branch br{M, N, nbases, row_scale_group, row_scale_group > 0 ? (N + row_scale_group - 1) / row_scale_group : 1,
              W, N, col_weight, signs_out, r_out, c_out};
    if ((int64_t)M * N > 0) fit_branch(br, iters);
    if (objective_out) *objective_out = (int64_t)M * N > 0 ? weighted_error(br) : 0.0;
    return FLUXBIN_OK;
}

extern "C" int fluxbin_fit_hybrid(int32_t M, int32_t N, int32_t Kb, int32_t row_scale_group, int32_t Ks,
                                  int32_t n_sal, const int32_t* sal_idx, int32_t sal_scale_group, int32_t iters,
                                  const double* W, const double* col_weight, int8_t* signs_out, double* r_out,
                                  double* c_out, int8_t* sal_signs_out, double* rs_out, double* cs_out,
                                  double* objective_out) {
    int st = check_fit_args(M, N, Kb, row_scale_group, iters);
    if (st != FLUXBIN_OK) return st;
    if (n_sal < 0 || n_sal > N || sal_scale_group < 0) return FLUXBIN_ERR_BAD_SHAPE;
    const bool sal = Ks > 0 && n_sal > 0;
    if (sal) {
        st = check_fit_args(M, n_sal, Ks, sal_scale_group, iters);
        if (st != FLUXBIN_OK) return st;
        if (!sal_idx || !sal_signs_out || !rs_out || !cs_out) return FLUXBIN_ERR_INVALID_ARG;
        for (int32_t t = 0; t < n_sal; ++t)
            if (sal_idx[t] < 0 || sal_idx[t] >= N || (t > 0 && sal_idx[t] <= sal_idx[t - 1])) return FLUXBIN_ERR_BAD_SHAPE;
    } else if (Ks < 0) {
        return FLUXBIN_ERR_BAD_SHAPE;
    }
    std::vector<double> ones;
    if (!col_weight) {
        ones.assign((size_t)N, 1.0);
        col_weight = ones.data();
    }
    st = fluxbin_fit(M, N, Kb, row_scale_group, iters, W, col_weight, signs_out, r_out, c_out, nullptr);
    if (st != FLUXBIN_OK) return st;
    if (!sal) {
        if (objective_out) {
            Branch br{M, N, Kb, row_scale_group, row_scale_group > 0 ? (N + row_scale_group - 1) / row_scale_group : 1,
                      W, N, col_weight, signs_out, r_out, c_out};
            *objective_out = (int64_t)M * N > 0 ? weighted_error(br) : 0.0;
        }
        return FLUXBIN_OK;
    }
    // the global residual gathered at the salient columns (dense M x n_sal)
    Branch gb{M, N, Kb, row_scale_group, row_scale_group > 0 ? (N + row_scale_group - 1) / row_scale_group : 1,
              W, N, col_weight, signs_out, r_out, c_out};
    std::vector<double> R((size_t)M * n_sal), hs((size_t)n_sal);
    for (int32_t t = 0; t < n_sal; ++t) hs[(size_t)t] = col_weight[sal_idx[t]];
    parallel_blocks(((int64_t)M + kRowBlock - 1) / kRowBlock, [&](int64_t blk) {
        for (int64_t i = blk * kRowBlock; i < std::min<int64_t>(M, (blk + 1) * kRowBlock); ++i)
            for (int32_t t = 0; t < n_sal; ++t) R[(size_t)(i * n_sal + t)] = gb.residual(i, sal_idx[t], -1);
    });
    st = fluxbin_fit(M, n_sal, Ks, sal_scale_group, iters, R.data(), hs.data(), sal_signs_out, rs_out, cs_out,
                     nullptr);
    if (st != FLUXBIN_OK) return st;
    if (objective_out) {
        // global error outside S plus the salient branch's error on S
        Branch sb{M, n_sal, Ks, sal_scale_group, sal_scale_group > 0 ? (n_sal + sal_scale_group - 1) / sal_scale_group : 1,
                  R.data(), n_sal, hs.data(), sal_signs_out, rs_out, cs_out};
        double e = weighted_error(sb);
        std::vector<char> in_s((size_t)N, 0);
        for (int32_t t = 0; t < n_sal; ++t) in_s[(size_t)sal_idx[t]] = 1;
        for (int64_t i = 0; i < M; ++i)
            for (int64_t j = 0; j < N; ++j)
                if (!in_s[(size_t)j]) {
                    const double v = gb.residual(i, j, -1);
                    e += col_weight[j] * v * v;
                }
        *objective_out = e;
    }
    return FLUXBIN_OK;
}
