/*
 * fluxbin.h -- C-ABI of the B200 (sm_100a) FluxBin LUT GEMV library, libfluxbin.so.
 *
 * FluxBin ("FluxBin: Flexible LUT-based Ultra-low-bit LLM Inference by
 * Algorithm-Kernel Synergy") stores a weight matrix W (M rows = output
 * features, N columns = input features) as
 *
 *     W = sum_{k < Kb} diag(r_k) B_k diag(c_k)                       (global branch)
 *       + salient refinement on a column set S, |S| = n_sal:
 *         sum_{s < Ks} diag(rs_s) Bs_s diag(cs_s), column t of Bs_s being column S[t] of W
 *
 * with B_k, Bs_s in {-1,+1} (summary, Section 3 "Quantization" and "Salient-
 * Aware Hybrid Bases").  The library evaluates y = W x for a batch of fp16
 * activations without ever forming a floating-point W: for every sub-vector
 * of mu activation columns it builds a table of the 2^mu signed partial sums
 * of c (.) x (scale fusion, Section 3 "LUT-Based GEMV Kernel", Appendix C.1),
 * streams the packed sign bits from HBM, uses each mu-bit pattern as a table
 * index, accumulates in fp32 and applies the row scale after accumulation.
 * The salient branch runs through the same kernel on its dense M x n_sal
 * sign matrix, its activations and scales gathered through S at run time
 * (Section 3 "Virtual Columnar Mapping").
 *
 * Conventions for every entry point:
 *   - Return value: FLUXBIN_OK (0) or a negative fluxbin_status.  No call
 *     throws, aborts or prints.  Arguments are validated before any CUDA call,
 *     so an argument error leaves the device and the stream untouched.
 *   - fp16 values travel as uint16_t bit patterns (IEEE binary16).
 *   - Pointers named d_* are device pointers, owned by the caller, never freed
 *     or retained after the call returns; no call allocates device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Device calls are asynchronous on that stream: they launch and
 *     return without synchronising.
 *   - Only one GPU architecture is built: sm_100a (B200).  Launch failures
 *     are reported as FLUXBIN_ERR_CUDA.
 *
 * ---------------------------------------------------------------------------
 * Packed sign layout (the device layout; a pure index function)
 * ---------------------------------------------------------------------------
 * One branch (the global one: nb = Kb bases over ncols = N columns; the
 * salient one: nb = Ks bases over ncols = n_sal dense columns) with
 * sub-vector length mu in {4, 8} and nb in {1, 2, 4} is stored as follows.
 *
 *   P  = 32 / nb            sub-vectors of one base in a unit
 *   U  = ceil(ncols / (P*mu)) units: column blocks of P*mu columns
 *   Ms = ceil(M / 32)       row slabs of 32 rows
 *   words: Ms * U chunks, chunk (s, u) at word offset (s*U + u) * 32*mu,
 *          each chunk 32*mu uint32 words (1 KiB for mu = 8, 512 B for mu = 4).
 *
 * The sign of base k at row i and column n (n < ncols) is one bit, set for
 * +1 and clear for -1; every padding bit (rows >= M, columns >= ncols) is 0:
 *   s = i / 32, L = i % 32                      row slab and lane
 *   jg = n / mu, t = n % mu                     sub-vector and bit within it
 *   u = jg / P, j = jg % P                      unit and sub-vector within it
 *   a = (k - L/P) mod nb                        (mod taken in 0..nb-1)
 *   q = a*P + ((j - L) mod P)                   step at which lane L visits it
 *   pos  = q*mu + t
 *   word = (s*U + u)*32*mu + ((pos / 128)*32 + L)*4 + (pos / 32) % 4
 *   bit  = pos % 32
 *
 * Grouped order.  A salient branch whose row scales change every Gs salient
 * columns with Gs a multiple of mu and gsv = Gs/mu in {1, 2, 4} dividing P
 * (sal_scale_group smaller than a unit) uses instead, with KG = 32/gsv and
 * NG = P/gsv, lane L = gsv*m + sg (m = L/gsv, sg = L%gsv):
 *   kg = k*NG + j/gsv,  a = (kg - m) mod KG,  q = a*gsv + ((j % gsv) xor sg)
 * so that the steps a*gsv .. a*gsv+gsv-1 of a lane cover one whole (base,
 * scale group) and the lane can apply that group's row scale once.
 *
 * Reading: lane L of a warp owns row 32*s + L.  Over its 32 steps q it visits
 * the unit's 32 (base, sub-vector) tables in the order
 *   base k = (q/P + L/P) mod nb, sub-vector j = (L + q) mod P,
 * so at every step the 32 lanes read 32 different tables.  Table (k, j) lives
 * in shared-memory bank k*P + j; no two lanes ever hit the same bank.  The
 * 32*mu bits a lane consumes for one unit are contiguous (mu/4 128-bit words,
 * interleaved across the warp's lanes so that every warp load is one
 * contiguous 512-byte line).
 *
 * ---------------------------------------------------------------------------
 * Scale layouts (fp16)
 * ---------------------------------------------------------------------------
 *   c  [Kb][N], cs [Ks][n_sal]                  column scales
 *   r  [Kb][M]            (row_scale_group == 0: one per row)
 *   r  [Kb][ceil(N/G)][M] (row_scale_group == G > 0: one per row per G-column
 *                          block, Appendix C.2 "block-wise row scales")
 *   rs [Ks][M] or [Ks][ceil(n_sal/Gs)][M]       (sal_scale_group == Gs: a multiple of
 *                                               the unit width, or Gs = gsv*mu as above)
 *   x  [B][N], y [B][M] (row-major; y fp16 or fp32)
 *   idx[n_sal] int32, strictly increasing, < N  (the salient column set S)
 */
#ifndef FLUXBIN_H
#define FLUXBIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fluxbin_status {
    FLUXBIN_OK = 0,
    FLUXBIN_ERR_INVALID_ARG = -1,  /* null pointer where data is needed, bad flag */
    FLUXBIN_ERR_BAD_SHAPE = -2,    /* negative or inconsistent sizes, bad salient index list */
    FLUXBIN_ERR_MISALIGNED = -3,   /* a device pointer lacks the alignment stated below */
    FLUXBIN_ERR_UNSUPPORTED = -4,  /* mu not in {4,8}; Kb not in {1,2,4}; Ks not in {0,1,2,4};
                                      B > 16; a row-scale block that does not hold whole units
                                      (salient: nor 1, 2 or 4 whole sub-vectors) */
    FLUXBIN_ERR_SMEM_BUDGET = -5,  /* the tables for this shape do not fit in shared memory */
    FLUXBIN_ERR_WORKSPACE = -6,    /* workspace missing or smaller than fluxbin_workspace_bytes() */
    FLUXBIN_ERR_CUDA = -7,         /* a CUDA runtime call or the kernel launch failed */
    FLUXBIN_ERR_SCRATCH_LIMIT = -8 /* the layer needs more scratch than FLUXBIN_STATIC_SCRATCH_BYTES */
} fluxbin_status;

/* Plain-old-data description of one layer. */
typedef struct fluxbin_layer_desc {
    int32_t M;                /* output features (rows of W), >= 0 */
    int32_t N;                /* input features (columns of W), >= 0 */
    int32_t Kb;               /* global bases: 1, 2 or 4 */
    int32_t Ks;               /* salient bases: 0 (no salient branch), 1, 2 or 4 */
    int32_t n_sal;            /* salient columns, 0 <= n_sal <= N (0 when Ks == 0) */
    int32_t mu;               /* LUT sub-vector length: 4 or 8 */
    int32_t row_scale_group;  /* 0: one row scale per row; G > 0: one per row per G columns */
    int32_t sal_scale_group;  /* 0: one salient row scale per row; Gs > 0: one per Gs salient columns
                                 (a multiple of the unit width (32/Ks)*mu, or mu, 2*mu or 4*mu
                                 dividing it: grouped visit order) */
} fluxbin_layer_desc;

/* Flags for the device entry points. */
#define FLUXBIN_FLAG_ACCUMULATE   1u  /* y += W x (else y = W x) */
#define FLUXBIN_FLAG_Y_FP32       2u  /* y is float32 (else fp16, round to nearest even) */
#define FLUXBIN_FLAG_EARLY_WEIGHTS 4u /* programmatic dependent launch: start streaming this
                                         layer's packed signs before the preceding kernel on the
                                         stream has finished.  The caller promises that no kernel
                                         still running before this call writes the layer's packed
                                         words.  x, y, scales and workspace are always read only
                                         after the preceding kernel has completed. */
#define FLUXBIN_FLAG_PATH_LUT     8u  /* always use the LUT path */
#define FLUXBIN_FLAG_PATH_TC      16u /* always use the tensor-core path (UNSUPPORTED when the layer
                                         does not qualify, WORKSPACE without a workspace) */
#define FLUXBIN_FLAG_SEPARATE_TABLES 64u /* batch 1, mu = 8, per-row scales: build every unit's tables
                                         once in a kernel of its own (the precompute as a separate
                                         operator) and look them up from shared-memory copies of the
                                         table buffer; needs fluxbin_layer_workspace_bytes() of
                                         workspace (WORKSPACE otherwise), UNSUPPORTED for other
                                         layers, INVALID_ARG with FLUXBIN_FLAG_PATH_TC.  The table
                                         buffer (the bytes from fluxbin_workspace_bytes(M, 1) on) is
                                         left holding the tables: only the bytes before it are left
                                         zero-filled, so a workspace shared with other calls must not
                                         put that buffer where they need zeros.  Measured slower
                                         than the default on B200 (see the batch-1 kernels). */
#define FLUXBIN_FLAG_TEST_WAIT_TIMEOUT 32u /* test hook, only together with FLUXBIN_FLAG_PATH_TC: the
                                         tensor-core kernel's preparing warps never report a buffer
                                         ready and every wait gives up after a few polls, so the
                                         give-up path runs: the outputs become NaN, bit 0 of
                                         fluxbin_device_status is set, no MMA is issued, tensor
                                         memory is released and the workspace is left zero-filled.
                                         INVALID_ARG without FLUXBIN_FLAG_PATH_TC. */
/*
 * Two execution paths compute the same layer.  The LUT path builds the 2^mu
 * signed partial sums of every activation sub-vector in shared memory and
 * looks them up with the packed bit patterns (FluxBin summary, Section 3
 * "LUT-Based GEMV Kernel").  At mu = 8 with per-row scales and a batch of 2 or
 * more (batch 2 only above 4096 x 4096), the LUT path keeps the tables of two
 * batch rows in one fp16 pair per entry (table quantisation to fp16, LUT Tensor
 * Core notes, Section 3.1.3): one lookup serves both rows; the entries are
 * rounded to fp16 once and the entries of two consecutive steps are added in
 * fp16 before the fp32 accumulation (relative error of y about 3e-4 on the
 * benchmark layers).  The tensor-core path expands the +-1 signs of each unit
 * into fp16 in shared memory only and contracts them with the fp16 products
 * c (.) x on the tensor cores (tcgen05.mma), fp32 accumulation in tensor
 * memory, row scales applied to the accumulators (the LUT Tensor Core notes,
 * Section 2.2, read LUT-based mixed-precision GEMM as a GEMM with one low-bit
 * operand).  It needs mu == 4 or 8, per-row scales (row_scale_group == 0 and
 * sal_scale_group == 0) and a workspace; it is taken by default only for
 * mu = 4 layers with B >= 16 and M * N > 4096 * 4096, or B >= 8 and
 * M >= 16384 (where it measured faster on B200), and may be forced either way
 * with the flags above.  Its products are rounded to fp16 before the
 * contraction (relative error below 2^-11 per product).
 */

/* Human-readable name of a status code (static storage, never NULL). */
const char* fluxbin_status_string(int status);

/* Name and description of the last CUDA failure (FLUXBIN_ERR_CUDA) seen by a
 * call on this host thread; "" if none.  Thread-local storage, never NULL. */
const char* fluxbin_last_error(void);

/*
 * Device-side status of the current device.  Bit 0: a tensor-core launch gave
 * up one of its bounded waits (never expected outside the test hook above;
 * the outputs it owned are then NaN).  Bit 1: a tensor-core launch could not
 * confirm that its matrix operations had finished and kept its tensor memory
 * instead of releasing it under them (never expected).  The LUT path has no
 * waits that can give up: its only cross-CTA wait is the hardware cluster
 * barrier.  Reads and clears the flags; synchronises with the device.
 * Errors: INVALID_ARG (null output), CUDA.
 */
int fluxbin_device_status(uint32_t* out_flags);

/* Library version: major*10000 + minor*100 + patch. */
int fluxbin_version(void);

/*
 * Sizes of the packed sign arrays of a layer, in bytes (words_bytes for the
 * global branch, swords_bytes for the salient branch; 0 when it is absent).
 * Follows the packed sign layout above.  Host only; no CUDA call.
 * Errors: INVALID_ARG (null desc or outputs), BAD_SHAPE, UNSUPPORTED.
 */
int fluxbin_packed_sizes(const fluxbin_layer_desc* desc, size_t* words_bytes, size_t* swords_bytes);

/*
 * Host packer: the binary bases as sign bits in uint32 words, streamed later
 * without ever being turned back into floats (summary, Section 3 "LUT-Based
 * GEMV Kernel"; news article: weights "streamed in a compressed Uint32
 * format").  It also validates the salient column list S that Virtual
 * Columnar Mapping gathers through (Section 3 "Virtual Columnar Mapping").
 *
 *   signs     host int8 [Kb][M][N], each +1 or -1
 *   sal_signs host int8 [Ks][M][n_sal], each +1 or -1 (NULL when Ks == 0 or n_sal == 0)
 *   sal_idx   host int32 [n_sal], strictly increasing, each in [0, N)
 *   words_out  host, caller-allocated, fluxbin_packed_sizes().words_bytes bytes
 *   swords_out host, caller-allocated, swords_bytes bytes (NULL when absent)
 * Every output word is written (padding bits 0).  Host only; no CUDA call.
 * Errors: INVALID_ARG (null arrays), BAD_SHAPE (a sign not +-1, S not strictly
 * increasing or out of range), UNSUPPORTED.  On error the outputs are unspecified.
 */
int fluxbin_pack(const fluxbin_layer_desc* desc, const int8_t* signs, const int8_t* sal_signs,
                 const int32_t* sal_idx, uint32_t* words_out, uint32_t* swords_out);

/*
 * Device workspace needed by fluxbin_linear / fluxbin_lut_gemv for a layer of
 * M rows at batch B: split-K partial sums (fp32 [B][ceil(M/32)*32]) and one
 * arrival counter per row group and batch chunk.  Host only.
 * The workspace must be zero-filled once before its first use (for example
 * with cudaMemsetAsync); every call leaves it zero-filled again.  Calls that
 * may run concurrently on the GPU must not share a workspace.  Given one, a
 * call may split long rows wider than a thread-block cluster and add the
 * partial sums through it (their order of summation then varies from call to
 * call); split-K reductions inside a cluster sum in a fixed order.
 * Errors: INVALID_ARG (null output), BAD_SHAPE (M < 0 or B < 0).
 */
int fluxbin_workspace_bytes(int32_t M, int32_t B, size_t* bytes);

/*
 * Workspace for one layer at batch B, in bytes: fluxbin_workspace_bytes(M, B)
 * plus, for a layer whose batch-1 calls can run the table precompute as a
 * separate kernel (B == 1, mu == 8, per-row scales in both branches), a table
 * buffer of 64 KiB per pair of units (a unit is (32/nb)*mu columns of a
 * branch).  Host only.
 *
 * With FLUXBIN_FLAG_SEPARATE_TABLES and at least this many bytes, a batch-1
 * mu = 8 call builds every unit's tables of signed partial sums once, in a
 * kernel of its own that writes them to the table buffer (the precompute as
 * a separate operator, LUT Tensor Core notes, Section 3.1.1), and the lookup
 * kernel copies each unit's tables into shared memory with bulk copies
 * instead of rebuilding them in every CTA.  Without the flag the tables are
 * built inside the lookup kernel.  Both give the same results up to fp32
 * summation order.  The first fluxbin_workspace_bytes(M, B) bytes keep the
 * zero-fill contract of fluxbin_workspace_bytes; the table buffer after them
 * holds scratch and needs no initialisation.
 * Errors: INVALID_ARG (null desc or output), BAD_SHAPE, UNSUPPORTED.
 */
int fluxbin_layer_workspace_bytes(const fluxbin_layer_desc* desc, int32_t B, size_t* bytes);

/*
 * One dense branch (the kernel that Virtual Columnar Mapping reuses):
 *   y[b][i] (+)= sum_k r_k(i) * sum_{n < ncols} B_k[i][n] c_k[n] x[b][col(n)]
 * with col(n) = d_gather[n] (or n when d_gather is NULL).
 *   M, N         rows of W and the length of every x row
 *   ncols, nbases, mu   geometry of the packed branch (nbases in {1,2,4})
 *   row_scale_group     0 (d_r is [nbases][M]) or G (d_r is [nbases][ceil(ncols/G)][M]);
 *                       G must be a multiple of the unit width (32/nbases)*mu
 *   d_words      packed signs, 16-byte aligned (layout above)
 *   d_r, d_c     fp16 scales; d_c is [nbases][ncols]
 *   d_gather     int32 [ncols] or NULL.  An entry outside [0, N) contributes 0.
 *   d_x          fp16 [B][N];  B in [0, 16]
 *   d_y          [B][M], fp16 or fp32 per FLUXBIN_FLAG_Y_FP32; 4-byte aligned for fp32
 *   flags        FLUXBIN_FLAG_*
 *   d_workspace, workspace_bytes   see fluxbin_workspace_bytes (may be NULL/0 only when
 *                the call needs none; FLUXBIN_FLAG_SEPARATE_TABLES needs
 *                fluxbin_workspace_bytes(M, 1) + 64 KiB per pair of units)
 * M == 0 or B == 0 returns FLUXBIN_OK without launching.
 * Errors: INVALID_ARG, BAD_SHAPE, MISALIGNED, UNSUPPORTED, SMEM_BUDGET, WORKSPACE, CUDA.
 */
int fluxbin_lut_gemv(int32_t M, int32_t N, int32_t ncols, int32_t nbases, int32_t mu,
                     int32_t row_scale_group,
                     const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c,
                     const int32_t* d_gather, const uint16_t* d_x, int32_t B,
                     void* d_y, uint32_t flags, void* d_workspace, size_t workspace_bytes,
                     void* stream);

/*
 * The full layer, global and salient branches in one launch:
 *   y[b] (+)= W x[b]   (W as at the top of this file)
 *   d_words  [global packed signs], d_r, d_c   global scales
 *   d_swords [salient packed signs], d_rs, d_cs, d_idx (S)   salient branch
 *            (all four ignored when Ks == 0 or n_sal == 0)
 * Other arguments as for fluxbin_lut_gemv.  Graph-capturable: no allocation,
 * no synchronisation, no host-device copy.
 * Errors: INVALID_ARG, BAD_SHAPE, MISALIGNED, UNSUPPORTED, SMEM_BUDGET, WORKSPACE, CUDA.
 */
int fluxbin_linear(const fluxbin_layer_desc* desc,
                   const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c,
                   const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs,
                   const int32_t* d_idx, const uint16_t* d_x, int32_t B,
                   void* d_y, uint32_t flags, void* d_workspace, size_t workspace_bytes,
                   void* stream);

/*
 * The layer with the table precompute fused into the element-wise operator
 * that precedes it (LUT Tensor Core notes, Section 3.1.1: the precompute as
 * an operator of its own, fused with the preceding element-wise operator).
 * The operator is taken to be the RMS normalisation of a LLaMA-style block:
 *   x = h (.) gamma / sqrt(mean_n(h[n]^2) + eps)
 *   y (+)= W x
 * for one activation row (batch 1).  The precompute kernel reads h, forms x
 * in fp32 and builds every unit's tables from it (x is never rounded on the
 * way to the tables); the lookup kernel of FLUXBIN_FLAG_SEPARATE_TABLES then
 * runs on those tables.
 *   d_h       fp16 [N], the un-normalised activation
 *   d_gamma   fp16 [N], the normalisation weight
 *   eps       >= 0, finite (with eps == 0 a row h == 0 divides by zero: x and y are NaN)
 *   d_x_out   fp16 [N] or NULL: if given, receives x rounded to fp16 (round to
 *             nearest even), e.g. for the other layers that read the same x;
 *             must not overlap d_h
 *   flags     FLUXBIN_FLAG_ACCUMULATE, FLUXBIN_FLAG_Y_FP32,
 *             FLUXBIN_FLAG_EARLY_WEIGHTS only
 *   d_workspace, workspace_bytes   at least fluxbin_layer_workspace_bytes(desc, 1)
 *             (the split-K scratch plus the table buffer), 16-byte aligned; as with
 *             FLUXBIN_FLAG_SEPARATE_TABLES the table buffer is left holding the tables
 * Other arguments as for fluxbin_linear.  Layers: mu = 8 with per-row scales
 * in both branches (else UNSUPPORTED).  M == 0 returns FLUXBIN_OK without
 * launching (x_out is then not written); N == 0 with M > 0 is BAD_SHAPE.
 * Graph-capturable like fluxbin_linear.
 * Errors: INVALID_ARG, BAD_SHAPE, MISALIGNED, UNSUPPORTED, WORKSPACE, CUDA.
 */
int fluxbin_linear_rmsnorm(const fluxbin_layer_desc* desc,
                           const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c,
                           const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs,
                           const int32_t* d_idx, const uint16_t* d_h, const uint16_t* d_gamma,
                           float eps, uint16_t* d_x_out,
                           void* d_y, uint32_t flags, void* d_workspace, size_t workspace_bytes,
                           void* stream);

/*
 * fluxbin_linear for callers that cannot allocate device memory.  (An
 * addition of this library; the FluxBin pages have no counterpart.)
 *
 * Some callers have no way to obtain a workspace: a plugin loaded into a host
 * program that owns every byte of device memory through its own pool and
 * forbids direct cudaMalloc, or a latency-critical loop that must never call
 * cudaMalloc / cudaFree because those calls synchronise the device.  This
 * entry point needs no workspace argument: its split-K scratch is a fixed
 * array of FLUXBIN_STATIC_SCRATCH_BYTES in the library's own device memory,
 * which every GPU that loads the library holds until the process exits.
 *
 *   - Same arguments and results as fluxbin_linear, without d_workspace and
 *     workspace_bytes.  Nothing is allocated: no cudaMalloc, cudaFree or
 *     allocating library routine is called.
 *   - The first call on each device looks up the scratch address for that
 *     device (with the device current); make that first call before any
 *     stream capture begins.
 *   - A call whose launch plan reduces its split-K partials through the
 *     scratch first clears, on `stream`, the part that must start at zero
 *     (fluxbin_workspace_bytes(M, B) bytes), then launches; a call whose plan
 *     does not touch the scratch launches the layer alone.
 *   - Every call on a device shares the one scratch array: calls that may
 *     overlap on the GPU (different streams without ordering between them)
 *     race and give wrong results.  Order them on one stream.
 *   - A layer whose scratch need fluxbin_workspace_bytes(M, B) exceeds
 *     FLUXBIN_STATIC_SCRATCH_BYTES is rejected with FLUXBIN_ERR_SCRATCH_LIMIT
 *     before anything is launched (4 MiB covers, for example, M = 32768 at B = 16).
 * Errors: as fluxbin_linear, plus SCRATCH_LIMIT; CUDA when the scratch address
 * cannot be obtained or cleared.
 */
#define FLUXBIN_STATIC_SCRATCH_BYTES (4u << 20)
int fluxbin_linear_static_scratch(const fluxbin_layer_desc* desc,
                                  const uint32_t* d_words, const uint16_t* d_r, const uint16_t* d_c,
                                  const uint32_t* d_swords, const uint16_t* d_rs, const uint16_t* d_cs,
                                  const int32_t* d_idx, const uint16_t* d_x, int32_t B,
                                  void* d_y, uint32_t flags, void* stream);

/*
 * ---------------------------------------------------------------------------
 * Decomposition fitting (host, offline): from a dense W to bases and scales
 * ---------------------------------------------------------------------------
 * FluxBin summary, Section 3 "Parameter Optimization": the bases B_k and the
 * scales r_k, c_k of one branch minimise the weighted reconstruction error
 *     E = sum_ij h_j (W_ij - sum_k r_k(i,j) B_k[i][j] c_k[j])^2
 * by alternating minimisation.  Appendix A.1: with the bases and the column
 * scales fixed, each row scale (each row block's scale when G > 0) has the
 * closed form sum_j h_j R_ij B_ij c_j / sum_j h_j c_j^2 over the residual R
 * of the other bases; symmetrically each column scale is
 * sum_i R_ij B_ij r_i / sum_i r_i^2.  Appendix A.2: with the scales fixed,
 * every element independently takes the best of its 2^nbases sign
 * combinations (exhaustive search, globally optimal for those scales).
 *
 * Procedure (fixed, so that results are reproducible):
 *   start: for k = 0 .. nbases-1, B_k = sign of the residual of the bases
 *          already placed (sign(0) = +1), c_k = 1, r_k by the row closed form;
 *   then `iters` times: for k = 0 .. nbases-1 the row scales of base k, then
 *          its column scales (the other bases fixed at their latest values);
 *          then the joint sign search over all elements.
 *   A scale whose denominator is zero is set to 0.  Among sign combinations
 *   with equal error the lowest p wins (bit k of p set means +1).
 * The error E never increases from one step to the next.  Work is spread over
 * the host's threads; results do not depend on the thread count.  The scales
 * are returned in fp64; round them to fp16 for the device entry points.
 *
 *   M, N           shape of W (M output rows, N input columns), >= 0
 *   nbases         bases of the branch, 1..8
 *   row_scale_group 0: r is [nbases][M]; G > 0: r is [nbases][ceil(N/G)][M]
 *   iters          alternating iterations after the start, >= 0
 *   W              host fp64 [M][N], row-major
 *   col_weight     host fp64 [N], every entry >= 0 (the h_j above), or NULL for all 1
 *   signs_out      host int8 [nbases][M][N], +1 / -1
 *   r_out, c_out   host fp64, layouts as above; c is [nbases][N]
 *   objective_out  host, the final E (may be NULL)
 * All buffers are the caller's.  Host only; no CUDA call.
 * Errors: INVALID_ARG (null array with M*N > 0), BAD_SHAPE (negative sizes or
 * iters, a negative or NaN weight), UNSUPPORTED (nbases outside 1..8).
 */
int fluxbin_fit(int32_t M, int32_t N, int32_t nbases, int32_t row_scale_group, int32_t iters,
                const double* W, const double* col_weight, int8_t* signs_out, double* r_out, double* c_out,
                double* objective_out);

/*
 * The hybrid layer (FluxBin summary, Section 3 "Salient-Aware Hybrid Bases"):
 * Kb global bases fitted to W as by fluxbin_fit, then Ks salient bases fitted
 * by the same procedure to the global residual gathered at the salient
 * columns S (a dense M x n_sal matrix -- the Virtual Columnar Mapping layout),
 * with the weights h_{S[t]} and their own row-scale group Gs.  The outputs
 * are the arrays fluxbin_pack and the device entry points take (after
 * rounding the scales to fp16):
 *   signs_out [Kb][M][N], r_out, c_out      as for fluxbin_fit
 *   sal_signs_out [Ks][M][n_sal], rs_out ([Ks][M] or [Ks][ceil(n_sal/Gs)][M]), cs_out [Ks][n_sal]
 *   sal_idx   host int32 [n_sal], strictly increasing, each in [0, N)
 *   objective_out  E of the whole reconstruction (global + salient)
 * With Ks == 0 or n_sal == 0 only the global branch is fitted (the salient
 * arrays may be NULL).
 * Errors: as fluxbin_fit; BAD_SHAPE for a bad salient column list.
 */
int fluxbin_fit_hybrid(int32_t M, int32_t N, int32_t Kb, int32_t row_scale_group, int32_t Ks, int32_t n_sal,
                       const int32_t* sal_idx, int32_t sal_scale_group, int32_t iters, const double* W,
                       const double* col_weight, int8_t* signs_out, double* r_out, double* c_out,
                       int8_t* sal_signs_out, double* rs_out, double* cs_out, double* objective_out);

#ifdef __cplusplus
}
#endif

#endif /* FLUXBIN_H */
