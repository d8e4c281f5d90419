/*
 * gq.h -- C ABI of the B200 Hessian-aware layer-wise weight quantization library (libgq.so).
 *
 * The library quantizes one linear layer W (m output rows x n input features) against
 * calibration activations X (T tokens x n features) by minimising tr(D H D^T), D = W - Q,
 * H = 2 X^T X, with GPTQ, i.e. Babai's nearest-plane algorithm on the lattice spanned by a
 * Cholesky factor of H ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
 * Algorithm", sections 2.1-2.2).  Three calls form the path:
 *
 *   gq_hessian_accumulate   H += 2 X^T X                                  (section 2.1)
 *   gq_prepare_hinv         dead fix, damping, U = upper factor of H_d^-1 (section 2.1, Thm 1)
 *   gq_quantize_layer       column loop + lazy updates, codes, grids, losses (sections 2.2-2.3)
 *
 * Conventions shared by every entry point:
 *  - All pointers named d_* are DEVICE pointers on the current CUDA device; h_* are host.
 *  - Matrices are dense, row-major, contiguous (leading dimension = number of columns).
 *  - The caller owns and allocates every buffer, including the workspace; the library never
 *    allocates or frees device memory and keeps no pointer after a call returns.
 *  - Calls are asynchronous on `stream` (0 = the legacy default stream) and return after the
 *    work is enqueued, except where a call's comment says it synchronizes.
 *  - Argument errors are reported synchronously by the return value and nothing is enqueued.
 *    Errors found on the device (non-positive pivot, scale ladder exhausted, a bounded wait
 *    that ran out) are written to a status word at the start of the workspace; read it with
 *    gq_workspace_status(), which synchronizes `stream`.
 *  - No C++ exception crosses this interface.  Every kernel's waits are bounded.
 *  - Inputs are never modified.
 */
#ifndef GQ_H_
#define GQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gq_stream_t; /* the same type as cudaStream_t */

typedef enum {
  GQ_OK = 0,
  GQ_ERR_INVALID_ARG = 1,  /* a size, pointer or setting is out of range (nothing enqueued) */
  GQ_ERR_NOT_PD = 2,       /* the damped Hessian has a non-positive Cholesky pivot */
  GQ_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, copy, attribute) */
  GQ_ERR_UNSUPPORTED = 4,  /* a valid but unimplemented combination of settings */
  GQ_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out */
  GQ_ERR_NO_FIT = 6,       /* clip-free: some row's codes still overflow after the ladder */
  GQ_ERR_WORKSPACE = 7     /* the workspace is smaller than the size query returned */
} gq_status;

typedef enum { GQ_BF16 = 0, GQ_FP32 = 1 } gq_dtype;

/* Column processing order ("The Geometry of LLM Quantization", section 2.3: Theorem 5's bound
 * is (1/4) sum s^2 D over the LDL pivots D of the Hessian permuted into the quantization
 * order, so the order changes the bound; the min-pivot order takes the smallest pivot at each
 * LDL step and "act-order" (descending Hessian diagonal) is its cheap approximation).  A
 * permutation perm lists the original columns in processing order: perm[k] = the column
 * processed k-th. */
typedef enum {
  GQ_ORDER_NATURAL = 0,   /* columns 0, 1, ..., n-1 (GPTQ order) */
  GQ_ORDER_REVERSE = 1,   /* columns n-1, ..., 0 (Babai order) */
  GQ_ORDER_ACT = 2,       /* descending diagonal of H after the dead fix; ties by column index */
  GQ_ORDER_MIN_PIVOT = 3, /* greedy min-pivot: the reverse of the elimination order of a
                             pivoted LDL of H_d that always eliminates the smallest remaining
                             Schur-complement pivot (ties: lowest column index) */
  GQ_ORDER_GIVEN = 4      /* the caller's permutation */
} gq_order;

/* Quantization settings of one call of gq_quantize_layer. */
typedef struct {
  int bits;       /* code width b, 2..8 */
  int group_size; /* 0: one grid per row; else the group width, which must divide 128 */
  int reverse;    /* 0: columns first to last (GPTQ order); 1: last to first (Babai order) */
  int clip;       /* 1: codes clamped to [0, 2^b-1] (GPTQ); 0: clip-free with a scale ladder;
                     2: unconstrained integer lattice ("The Geometry of LLM Quantization",
                     section 3, HPTQ): step s = (hi - lo) / (2^b - 1) of the row, zero point 0,
                     codes any int32 (for entropy coding, gq_huffman_encode); needs
                     group_size 0 and reverse 0 */
  float ladder;   /* clip-free: factor applied to a row's step when its codes overflow (1.25) */
  int ladder_max; /* clip-free: at most this many widenings per row (8) */
  int spacing;    /* 0: one step per row or group; 1: ZSIC ("WaterSIC", section 2: grid spacing
                     proportional to 1/|l_jj|): column j's step is the row step times
                     kappa_j = U_jj / geomean(U_kk), U in the processing order.  Needs
                     group_size 0 and reverse 0 (use an order for last-to-first). */
} gq_quant_cfg;

/* Library version string, e.g. "gq 0.1 sm_100a". */
const char* gq_version(void);

/* Number of CUDA kernels this library has launched in this process (all devices, all calls).
 * Instrumentation for benchmarks: the difference around a region counts its launches. */
unsigned long long gq_kernel_launches(void);

/* Human-readable text of a status code (static storage). */
const char* gq_status_string(gq_status s);

/* Workspace bytes gq_hessian_accumulate needs for T tokens of width n. */
size_t gq_hessian_workspace_size(int64_t T, int64_t n);

/*
 * H = 2 X^T X, or H += 2 X^T X  ("The Geometry of LLM Quantization", section 2.1: the lattice
 * basis comes from the calibration inputs and the CVP's Gram matrix is X^T X).
 *
 *   d_H        n x n, fp64, device.  accumulate = 0 overwrites it with 2 X^T X; accumulate = 1
 *              adds 2 X^T X (streaming over token chunks).  Both triangles are written (H stays
 *              exactly symmetric).
 *   d_X     T x n, row-major (tokens x features), dtype x_dtype (bf16 or fp32), device.
 *   T, n    T >= 0 (T = 0: H = 0 when accumulate = 0, H unchanged when accumulate = 1),
 *           1 <= n <= 32768.
 *   d_ws    workspace of at least gq_hessian_workspace_size(T, n) bytes (256-byte aligned).
 *
 * Precision: the products are formed from exact pieces (each value as four 7-bit digits
 * against a power-of-two scale per input column, int8 tensor-core products of the 13 digit
 * pairs that weigh at least 2^-42 of the scales, int32 sums) and combined in fp64; besides fp64
 * rounding, the errors are the rounding of entries smaller than 2^-21 of their column's
 * largest, at 2^-29 of that largest, and the three dropped digit pairs, below 2^-35 of a
 * product's scale (H within about 1e-12 relative of the exact 2 X^T X on the layer recipes).  H is fp64 because the
 * column loop's codes depend on H to about 1e-9 relative for the ill-conditioned Hessians of
 * LLM layers.
 */
gq_status gq_hessian_accumulate(double* d_H, const void* d_X, gq_dtype x_dtype, int64_t T,
                                int64_t n, int accumulate, void* d_ws, size_t ws_bytes,
                                gq_stream_t stream);

/* Workspace bytes gq_prepare_hinv needs for width n (256-byte aligned base required): two fp64
 * n x n work matrices (the factor and its inverse in place, and the inverse's accumulated block
 * products), about 16 n^2 bytes, and from n = 1536 about 3 n^2 bytes more of int8 digit planes
 * (the large products of the factorisation run as exact int8 digit products on the tensor
 * cores, combined in fp64). */
size_t gq_prepare_workspace_size(int64_t n);

/*
 * Factor preparation: dead-feature fix (WaterSIC, "dead feature erasure": H_ii == 0 ->
 * H_ii = 1 and the column's weights are zeroed), relative damping
 * H_d = H + damp * mean(diag H) * I, then U = the upper Cholesky factor of (P H_d P)^-1, i.e.
 * U upper triangular with positive diagonal and U^T U = (P H_d P)^-1, where P is the identity
 * (reverse = 0) or the column reversal (reverse = 1).  U is the factor in the order the
 * columns are processed.  Computed as P H_d P = R R^T (R upper, a Cholesky factorisation
 * from the last pivot) and U = R^-1, in fp64; U is stored rounded to fp32.
 *
 *   d_H        n x n fp64 (from gq_hessian_accumulate), device, read only.
 *   n          1 <= n <= 32768.
 *   damp       >= 0 (0.01 in the usual setting).
 *   reverse    0 or 1, as above; pass the same value to gq_quantize_layer.
 *   d_U        n x n fp32, device, written in full (strict lower triangle set to 0).
 *   d_dead     n bytes, device, written: 1 where H_ii == 0, else 0.
 *   d_delta    1 double, device, written: the damping amount damp * mean(diag H) (after the
 *              dead fix).  gq_quantize_layer uses it for the undamped proxy loss.
 *   d_ws       workspace of at least gq_prepare_workspace_size(n) bytes.
 * Device-detected error: GQ_ERR_NOT_PD (non-positive pivot; U is then undefined).
 */
gq_status gq_prepare_hinv(const double* d_H, int64_t n, double damp, int reverse, float* d_U,
                          uint8_t* d_dead, double* d_delta, void* d_ws, size_t ws_bytes,
                          gq_stream_t stream);

/*
 * gq_prepare_hinv without a workspace, for callers that cannot allocate device memory at call
 * time (a plugin whose memory plan is fixed in advance, code recorded into a CUDA graph under
 * a capture mode that forbids cudaMalloc, a host that hands this library only its inputs and
 * outputs).  The papers have no counterpart of this call; it exists for such callers.
 *
 * Same arguments and results as gq_prepare_hinv, minus the workspace: the scratch is a static
 * device array inside the library (about 17 MB per device that loads the library, held until
 * the process exits), so n is limited to 1 <= n <= 1024; larger n returns GQ_ERR_INVALID_ARG
 * and enqueues nothing.  No device memory is allocated or freed.
 *
 *   d_status   optional (may be NULL) device int, written on `stream` with the device-side
 *              status of this call (GQ_OK, or GQ_ERR_NOT_PD for a non-positive pivot).
 *
 * The first call on a device looks up the scratch array's device address (once per device).
 * With CUDA's lazy module loading (the default) that lookup is also when the driver loads this
 * part of the library and reserves the ~17 MB array on that device; and the first call from
 * each host thread creates the library's private streams and events for that thread and
 * device.  So make the first call per device, and per calling thread, outside any stream
 * capture and at a point where that one-time setup is acceptable.  Every call on a device shares the one
 * scratch array and leaves its contents behind; each call clears what it needs cleared.  Two
 * calls whose work overlaps on the GPU (different streams, no ordering between them) race on
 * the scratch and give undefined results: order them on one stream or with events.
 */
gq_status gq_prepare_hinv_static(const double* d_H, int64_t n, double damp, int reverse,
                                 float* d_U, uint8_t* d_dead, double* d_delta, int* d_status,
                                 gq_stream_t stream);

/*
 * gq_prepare_hinv in a chosen column order: U = the upper Cholesky factor of (P H_d P^T)^-1,
 * P the permutation matrix of the processing order (row k of P H_d P^T is column perm[k] of
 * H_d).  Same arguments, results and workspace as gq_prepare_hinv, plus:
 *
 *   order    a gq_order.  NATURAL and REVERSE give exactly gq_prepare_hinv's U with
 *            reverse = 0 / 1 (d_perm is then not touched and may be NULL).
 *   d_perm   n int32, device.  ACT and MIN_PIVOT write the order computed on the device from
 *            H; GIVEN reads it.  Pass the same array to gq_quantize_layer_ordered.  MIN_PIVOT
 *            runs a pivoted elimination of H_d before the factor (about n/32 one-CTA panel
 *            launches and as many n x n fp64 rank-32 updates).
 * Device-detected errors: GQ_ERR_INVALID_ARG (GIVEN: d_perm is not a permutation of 0..n-1;
 * every access stays in bounds and U is then undefined), GQ_ERR_NOT_PD.
 */
gq_status gq_prepare_hinv_ordered(const double* d_H, int64_t n, double damp, gq_order order,
                                  int32_t* d_perm, float* d_U, uint8_t* d_dead, double* d_delta,
                                  void* d_ws, size_t ws_bytes, gq_stream_t stream);

/* Workspace bytes gq_quantize_layer needs for an m x n layer under cfg. */
size_t gq_quantize_workspace_size(int64_t m, int64_t n, const gq_quant_cfg* cfg);

/*
 * Quantize one layer ("The Geometry of LLM Quantization", section 2.2: GPTQ's error feedback
 * is the nearest-plane step; section 2.3: the no-clipping setting and Theorem 5's bound).
 *
 * Columns are processed in blocks of 128: inside a block, column by column (grid, round,
 * error e = (w_j - q_j) / U_jj, feedback to the block's later columns); between blocks, a
 * lazy rank-128 update W[:, j+128:] -= E U[j:j+128, j+128:].  Grids are asymmetric min-max:
 * per row from the input row (group_size = 0) or per group, from the error-fed weights at
 * the group's first column.  clip = 0 runs unclamped on a per-row step
 * ladder^k (hi - lo) / (2^b - 1), k raised for each row whose codes leave [0, 2^b - 1]
 * (at most ladder_max times); this call then SYNCHRONIZES `stream` once per ladder round.
 *
 *   d_W       m x n, dtype w_dtype, device, read only.
 *   d_U       n x n fp32 from gq_prepare_hinv with the same `reverse`.
 *   d_dead    n bytes from gq_prepare_hinv (may be NULL: no dead columns).
 *   d_delta   1 double from gq_prepare_hinv (may be NULL: loss[0] is then not computed).
 *   d_codes   m x ceil(n*b/32) uint32, written: per row an LSB-first bitstream of b-bit
 *             codes, the code of ORIGINAL column c at bits [b*c, b*c+b); unused bits are 0.
 *             With clip = 2: m x n int32, the code of original column c at [row][c]
 *             (dequantized weight = scale * code).
 *   d_scales  m x G fp32, written, G = 1 (group_size 0) or ceil(n / group_size); group g
 *             covers original columns [g*group_size, (g+1)*group_size).
 *   d_zeros   m x G uint8, written; dequantized weight = scale * (code - zero).
 *   d_loss    3 doubles, written: [0] ||(W0 - Q) X^T||_F^2 = (loss[1] - delta ||W0 - Q||^2)/2
 *             (W0 = W with dead columns zeroed), [1] tr(D H_d D^T) = sum of e^2,
 *             [2] Theorem 5 bound sum_r sum_j s_rj^2 / (4 U_jj^2) (a guarantee for clip = 0).
 *   d_ws      workspace of at least gq_quantize_workspace_size(m, n, cfg) bytes.
 * Limits: 1 <= m <= 2^24, 1 <= n <= 32768, 2 <= bits <= 8; reverse = 1 needs group_size 0;
 * spacing = 1 needs group_size 0 and reverse 0.  With spacing = 1 the Theorem 5 bound and the
 * losses use the per-column steps.
 * Device-detected error: GQ_ERR_NO_FIT.
 */
gq_status gq_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                            const float* d_U, const uint8_t* d_dead, const double* d_delta,
                            const gq_quant_cfg* cfg, uint32_t* d_codes, float* d_scales,
                            uint8_t* d_zeros, double* d_loss, void* d_ws, size_t ws_bytes,
                            gq_stream_t stream);

/*
 * gq_quantize_layer with the columns processed in the order d_perm (n int32, device, from
 * gq_prepare_hinv_ordered; d_U must be the factor of that order).  cfg->reverse must be 0.
 * The packed codes are still indexed by ORIGINAL column.  Group grids cover consecutive
 * columns of the processing order: group g of a row covers original columns
 * d_perm[g*group_size .. (g+1)*group_size - 1] (the usual act-order convention; for a
 * dequantizer, the group of original column c is (position of c in d_perm) / group_size).
 * The Theorem 5 bound uses the pivots of the processing order.
 * Device-detected errors: GQ_ERR_INVALID_ARG (d_perm is not a permutation; every access stays
 * in bounds and the outputs are then undefined), GQ_ERR_NO_FIT.
 */
gq_status gq_quantize_layer_ordered(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                    const float* d_U, const uint8_t* d_dead,
                                    const double* d_delta, const gq_quant_cfg* cfg,
                                    const int32_t* d_perm, uint32_t* d_codes, float* d_scales,
                                    uint8_t* d_zeros, double* d_loss, void* d_ws,
                                    size_t ws_bytes, gq_stream_t stream);

/* Workspace bytes gq_ssqr_quantize_layer needs for an m x n layer (0 if out of range). */
size_t gq_ssqr_workspace_size(int64_t m, int64_t n);

/*
 * SSQR ("The Geometry of LLM Quantization", section 3, scale-adjusted SpQR): the layer is
 * quantized with the GPTQ column loop on one clip-free grid per row, centred on the row's range
 * [lo, hi] (lo <= 0 <= hi) with step s = alpha (hi - lo) / (2^b - 1); an entry whose code would
 * leave [0, 2^b - 1] is an outlier: it keeps its current (error-fed) value in full precision,
 * feeds no error forward, and gets code 0 in the packed stream.  Each row's alpha is found by a
 * search for the target outlier density: the smallest alpha (finest grid) with at most
 * floor(density n) outliers, by doubling alpha from 1 until the row is feasible (at most
 * max_doublings times) and then `steps` bisection steps in log2 alpha between the last
 * infeasible value (2^-8 when alpha = 1 is already feasible) and the feasible one; the result
 * is always a feasible alpha.  Natural column order, one grid per row.  SYNCHRONIZES `stream`
 * once per doubling round.
 *
 *   d_W, w_dtype, m, n, d_U, d_dead, d_delta   as gq_quantize_layer (reverse = 0).
 *   bits          2..8.   density  0..1.   steps  0..60 (20 usual).   max_doublings  0..30.
 *   d_codes       m x ceil(n*b/32) uint32, written (outliers have code 0).
 *   d_scales      m fp32, written (the step s of each row).   d_zeros  m uint8, written.
 *   d_alpha       m doubles, written: the chosen alpha of each row.
 *   d_row_ptr     m + 1 int64, written: CSR row offsets of the outliers.
 *   d_col_idx     nnz_capacity int32, written: column of each outlier (ascending in a row).
 *   d_values      nnz_capacity fp32, written: the kept value of each outlier (dequantized
 *                 weight = value there, scale * (code - zero) elsewhere).
 *   nnz_capacity  room in d_col_idx / d_values; m * floor(density n) always suffices.
 *   d_loss        3 doubles, written as by gq_quantize_layer ([2], the Theorem 5 sum over all
 *                 columns, is not a bound here).
 *   d_ws          workspace of at least gq_ssqr_workspace_size(m, n) bytes.
 * Device-detected errors: GQ_ERR_NO_FIT (some row is still infeasible after max_doublings),
 * GQ_ERR_WORKSPACE (more outliers than nnz_capacity; the CSR arrays then hold the first ones).
 */
gq_status gq_ssqr_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                 const float* d_U, const uint8_t* d_dead, const double* d_delta,
                                 int bits, double density, int steps, int max_doublings,
                                 uint32_t* d_codes, float* d_scales, uint8_t* d_zeros,
                                 double* d_alpha, int64_t* d_row_ptr, int32_t* d_col_idx,
                                 float* d_values, int64_t nnz_capacity, double* d_loss,
                                 void* d_ws, size_t ws_bytes, gq_stream_t stream);

/* Workspace bytes gq_hptq_quantize_layer needs for an m x n layer (0 if out of range). */
size_t gq_hptq_workspace_size(int64_t m, int64_t n);

/*
 * HPTQ rate control ("The Geometry of LLM Quantization", section 3, HPTQ: normal and outlier
 * weights share one unconstrained integer lattice, and Huffman coding of the integers gives a
 * variable bit width that meets a compression budget).  The layer is quantized with the GPTQ
 * column loop on the lattice s Z of each row (zero point 0, no clamp), s = alpha (hi - lo) /
 * (2^b - 1) with [lo, hi] (lo <= 0 <= hi) the row's range and ONE factor alpha for the whole
 * layer.  The budget counts the canonical Huffman code of all m n integers alone (as
 * gq_huffman_encode writes it; scales and the code table are not counted), in bits per weight:
 * alpha is the smallest factor (finest lattice) whose coded size is at most budget * m * n
 * bits, found by doubling alpha from 1 until the layer fits (at most max_doublings times) and
 * then `steps` bisection steps in log2 alpha between the last value that did not fit (2^-8
 * when alpha = 1 already fits) and the one that does; the result always fits.  alpha = 2^t is
 * computed on the host as pow(2, t).  Natural column order.  SYNCHRONIZES `stream` once per
 * pass of the search (1 + doublings + steps + 1 passes).
 *
 *   d_W, w_dtype, m, n, d_U, d_dead, d_delta   as gq_quantize_layer (reverse = 0).
 *   bits          2..8 (the min-max step the factor multiplies).   budget  > 0, bits/weight.
 *   steps         0..60 (12 usual).   max_doublings  0..30.
 *   d_codes       m x n int32, written: the integers, original column order.
 *   d_scales      m fp32, written: the step s of each row (dequantized weight = s * code).
 *   d_alpha       1 double, written: the chosen factor.
 *   d_total_bits  1 int64, written: the coded size at that factor.
 *   d_loss        3 doubles, written as by gq_quantize_layer ([2], the Theorem 5 sum, is the
 *                 no-clipping bound of the chosen lattice).
 *   d_ws          workspace of at least gq_hptq_workspace_size(m, n) bytes.
 * Device-detected errors: GQ_ERR_NO_FIT (the layer does not fit even after max_doublings),
 * GQ_ERR_UNSUPPORTED (a pass spans more than 4096 distinct integers).
 */
gq_status gq_hptq_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                 const float* d_U, const uint8_t* d_dead, const double* d_delta,
                                 int bits, double budget, int steps, int max_doublings,
                                 int32_t* d_codes, float* d_scales, double* d_alpha,
                                 int64_t* d_total_bits, double* d_loss, void* d_ws,
                                 size_t ws_bytes, gq_stream_t stream);

/*
 * The ZSIC column factors kappa_j = U_jj / geomean(U_kk) ("WaterSIC", section 2) of a factor
 * from gq_prepare_hinv(_ordered), exactly as gq_quantize_layer uses them with spacing = 1; a
 * dequantizer takes column j's step as (row step) x kappa_j, j in the processing order.
 *
 *   d_U      n x n fp32, device.   d_kappa  n fp64, device, written.   1 <= n <= 32768.
 */
gq_status gq_zsic_spacing(const float* d_U, int64_t n, double* d_kappa, gq_stream_t stream);

/* Workspace bytes gq_huffman_encode needs for `count` codes (0 if count is out of range). */
size_t gq_huffman_workspace_size(int64_t count);

/*
 * Canonical Huffman coding of integer codes ("The Geometry of LLM Quantization", section 3,
 * HPTQ: the integers of one unconstrained grid are Huffman-coded, so the bit width follows the
 * weight distribution; "WaterSIC", section 2: entropy coding of the ZSIC integers).  Typical
 * input: the int32 codes of gq_quantize_layer with clip = 2; rate = total bits / count.
 *
 *   d_codes      count int32, device, read.  1 <= count <= 2^31 - 1.  The values may span at
 *                most 4096 consecutive integers (symbol k is the value min + k).
 *   d_stream     stream_words uint64, device: the codewords of d_codes in order, MSB first
 *                (stream bit i is bit 63 - i % 64 of word i / 64), in the first
 *                ceil(total bits / 64) words (zeroed, then written); later words are not
 *                touched.  Room for count words (64 bits a code) always suffices.
 *   d_lengths    4096 uint8, device, written: the codeword length of symbol k (0 = unused).
 *   d_codewords  4096 uint64, device, written: the canonical codeword of symbol k (symbols in
 *                order of (length, k) take consecutive values, shifted left at each new length).
 *   d_info       4 int64, device, written: [min value, number of symbols spanned, total bits,
 *                longest codeword].
 *   d_ws         workspace of at least gq_huffman_workspace_size(count) bytes.
 * Device-detected errors (nothing is encoded): GQ_ERR_UNSUPPORTED (more than 4096 values
 * spanned, or a codeword longer than 63 bits), GQ_ERR_WORKSPACE (the total exceeds
 * 64 * stream_words bits).
 */
gq_status gq_huffman_encode(const int32_t* d_codes, int64_t count, uint64_t* d_stream,
                            int64_t stream_words, uint8_t* d_lengths, uint64_t* d_codewords,
                            int64_t* d_info, void* d_ws, size_t ws_bytes, gq_stream_t stream);

/*
 * Test setting of the bounded device waits, for tests of the timeout path (process-wide, read
 * when a call is enqueued; default off).  poll_limit > 0 replaces the poll budget of the
 * factor's per-pivot waits in gq_prepare_hinv(_ordered) (0 restores the default of about 2^26
 * polls, well over a second); withhold_arrival = 1 makes the factor's leaf kernel withhold one
 * thread's first barrier arrival, so that every wait of that phase runs out: the kernel records
 * GQ_ERR_TIMEOUT in the workspace and returns (no copy or tensor-core operation is in flight in
 * that kernel), and the call's U is undefined.  withhold_arrival must be 0 or 1.  The setting is
 * part of the key under which a call's launch sequence is cached, so calls made under it never
 * replay as clean calls.
 */
gq_status gq_debug_wait_test(uint32_t poll_limit, int withhold_arrival);

/*
 * Synchronize `stream` and return the device-side status recorded in a workspace by the last
 * gq_prepare_hinv / gq_quantize_layer that used it (GQ_OK if none), then clear it.
 * For gq_quantize_layer's clip-free ladder, h_ladder_rounds (may be NULL) receives the number
 * of ladder rounds the last call ran.
 */
gq_status gq_workspace_status(void* d_ws, int* h_ladder_rounds, gq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GQ_H_ */
