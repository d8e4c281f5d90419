// Factor preparation: dead-feature fix, relative damping, and U = upper factor of (P H_d P)^-1.
//
// Sources: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 2.1 (Theorem 1: any factor of the Hessian gives an equivalent CVP, so a square
// Cholesky factor is used); "WaterSIC", section 2 (Cholesky Sigma = L L^T) and its "dead feature
// erasure"; "Initialisation Determines the Basin", OA-EM section (H + lambda I).
//
// Route (differs from the three-step Cholesky -> inverse -> Cholesky-of-inverse route, same
// result): with M = J (P H_d P) J (J = column reversal), the lower Cholesky factor L of M and
// its inverse give U = J L^-1 J, which is upper triangular with positive diagonal and satisfies
// U^T U = (P H_d P)^-1; the upper Cholesky factor of a positive definite matrix is unique, so
// this is the same U.  Cost n^3/3 (Cholesky) + n^3/3 (triangular inverse) instead of ~4n^3/3.
//
// Everything is fp64: the damped Hessians of LLM layers have condition numbers ~1e5 and the
// codes downstream change when U carries fp32-level errors.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <math.h>
#include <vector>
#include <algorithm>

namespace gq {

constexpr int kNB = 64;      // Cholesky panel width (the leaf)
constexpr int kSuper = 256;  // super-panel width (trailing-update depth) of the fp64 path
constexpr int kPnPitch = 68;  // shared-memory pitch (doubles) of the panel kernel's tiles
// the leaf's L11^-1 (64 rows), a chunk of the panel (32), the previous panel's rows of the
// diagonal block (64) and of the chunk (32)
constexpr size_t kPnSmem = (size_t)(2 * kNB + 64) * kPnPitch * sizeof(double);

// ---------------------------------------------------------------------------------------
// dead fix + damping statistics (one CTA)
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) diag_stats_kernel(const double* H, int64_t n, double damp,
                                                          uint8_t* dead, double* delta_out,
                                                          WsHeader* hdr) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    double d = H[i * n + i];
    bool isdead = (d == 0.0);
    dead[i] = isdead ? 1 : 0;
    acc += isdead ? 1.0 : d;
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    acc = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (threadIdx.x == 0) {
      double delta = damp * (acc / (double)n);
      *delta_out = delta;
      hdr->scratch[0] = delta;
    }
  }
}

// M[i][j] (j <= i) = Hfix[pi(i)][pi(j)] + (i == j) * delta, pi(i) = n-1-i (forward) or i.
__global__ void build_m_kernel(const double* H, int64_t n, int64_t ldm, int reverse,
                               const WsHeader* hdr, double* M) {
  int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  int64_t i = blockIdx.y;
  if (j > i || i >= n) return;
  int64_t pi = reverse ? i : n - 1 - i;
  int64_t pj = reverse ? j : n - 1 - j;
  double v = H[pi * n + pj];
  if (i == j) {
    if (v == 0.0) v = 1.0;
    v += hdr->scratch[0];
  }
  M[i * ldm + j] = v;
}

// ---------------------------------------------------------------------------------------
// Column orders ("The Geometry of LLM Quantization", section 2.3, the role of the order)
// ---------------------------------------------------------------------------------------
// act-order sort key: the diagonal after the dead fix (0 -> 1); NaN sorts last, so the keys
// are totally ordered and the ranks below always form a permutation.
__device__ __forceinline__ double act_key(double v) {
  if (v == 0.0) return 1.0;
  return (v == v) ? v : -INFINITY;
}

constexpr int kActCols = 128;  // columns ranked per CTA (8 threads each)

// perm[rank(i)] = i, rank(i) = #{j : key_j > key_i} + #{j < i : key_j == key_i}: the columns
// by descending Hessian diagonal, ties in column order.  O(n^2) comparisons, each CTA ranking
// 128 columns against all n keys staged through shared memory.
__global__ void __launch_bounds__(1024) act_order_kernel(const double* H, int64_t n, int* perm) {
  __shared__ double keys[1024];
  const int sub = threadIdx.x & 7;
  const int64_t i = blockIdx.x * (int64_t)kActCols + (threadIdx.x >> 3);
  const double ki = (i < n) ? act_key(H[i * n + i]) : 0.0;
  int rank = 0;
  for (int64_t j0 = 0; j0 < n; j0 += 1024) {
    __syncthreads();
    const int64_t jj = j0 + threadIdx.x;
    keys[threadIdx.x] = (jj < n) ? act_key(H[jj * n + jj]) : 0.0;
    __syncthreads();
    const int lim = (int)((n - j0) < 1024 ? (n - j0) : 1024);
    for (int k = sub; k < lim; k += 8) {
      const double kj = keys[k];
      rank += (kj > ki) || (kj == ki && j0 + k < i);
    }
  }
  rank += __shfl_xor_sync(0xffffffffu, rank, 1);
  rank += __shfl_xor_sync(0xffffffffu, rank, 2);
  rank += __shfl_xor_sync(0xffffffffu, rank, 4);
  if (sub == 0 && i < n) perm[rank] = (int)i;
}

// A caller's permutation: every entry in [0, n) and none repeated (mark zeroed beforehand);
// otherwise GQ_ERR_INVALID_ARG is recorded.
__global__ void perm_check_kernel(const int* perm, int64_t n, int* mark, WsHeader* hdr) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x) {
    const unsigned p = (unsigned)perm[k];
    if (p >= (unsigned long long)n || atomicExch(&mark[p], 1) != 0)
      record_status(hdr, GQ_ERR_INVALID_ARG);
  }
}

// M[i][j] (j <= i) = Hfix[pi(i)][pi(j)] + (i == j) * delta with pi(i) = perm[n-1-i]: M is the
// permuted Hessian in the reverse of the processing order.  One CTA per row of M; the row
// pi(i) of H is staged in shared memory (coalesced) when `stage`, so the gather of its
// columns reads shared memory.
constexpr int64_t kStageMaxN = 25600;  // 200 KB of shared memory per staged row
__global__ void __launch_bounds__(256) build_m_perm_kernel(const double* H, int64_t n,
                                                           int64_t ldm, const int* perm,
                                                           int stage, const WsHeader* hdr,
                                                           double* M) {
  extern __shared__ double srow[];
  const int64_t i = blockIdx.x;
  const double* hrow = H + perm_at(perm, n - 1 - i, n) * n;
  if (stage) {
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) srow[c] = hrow[c];
    __syncthreads();
  }
  const double delta = hdr->scratch[0];
  for (int64_t j = threadIdx.x; j <= i; j += blockDim.x) {
    const int64_t pj = perm_at(perm, n - 1 - j, n);
    double v = stage ? srow[pj] : hrow[pj];
    if (i == j) {
      if (v == 0.0) v = 1.0;
      v += delta;
    }
    M[i * ldm + j] = v;
  }
}

// ---------------------------------------------------------------------------------------
// Greedy min-pivot order ("The Geometry of LLM Quantization", section 2.3: Theorem 5's bound is
// (1/4) sum s^2 D over the LDL pivots D of the Hessian in the quantization order, so taking
// the smallest remaining Schur-complement pivot at every elimination step tightens it).  The
// elimination runs in panels of kMpW pivots on the full symmetric H_d in original indexing:
// one CTA per panel does the pivot steps (argmin of the current Schur diagonal over the
// remaining columns, ties to the lowest index; the Schur column at the pivot from the panel's
// earlier columns; the diagonal updated in place), then one fp64 GEMM applies the panel's
// rank-kMpW update to the whole matrix.  Eliminated rows and columns become zero, as in the
// rank-one form.  Babai decides the columns in the reverse of the elimination order, so that
// reversal is the processing order.  No kernel waits on another: the CTAs of one launch never
// depend on each other, and consecutive launches are ordered by the stream.
// ---------------------------------------------------------------------------------------
constexpr int kMpW = 32;  // pivots per panel

// A (full symmetric, n x lda) = H with the dead fix and the damping, both triangles
__global__ void build_full_kernel(const double* H, int64_t n, int64_t lda, const WsHeader* hdr,
                                  double* A) {
  const int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t i = blockIdx.y;
  if (j >= n) return;
  double v = H[i * n + j];
  if (i == j) {
    if (v == 0.0) v = 1.0;
    v += hdr->scratch[0];
  }
  A[i * lda + j] = v;
}

// The w pivot steps of one panel.  Lp[i][kk] holds the Schur column of the kk-th pivot of the
// panel (row i; 0 for rows eliminated before it, the pivot itself on the pivot's row), Dp[kk]
// the pivot; d[i] the current Schur diagonal, elim[i] whether column i is eliminated.
__global__ void __launch_bounds__(1024, 1) minpivot_panel_kernel(const double* A, int64_t lda,
                                                                 int64_t n, int64_t k0, int w,
                                                                 double* d, int* elim,
                                                                 double* Lp, double* Dp,
                                                                 int* order, WsHeader* hdr) {
  __shared__ double s_v[32];
  __shared__ int s_i[32];
  __shared__ int s_p;
  __shared__ double s_d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int64_t i = tid; i < n; i += 1024)
    if (!elim[i]) d[i] = A[i * lda + i];
  __syncthreads();
  for (int kk = 0; kk < w; ++kk) {
    double best = INFINITY;
    int bi = 0x7fffffff;
    for (int64_t i = tid; i < n; i += 1024) {
      if (elim[i]) continue;
      // NaN compares as +inf, so every remaining column is a candidate and the winner is
      // always a remaining index (at least one remains at every step)
      const double v = d[i] == d[i] ? d[i] : INFINITY;
      if (v < best || (v == best && (int)i < bi)) { best = v; bi = (int)i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov < best || (ov == best && oi < bi)) { best = ov; bi = oi; }
    }
    if (lane == 0) { s_v[warp] = best; s_i[warp] = bi; }
    __syncthreads();
    if (warp == 0) {
      best = s_v[lane];
      bi = s_i[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov < best || (ov == best && oi < bi)) { best = ov; bi = oi; }
      }
      if (lane == 0) { s_p = bi; s_d = best; }
    }
    __syncthreads();
    const int p = s_p;
    double D = s_d;
    if (!(D > 0.0) || !(D < INFINITY)) {  // reported; the rest of the order is then undefined
      if (tid == 0) record_status(hdr, GQ_ERR_NOT_PD);
      D = 1.0;
    }
    const double rD = 1.0 / D;
    for (int64_t i = tid; i < n; i += 1024) {
      double c = 0.0;
      if (!elim[i]) {
        c = A[(int64_t)p * lda + i];  // = A[i][p] (both triangles are kept)
        for (int j = 0; j < kk; ++j) c -= Lp[i * kMpW + j] * Lp[(int64_t)p * kMpW + j] / Dp[j];
        if (i != p) d[i] -= c * c * rD;
      }
      Lp[i * kMpW + kk] = c;
    }
    __syncthreads();
    if (tid == 0) {
      Lp[(int64_t)p * kMpW + kk] = D;
      Dp[kk] = D;
      elim[p] = 1;
      order[k0 + kk] = p;
    }
    __syncthreads();
  }
}

// Ls[i][j] = Lp[i][j] / Dp[j] (the left factor of the panel's update A -= Ls Lp^T)
__global__ void minpivot_scale_kernel(const double* Lp, const double* Dp, int64_t n, int w,
                                      double* Ls) {
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= n * kMpW) return;
  const int j = (int)(e % kMpW);
  Ls[e] = j < w ? Lp[e] / Dp[j] : 0.0;
}

// processing order = elimination order reversed
__global__ void reverse_order_kernel(const int* order, int64_t n, int* perm) {
  const int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (k < n) perm[k] = order[n - 1 - k];
}

// 1/p for p > 0: the hardware reciprocal estimate (rcp.approx.ftz.f64, about 2^-22 relative)
// refined by two Newton-Raphson steps r <- r + r (1 - p r), each squaring the relative error,
// to fp64 precision.  It replaces an IEEE division on the leaf's per-pivot critical path; the
// result may differ from 1.0/p in the last bit, far inside the factor's tolerance.
__device__ __forceinline__ double recip_newton(double p) {
  double r;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(r) : "d"(p));
  double e = fma(-p, r, 1.0);
  r = fma(r, e, r);
  e = fma(-p, r, 1.0);
  return fma(r, e, r);
}

// ---------------------------------------------------------------------------------------
// Diagonal block (w <= 64): the inverse of its Cholesky factor, in place (lower part).
// Unnormalised elimination of [S | I] (S the block, rows >= w padded with the identity): at
// pivot c, rows r > c take S[r][q] -= f_r S[q][c] (q in (c, r]) and A[r][j] -= f_r A[c][j]
// (j <= c), f_r = S[r][c] / S[c][c].  Then A = L_unit^-1, the pivots are D of
// S = L_unit D L_unit^T, and L^-1 = D^-1/2 A.
// 256 threads; thread (a, b) = (tid / 16, tid % 16) keeps the 4 x 4 blocks S[4a..4a+3][4b..4b+3]
// and A[4a..4a+3][4b..4b+3] in registers.  Column c of S and row c of A travel through
// double-buffered shared memory; a thread reads 4 multipliers, 4 column values and 4 row values
// there with 16-byte loads.
// The updates run on whole 4 x 4 blocks without per-entry conditions: after pivot c only the
// trailing lower triangle S[r][q], c < q <= r, the pivots S[r][r] and A[r][j], j <= c < r, are
// read again, and every entry outside them (columns <= c, the upper part) only ever feeds other
// such entries, so whatever they hold does not matter.  Rows r <= c must stay fixed (their
// pivots are final), so their multipliers are set to 0; A[c][j] is exactly 0 for j > c.
// Synchronisation is one mbarrier phase per pivot, split into arrive and wait: at pivot c the
// owners of column c+1 of S and row c+1 of A update those entries first, publish them and
// arrive; every thread then does the rest of its block update while the phase completes, and
// waits for it only when it needs pivot c+1.  The per-pivot critical path is load, reciprocal,
// one FMA and a store.  A row block whose rows are all eliminated leaves with arrive_drop.
// The pivot loop is unrolled 4 deep (register indices fixed, the body small enough to stay in
// the instruction cache).  Waits are bounded: a timeout is recorded and the kernel finishes.
// Look-ahead inside a super-panel (cp >= 0, the previous panel's first column): the previous
// panel's update of this panel's columns is applied here, not by a separate product, so the
// chain runs one kernel per panel.  Every CTA subtracts Lp Lp^T from its copy of the diagonal
// block (Lp = L[c0 .. c0 + 63][cp .. cp + 63], fp64 MMAs into shared memory) and, for each of
// its chunks, Lr Lp^T from the chunk before the solve (Lr = the chunk's rows of L in the
// previous panel's columns).  The later columns of the super-panel take the previous panel's
// update on another stream, overlapped with this kernel.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 1) potrf_panel_kernel(double* M, int64_t ldm, int64_t n,
                                                             int64_t c0, int w, int64_t cp,
                                                             double* Dinv, WsHeader* hdr,
                                                             uint32_t polls, int withhold) {
  extern __shared__ __align__(16) double pn_smem[];
  __shared__ __align__(16) double colbuf[2][kNB];
  __shared__ __align__(16) double rowbuf[2][kNB];
  __shared__ double dbuf[kNB];
  __shared__ __align__(8) uint64_t bar;
  const int tid = threadIdx.x;
  const int a = tid >> 4, b = tid & 15;
  double sv[4][4], av[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = 4 * a + i, q = 4 * b + j;
      double v = 0.0;
      if (r < w && q < w) {
        if (q <= r) v = M[(c0 + r) * ldm + c0 + q];
      } else if (q == r) {
        v = 1.0;
      }
      sv[i][j] = v;
      av[i][j] = (q == r) ? 1.0 : 0.0;
    }
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  double* sQ = pn_smem + (kNB + 32) * kPnPitch;   // 64 x kPnPitch: Lp
  double* sR = pn_smem + (2 * kNB + 32) * kPnPitch;  // 32 x kPnPitch: a chunk's Lr
  if (cp >= 0) {  // diagonal block -= Lp Lp^T
    double* sG = pn_smem;  // 64 x kPnPitch, free until the leaf's result is written
    for (int e = tid; e < kNB * 32; e += 256) {
      const int rr = e >> 5, cc2 = (e & 31) * 2;
      double2 v = make_double2(0.0, 0.0);
      if (rr < w) v = *reinterpret_cast<const double2*>(M + (c0 + rr) * ldm + cp + cc2);
      *reinterpret_cast<double2*>(sQ + rr * kPnPitch + cc2) = v;
    }
    __syncthreads();
    const int gm = warp & 3, gn = warp >> 2;  // rows 16 gm .., columns 32 gn ..
    double acc[4][4] = {};
#pragma unroll
    for (int kb = 0; kb < kNB; kb += 8) {
      const double* pa = sQ + (gm * 16 + g) * kPnPitch + kb + t;
      const double af[4] = {pa[0], pa[8 * kPnPitch], pa[4], pa[8 * kPnPitch + 4]};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const double* pb = sQ + (gn * 32 + u * 8 + g) * kPnPitch + kb + t;
        const double bf[2] = {pb[0], pb[4]};
        tc::dmma_m16n8k8(acc[u], af, bf);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        *reinterpret_cast<double2*>(sG + (gm * 16 + g + 8 * h) * kPnPitch + gn * 32 + u * 8 +
                                    2 * t) = make_double2(acc[u][2 * h], acc[u][2 * h + 1]);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 4 * a + i, q = 4 * b + j;
        if (r < w && q <= r) sv[i][j] -= sG[r * kPnPitch + q];
      }
  }
  if (tid == 0) tc::mbar_init(&bar, 256);
  __syncthreads();
  // pivot 0's column and row, then phase 0
  if (b == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) colbuf[0][4 * a + i] = sv[i][0];
  }
  if (a == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) rowbuf[0][4 * b + j] = av[0][j];
  }
  // (test setting: thread 0 withholds this arrival, so phase 0 never completes and every wait
  // below runs out after `polls` polls)
  if (!(withhold && tid == 0)) tc::mbar_arrive(&bar);
  bool live = true;
#pragma unroll 1
  for (int c4 = 0; c4 < kNB / 4 && live; ++c4) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = 4 * c4 + cc;
      if (!live || c == kNB - 1) break;
      if (!tc::mbar_wait_polls(&bar, c & 1, polls)) {  // pivot c published
        record_status(hdr, GQ_ERR_TIMEOUT);
        live = false;
        break;
      }
      if (4 * a + 3 == c) {  // every row of this block is eliminated: leave the protocol
        tc::mbar_arrive_drop(&bar);
        live = false;
        break;
      }
      const int buf = cc & 1, nbuf = buf ^ 1;
      const int cn = (cc + 1) & 3;  // column / row index of pivot c+1 inside its 4-block
      double p = colbuf[buf][c];
      if (!(p > 0.0)) p = 1.0;  // reported below from the final pivots
      const double rp = recip_newton(p);
      const double2 f01 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * a]);
      const double2 f23 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * a + 2]);
      const double2 q01 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * b]);
      const double2 q23 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * b + 2]);
      const double2 r01 = *reinterpret_cast<const double2*>(&rowbuf[buf][4 * b]);
      const double2 r23 = *reinterpret_cast<const double2*>(&rowbuf[buf][4 * b + 2]);
      const double fr[4] = {4 * a + 0 > c ? f01.x * rp : 0.0, 4 * a + 1 > c ? f01.y * rp : 0.0,
                            4 * a + 2 > c ? f23.x * rp : 0.0, 4 * a + 3 > c ? f23.y * rp : 0.0};
      const double cq[4] = {q01.x, q01.y, q23.x, q23.y};
      const double rq[4] = {r01.x, r01.y, r23.x, r23.y};
      // critical: column c+1 of S and row c+1 of A, published before the rest
      const bool own_col = (b == ((c + 1) >> 2)), own_row = (a == ((c + 1) >> 2));
      if (own_col) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sv[i][cn] = fma(-fr[i], cq[cn], sv[i][cn]);
          colbuf[nbuf][4 * a + i] = sv[i][cn];
        }
      }
      if (own_row) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          av[cn][j] = fma(-fr[cn], rq[j], av[cn][j]);
          rowbuf[nbuf][4 * b + j] = av[cn][j];
        }
      }
      tc::mbar_arrive(&bar);
      // the rest of the block update, overlapped with the next phase
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (!(own_col && j == cn)) sv[i][j] = fma(-fr[i], cq[j], sv[i][j]);
          if (!(own_row && i == cn)) av[i][j] = fma(-fr[i], rq[j], av[i][j]);
        }
    }
  }
  __syncthreads();
  // pivots D_r = S[r][r], held by the diagonal threads
  if (a == b) {
#pragma unroll
    for (int i = 0; i < 4; ++i) dbuf[4 * a + i] = sv[i][i];
  }
  __syncthreads();
  // L11^-1 = D^-1/2 A (lower; zero above) into shared memory, and by CTA 0 into the leaf
  // buffer (not into the diagonal block itself: other CTAs may still be reading that block for
  // their own copy of the leaf)
  double* sL = pn_smem;                   // 64 x kPnPitch
  double* sP = pn_smem + kNB * kPnPitch;  // 32 x kPnPitch: a chunk of the panel below
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 4 * a + i;
    double d = dbuf[r];
    if (!(d > 0.0)) {
      if (r < w && b == 0 && blockIdx.x == 0) record_status(hdr, GQ_ERR_NOT_PD);
      d = 1.0;
    }
    const double rs = 1.0 / sqrt(d);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = 4 * b + j;
      const double v = q <= r ? av[i][j] * rs : 0.0;
      sL[r * kPnPitch + q] = v;
      if (blockIdx.x == 0) Dinv[r * kNB + q] = v;
    }
  }
  // Panel below (w == 64 whenever rows remain): P <- P L11^-T, in place, in chunks of 32 rows
  // spread over the CTAs.  Each warp computes one m16 x (2 x n8) part of the 32 x 64 chunk with
  // fp64 MMAs; the padded pitch makes the fragment loads conflict-free.
  const int64_t rem = n - c0 - w;
  if (rem <= 0) return;
  const int mi = warp & 1, np = warp >> 1;
  const int64_t nch = (rem + 31) / 32;
  for (int64_t ch = blockIdx.x; ch < nch; ch += gridDim.x) {
    const int64_t r0 = c0 + w + ch * 32;
    __syncthreads();  // sL written / the previous chunk consumed
    for (int e = tid; e < 32 * 32; e += 256) {
      const int rr = e >> 5, cc2 = (e & 31) * 2;
      double2 v = make_double2(0.0, 0.0), vr = make_double2(0.0, 0.0);
      if (r0 + rr < n) {
        v = *reinterpret_cast<const double2*>(M + (r0 + rr) * ldm + c0 + cc2);
        if (cp >= 0) vr = *reinterpret_cast<const double2*>(M + (r0 + rr) * ldm + cp + cc2);
      }
      *reinterpret_cast<double2*>(sP + rr * kPnPitch + cc2) = v;
      if (cp >= 0) *reinterpret_cast<double2*>(sR + rr * kPnPitch + cc2) = vr;
    }
    __syncthreads();
    if (cp >= 0) {  // chunk -= Lr Lp^T (each entry of the chunk owned by one thread)
      double up[2][4] = {{0.0, 0.0, 0.0, 0.0}, {0.0, 0.0, 0.0, 0.0}};
#pragma unroll
      for (int kb = 0; kb < kNB; kb += 8) {
        const double* pa = sR + (mi * 16 + g) * kPnPitch + kb + t;
        const double af[4] = {pa[0], pa[8 * kPnPitch], pa[4], pa[8 * kPnPitch + 4]};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const double* pb = sQ + ((2 * np + u) * 8 + g) * kPnPitch + kb + t;
          const double bf[2] = {pb[0], pb[4]};
          tc::dmma_m16n8k8(up[u], af, bf);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          double* pp = sP + (mi * 16 + g + 8 * h) * kPnPitch + (2 * np + u) * 8 + 2 * t;
          pp[0] -= up[u][2 * h];
          pp[1] -= up[u][2 * h + 1];
        }
      __syncthreads();
    }
    double acc[2][4] = {{0.0, 0.0, 0.0, 0.0}, {0.0, 0.0, 0.0, 0.0}};
#pragma unroll
    for (int kb = 0; kb < kNB; kb += 8) {
      const double* pa = sP + (mi * 16 + g) * kPnPitch + kb + t;
      const double af[4] = {pa[0], pa[8 * kPnPitch], pa[4], pa[8 * kPnPitch + 4]};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const double* pb = sL + ((2 * np + u) * 8 + g) * kPnPitch + kb + t;
        const double bf[2] = {pb[0], pb[4]};
        tc::dmma_m16n8k8(acc[u], af, bf);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = r0 + mi * 16 + g + 8 * h;
        if (row < n)
          *reinterpret_cast<double2*>(M + row * ldm + c0 + (2 * np + u) * 8 + 2 * t) =
              make_double2(acc[u][2 * h], acc[u][2 * h + 1]);
      }
  }
}

// Diagonal 64-blocks of [r0, r0 + w) <- the inverted leaves (lower parts), once every panel
// kernel of the range has finished.
__global__ void place_leaves_kernel(double* M, int64_t ldm, const double* Dinv, int64_t r0,
                                    int64_t w) {
  const int64_t r = blockIdx.x;  // row inside the range
  const int q = threadIdx.x;     // column inside the row's 64-block
  if (r >= w) return;
  const int64_t b0 = (r / kNB) * kNB;  // block start inside the range
  const int64_t rr = r - b0;
  if (q <= rr) M[(r0 + r) * ldm + r0 + b0 + q] = Dinv[((r0 + b0) / kNB) * kNB * kNB + rr * kNB + q];
}

// U[i][j] = (i <= j) ? (float) Linv[n-1-i][n-1-j] : 0
__global__ void flip_to_u_kernel(const double* M, int64_t n, int64_t ldm, float* U) {
  int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  int64_t i = blockIdx.y;
  if (j >= n) return;
  float v = 0.f;
  if (i <= j) v = (float)M[(n - 1 - i) * ldm + (n - 1 - j)];
  U[i * n + j] = v;
}

// ---------------------------------------------------------------------------------------
// host orchestration
// ---------------------------------------------------------------------------------------
// Leading dimension of the factor's work matrix: rows start on 128-byte boundaries (TMA needs
// 16-byte multiples).
static int64_t m_ld(int64_t n) { return (n + 15) / 16 * 16; }

// Widths from which the large products run on the int8 tensor cores (gq_split.cu); below it
// every product stays on the fp64 units (the products are small and the chain dominates).
constexpr int64_t kSplitMinN = 1536;
static bool use_split(int64_t n) { return n >= kSplitMinN; }
// Super-panel width: the split path's products are as deep as a super-panel (kSplitK = 512,
// which keeps the fp64 read-modify-write of each output tile under its products); the fp64
// path keeps 256 (a shorter chain of in-panel updates).
static int64_t super_width(int64_t n) { return use_split(n) ? kSplitK : kSuper; }

struct PrepLayout {
  WsHeader* hdr;
  double* M;     // n x ldm: lower triangle = J P H_d P J, then the inverse of its Cholesky factor
  double* T;     // n x ldm: block rows of L X accumulated for the inverse (lower blocks)
  double* Dinv;  // ceil(n / 64) x 64 x 64: the inverted 64-wide leaves
  double* tbuf;  // doubling scratch of the diagonal super-block inverses
  int* pmark;    // n ints: occurrence marks when checking a caller's permutation
  // min-pivot elimination (before M is built; A lives in T): panel columns Lp and Ls (n x 32),
  // Schur diagonal d, elimination flags, panel pivots, elimination order
  double* mpL;
  double* mpLs;
  double* mpd;
  double* mpD;
  int* mpelim;
  int* mporder;
  // int8 digit planes (split path only): for every super-panel K with rows below it, the rows
  // sp1..n-1 of its columns of L (kept until the call ends, read by three streams), and one
  // block row of the inverse as the second operand of the inverse's products
  int8_t* ldig;
  int* lex;
  int8_t* xdig;
  int* xex;
  int8_t* kdig;  // the diagonal block X_KK of the inverse: its rows, then its columns
  int* kex;
  size_t bytes;
};

// rows of the L digit planes of the super-panels before super-panel K
static int64_t lrow_offset(int64_t n, int64_t K) {
  int64_t off = 0;
  const int64_t sw = super_width(n);
  for (int64_t k = 0; k < K; ++k) off += std::max<int64_t>(n - (k + 1) * sw, 0);
  return off;
}

// doubling scratch for one diagonal block of width w (<= 512)
static size_t trtri_tbuf_elems(int64_t w) {
  size_t best = 0;
  for (int64_t bs = kNB; bs < w; bs *= 2) {
    size_t tot = 0;
    for (int64_t r = 0; r + bs < w; r += 2 * bs) tot += (size_t)bs * bs;
    best = std::max(best, tot);
  }
  return best;
}

static PrepLayout prep_layout(void* ws, int64_t n) {
  Carver c(ws);
  PrepLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.M = c.take<double>((size_t)n * m_ld(n));
  L.T = c.take<double>((size_t)n * m_ld(n));
  L.Dinv = c.take<double>((size_t)((n + kNB - 1) / kNB) * kNB * kNB);
  L.tbuf = c.take<double>(trtri_tbuf_elems(super_width(n)) + 1);
  L.pmark = c.take<int>((size_t)n);
  {
    const size_t need = (size_t)n * kMpW * 2 + (size_t)n + kMpW + (size_t)n;  // doubles
    if ((size_t)n * m_ld(n) >= need) {  // inside M
      double* b = L.M;
      L.mpL = b; L.mpLs = b + (size_t)n * kMpW; L.mpd = L.mpLs + (size_t)n * kMpW;
      L.mpD = L.mpd + n;
      L.mpelim = reinterpret_cast<int*>(L.mpD + kMpW);
      L.mporder = L.mpelim + n;
    } else {
      L.mpL = c.take<double>((size_t)n * kMpW);
      L.mpLs = c.take<double>((size_t)n * kMpW);
      L.mpd = c.take<double>((size_t)n);
      L.mpD = c.take<double>(kMpW);
      L.mpelim = c.take<int>((size_t)n);
      L.mporder = c.take<int>((size_t)n);
    }
  }
  L.ldig = nullptr; L.lex = nullptr; L.xdig = nullptr; L.xex = nullptr;
  L.kdig = nullptr; L.kex = nullptr;
  if (use_split(n)) {
    const int64_t lrows = lrow_offset(n, (n + kSplitK - 1) / kSplitK);
    L.ldig = c.take<int8_t>((size_t)kSplitDigits * kSplitK * (size_t)lrows);
    L.lex = c.take<int>((size_t)lrows);
    L.xdig = c.take<int8_t>((size_t)kSplitDigits * kSplitK * (size_t)n);
    L.xex = c.take<int>((size_t)n);
    L.kdig = c.take<int8_t>((size_t)2 * kSplitDigits * kSplitK * kSplitK);
    L.kex = c.take<int>((size_t)2 * kSplitK);
  }
  L.bytes = c.off;
  return L;
}

size_t prepare_ws_bytes(int64_t n) { return prep_layout(nullptr, n).bytes; }

cudaError_t factor_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(potrf_panel_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPnSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(build_m_perm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(kStageMaxN * sizeof(double)));
  if (e != cudaSuccess) return e;
  if ((e = split_init_attributes()) != cudaSuccess) return e;
  return dgemm_init_attributes();
}

#define GQ_TRY(x)                               \
  do {                                          \
    cudaError_t _e = (x);                       \
    if (_e != cudaSuccess) return _e;           \
  } while (0)

// Inverse of the diagonal block [r0, r0 + w) of L (w <= 512) from its inverted 64-wide
// leaves, by doubling: inv([[A, 0], [B, C]]) = [[A^-1, 0], [-C^-1 B A^-1, C^-1]], all pairs of
// a level batched.
static cudaError_t invert_diag_block(double* M, int64_t n, int64_t ldm, int64_t r0, int64_t w,
                                     const double* Dinv, double* tbuf, WsHeader* hdr,
                                     cudaStream_t s) {
  place_leaves_kernel<<<(unsigned)w, kNB, 0, s>>>(M, ldm, Dinv, r0, w);
  count_launches(1);
  {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  for (int64_t bs = kNB; bs < w; bs *= 2) {
    const int64_t npairs_full = w / (2 * bs);
    const int64_t rtail = npairs_full * 2 * bs;
    const int64_t cw_tail = w - rtail - bs;
    for (int pass = 0; pass < 2; ++pass) {
      const int64_t r = r0 + (pass == 0 ? 0 : rtail);
      const int64_t cw = pass == 0 ? bs : cw_tail;
      const int64_t batch = pass == 0 ? npairs_full : (cw_tail > 0 ? 1 : 0);
      if (batch <= 0 || cw <= 0) continue;
      double* tb = tbuf + (pass == 0 ? 0 : npairs_full * bs * bs);
      {  // T = B A^-1
        DgemmCall g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)bs; g.batch = (int)batch; g.alpha = 1.0;
        g.beta_one = 0;
        g.A = DgemmOperand{M, n, n, ldm, r + bs, r, 2 * bs, 2 * bs};
        g.B = DgemmOperand{M, n, n, ldm, r, r, 2 * bs, 2 * bs}; g.b_nmajor = 1; g.b_lower = 1;
        g.C = tb; g.ldc = bs; g.strideC = bs * bs; g.hdr = hdr;
        cudaError_t e = launch_dgemm(g, s);
        if (e != cudaSuccess) return e;
      }
      {  // B <- -C^-1 T
        DgemmCall g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)cw; g.batch = (int)batch; g.alpha = -1.0;
        g.beta_one = 0;
        g.A = DgemmOperand{M, n, n, ldm, r + bs, r + bs, 2 * bs, 2 * bs}; g.a_lower = 1;
        g.B = DgemmOperand{tb, batch * bs, bs, bs, 0, 0, bs, 0}; g.b_nmajor = 1;
        g.C = M + (r + bs) * ldm + r; g.ldc = ldm; g.strideC = 2 * bs * ldm + 2 * bs;
        g.hdr = hdr;
        cudaError_t e = launch_dgemm(g, s);
        if (e != cudaSuccess) return e;
      }
    }
  }
  return cudaSuccess;
}

// Three streams per call, forked from and joined back into the caller's stream:
//   A (highest priority): the latency-bound chain (leaf + panel solve kernels, the in-panel
//     updates, and the trailing update of the next super-panel's columns);
//   B: the trailing update of all later columns, overlapped with the next super-panel's chain;
//   C (lowest priority): the block rows of the triangular inverse, each started as soon as
//     its super-panel is factored.
// One set per host thread and device, created on first use and kept.
struct PrepStreams {
  bool ready = false;
  cudaStream_t a = nullptr, b = nullptr, c = nullptr, d = nullptr;
  cudaEvent_t fork = nullptr, panel[2] = {}, far[2] = {}, join[4] = {}, pk = nullptr,
              upd[2] = {};
};
thread_local PrepStreams t_prep_streams[128];

static cudaError_t prep_streams(PrepStreams** out) {
  int dev = 0;
  GQ_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  PrepStreams& p = t_prep_streams[dev];
  if (!p.ready) {
    int least = 0, greatest = 0;
    GQ_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    GQ_TRY(cudaStreamCreateWithPriority(&p.a, cudaStreamNonBlocking, greatest));
    GQ_TRY(cudaStreamCreateWithPriority(&p.b, cudaStreamNonBlocking, (least + greatest) / 2));
    GQ_TRY(cudaStreamCreateWithPriority(&p.c, cudaStreamNonBlocking, least));
    GQ_TRY(cudaStreamCreateWithPriority(&p.d, cudaStreamNonBlocking, greatest));
    cudaEvent_t* evs[] = {&p.fork, &p.panel[0], &p.panel[1], &p.far[0], &p.far[1],
                          &p.join[0], &p.join[1], &p.join[2], &p.join[3], &p.pk,
                          &p.upd[0], &p.upd[1]};
    for (cudaEvent_t* e : evs) GQ_TRY(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    p.ready = true;
  }
  *out = &p;
  return cudaSuccess;
}

cudaError_t launch_prepare(const double* H, int64_t n, double damp, int order, int* perm,
                           float* U, uint8_t* dead, double* delta, void* ws, cudaStream_t s0) {
  PrepLayout L = prep_layout(ws, n);
  const int64_t ldm = m_ld(n);
  int dev = 0, sms = 148;
  GQ_TRY(cudaGetDevice(&dev));
  GQ_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  PrepStreams* ps = nullptr;
  GQ_TRY(prep_streams(&ps));
  const WaitTest wt = wait_test();
  cudaStream_t s = ps->a, sb = ps->b, sc = ps->c, sd = ps->d;
  GQ_TRY(cudaEventRecord(ps->fork, s0));
  GQ_TRY(cudaStreamWaitEvent(s, ps->fork, 0));
  GQ_TRY(cudaStreamWaitEvent(sb, ps->fork, 0));
  GQ_TRY(cudaStreamWaitEvent(sc, ps->fork, 0));
  GQ_TRY(cudaStreamWaitEvent(sd, ps->fork, 0));
  GQ_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s));
  diag_stats_kernel<<<1, 1024, 0, s>>>(H, n, damp, dead, delta, L.hdr);
  count_launches(1);
  GQ_TRY(cudaGetLastError());
  if (order == GQ_ORDER_ACT) {
    act_order_kernel<<<(unsigned)((n + kActCols - 1) / kActCols), 1024, 0, s>>>(H, n, perm);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  } else if (order == GQ_ORDER_MIN_PIVOT) {
    const int64_t ldm = m_ld(n);
    double* A = L.T;  // full symmetric H_d (T is not used before the inverse writes it)
    {
      dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
      build_full_kernel<<<grid, 256, 0, s>>>(H, n, ldm, L.hdr, A);
      count_launches(1);
      GQ_TRY(cudaGetLastError());
    }
    GQ_TRY(cudaMemsetAsync(L.mpelim, 0, (size_t)n * sizeof(int), s));
    for (int64_t k0 = 0; k0 < n; k0 += kMpW) {
      const int w = (int)std::min<int64_t>(kMpW, n - k0);
      minpivot_panel_kernel<<<1, 1024, 0, s>>>(A, ldm, n, k0, w, L.mpd, L.mpelim, L.mpL, L.mpD,
                                               L.mporder, L.hdr);
      count_launches(1);
      GQ_TRY(cudaGetLastError());
      if (k0 + w >= n) break;
      minpivot_scale_kernel<<<(unsigned)((n * kMpW + 255) / 256), 256, 0, s>>>(L.mpL, L.mpD, n,
                                                                               w, L.mpLs);
      count_launches(1);
      GQ_TRY(cudaGetLastError());
      DgemmCall g{};  // A -= Ls Lp^T over the whole matrix
      g.M = (int)n; g.N = (int)n; g.K = w; g.batch = 1; g.alpha = -1.0; g.beta_one = 1;
      g.A = DgemmOperand{L.mpLs, n, kMpW, kMpW, 0, 0, 0, 0};
      g.B = DgemmOperand{L.mpL, n, kMpW, kMpW, 0, 0, 0, 0}; g.b_nmajor = 0;
      g.C = A; g.ldc = ldm; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, s));
    }
    reverse_order_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L.mporder, n, perm);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  } else if (order == GQ_ORDER_GIVEN) {
    GQ_TRY(cudaMemsetAsync(L.pmark, 0, (size_t)n * sizeof(int), s));
    perm_check_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 1024), 256, 0, s>>>(
        perm, n, L.pmark, L.hdr);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  if (order == GQ_ORDER_NATURAL || order == GQ_ORDER_REVERSE) {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    build_m_kernel<<<grid, 256, 0, s>>>(H, n, ldm, order == GQ_ORDER_REVERSE, L.hdr, L.M);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  } else {
    const int stage = n <= kStageMaxN;
    build_m_perm_kernel<<<(unsigned)n, 256, stage ? (size_t)n * sizeof(double) : 0, s>>>(
        H, n, ldm, perm, stage, L.hdr, L.M);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  // The work matrix as a GEMM operand (its upper triangle is scratch: the GEMM never multiplies
  // entries outside an operand's triangle).
  auto Mop = [&](int64_t row0, int64_t col0, int64_t zrow = 0, int64_t zcol = 0) {
    return DgemmOperand{L.M, n, n, ldm, row0, col0, zrow, zcol};
  };
  auto Top = [&](int64_t row0, int64_t col0) {
    return DgemmOperand{L.T, n, n, ldm, row0, col0, 0, 0};
  };
  // Block row [k0, k1) of the triangular inverse X = L^-1 (stream C):
  //   X_KK = L_KK^-1 (doubling over the inverted 64-wide leaves inside the block),
  //   X[K, :k0] = -X_KK T[K, :k0],   T[K, J] = sum_{J <= I < K} L[K, I] X[I, J],
  // with T accumulated right-looking once X's block row K is known:
  //   T[i >= k1, K] = L[i, K] X_KK,   T[i >= k1, :k0] += L[i, K] X[K, :k0].
  // X overwrites L in place: block row K of L is not read by the Cholesky after block K.
  // On the split path a full-width block row (512) takes its three products on the int8
  // tensor cores; X_KK's rows and columns are split with its upper triangle counted as zero,
  // and the two products that assign (rather than add) write into zeroed blocks.
  const bool split = use_split(n);
  const int64_t sup = super_width(n);
  // digit planes of super-panel K's columns of L, rows sp1 .. n-1 (plane row r = row sp1 + r)
  auto l_operand = [&](int64_t K) {
    const int64_t off = lrow_offset(n, K);
    return SplitOperand{L.ldig + off * kSplitDigits * kSplitK, L.lex + off,
                        n - std::min<int64_t>((K + 1) * sup, n)};
  };
  auto inverse_block_row = [&](int64_t k0, int64_t k1) -> cudaError_t {
    const int64_t kw = k1 - k0;
    GQ_TRY(invert_diag_block(L.M, n, ldm, k0, kw, L.Dinv, L.tbuf, L.hdr, sc));
    const bool ksplit = split && kw == kSplitK;
    const SplitOperand krows{L.kdig, L.kex, kSplitK};  // rows of X_KK
    const SplitOperand kcols{L.kdig + (size_t)kSplitDigits * kSplitK * kSplitK, L.kex + kSplitK,
                             kSplitK};                  // columns of X_KK
    if (k0 > 0 && ksplit) {  // X[K, :k0] = -X_KK T[K, :k0] (block row K of L is not needed)
      const SplitOperand top{L.xdig, L.xex, k0};
      GQ_TRY(launch_split_rows(L.M + k0 * ldm + k0, ldm, (int)kw, krows, sc, 1));
      GQ_TRY(launch_split_cols(L.T + k0 * ldm, ldm, (int)k0, top, sc));
      GQ_TRY(cudaMemset2DAsync(L.M + k0 * ldm, ldm * sizeof(double), 0, k0 * sizeof(double),
                               kw, sc));
      GQ_TRY(launch_split_gemm(L.M + k0 * ldm, ldm, (int)kw, (int)k0, krows, 0, top, 0, -1.0, 0,
                               L.hdr, sc));
    } else if (k0 > 0) {  // X[K, :k0] = -X_KK T[K, :k0]
      DgemmCall g{};
      g.M = (int)kw; g.N = (int)k0; g.K = (int)kw; g.batch = 1; g.alpha = -1.0; g.beta_one = 0;
      g.A = Mop(k0, k0); g.a_lower = 1;
      g.B = Top(k0, 0); g.b_nmajor = 1;
      g.C = L.M + k0 * ldm; g.ldc = ldm; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, sc));
    }
    if (k1 < n) {
      if (ksplit) {  // T[k1:, K] = L[k1:, K] X_KK
        GQ_TRY(launch_split_cols(L.M + k0 * ldm + k0, ldm, (int)kw, kcols, sc, 1));
        GQ_TRY(cudaMemset2DAsync(L.T + k1 * ldm + k0, ldm * sizeof(double), 0,
                                 kw * sizeof(double), n - k1, sc));
        GQ_TRY(launch_split_gemm(L.T + k1 * ldm + k0, ldm, (int)(n - k1), (int)kw,
                                 l_operand(k0 / sup), 0, kcols, 0, 1.0, 0, L.hdr, sc));
      } else {  // T[k1:, K] = L[k1:, K] X_KK
        DgemmCall g{};
        g.M = (int)(n - k1); g.N = (int)kw; g.K = (int)kw; g.batch = 1; g.alpha = 1.0;
        g.beta_one = 0;
        g.A = Mop(k1, k0);
        g.B = Mop(k0, k0); g.b_nmajor = 1; g.b_lower = 1;
        g.C = L.T + k1 * ldm + k0; g.ldc = ldm; g.hdr = L.hdr;
        GQ_TRY(launch_dgemm(g, sc));
      }
      if (k0 > 0 && split) {  // T[k1:, :k0] += L[k1:, K] X[K, :k0] on the int8 tensor cores
        const SplitOperand xop{L.xdig, L.xex, k0};
        GQ_TRY(launch_split_cols(L.M + k0 * ldm, ldm, (int)k0, xop, sc));
        GQ_TRY(launch_split_gemm(L.T + k1 * ldm, ldm, (int)(n - k1), (int)k0, l_operand(k0 / sup),
                                 0, xop, 0, 1.0, 0, L.hdr, sc));
      } else if (k0 > 0) {  // T[k1:, :k0] += L[k1:, K] X[K, :k0]
        DgemmCall g{};
        g.M = (int)(n - k1); g.N = (int)k0; g.K = (int)kw; g.batch = 1; g.alpha = 1.0;
        g.beta_one = 1;
        g.A = Mop(k1, k0);
        g.B = Mop(k0, 0); g.b_nmajor = 1;
        g.C = L.T + k1 * ldm; g.ldc = ldm; g.hdr = L.hdr;
        GQ_TRY(launch_dgemm(g, sc));
      }
    }
    return cudaSuccess;
  };
  // Blocked right-looking Cholesky of M (lower, in place), 64-wide panels grouped into
  // 256-wide super-panels (stream A).  For each 64-wide panel one kernel replaces the diagonal
  // block by the inverse of its factor (leaf) and the rows below by L21 = A21 L11^-T; then only
  // the rest of the super-panel takes the update A -= L21 L21^T.  After a super-panel, the
  // trailing matrix takes one K = 256 update: the next super-panel's columns on A, all later
  // columns on B, overlapped with the next super-panel's chain (look-ahead of one).
  const int64_t nb = (n + kNB - 1) / kNB;
  int sidx = 0;
  bool far_pending = false;
  for (int64_t k = 0; k < nb; ++k) {
    const int64_t c0 = k * kNB;
    const int w = (int)std::min<int64_t>(kNB, n - c0);
    const int64_t sp0 = (c0 / sup) * sup;                       // super-panel start
    const int64_t sp1 = std::min<int64_t>(sp0 + sup, n);        // super-panel end
    const int64_t rem = n - c0 - w;
    // Look-ahead inside the super-panel: the panel kernel applies the previous panel's update
    // to its own columns; the previous panel's update of the columns two panels on and later
    // runs on stream D beside it, and this panel waits for the one two panels back.
    const int64_t cp = c0 > sp0 ? c0 - kNB : -1;
    if (c0 - sp0 >= 2 * kNB) GQ_TRY(cudaStreamWaitEvent(s, ps->upd[(k - 2) & 1], 0));
    {  // leaf (every CTA) + P <- P L11^-T for the rows below, one wave of CTAs
      const int64_t nch = rem > 0 ? (rem + 31) / 32 : 1;
      const int grid = (int)std::min<int64_t>(nch, sms);
      potrf_panel_kernel<<<grid, 256, kPnSmem, s>>>(L.M, ldm, n, c0, w, cp,
                                                    L.Dinv + (c0 / kNB) * kNB * kNB, L.hdr,
                                                    wt.polls, wt.withhold);
      count_launches(1);
      GQ_TRY(cudaGetLastError());
    }
    const int64_t c2 = c0 + 2 * kNB;  // first column this panel updates on stream D
    if (rem > 0 && c2 < sp1) {  // A[c2:, c2 : sp1] -= L21[c2:] L21[c2 : sp1]^T (stream D)
      GQ_TRY(cudaEventRecord(ps->pk, s));
      GQ_TRY(cudaStreamWaitEvent(sd, ps->pk, 0));
      DgemmCall g{};
      g.M = (int)(n - c2); g.N = (int)(sp1 - c2); g.K = w; g.batch = 1; g.alpha = -1.0;
      g.beta_one = 1;
      g.A = Mop(c2, c0);
      g.B = Mop(c2, c0); g.b_nmajor = 0;
      g.C = L.M + c2 * ldm + c2; g.ldc = ldm; g.lower_tiles = 1; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, sd));
      GQ_TRY(cudaEventRecord(ps->upd[k & 1], sd));
    }
    if (c0 + w != sp1) continue;
    // super-panel [sp0, sp1) factored; on the split path its columns of L below it become
    // digit planes once, for the two trailing updates and the inverse's block product
    const bool sp_split = split && sp1 < n;
    const SplitOperand lop = sp_split ? l_operand(sp0 / sup) : SplitOperand{};
    if (sp_split) GQ_TRY(launch_split_rows(L.M + sp1 * ldm + sp0, ldm, (int)(n - sp1), lop, s));
    cudaEvent_t ev_panel = ps->panel[sidx & 1];
    GQ_TRY(cudaEventRecord(ev_panel, s));
    GQ_TRY(cudaStreamWaitEvent(sc, ev_panel, 0));
    GQ_TRY(inverse_block_row(sp0, sp1));
    if (sp1 < n) {
      const int64_t sp2 = std::min<int64_t>(sp1 + sup, n), kw = sp1 - sp0;
      if (far_pending) GQ_TRY(cudaStreamWaitEvent(s, ps->far[(sidx - 1) & 1], 0));
      if (sp_split) {  // next super-panel's columns: A[sp1:, sp1:sp2] -= L[sp1:, SP] L[sp1:sp2, SP]^T
        GQ_TRY(launch_split_gemm(L.M + sp1 * ldm + sp1, ldm, (int)(n - sp1), (int)(sp2 - sp1),
                                 lop, 0, lop, 0, -1.0, 1, L.hdr, s));
      } else {  // next super-panel's columns: A[sp1:, sp1:sp2] -= L[sp1:, SP] L[sp1:sp2, SP]^T
        DgemmCall g{};
        g.M = (int)(n - sp1); g.N = (int)(sp2 - sp1); g.K = (int)kw; g.batch = 1;
        g.alpha = -1.0; g.beta_one = 1;
        g.A = Mop(sp1, sp0);
        g.B = Mop(sp1, sp0); g.b_nmajor = 0;
        g.C = L.M + sp1 * ldm + sp1; g.ldc = ldm; g.lower_tiles = 1; g.hdr = L.hdr;
        GQ_TRY(launch_dgemm(g, s));
      }
      far_pending = false;
      if (sp2 < n) {  // later columns, stream B: A[sp2:, sp2:] -= L[sp2:, SP] L[sp2:, SP]^T
        GQ_TRY(cudaStreamWaitEvent(sb, ev_panel, 0));
        if (sp_split) {
          GQ_TRY(launch_split_gemm(L.M + sp2 * ldm + sp2, ldm, (int)(n - sp2), (int)(n - sp2),
                                   lop, (int)(sp2 - sp1), lop, (int)(sp2 - sp1), -1.0, 1, L.hdr,
                                   sb));
        } else {
          DgemmCall g{};
          g.M = (int)(n - sp2); g.N = (int)(n - sp2); g.K = (int)kw; g.batch = 1;
          g.alpha = -1.0; g.beta_one = 1;
          g.A = Mop(sp2, sp0);
          g.B = Mop(sp2, sp0); g.b_nmajor = 0;
          g.C = L.M + sp2 * ldm + sp2; g.ldc = ldm; g.lower_tiles = 1; g.hdr = L.hdr;
          GQ_TRY(launch_dgemm(g, sb));
        }
        GQ_TRY(cudaEventRecord(ps->far[sidx & 1], sb));
        far_pending = true;
      }
    }
    ++sidx;
  }
  GQ_TRY(cudaEventRecord(ps->join[1], sb));
  GQ_TRY(cudaEventRecord(ps->join[2], sc));
  GQ_TRY(cudaEventRecord(ps->join[3], sd));
  GQ_TRY(cudaStreamWaitEvent(s, ps->join[1], 0));
  GQ_TRY(cudaStreamWaitEvent(s, ps->join[2], 0));
  GQ_TRY(cudaStreamWaitEvent(s, ps->join[3], 0));
  {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    flip_to_u_kernel<<<grid, 256, 0, s>>>(L.M, n, ldm, U);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  GQ_TRY(cudaEventRecord(ps->join[0], s));
  GQ_TRY(cudaStreamWaitEvent(s0, ps->join[0], 0));
  return cudaSuccess;
}

}  // namespace gq
