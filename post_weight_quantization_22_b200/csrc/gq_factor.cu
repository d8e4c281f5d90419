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
#include "gq_f64gemm.cuh"

#include <math.h>
#include <vector>
#include <algorithm>

namespace gq {

constexpr int kNB = 64;      // Cholesky panel width (the leaf)
constexpr int kSuper = 256;  // super-panel width (trailing-update depth)

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
__global__ void build_m_kernel(const double* H, int64_t n, int reverse, const WsHeader* hdr,
                               double* M) {
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
  M[i * n + j] = v;
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
// 256 threads, 4 per row; thread (r, part) keeps S[r][4i+part] and A[r][4i+part] (i < 16) in
// registers.  Per pivot only column c of S and row c of A travel, through double-buffered
// shared memory, with one barrier; the pivot loop is unrolled so every register index is fixed.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 1) potrf_diag_kernel(double* M, int64_t n, int64_t c0,
                                                            int w, WsHeader* hdr) {
  __shared__ double colbuf[2][kNB];
  __shared__ double rowbuf[2][kNB];
  const int tid = threadIdx.x;
  const int r = tid >> 2, part = tid & 3;
  double sv[16], av[16];
  // all loads of the block issue before any use
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int q = 4 * i + part;
    double v = 0.0;
    if (r < w && q < w) {
      if (q <= r) v = M[(c0 + r) * n + c0 + q];
    } else if (q == r) {
      v = 1.0;
    }
    sv[i] = v;
    av[i] = (q == r) ? 1.0 : 0.0;
  }
#pragma unroll
  for (int c = 0; c < kNB - 1; ++c) {
    const int buf = c & 1;
    if (part == (c & 3)) colbuf[buf][r] = sv[c >> 2];  // S[r][c]
    if (r == c) {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (4 * i + part <= c) rowbuf[buf][4 * i + part] = av[i];  // A[c][j]
    }
    __syncthreads();
    if (r > c) {
      double p = colbuf[buf][c];
      if (!(p > 0.0)) p = 1.0;  // reported below from the final pivots
      const double f = colbuf[buf][r] * recip_newton(p);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = 4 * i + part;
        if (q > c && q <= r) sv[i] = fma(-f, colbuf[buf][q], sv[i]);
        if (q <= c) av[i] = fma(-f, rowbuf[buf][q], av[i]);
      }
    }
  }
  // pivot D_r = S[r][r], held by part r % 4
  double d = 0.0;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (4 * i + part == r) d = sv[i];
  d = __shfl_sync(0xffffffffu, d, (tid & 31 & ~3) | (r & 3));
  if (!(d > 0.0)) {
    if (r < w && part == 0) record_status(hdr, GQ_ERR_NOT_PD);
    d = 1.0;
  }
  const double rs = 1.0 / sqrt(d);
  if (r < w) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int q = 4 * i + part;
      if (q <= r) M[(c0 + r) * n + c0 + q] = av[i] * rs;
    }
  }
}

// U[i][j] = (i <= j) ? (float) Linv[n-1-i][n-1-j] : 0
__global__ void flip_to_u_kernel(const double* M, int64_t n, float* U) {
  int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  int64_t i = blockIdx.y;
  if (j >= n) return;
  float v = 0.f;
  if (i <= j) v = (float)M[(n - 1 - i) * n + (n - 1 - j)];
  U[i * n + j] = v;
}

// ---------------------------------------------------------------------------------------
// host orchestration
// ---------------------------------------------------------------------------------------
struct PrepLayout {
  WsHeader* hdr;
  double* M;     // n x n: lower triangle = J P H_d P J, then the inverse of its Cholesky factor
  double* tbuf;  // doubling scratch of the triangular inverse
  size_t bytes;
};

static size_t trtri_tbuf_elems(int64_t n) {
  size_t best = 0;
  for (int64_t bs = kNB; bs < n; bs *= 2) {
    size_t tot = 0;
    for (int64_t r = 0; r + bs < n; r += 2 * bs) tot += (size_t)bs * bs;
    best = std::max(best, tot);
  }
  return best;
}

static PrepLayout prep_layout(void* ws, int64_t n) {
  Carver c(ws);
  PrepLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.M = c.take<double>((size_t)n * n);
  L.tbuf = c.take<double>(trtri_tbuf_elems(n) + 1);
  L.bytes = c.off;
  return L;
}

size_t prepare_ws_bytes(int64_t n) { return prep_layout(nullptr, n).bytes; }

cudaError_t factor_init_attributes() { return cudaSuccess; }

#define GQ_TRY(x)                               \
  do {                                          \
    cudaError_t _e = (x);                       \
    if (_e != cudaSuccess) return _e;           \
  } while (0)

cudaError_t launch_prepare(const double* H, int64_t n, double damp, int reverse, float* U,
                           uint8_t* dead, double* delta, void* ws, cudaStream_t s) {
  PrepLayout L = prep_layout(ws, n);
  GQ_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s));
  diag_stats_kernel<<<1, 1024, 0, s>>>(H, n, damp, dead, delta, L.hdr);
  count_launches(1);
  GQ_TRY(cudaGetLastError());
  {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    build_m_kernel<<<grid, 256, 0, s>>>(H, n, reverse, L.hdr, L.M);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  // Blocked right-looking Cholesky of M (lower, in place), 64-wide panels grouped into
  // 256-wide super-panels.  For each 64-wide panel: the diagonal block is replaced by the
  // inverse of its factor (leaf), the rows below become L21 = A21 L11^-T, and only the rest of
  // the super-panel takes the update A -= L21 L21^T.  The columns after the super-panel take
  // one K = 256 update per super-panel (fewer, larger fp64 tensor-core GEMMs, 4x less
  // read-modify-write traffic on the trailing matrix than 64-wide steps).
  const int64_t nb = (n + kNB - 1) / kNB;
  for (int64_t k = 0; k < nb; ++k) {
    const int64_t c0 = k * kNB;
    const int w = (int)std::min<int64_t>(kNB, n - c0);
    const int64_t sp0 = (c0 / kSuper) * kSuper;                 // super-panel start
    const int64_t sp1 = std::min<int64_t>(sp0 + kSuper, n);     // super-panel end
    potrf_diag_kernel<<<1, 256, 0, s>>>(L.M, n, c0, w, L.hdr);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
    const int64_t rem = n - c0 - w;
    if (rem <= 0) continue;
    double* P = L.M + (c0 + w) * n + c0;
    {  // P <- P (L11^-1)^T  (in place: one output tile column, each CTA owns its rows)
      F64GemmArgs g{};
      g.M = (int)rem; g.N = w; g.K = w; g.alpha = 1.0; g.beta_one = 0;
      g.A = P; g.lda = n; g.B = L.M + c0 * n + c0; g.ldb = n; g.b_upper = 1;
      g.C = P; g.ldc = n;
      GQ_TRY((f64_gemm<double, double, false, true>(g, 1, s)));
    }
    const int64_t inw = sp1 - (c0 + w);  // columns of the super-panel after this panel
    if (inw > 0) {  // A[:, c0+w : sp1] -= L21 L21[c0+w : sp1]^T for every row below
      F64GemmArgs g{};
      g.M = (int)rem; g.N = (int)inw; g.K = w; g.alpha = -1.0; g.beta_one = 1;
      g.A = P; g.lda = n; g.B = P; g.ldb = n;
      g.C = L.M + (c0 + w) * n + (c0 + w); g.ldc = n; g.lower_tiles = 1;
      GQ_TRY((f64_gemm<double, double, false, true>(g, 1, s)));
    }
    if (c0 + w == sp1 && sp1 < n) {  // super-panel done: trailing update with K = its width
      const int64_t trem = n - sp1, kw = sp1 - sp0;
      double* PS = L.M + sp1 * n + sp0;  // L of the super-panel, rows sp1..n-1
      F64GemmArgs g{};
      g.M = (int)trem; g.N = (int)trem; g.K = (int)kw; g.alpha = -1.0; g.beta_one = 1;
      g.A = PS; g.lda = n; g.B = PS; g.ldb = n;
      g.C = L.M + sp1 * n + sp1; g.ldc = n; g.lower_tiles = 1;
      GQ_TRY((f64_gemm<double, double, false, true>(g, 1, s)));
    }
  }
  // Triangular inverse by doubling over the diagonal blocks (already inverted):
  //   inv([[A, 0], [B, C]]) = [[A^-1, 0], [-C^-1 B A^-1, C^-1]], all pairs of a level batched.
  for (int64_t bs = kNB; bs < n; bs *= 2) {
    const int64_t npairs_full = n / (2 * bs);
    const int64_t rtail = npairs_full * 2 * bs;
    const int64_t cw_tail = n - rtail - bs;
    for (int pass = 0; pass < 2; ++pass) {
      int64_t r = pass == 0 ? 0 : rtail;
      int64_t cw = pass == 0 ? bs : cw_tail;
      int64_t batch = pass == 0 ? npairs_full : (cw_tail > 0 ? 1 : 0);
      if (batch <= 0 || cw <= 0) continue;
      double* tb = L.tbuf + (pass == 0 ? 0 : npairs_full * bs * bs);
      {  // T = B A^-1
        F64GemmArgs g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)bs; g.alpha = 1.0; g.beta_one = 0;
        g.A = L.M + (r + bs) * n + r; g.lda = n; g.strideA = 2 * bs * n + 2 * bs;
        g.B = L.M + r * n + r; g.ldb = n; g.strideB = 2 * bs * n + 2 * bs; g.b_lower = 1;
        g.C = tb; g.ldc = bs; g.strideC = bs * bs;
        GQ_TRY((f64_gemm<double, double, false, false>(g, (int)batch, s)));
      }
      {  // B <- -C^-1 T
        F64GemmArgs g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)cw; g.alpha = -1.0; g.beta_one = 0;
        g.A = L.M + (r + bs) * n + (r + bs); g.lda = n; g.strideA = 2 * bs * n + 2 * bs;
        g.a_lower = 1;
        g.B = tb; g.ldb = bs; g.strideB = bs * bs;
        g.C = L.M + (r + bs) * n + r; g.ldc = n; g.strideC = 2 * bs * n + 2 * bs;
        GQ_TRY((f64_gemm<double, double, false, false>(g, (int)batch, s)));
      }
    }
  }
  {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    flip_to_u_kernel<<<grid, 256, 0, s>>>(L.M, n, U);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

}  // namespace gq
