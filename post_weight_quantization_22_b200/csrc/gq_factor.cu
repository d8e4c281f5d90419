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
// and A[4a..4a+3][4b..4b+3] in registers.  Per pivot, column c of S and row c of A travel
// through double-buffered shared memory (one barrier); a thread reads 4 multipliers, 4 column
// values and 4 row values there with 16-byte loads.  The pivot loop is unrolled 4 deep (register
// indices fixed, the body small enough to stay in the instruction cache).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 1) potrf_diag_kernel(double* M, int64_t ldm, int64_t c0,
                                                            int w, WsHeader* hdr) {
  __shared__ __align__(16) double colbuf[2][kNB];
  __shared__ __align__(16) double rowbuf[2][kNB];
  __shared__ double dbuf[kNB];
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
#pragma unroll 1
  for (int c4 = 0; c4 < kNB / 4; ++c4) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int c = 4 * c4 + cc;
      const int buf = cc & 1;
      if (b == c4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) colbuf[buf][4 * a + i] = sv[i][cc];  // S[.][c]
      }
      if (a == c4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) rowbuf[buf][4 * b + j] = av[cc][j];  // A[c][.]
      }
      __syncthreads();
      if (4 * a + 3 > c) {
        double p = colbuf[buf][c];
        if (!(p > 0.0)) p = 1.0;  // reported below from the final pivots
        const double rp = recip_newton(p);
        const double2 f01 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * a]);
        const double2 f23 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * a + 2]);
        const double fr[4] = {f01.x * rp, f01.y * rp, f23.x * rp, f23.y * rp};
        if (4 * b + 3 > c) {  // S: entries with c < q <= r
          const double2 q01 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * b]);
          const double2 q23 = *reinterpret_cast<const double2*>(&colbuf[buf][4 * b + 2]);
          const double cq[4] = {q01.x, q01.y, q23.x, q23.y};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (4 * b + j > c && 4 * b + j <= 4 * a + i) sv[i][j] = fma(-fr[i], cq[j], sv[i][j]);
        }
        if (4 * b <= c) {  // A: entries with q <= c < r
          const double2 r01 = *reinterpret_cast<const double2*>(&rowbuf[buf][4 * b]);
          const double2 r23 = *reinterpret_cast<const double2*>(&rowbuf[buf][4 * b + 2]);
          const double rq[4] = {r01.x, r01.y, r23.x, r23.y};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (4 * b + j <= c && 4 * a + i > c) av[i][j] = fma(-fr[i], rq[j], av[i][j]);
        }
      }
    }
  }
  // pivots D_r = S[r][r], held by the diagonal threads
  if (a == b) {
#pragma unroll
    for (int i = 0; i < 4; ++i) dbuf[4 * a + i] = sv[i][i];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 4 * a + i;
    double d = dbuf[r];
    if (!(d > 0.0)) {
      if (r < w && b == 0) record_status(hdr, GQ_ERR_NOT_PD);
      d = 1.0;
    }
    const double rs = 1.0 / sqrt(d);
    if (r < w) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = 4 * b + j;
        if (q <= r) M[(c0 + r) * ldm + c0 + q] = av[i][j] * rs;
      }
    }
  }
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

struct PrepLayout {
  WsHeader* hdr;
  double* M;     // n x ldm: lower triangle = J P H_d P J, then the inverse of its Cholesky factor
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
  L.M = c.take<double>((size_t)n * m_ld(n));
  L.tbuf = c.take<double>(trtri_tbuf_elems(n) + 1);
  L.bytes = c.off;
  return L;
}

size_t prepare_ws_bytes(int64_t n) { return prep_layout(nullptr, n).bytes; }

cudaError_t factor_init_attributes() { return dgemm_init_attributes(); }

#define GQ_TRY(x)                               \
  do {                                          \
    cudaError_t _e = (x);                       \
    if (_e != cudaSuccess) return _e;           \
  } while (0)

cudaError_t launch_prepare(const double* H, int64_t n, double damp, int reverse, float* U,
                           uint8_t* dead, double* delta, void* ws, cudaStream_t s) {
  PrepLayout L = prep_layout(ws, n);
  const int64_t ldm = m_ld(n);
  GQ_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s));
  diag_stats_kernel<<<1, 1024, 0, s>>>(H, n, damp, dead, delta, L.hdr);
  count_launches(1);
  GQ_TRY(cudaGetLastError());
  {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    build_m_kernel<<<grid, 256, 0, s>>>(H, n, ldm, reverse, L.hdr, L.M);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  // The work matrix as a GEMM operand (its upper triangle is scratch: the GEMM never multiplies
  // entries outside an operand's triangle).
  auto Mop = [&](int64_t row0, int64_t col0, int64_t zrow = 0, int64_t zcol = 0) {
    return DgemmOperand{L.M, n, n, ldm, row0, col0, zrow, zcol};
  };
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
    potrf_diag_kernel<<<1, 256, 0, s>>>(L.M, ldm, c0, w, L.hdr);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
    const int64_t rem = n - c0 - w;
    if (rem <= 0) continue;
    {  // P <- P (L11^-1)^T, in place: each CTA owns whole rows of P (N = w = one tile)
      DgemmCall g{};
      g.M = (int)rem; g.N = w; g.K = w; g.batch = 1; g.alpha = 1.0; g.beta_one = 0;
      g.A = Mop(c0 + w, c0);
      g.B = Mop(c0, c0); g.b_nmajor = 0; g.b_upper = 1;  // opB[k][j] = L11^-1[j][k]
      g.C = L.M + (c0 + w) * ldm + c0; g.ldc = ldm; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, s));
    }
    const int64_t inw = sp1 - (c0 + w);  // columns of the super-panel after this panel
    if (inw > 0) {  // A[:, c0+w : sp1] -= L21 L21[c0+w : sp1]^T for every row below
      DgemmCall g{};
      g.M = (int)rem; g.N = (int)inw; g.K = w; g.batch = 1; g.alpha = -1.0; g.beta_one = 1;
      g.A = Mop(c0 + w, c0);
      g.B = Mop(c0 + w, c0); g.b_nmajor = 0;
      g.C = L.M + (c0 + w) * ldm + (c0 + w); g.ldc = ldm; g.lower_tiles = 1; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, s));
    }
    if (c0 + w == sp1 && sp1 < n) {  // super-panel done: trailing update with K = its width
      const int64_t trem = n - sp1, kw = sp1 - sp0;
      DgemmCall g{};
      g.M = (int)trem; g.N = (int)trem; g.K = (int)kw; g.batch = 1; g.alpha = -1.0;
      g.beta_one = 1;
      g.A = Mop(sp1, sp0);
      g.B = Mop(sp1, sp0); g.b_nmajor = 0;
      g.C = L.M + sp1 * ldm + sp1; g.ldc = ldm; g.lower_tiles = 1; g.hdr = L.hdr;
      GQ_TRY(launch_dgemm(g, s));
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
        DgemmCall g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)bs; g.batch = (int)batch; g.alpha = 1.0;
        g.beta_one = 0;
        g.A = Mop(r + bs, r, 2 * bs, 2 * bs);
        g.B = Mop(r, r, 2 * bs, 2 * bs); g.b_nmajor = 1; g.b_lower = 1;
        g.C = tb; g.ldc = bs; g.strideC = bs * bs; g.hdr = L.hdr;
        GQ_TRY(launch_dgemm(g, s));
      }
      {  // B <- -C^-1 T
        DgemmCall g{};
        g.M = (int)cw; g.N = (int)bs; g.K = (int)cw; g.batch = (int)batch; g.alpha = -1.0;
        g.beta_one = 0;
        g.A = Mop(r + bs, r + bs, 2 * bs, 2 * bs); g.a_lower = 1;
        g.B = DgemmOperand{tb, batch * bs, bs, bs, 0, 0, bs, 0}; g.b_nmajor = 1;
        g.C = L.M + (r + bs) * ldm + r; g.ldc = ldm; g.strideC = 2 * bs * ldm + 2 * bs;
        g.hdr = L.hdr;
        GQ_TRY(launch_dgemm(g, s));
      }
    }
  }
  {
    dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
    flip_to_u_kernel<<<grid, 256, 0, s>>>(L.M, n, ldm, U);
    count_launches(1);
    GQ_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

}  // namespace gq
