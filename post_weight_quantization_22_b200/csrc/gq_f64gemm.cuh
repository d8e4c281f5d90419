// fp64 SIMT GEMM used by the Hessian and the factorisation (accuracy-critical stages).
//
//   C[i][j] = (beta_one ? C[i][j] : 0) + alpha * sum_k opA[i][k] * opB[k][j]
//   opA[i][k] = A_T ? A[k*lda + i] : A[i*lda + k]      (A element type TA, converted to fp64)
//   opB[k][j] = B_T ? B[j*ldb + k] : B[k*ldb + j]
//
// Optional structure (skipped work and masked loads, never reads of the masked entries):
//   a_lower:  opA[i][k] = 0 for k > i        b_lower: opB[k][j] = 0 for k < j
//   b_upper:  opB[k][j] = 0 for k > j        lower_tiles: skip output tiles above the diagonal
// Batched over blockIdx.z with element strides.
//
// Two kernels: f64_gemm_kernel (SIMT fp64 FMA, kept for reference) and f64_mma_gemm_kernel (fp64
// tensor cores, mma.sync m8n8k4), which the launcher uses.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "gq_internal.cuh"

namespace gq {

constexpr int kGK = 8;    // k step

template <class T>
__device__ __forceinline__ double to_f64(T v);
template <>
__device__ __forceinline__ double to_f64<double>(double v) { return v; }
template <>
__device__ __forceinline__ double to_f64<float>(float v) { return (double)v; }
template <>
__device__ __forceinline__ double to_f64<__nv_bfloat16>(__nv_bfloat16 v) {
  return (double)__bfloat162float(v);
}

struct F64GemmArgs {
  int M, N, K;
  double alpha;
  int beta_one;
  const void* A;
  int64_t lda, strideA;
  const void* B;
  int64_t ldb, strideB;
  double* C;
  int64_t ldc, strideC;
  int a_lower, b_lower, b_upper, lower_tiles;
};

template <class TA, class TB, bool A_T, bool B_T, int kGB>
__global__ void __launch_bounds__(256) f64_gemm_kernel(F64GemmArgs g) {
  constexpr int TM = kGB / 16;   // outputs per thread per dimension
  constexpr int LPT = kGB / 32;  // tile elements loaded per thread per operand and k step
  __shared__ double As[2][kGK][kGB];
  __shared__ double Bs[2][kGK][kGB];
  const int ti = blockIdx.y, tj = blockIdx.x;
  if (g.lower_tiles && tj > ti) return;
  const int i0 = ti * kGB, j0 = tj * kGB;
  if (i0 >= g.M || j0 >= g.N) return;
  const TA* A = static_cast<const TA*>(g.A) + (int64_t)blockIdx.z * g.strideA;
  const TB* B = static_cast<const TB*>(g.B) + (int64_t)blockIdx.z * g.strideB;
  double* C = g.C + (int64_t)blockIdx.z * g.strideC;

  int k_lo = 0, k_hi = g.K;
  if (g.a_lower) k_hi = min(k_hi, i0 + kGB);
  if (g.b_upper) k_hi = min(k_hi, j0 + kGB);
  if (g.b_lower) k_lo = (j0 / kGK) * kGK;

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  double acc[TM][TM];
#pragma unroll
  for (int a = 0; a < TM; ++a)
#pragma unroll
    for (int b = 0; b < TM; ++b) acc[a][b] = 0.0;

  double ra[LPT], rb[LPT];
  auto load_tiles = [&](int k0) {
#pragma unroll
    for (int r = 0; r < LPT; ++r) {
      int e = tid + 256 * r;
      int ii, kk;
      if (A_T) { kk = e / kGB; ii = e % kGB; } else { ii = e / kGK; kk = e % kGK; }
      int gi = i0 + ii, gk = k0 + kk;
      double v = 0.0;
      if (gi < g.M && gk < k_hi && !(g.a_lower && gk > gi))
        v = A_T ? to_f64<TA>(A[(int64_t)gk * g.lda + gi]) : to_f64<TA>(A[(int64_t)gi * g.lda + gk]);
      ra[r] = v;
      int jj;
      if (B_T) { jj = e / kGK; kk = e % kGK; } else { kk = e / kGB; jj = e % kGB; }
      int gj = j0 + jj;
      gk = k0 + kk;
      v = 0.0;
      if (gj < g.N && gk < k_hi && gk >= k_lo && !(g.b_lower && gk < gj) &&
          !(g.b_upper && gk > gj))
        v = B_T ? to_f64<TB>(B[(int64_t)gj * g.ldb + gk]) : to_f64<TB>(B[(int64_t)gk * g.ldb + gj]);
      rb[r] = v;
    }
  };
  auto store_tiles = [&](int buf) {
#pragma unroll
    for (int r = 0; r < LPT; ++r) {
      int e = tid + 256 * r;
      int ii, kk;
      if (A_T) { kk = e / kGB; ii = e % kGB; } else { ii = e / kGK; kk = e % kGK; }
      As[buf][kk][ii] = ra[r];
      int jj;
      if (B_T) { jj = e / kGK; kk = e % kGK; } else { kk = e / kGB; jj = e % kGB; }
      Bs[buf][kk][jj] = rb[r];
    }
  };

  if (k_lo < k_hi) {
    load_tiles(k_lo);
    store_tiles(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = k_lo; k0 < k_hi; k0 += kGK) {
      const bool more = k0 + kGK < k_hi;
      if (more) load_tiles(k0 + kGK);
#pragma unroll
      for (int kk = 0; kk < kGK; ++kk) {
        double a[TM], b[TM];
#pragma unroll
        for (int q = 0; q < TM; ++q) { a[q] = As[buf][kk][ty + 16 * q]; b[q] = Bs[buf][kk][tx + 16 * q]; }
#pragma unroll
        for (int p = 0; p < TM; ++p)
#pragma unroll
          for (int q = 0; q < TM; ++q) acc[p][q] = fma(a[p], b[q], acc[p][q]);
      }
      if (more) {
        store_tiles(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int p = 0; p < TM; ++p) {
    int gi = i0 + ty + 16 * p;
    if (gi >= g.M) continue;
#pragma unroll
    for (int q = 0; q < TM; ++q) {
      int gj = j0 + tx + 16 * q;
      if (gj >= g.N) continue;
      double* c = C + (int64_t)gi * g.ldc + gj;
      double v = g.alpha * acc[p][q];
      *c = g.beta_one ? (*c + v) : v;
    }
  }
}

// fp64 tensor-core variant: 64 x 64 x 16 tiles, 4 warps (2 x 2) of 32 x 32, each a 4 x 4 grid of
// mma.sync m8n8k4 f64 tiles.  Fragments (m8n8k4, f64): A holds A[lane/4][lane%4], B holds
// B[lane%4][lane/4], C holds C[lane/4][2 (lane%4) + {0,1}].  Shared tiles are k-major with a
// row pitch of 72 doubles (576 B = 64 mod 128) so each fragment load takes two wavefronts.
constexpr int kMB = 64, kMK = 16, kMPitch = kMB + 8;

__device__ __forceinline__ void dmma(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};\n"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

template <class TA, class TB, bool A_T, bool B_T>
__global__ void __launch_bounds__(128) f64_mma_gemm_kernel(F64GemmArgs g) {
  __shared__ __align__(16) double As[2][kMK][kMPitch];
  __shared__ __align__(16) double Bs[2][kMK][kMPitch];
  const int ti = blockIdx.y, tj = blockIdx.x;
  if (g.lower_tiles && tj > ti) return;
  const int i0 = ti * kMB, j0 = tj * kMB;
  if (i0 >= g.M || j0 >= g.N) return;
  const TA* A = static_cast<const TA*>(g.A) + (int64_t)blockIdx.z * g.strideA;
  const TB* B = static_cast<const TB*>(g.B) + (int64_t)blockIdx.z * g.strideB;
  double* C = g.C + (int64_t)blockIdx.z * g.strideC;

  int k_lo = 0, k_hi = g.K;
  if (g.a_lower) k_hi = min(k_hi, i0 + kMB);
  if (g.b_upper) k_hi = min(k_hi, j0 + kMB);
  if (g.b_lower) k_lo = (j0 / kMK) * kMK;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 1, wn = warp & 1;
  double acc[4][4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;

  constexpr int LPT = kMB * kMK / 128;  // 8 elements per thread per operand
  double ra[LPT], rb[LPT];
  auto load_tiles = [&](int k0) {
#pragma unroll
    for (int r = 0; r < LPT; ++r) {
      int e = tid + 128 * r;
      int ii, kk;
      if (A_T) { kk = e / kMB; ii = e % kMB; } else { ii = e / kMK; kk = e % kMK; }
      int gi = i0 + ii, gk = k0 + kk;
      double v = 0.0;
      if (gi < g.M && gk < k_hi && !(g.a_lower && gk > gi))
        v = A_T ? to_f64<TA>(A[(int64_t)gk * g.lda + gi]) : to_f64<TA>(A[(int64_t)gi * g.lda + gk]);
      ra[r] = v;
      int jj;
      if (B_T) { jj = e / kMK; kk = e % kMK; } else { kk = e / kMB; jj = e % kMB; }
      int gj = j0 + jj;
      gk = k0 + kk;
      v = 0.0;
      if (gj < g.N && gk < k_hi && gk >= k_lo && !(g.b_lower && gk < gj) &&
          !(g.b_upper && gk > gj))
        v = B_T ? to_f64<TB>(B[(int64_t)gj * g.ldb + gk]) : to_f64<TB>(B[(int64_t)gk * g.ldb + gj]);
      rb[r] = v;
    }
  };
  auto store_tiles = [&](int buf) {
#pragma unroll
    for (int r = 0; r < LPT; ++r) {
      int e = tid + 128 * r;
      int ii, kk;
      if (A_T) { kk = e / kMB; ii = e % kMB; } else { ii = e / kMK; kk = e % kMK; }
      As[buf][kk][ii] = ra[r];
      int jj;
      if (B_T) { jj = e / kMK; kk = e % kMK; } else { kk = e / kMB; jj = e % kMB; }
      Bs[buf][kk][jj] = rb[r];
    }
  };

  if (k_lo < k_hi) {
    load_tiles(k_lo);
    store_tiles(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = k_lo; k0 < k_hi; k0 += kMK) {
      const bool more = k0 + kMK < k_hi;
      if (more) load_tiles(k0 + kMK);
#pragma unroll
      for (int k4 = 0; k4 < kMK; k4 += 4) {
        double fa[4], fb[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          fa[q] = As[buf][k4 + (lane & 3)][wm * 32 + q * 8 + (lane >> 2)];
          fb[q] = Bs[buf][k4 + (lane & 3)][wn * 32 + q * 8 + (lane >> 2)];
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) dmma(acc[p][q][0], acc[p][q][1], fa[p], fb[q]);
      }
      if (more) {
        store_tiles(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int gi = i0 + wm * 32 + p * 8 + (lane >> 2);
    if (gi >= g.M) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int gj = j0 + wn * 32 + q * 8 + 2 * (lane & 3) + h;
        if (gj >= g.N) continue;
        double* c = C + (int64_t)gi * g.ldc + gj;
        const double v = g.alpha * acc[p][q][h];
        *c = g.beta_one ? (*c + v) : v;
      }
    }
  }
}

template <class TA, class TB, bool A_T, bool B_T>
inline cudaError_t f64_gemm(const F64GemmArgs& g, int batch, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || batch <= 0) return cudaSuccess;
  dim3 grid((g.N + kMB - 1) / kMB, (g.M + kMB - 1) / kMB, batch);
  f64_mma_gemm_kernel<TA, TB, A_T, B_T><<<grid, 128, 0, s>>>(g);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
