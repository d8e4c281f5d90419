// H += 2 X^T X  ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 2.1: the CVP's Gram matrix is X^T X; the factor 2 is the Hessian of the squared
// output error).
//
// Every product of two bf16 (or fp32) inputs is exact in fp64 and the token sums accumulate in
// fp64, so H carries ~1e-15 relative error.  Lower 64x64 tiles are computed, the upper
// triangle is then mirrored so H stays exactly symmetric.
#include "gq_internal.cuh"
#include "gq_f64gemm.cuh"

namespace gq {

__global__ void mirror_lower_kernel(double* H, int64_t n) {
  int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // column (fast)
  int64_t i = blockIdx.y;                                      // row
  if (j < n && i < j) H[i * n + j] = H[j * n + i];
}

cudaError_t launch_hessian(double* H, const void* X, gq_dtype xt, int64_t T, int64_t n,
                           cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  F64GemmArgs g{};
  g.M = (int)n; g.N = (int)n; g.K = (int)T;
  g.alpha = 2.0; g.beta_one = 1;
  g.A = X; g.lda = n; g.B = X; g.ldb = n;
  g.C = H; g.ldc = n;
  g.lower_tiles = 1;
  cudaError_t e;
  if (xt == GQ_BF16)
    e = f64_gemm<__nv_bfloat16, __nv_bfloat16, true, false>(g, 1, s);
  else
    e = f64_gemm<float, float, true, false>(g, 1, s);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
  mirror_lower_kernel<<<grid, 256, 0, s>>>(H, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
