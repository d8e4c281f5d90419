// H (+)= 2 X^T X  ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 2.1: the CVP's Gram matrix is X^T X; the factor 2 is the Hessian of the squared
// output error), accumulated to fp64 accuracy on the int8 tensor cores.
//
// Exact-digit scheme (the splitting idea of Ozaki et al., "Error-free transformations of
// matrix multiplication by using fast routines of matrix multiplication and its applications",
// Numer. Algorithms 59 (2012)): every input column i (a feature, over the tokens of this call)
// gets a power-of-two scale 2^e_i with |X_ti| 2^-e_i <= 1/2, and x = X_ti 2^-e_i is written
// as four signed 7-bit digits, x = sum_s d_s 2^-7(s+1), d_s in [-64, 64] (round to nearest at
// every step; exact for every entry within 2^21 of its column's largest, a rounding at 2^-29
// of the column's largest below that).  Then
//   sum_t x_ti x_tj = sum_{a,b} 2^-7(a+b+2) sum_t d_a,ti d_b,tj,
// each inner sum an exact int8 x int8 -> int32 tensor-core product, grouped by a + b into
// int32 accumulators in tensor memory and combined in fp64 in the epilogue.  Only the 13 digit
// pairs with a + b <= 4 are multiplied: the other three weigh at most 3 x 2^12 x 2^-56 of the
// column scales, below 2^-35 of the leading pair (measured on the layer recipes: H within
// 6e-13 relative Frobenius of the exact product with or without them).  The errors besides
// fp64 rounding are that and the digit rounding of the very small entries (about 1e-10 of H
// relative for LLM-like activations), far below what the factorisation needs (about 1e-9; a
// plain fp32 accumulation is about 3e-7).
//
// Kernels: per token chunk, a column-max pass, a digit pass (32 x 32 transpose tiles into four
// K-major int8 planes [feature][token]), and the tcgen05 kernel over 128 x 64 tiles of the lower
// triangle; a final pass mirrors the lower triangle.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <cudaTypedefs.h>
#include <algorithm>
#include <mutex>

namespace gq {

namespace {
constexpr int kHS = 4;                 // digits per value
constexpr int kHBM = 128, kHBN = 64;   // output tile (rows i, columns j)
constexpr int kHBK = 64;               // tokens per stage (64-byte int8 rows)
constexpr int kHStages = 4;
constexpr uint32_t kHATile = kHBM * kHBK;              // 8 KB per digit plane
constexpr uint32_t kHBTile = kHBN * kHBK;              // 4 KB per digit plane
constexpr uint32_t kHStage = kHS * (kHATile + kHBTile);  // 48 KB
constexpr size_t kHSmem = kHStages * kHStage + 1024 + 256;
constexpr int kHClasses = 5;                           // a + b in [0, 4] (13 digit pairs)
constexpr int64_t kHChunk = 65536;                     // tokens per pass (int32 headroom)
// int8 x int8 -> s32, A and B K-major, M 128, N columns (a multiple of 16, at most 256)
__host__ __device__ constexpr uint32_t hess_idesc(uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((uint32_t)(kHBM >> 4) << 24);
}
}  // namespace

// ---------------------------------------------------------------------------------------
// column max |X| over the chunk (as float bits; non-negative floats order like their bits)
// ---------------------------------------------------------------------------------------
template <class TX>
__global__ void colmax_kernel(const TX* X, int64_t n, int64_t t0, int64_t tc, int* maxbits) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t tb = blockIdx.y, nt = gridDim.y;
  float mx = 0.f;
  for (int64_t t = tb; t < tc; t += nt) {
    float v;
    if constexpr (sizeof(TX) == 2) v = __bfloat162float(X[(t0 + t) * n + i]);
    else v = X[(t0 + t) * n + i];
    mx = fmaxf(mx, fabsf(v));
  }
  atomicMax(&maxbits[i], __float_as_int(mx));
}

__device__ __forceinline__ int digit_exponent(int maxbits) {
  const float mx = __int_as_float(maxbits);
  return mx == 0.f ? 0 : ilogbf(mx) + 2;  // |x| 2^-e <= 1/2
}

// ---------------------------------------------------------------------------------------
// digits: D[s][i][t] for features i, tokens t of the chunk (zero past tc up to tp)
// ---------------------------------------------------------------------------------------
template <class TX>
__global__ void __launch_bounds__(256) digits_kernel(const TX* X, int64_t n, int64_t t0,
                                                      int64_t tc, int64_t tp, const int* maxbits,
                                                      int8_t* D) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int64_t tb = (int64_t)blockIdx.x * 32, ib = (int64_t)blockIdx.y * 32;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t t = tb + ty * 4 + r, i = ib + tx;
    float v = 0.f;
    if (t < tc && i < n) {
      if constexpr (sizeof(TX) == 2) v = __bfloat162float(X[(t0 + t) * n + i]);
      else v = X[(t0 + t) * n + i];
    }
    tile[ty * 4 + r][tx] = v;
  }
  __syncthreads();
  const size_t plane = (size_t)n * (size_t)tp;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = ib + ty * 4 + r, t = tb + tx;
    if (i >= n || t >= tp) continue;
    const int e = digit_exponent(maxbits[i]);
    double x = ldexp((double)tile[tx][ty * 4 + r], -e);
    int8_t d[kHS];
#pragma unroll
    for (int s = 0; s < kHS; ++s) {
      x *= 128.0;
      const double q = rint(x);
      d[s] = (int8_t)(int)q;
      x -= q;
    }
#pragma unroll
    for (int s = 0; s < kHS; ++s) D[s * plane + (size_t)i * tp + t] = d[s];
  }
}

// ---------------------------------------------------------------------------------------
// tcgen05 int8 kernel: H[i][j] += 2 2^(e_i + e_j) sum_c 2^-7(c+2) acc_c[i][j], j <= i
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1)
    hessian_tc_kernel(const __grid_constant__ CUtensorMap m_a, const __grid_constant__ CUtensorMap m_b,
                      double* H, int64_t n, int64_t tp, const int* maxbits, int add,
                      WsHeader* hdr) {
  const int bj = blockIdx.x, bi = blockIdx.y;
  if ((int64_t)bj * kHBN > (int64_t)bi * kHBM + kHBM - 1) return;  // tile above the diagonal
  extern __shared__ uint8_t hs_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hs_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kHStages * kHStage);
  uint64_t* empty = full + kHStages;
  uint64_t* accum = empty + kHStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accum + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kHStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    tc::mbar_init(accum, 1);
    tc::fence_barrier_init();
    tc::prefetch_tmap(&m_a);
    tc::prefetch_tmap(&m_b);
  }
  if (warp == 1) tc::tmem_alloc(tslot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const int nk = (int)(tp / kHBK);

  if (warp == 0 && lane == 0) {
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kHStages;
      if (kc >= kHStages && !tc::mbar_wait(&empty[s], ((kc / kHStages) - 1) & 1)) {
        record_status(hdr, GQ_ERR_TIMEOUT);
        break;
      }
      uint8_t* st = base + s * kHStage;
      tc::mbar_arrive_expect_tx(&full[s], kHStage);
#pragma unroll
      for (int d = 0; d < kHS; ++d) {
        tc::tma_load_2d(st + d * kHATile, &m_a, &full[s], kc * kHBK, (int)(d * n + (int64_t)bi * kHBM));
        tc::tma_load_2d(st + kHS * kHATile + d * kHBTile, &m_b, &full[s], kc * kHBK,
                        (int)(d * n + (int64_t)bj * kHBN));
      }
    }
  } else if (warp == 1 && lane == 0) {
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kHStages;
      if (!tc::mbar_wait(&full[s], (kc / kHStages) & 1)) {
        record_status(hdr, GQ_ERR_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const uint32_t a0 = tc::smem_u32(base + s * kHStage);
      const uint32_t b0 = a0 + kHS * kHATile;
      // the stage's descriptors once; operands at constant offsets add offset / 16 to the
      // start-address field (address / 16 in 14 bits; no address here reaches 2^18)
      const uint64_t ad0 = tc::sdesc(a0, 16, 512, tc::kLayoutSW64);
      const uint64_t bd0 = tc::sdesc(b0, 16, 512, tc::kLayoutSW64);
      // Digit pairs (da, db) with da + db < 5 (pairs below 2^-35 of the leading one are
      // dropped).  For one da the products with consecutive db go to consecutive classes,
      // side by side in TMEM, and the B planes sit back to back in shared memory (64 rows
      // each, the same swizzle phase): one product A_da [B_db0; B_db0+1; ..] covers them.
      // One instruction has one accumulate flag, so the pair that opens class 4, (1, 3), is
      // issued on its own: 5 instructions per k-step instead of 13.
      struct Run { int da, db0, nb, open; };
      constexpr Run kRuns[5] = {{0, 0, 4, 1}, {1, 0, 3, 0}, {1, 3, 1, 1}, {2, 0, 3, 0}, {3, 0, 2, 0}};
      static_assert(kHS == 4 && kHClasses == 5, "the runs list the 13 pairs of 4 digits");
#pragma unroll
      for (int k = 0; k < kHBK / 32; ++k) {
#pragma unroll
        for (int r = 0; r < 5; ++r) {
          const Run u = kRuns[r];
          const uint32_t acc = (kc == 0 && k == 0 && u.open) ? 0u : 1u;
          tc::mma_i8(tmem + (u.da + u.db0) * kHBN, ad0 + (uint64_t)((u.da * kHATile + k * 32) >> 4),
                     bd0 + (uint64_t)((u.db0 * kHBTile + k * 32) >> 4),
                     hess_idesc((uint32_t)(u.nb * kHBN)), acc);
        }
      }
      tc::mma_commit(&empty[s]);
    }
    tc::mma_commit(accum);
  }
  __syncwarp();

  const bool ok = tc::mbar_wait(accum, 0);
  if (!ok && lane == 0) record_status(hdr, GQ_ERR_TIMEOUT);
  tc::fence_after_sync();
  const int64_t i = (int64_t)bi * kHBM + warp * 32 + lane;
  const double si = (i < n) ? 2.0 * ldexp(1.0, digit_exponent(maxbits[i])) : 0.0;
  if (ok) {
#pragma unroll 1
    for (int ch = 0; ch < kHBN / 32; ++ch) {
      double acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0.0;
#pragma unroll 1
      for (int c = 0; c < kHClasses; ++c) {
        float v[32];
        tc::tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c * kHBN + ch * 32, v);
        const double w = ldexp(1.0, -7 * (c + 2));
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = fma((double)__float_as_int(v[j]), w, acc[j]);
      }
      const int64_t j0 = (int64_t)bj * kHBN + ch * 32;
      if (i < n) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int64_t col = j0 + j;
          if (col < n && col <= i) {
            const double sj = ldexp(1.0, digit_exponent(maxbits[col]));
            const double v = si * sj * acc[j];
            H[i * n + col] = add ? H[i * n + col] + v : v;
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

__global__ void mirror_lower_kernel(double* H, int64_t n) {
  int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // column (fast)
  int64_t i = blockIdx.y;                                      // row
  if (j < n && i < j) H[i * n + j] = H[j * n + i];
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode_h = nullptr;
std::mutex g_encode_h_mu;

cudaError_t get_encode_h() {
  std::lock_guard<std::mutex> lk(g_encode_h_mu);
  if (g_encode_h) return cudaSuccess;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode_h = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

cudaError_t encode_digits(CUtensorMap* map, const int8_t* D, int64_t rows, int64_t tp,
                          uint32_t box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)tp, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)tp};
  cuuint32_t box[2] = {(cuuint32_t)kHBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode_h(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(D), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int64_t chunk_tokens(int64_t T) { return std::min<int64_t>(T, kHChunk); }
int64_t padded(int64_t t) { return (t + kHBK - 1) / kHBK * kHBK; }

struct HessLayout {
  WsHeader* hdr;
  int* maxbits;
  int8_t* D;
  size_t bytes;
};
HessLayout hess_layout(void* ws, int64_t T, int64_t n) {
  Carver c(ws);
  HessLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.maxbits = c.take<int>(n);
  // rows padded to the 128-row tile so the last tile's loads stay inside the planes
  const int64_t rows = (int64_t)kHS * n + kHBM;
  L.D = c.take<int8_t>((size_t)rows * (size_t)padded(std::max<int64_t>(chunk_tokens(T), 1)));
  L.bytes = c.off;
  return L;
}
}  // namespace

#define H_TRY(x)                        \
  do {                                  \
    cudaError_t _e = (x);               \
    if (_e != cudaSuccess) return _e;   \
  } while (0)

size_t hessian_ws_bytes(int64_t T, int64_t n) { return hess_layout(nullptr, T, n).bytes; }

cudaError_t hessian_init_attributes() {
  return cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kHSmem);
}

cudaError_t launch_hessian(double* H, const void* X, gq_dtype xt, int64_t T, int64_t n,
                           int accumulate, void* ws, cudaStream_t s) {
  if (T == 0) return accumulate ? cudaSuccess : cudaMemsetAsync(H, 0, sizeof(double) * n * n, s);
  H_TRY(get_encode_h());
  HessLayout L = hess_layout(ws, T, n);
  H_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s));
  const int64_t chunk = chunk_tokens(T);
  for (int64_t t0 = 0; t0 < T; t0 += chunk) {
    const int64_t tc = std::min<int64_t>(chunk, T - t0), tp = padded(tc);
    H_TRY(cudaMemsetAsync(L.maxbits, 0, sizeof(int) * n, s));
    {
      dim3 grid((unsigned)((n + 255) / 256), (unsigned)std::min<int64_t>(64, (tc + 63) / 64));
      if (xt == GQ_BF16)
        colmax_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), n, t0, tc, L.maxbits);
      else
        colmax_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(X), n, t0, tc, L.maxbits);
      count_launches(1);
      H_TRY(cudaGetLastError());
    }
    {
      dim3 grid((unsigned)(tp / 32), (unsigned)((n + 31) / 32));
      if (xt == GQ_BF16)
        digits_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), n, t0, tc, tp, L.maxbits, L.D);
      else
        digits_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(X), n, t0, tc, tp, L.maxbits, L.D);
      count_launches(1);
      H_TRY(cudaGetLastError());
    }
    CUtensorMap ma, mb;
    const int64_t rows = (int64_t)kHS * n + kHBM;
    H_TRY(encode_digits(&ma, L.D, rows, tp, kHBM));
    H_TRY(encode_digits(&mb, L.D, rows, tp, kHBN));
    dim3 grid((unsigned)((n + kHBN - 1) / kHBN), (unsigned)((n + kHBM - 1) / kHBM));
    const int add = (t0 > 0 || accumulate) ? 1 : 0;
    hessian_tc_kernel<<<grid, 128, kHSmem, s>>>(ma, mb, H, n, tp, L.maxbits, add, L.hdr);
    count_launches(1);
    H_TRY(cudaGetLastError());
  }
  dim3 grid((unsigned)((n + 255) / 256), (unsigned)n);
  mirror_lower_kernel<<<grid, 256, 0, s>>>(H, n);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
