// Internal declarations shared by the libgq translation units (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/gq.h"

namespace gq {

// Workspace header: the first 256 bytes of every workspace.  Device kernels record the first
// error they detect in `status` (atomicCAS from 0); gq_workspace_status reads and clears it.
struct WsHeader {
  int status;
  int ladder_rounds;
  int overflow_rows;
  int pad0;
  double scratch[8];
};

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Carve consecutive aligned sub-buffers out of a workspace.
struct Carver {
  char* base;
  size_t off;
  explicit Carver(void* b) : base(static_cast<char*>(b)), off(0) {}
  template <class T>
  T* take(size_t count) {
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

__device__ __forceinline__ void record_status(WsHeader* h, int code) {
  if (h) atomicCAS(&h->status, 0, code);
}

// ---- Hessian (H += 2 X^T X, fp64-accurate) ----
size_t hessian_ws_bytes(int64_t T, int64_t n);
cudaError_t hessian_init_attributes();
cudaError_t launch_hessian(double* H, const void* X, gq_dtype xt, int64_t T, int64_t n,
                           int accumulate, void* ws, cudaStream_t s);

// ---- factor preparation ----
size_t prepare_ws_bytes(int64_t n);
// order: a gq_order value other than MIN_PIVOT; perm (n ints) is written for ACT, read for
// GIVEN and not used for NATURAL / REVERSE (may be null there).
cudaError_t launch_prepare(const double* H, int64_t n, double damp, int order, int* perm,
                           float* U, uint8_t* dead, double* delta, void* ws, cudaStream_t s);

// perm[k] as an index that is always in [0, n) (0 for an out-of-range entry; a caller-given
// permutation is validated separately and reported through the workspace status).
__device__ __forceinline__ int64_t perm_at(const int* perm, int64_t k, int64_t n) {
  unsigned p = (unsigned)perm[k];
  return p < (unsigned long long)n ? (int64_t)p : 0;
}

// ---- quantization ----
struct QuantArgs {
  const void* W;
  gq_dtype wt;
  int64_t m, n;
  const float* U;
  const uint8_t* dead;
  const double* delta;
  gq_quant_cfg cfg;
  uint32_t* codes;
  float* scales;
  uint8_t* zeros;
  double* loss;
  void* ws;
  const int* perm;  // processing order (null: natural, or reversed when cfg.reverse)
  double lattice_alpha = 1.0;  // unconstrained lattice (clip 2): step = min-max step x this
};
size_t quantize_ws_bytes(int64_t m, int64_t n, const gq_quant_cfg& cfg);
// SSQR outlier search (cfg.clip = 3, one grid per row, natural order): its workspace, and the
// search + final pass with the outliers written as CSR.
size_t ssqr_ws_bytes(int64_t m, int64_t n);
struct SsqrArgs {
  double density;
  int steps, max_doublings;
  double* alpha;        // m, out
  long long* row_ptr;   // m + 1, out
  int* col_idx;         // capacity, out
  float* values;        // capacity, out
  int64_t capacity;
};
cudaError_t launch_zsic_spacing(const float* U, int64_t n, double* kappa, cudaStream_t s);

// ---- canonical Huffman coding of int32 codes ----
size_t huffman_ws_bytes(int64_t count);
cudaError_t huffman_init_attributes();
cudaError_t launch_huffman(const int* codes, int64_t count, unsigned long long* stream_words,
                           int64_t nwords, uint8_t* lengths, unsigned long long* words,
                           long long* info, void* ws, cudaStream_t s);
// range, histogram and canonical code only: info[2] = total bits of the coded stream
cudaError_t launch_huffman_stats(const int* codes, int64_t count, uint8_t* lengths,
                                 unsigned long long* words, long long* info, void* ws,
                                 cudaStream_t s);
// HPTQ rate control (cfg.clip = 2, one grid per row, natural order): the smallest lattice
// factor alpha whose Huffman-coded codes fit a budget in bits per weight.
size_t hptq_ws_bytes(int64_t m, int64_t n);
struct HptqArgs {
  double budget;          // bits per weight
  int steps, max_doublings;
  double* alpha;          // 1, out
  long long* total_bits;  // 1, out: coded size of the codes at alpha
};
// Synchronizes the stream once per pass of the search.
gq_status run_hptq(const QuantArgs& a, const HptqArgs& o, cudaStream_t s);
// Returns GQ_OK or an error; the clip-free ladder synchronizes the stream per round.
gq_status run_quantize(const QuantArgs& a, cudaStream_t s);
// Synchronizes the stream once per doubling round of the search.
gq_status run_ssqr(const QuantArgs& a, const SsqrArgs& o, cudaStream_t s);

constexpr int kBlock = 128;  // columns per GPTQ block (lazy-update rank)

// Kernel launches issued by this library since load (instrumentation; see gq_kernel_launches).
void count_launches(long k);

// Test setting of the bounded waits (gq_debug_wait_test): the poll budget of the factor leaf
// kernel's per-pivot waits and whether that kernel withholds one thread's first arrival.
struct WaitTest {
  uint32_t polls;
  int withhold;
};
WaitTest wait_test();

// one-time per-device kernel attribute setup (dynamic shared memory above 48 KB)
cudaError_t factor_init_attributes();
cudaError_t quant_init_attributes();
cudaError_t lazy_tc_init_attributes();

// ---- TMA tensor maps (gq_lazy_tc.cu) ----
// Row-major matrix (rows x cols elements of elem_bytes, leading dimension ld elements) as a 2-D
// tensor map with a box of box_cols x box_rows elements, zero fill outside the matrix.
cudaError_t encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, size_t elem_bytes,
                           const void* p, int64_t rows, int64_t cols, int64_t ld,
                           uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

// ---- fp64 GEMM on the fp64 tensor cores (gq_dgemm.cu) ----
// A matrix operand: a row-major fp64 matrix (rows x cols, leading dimension ld, 16-byte aligned
// base, ld even) and the position of the GEMM's operand block inside it; batch z adds
// (zrow, zcol) to the position.
struct DgemmOperand {
  const double* base;
  int64_t rows, cols, ld;
  int64_t row0, col0, zrow, zcol;
};
// C[i][j] = (beta_one ? C[i][j] : 0) + alpha * sum_k opA[i][k] opB[k][j], i < M, j < N, k < K.
//   opA[i][k] = A(row0 + i, col0 + k)                      (contraction index contiguous)
//   opB[k][j] = B(row0 + j, col0 + k)  if !b_nmajor         ("NT": contraction contiguous)
//             = B(row0 + k, col0 + j)  if  b_nmajor         ("NN": output index contiguous)
// Structure: a_lower (opA[i][k] = 0 for k > i), b_lower (opB[k][j] = 0 for k < j), b_upper
// (opB[k][j] = 0 for k > j): the zero parts are never multiplied, whatever memory holds there.
// lower_tiles: only output tiles that reach the diagonal i >= j are computed.
struct DgemmCall {
  int M, N, K, batch;
  double alpha;
  int beta_one;
  DgemmOperand A, B;
  int b_nmajor;
  double* C;
  int64_t ldc, strideC;
  int a_lower, b_lower, b_upper, lower_tiles;
  WsHeader* hdr;
};
cudaError_t dgemm_init_attributes();
cudaError_t launch_dgemm(const DgemmCall& c, cudaStream_t s);

// ---- fp64-accurate products from int8 digit products (gq_split.cu) ----
constexpr int kSplitDigits = 6;  // signed 7-bit digits per value
constexpr int kSplitK = 512;     // depth of every split product (one super-panel of the split path)
// Digit planes of an operand: plane s is plane_rows x kSplitK int8 (K-major rows), planes
// stacked at plane_rows x kSplitK bytes; ex[r] is the power-of-two scale exponent of row r.
struct SplitOperand {
  int8_t* digits;
  int* ex;
  int64_t plane_rows;
};
cudaError_t split_init_attributes();
// digits of the rows of A (rows x kSplitK fp64, leading dimension lda, 16-byte aligned);
// tri: A is lower triangular from (0, 0), entries right of the diagonal count as zero
cudaError_t launch_split_rows(const double* A, int64_t lda, int rows, SplitOperand op,
                              cudaStream_t s, int tri = 0);
// digits of the columns of X (kSplitK rows x cols fp64, leading dimension ldx) as operand rows;
// tri: X is lower triangular from (0, 0), entries above the diagonal count as zero
cudaError_t launch_split_cols(const double* X, int64_t ldx, int cols, SplitOperand op,
                              cudaStream_t s, int tri = 0);
// C[i][j] += alpha sum_k A(a_row0 + i, k) B(b_row0 + j, k), i < M, j < N (only j <= i when
// lower), C fp64 row-major with leading dimension ldc.
cudaError_t launch_split_gemm(double* C, int64_t ldc, int M, int N, const SplitOperand& A,
                              int a_row0, const SplitOperand& B, int b_row0, double alpha,
                              int lower, WsHeader* hdr, cudaStream_t s);

// ---- lazy block update on tensor cores (gq_lazy_tc.cu) ----
struct LazyTcMaps {
  CUtensorMap ahi, alo, bhi, blo;
};
// E_hi / E_lo: rows x n fp32 with leading dimension ldE (multiple of 4); U_hi / U_lo: n x n
// fp32 with leading dimension ldu (multiple of 4)
cudaError_t lazy_tc_make_maps(LazyTcMaps* maps, const float* Ehi, const float* Elo, int64_t rows,
                              int64_t ldE, const float* Uhi, const float* Ulo, int64_t n,
                              int64_t ldu);
// Wf[:, j1:jend] -= (E_hi + E_lo)[:, k0:k0+K] (U_hi + U_lo)[k0:k0+K, j1:jend]  (3xTF32),
// rows < k_rows; K and k0 multiples of 16, k0 + K <= n.
cudaError_t launch_lazy_tc(const LazyTcMaps& maps, float* Wf, int64_t n, int64_t k_rows,
                           int64_t k0, int K, int64_t j1, int64_t jend, WsHeader* hdr,
                           cudaStream_t s);

}  // namespace gq
