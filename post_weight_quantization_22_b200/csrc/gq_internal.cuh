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
cudaError_t launch_prepare(const double* H, int64_t n, double damp, int reverse, float* U,
                           uint8_t* dead, double* delta, void* ws, cudaStream_t s);

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
};
size_t quantize_ws_bytes(int64_t m, int64_t n, const gq_quant_cfg& cfg);
// Returns GQ_OK or an error; the clip-free ladder synchronizes the stream per round.
gq_status run_quantize(const QuantArgs& a, cudaStream_t s);

constexpr int kBlock = 128;  // columns per GPTQ block (lazy-update rank)

// Kernel launches issued by this library since load (instrumentation; see gq_kernel_launches).
void count_launches(long k);

// one-time per-device kernel attribute setup (dynamic shared memory above 48 KB)
cudaError_t factor_init_attributes();
cudaError_t quant_init_attributes();
cudaError_t lazy_tc_init_attributes();

// ---- lazy block update on tensor cores (gq_lazy_tc.cu) ----
struct LazyTcMaps {
  CUtensorMap ahi, alo, bhi, blo;
};
// E_hi / E_lo: rows x 128 fp32; U_hi / U_lo: n x n fp32 with leading dimension ldu (mult. of 4)
cudaError_t lazy_tc_make_maps(LazyTcMaps* maps, const float* Ehi, const float* Elo, int64_t rows,
                              const float* Uhi, const float* Ulo, int64_t n, int64_t ldu);
// Wf[:, j1:] -= (E_hi + E_lo) (U_hi + U_lo)[j0:j0+128, j1:]  (3xTF32), rows < k_rows
cudaError_t launch_lazy_tc(const LazyTcMaps& maps, float* Wf, int64_t n, int64_t k_rows,
                           int64_t j0, int64_t j1, WsHeader* hdr, cudaStream_t s);

}  // namespace gq
