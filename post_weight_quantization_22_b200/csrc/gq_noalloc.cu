// gq_prepare_hinv_static: the factor preparation for callers that must not allocate device
// memory.
//
// Some hosts run this library where a device allocation is not allowed or not possible at the
// moment of the call: an inference engine's plugin whose memory plan was fixed before it ran,
// code recorded into a CUDA graph under a capture mode that forbids cudaMalloc, or a service
// that owns all device memory through its own pool and hands out only input and output
// buffers.  Such a caller cannot provide the n x n fp64 workspace gq_prepare_hinv needs.  This
// entry point uses a scratch area compiled into the library instead: a file-scope static
// device array, sized for layers up to kStaticMaxN input features.  Every GPU that loads the
// library holds that array (about 17 MB) until the process exits.
//
// The same kernels run as in gq_prepare_hinv, in the same order, on the caller's stream; only
// the scratch address differs.
#include "gq_internal.cuh"

#include <mutex>

namespace {

constexpr int64_t kStaticMaxN = 1024;
constexpr size_t kStaticBytes = size_t(17) << 20;  // >= the workspace of width kStaticMaxN

// One scratch area per device that loads the library, shared by every call on that device.
static __device__ __align__(256) unsigned char g_prepare_scratch[kStaticBytes];

std::mutex g_addr_mu;
void* g_addr[128] = {};

// Device address of the scratch array on the current device.  In host code the array's name
// only stands in for the device object, so the address is looked up once per device with that
// device current.
gq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return GQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_addr_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_prepare_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return GQ_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return GQ_OK;
}

}  // namespace

extern "C" gq_status gq_prepare_hinv_static(const double* d_H, int64_t n, double damp,
                                            int reverse, float* d_U, uint8_t* d_dead,
                                            double* d_delta, int* d_status, gq_stream_t stream) {
  if (n < 1 || n > kStaticMaxN || !(damp >= 0.0) || (reverse != 0 && reverse != 1))
    return GQ_ERR_INVALID_ARG;
  if (!d_H || !d_U || !d_dead || !d_delta) return GQ_ERR_INVALID_ARG;
  if (gq::prepare_ws_bytes(n) > kStaticBytes) return GQ_ERR_INVALID_ARG;
  void* scratch = nullptr;
  gq_status st = scratch_address(&scratch);
  if (st != GQ_OK) return st;
  if (gq::factor_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // launch_prepare clears the scratch's status word first and writes every other scratch
  // element it reads before reading it, so the previous call's contents do not leak in.
  if (gq::launch_prepare(d_H, n, damp, reverse, nullptr, d_U, d_dead, d_delta, scratch, s) != cudaSuccess)
    return GQ_ERR_CUDA;
  if (d_status &&
      cudaMemcpyAsync(d_status, scratch, sizeof(int), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return GQ_ERR_CUDA;
  return GQ_OK;
}
