// C ABI entry points of libgq: argument validation, per-device setup, dispatch.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <atomic>
#include <cstring>
#include <list>
#include <mutex>
#include <vector>

using namespace gq;

namespace gq {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(long k) { g_launches.fetch_add((unsigned long long)k, std::memory_order_relaxed); }

static std::atomic<uint32_t> g_wait_polls{0};  // 0: the default budget
static std::atomic<int> g_wait_withhold{0};
WaitTest wait_test() {
  const uint32_t p = g_wait_polls.load();
  return WaitTest{p ? p : tc::kDefaultPolls, g_wait_withhold.load()};
}
}  // namespace gq

namespace {

constexpr int64_t kMaxN = 32768;
constexpr int64_t kMaxM = int64_t(1) << 24;

std::mutex g_init_mu;
bool g_init_done[128] = {};

gq_status ensure_device_setup() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return GQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_init_mu);
  if (g_init_done[dev]) return GQ_OK;
  if (factor_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  if (quant_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  if (lazy_tc_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  if (hessian_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  if (huffman_init_attributes() != cudaSuccess) return GQ_ERR_CUDA;
  g_init_done[dev] = true;
  return GQ_OK;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// ---- launch-sequence graphs -------------------------------------------------------------
// A call's kernel sequence (hundreds of small dependent launches for the factorisation) is
// captured once per distinct argument list on a private stream, instantiated, and replayed on
// the caller's stream; replay costs one graph launch instead of one launch per kernel.  A
// caller that is itself capturing gets the plain launches recorded into its own graph.
struct GraphEntry {
  int device;
  std::vector<uint64_t> key;
  cudaGraphExec_t exec;
  unsigned long long kernels;  // kernel nodes, counted in gq_kernel_launches per replay
};
std::mutex g_graph_mu;
std::list<GraphEntry> g_graphs;  // most recently used first
constexpr size_t kMaxGraphs = 32;
cudaStream_t g_capture_stream[128] = {};

template <class Enqueue>
gq_status run_graphed(std::vector<uint64_t> key, cudaStream_t user, Enqueue enqueue) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(user, &cs) != cudaSuccess) return GQ_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return enqueue(user);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_graph_mu);
  for (auto it = g_graphs.begin(); it != g_graphs.end(); ++it) {
    if (it->device == dev && it->key == key) {
      g_graphs.splice(g_graphs.begin(), g_graphs, it);
      if (cudaGraphLaunch(it->exec, user) != cudaSuccess) return GQ_ERR_CUDA;
      count_launches((long)it->kernels);
      return GQ_OK;
    }
  }
  if (!g_capture_stream[dev] &&
      cudaStreamCreateWithFlags(&g_capture_stream[dev], cudaStreamNonBlocking) != cudaSuccess)
    return GQ_ERR_CUDA;
  cudaStream_t cap = g_capture_stream[dev];
  if (cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return GQ_ERR_CUDA;
  const unsigned long long before = g_launches.load();
  gq_status st = enqueue(cap);
  const unsigned long long kernels = g_launches.load() - before;
  g_launches.fetch_sub(kernels);  // captured, not yet run
  cudaGraph_t graph = nullptr;
  cudaError_t ec = cudaStreamEndCapture(cap, &graph);
  if (st != GQ_OK || ec != cudaSuccess || !graph) {
    if (graph) cudaGraphDestroy(graph);
    (void)cudaGetLastError();
    return st != GQ_OK ? st : GQ_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  ec = cudaGraphInstantiateWithFlags(&exec, graph, cudaGraphInstantiateFlagUseNodePriority);
  cudaGraphDestroy(graph);
  if (ec != cudaSuccess) {
    (void)cudaGetLastError();
    return enqueue(user);  // not instantiable: plain launches on the caller's stream
  }
  if (g_graphs.size() >= kMaxGraphs) {
    cudaGraphExecDestroy(g_graphs.back().exec);
    g_graphs.pop_back();
  }
  g_graphs.push_front(GraphEntry{dev, std::move(key), exec, kernels});
  if (cudaGraphLaunch(exec, user) != cudaSuccess) return GQ_ERR_CUDA;
  count_launches((long)kernels);
  return GQ_OK;
}

uint64_t bits_of(double d) {
  uint64_t u;
  std::memcpy(&u, &d, sizeof u);
  return u;
}
uint64_t P(const void* p) { return (uint64_t)(uintptr_t)p; }

}  // namespace

extern "C" {

const char* gq_version(void) { return "gq 0.1 sm_100a"; }

unsigned long long gq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gq_status_string(gq_status s) {
  switch (s) {
    case GQ_OK: return "ok";
    case GQ_ERR_INVALID_ARG: return "invalid argument";
    case GQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case GQ_ERR_CUDA: return "CUDA runtime error";
    case GQ_ERR_UNSUPPORTED: return "unsupported combination of settings";
    case GQ_ERR_TIMEOUT: return "bounded device wait ran out";
    case GQ_ERR_NO_FIT: return "clip-free scale ladder exhausted";
    case GQ_ERR_WORKSPACE: return "workspace too small or misaligned";
  }
  return "unknown status";
}

size_t gq_hessian_workspace_size(int64_t T, int64_t n) {
  if (T < 0 || n < 1 || n > kMaxN || T > (int64_t(1) << 31) - 1) return 0;
  return hessian_ws_bytes(T, n);
}

gq_status gq_hessian_accumulate(double* d_H, const void* d_X, gq_dtype x_dtype, int64_t T,
                                int64_t n, int accumulate, void* d_ws, size_t ws_bytes,
                                gq_stream_t stream) {
  if (T < 0 || n < 1 || n > kMaxN || T > (int64_t(1) << 31) - 1) return GQ_ERR_INVALID_ARG;
  if (x_dtype != GQ_BF16 && x_dtype != GQ_FP32) return GQ_ERR_INVALID_ARG;
  if (!d_H || (T > 0 && !d_X) || !d_ws) return GQ_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < hessian_ws_bytes(T, n)) return GQ_ERR_WORKSPACE;
  if (T == 0 && accumulate) return GQ_OK;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  auto enqueue = [&](cudaStream_t s) {
    return launch_hessian(d_H, d_X, x_dtype, T, n, accumulate, d_ws, s) == cudaSuccess
               ? GQ_OK : GQ_ERR_CUDA;
  };
  return run_graphed({3, P(d_H), P(d_X), (uint64_t)x_dtype, (uint64_t)T, (uint64_t)n,
                      (uint64_t)accumulate, P(d_ws)},
                     (cudaStream_t)stream, enqueue);
}

size_t gq_prepare_workspace_size(int64_t n) {
  if (n < 1 || n > kMaxN) return 0;
  return prepare_ws_bytes(n);
}

gq_status gq_prepare_hinv(const double* d_H, int64_t n, double damp, int reverse, float* d_U,
                          uint8_t* d_dead, double* d_delta, void* d_ws, size_t ws_bytes,
                          gq_stream_t stream) {
  if (n < 1 || n > kMaxN || !(damp >= 0.0) || (reverse != 0 && reverse != 1))
    return GQ_ERR_INVALID_ARG;
  if (!d_H || !d_U || !d_dead || !d_delta || !d_ws) return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < prepare_ws_bytes(n)) return GQ_ERR_WORKSPACE;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  auto enqueue = [&](cudaStream_t s) {
    return launch_prepare(d_H, n, damp, reverse, nullptr, d_U, d_dead, d_delta, d_ws, s) ==
                   cudaSuccess
               ? GQ_OK : GQ_ERR_CUDA;
  };
  const WaitTest wt = wait_test();
  return run_graphed({1, P(d_H), (uint64_t)n, bits_of(damp), (uint64_t)reverse, P(d_U),
                      P(d_dead), P(d_delta), P(d_ws), wt.polls, (uint64_t)wt.withhold},
                     (cudaStream_t)stream, enqueue);
}

gq_status gq_prepare_hinv_ordered(const double* d_H, int64_t n, double damp, gq_order order,
                                  int32_t* d_perm, float* d_U, uint8_t* d_dead, double* d_delta,
                                  void* d_ws, size_t ws_bytes, gq_stream_t stream) {
  const int o = (int)order;
  if (o < GQ_ORDER_NATURAL || o > GQ_ORDER_GIVEN) return GQ_ERR_INVALID_ARG;
  if (o == GQ_ORDER_NATURAL || o == GQ_ORDER_REVERSE)
    return gq_prepare_hinv(d_H, n, damp, o, d_U, d_dead, d_delta, d_ws, ws_bytes, stream);
  if (n < 1 || n > kMaxN || !(damp >= 0.0)) return GQ_ERR_INVALID_ARG;
  if (!d_H || !d_U || !d_dead || !d_delta || !d_ws || !d_perm) return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < prepare_ws_bytes(n)) return GQ_ERR_WORKSPACE;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  auto enqueue = [&](cudaStream_t s) {
    return launch_prepare(d_H, n, damp, o, d_perm, d_U, d_dead, d_delta, d_ws, s) == cudaSuccess
               ? GQ_OK : GQ_ERR_CUDA;
  };
  const WaitTest wt = wait_test();
  return run_graphed({4, P(d_H), (uint64_t)n, bits_of(damp), (uint64_t)o, P(d_perm), P(d_U),
                      P(d_dead), P(d_delta), P(d_ws), wt.polls, (uint64_t)wt.withhold},
                     (cudaStream_t)stream, enqueue);
}

static gq_status check_cfg(const gq_quant_cfg* cfg) {
  if (!cfg) return GQ_ERR_INVALID_ARG;
  if (cfg->bits < 2 || cfg->bits > 8) return GQ_ERR_INVALID_ARG;
  if (cfg->reverse != 0 && cfg->reverse != 1) return GQ_ERR_INVALID_ARG;
  if (cfg->clip < 0 || cfg->clip > 2) return GQ_ERR_INVALID_ARG;
  const int g = cfg->group_size;
  if (g != 0 && g != 16 && g != 32 && g != 64 && g != 128) {
    return (g > 0 && g <= 128 && kBlock % g == 0) ? GQ_ERR_UNSUPPORTED : GQ_ERR_INVALID_ARG;
  }
  if (g != 0 && (cfg->reverse || cfg->clip != 1)) return GQ_ERR_UNSUPPORTED;
  if (cfg->clip == 2 && cfg->reverse) return GQ_ERR_UNSUPPORTED;
  if (cfg->spacing != 0 && cfg->spacing != 1) return GQ_ERR_INVALID_ARG;
  if (cfg->spacing && (g != 0 || cfg->reverse)) return GQ_ERR_UNSUPPORTED;
  if (!cfg->clip) {
    if (!(cfg->ladder > 1.f) || cfg->ladder_max < 0 || cfg->ladder_max > 64)
      return GQ_ERR_INVALID_ARG;
  }
  return GQ_OK;
}

size_t gq_quantize_workspace_size(int64_t m, int64_t n, const gq_quant_cfg* cfg) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN || check_cfg(cfg) != GQ_OK) return 0;
  return quantize_ws_bytes(m, n, *cfg);
}

static gq_status quantize_common(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                 const float* d_U, const uint8_t* d_dead, const double* d_delta,
                                 const gq_quant_cfg* cfg, const int32_t* d_perm,
                                 uint32_t* d_codes, float* d_scales, uint8_t* d_zeros,
                                 double* d_loss, void* d_ws, size_t ws_bytes,
                                 gq_stream_t stream) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN) return GQ_ERR_INVALID_ARG;
  if (w_dtype != GQ_BF16 && w_dtype != GQ_FP32) return GQ_ERR_INVALID_ARG;
  gq_status st = check_cfg(cfg);
  if (st != GQ_OK) return st;
  if (!d_W || !d_U || !d_codes || !d_scales || !d_zeros || !d_loss || !d_ws)
    return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < quantize_ws_bytes(m, n, *cfg)) return GQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(d_U) & 15u) != 0) return GQ_ERR_INVALID_ARG;
  st = ensure_device_setup();
  if (st != GQ_OK) return st;
  QuantArgs a{};
  a.W = d_W; a.wt = w_dtype; a.m = m; a.n = n; a.U = d_U; a.dead = d_dead; a.delta = d_delta;
  a.cfg = *cfg; a.codes = d_codes; a.scales = d_scales; a.zeros = d_zeros; a.loss = d_loss;
  a.ws = d_ws; a.perm = d_perm;
  if (!cfg->clip) return run_quantize(a, (cudaStream_t)stream);  // the ladder reads back counts
  auto enqueue = [&](cudaStream_t s) { return run_quantize(a, s); };
  return run_graphed({2, P(d_W), (uint64_t)w_dtype, (uint64_t)m, (uint64_t)n, P(d_U), P(d_dead),
                      P(d_delta), (uint64_t)cfg->bits, (uint64_t)cfg->group_size,
                      (uint64_t)cfg->reverse, (uint64_t)cfg->clip, (uint64_t)cfg->spacing,
                      P(d_perm), P(d_codes),
                      P(d_scales), P(d_zeros), P(d_loss), P(d_ws)},
                     (cudaStream_t)stream, enqueue);
}

gq_status gq_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                            const float* d_U, const uint8_t* d_dead, const double* d_delta,
                            const gq_quant_cfg* cfg, uint32_t* d_codes, float* d_scales,
                            uint8_t* d_zeros, double* d_loss, void* d_ws, size_t ws_bytes,
                            gq_stream_t stream) {
  return quantize_common(d_W, w_dtype, m, n, d_U, d_dead, d_delta, cfg, nullptr, d_codes,
                         d_scales, d_zeros, d_loss, d_ws, ws_bytes, stream);
}

gq_status gq_quantize_layer_ordered(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                    const float* d_U, const uint8_t* d_dead,
                                    const double* d_delta, const gq_quant_cfg* cfg,
                                    const int32_t* d_perm, uint32_t* d_codes, float* d_scales,
                                    uint8_t* d_zeros, double* d_loss, void* d_ws,
                                    size_t ws_bytes, gq_stream_t stream) {
  if (!d_perm || !cfg || cfg->reverse) return GQ_ERR_INVALID_ARG;
  return quantize_common(d_W, w_dtype, m, n, d_U, d_dead, d_delta, cfg, d_perm, d_codes,
                         d_scales, d_zeros, d_loss, d_ws, ws_bytes, stream);
}

size_t gq_ssqr_workspace_size(int64_t m, int64_t n) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN) return 0;
  return ssqr_ws_bytes(m, n);
}

gq_status gq_ssqr_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                 const float* d_U, const uint8_t* d_dead, const double* d_delta,
                                 int bits, double density, int steps, int max_doublings,
                                 uint32_t* d_codes, float* d_scales, uint8_t* d_zeros,
                                 double* d_alpha, int64_t* d_row_ptr, int32_t* d_col_idx,
                                 float* d_values, int64_t nnz_capacity, double* d_loss,
                                 void* d_ws, size_t ws_bytes, gq_stream_t stream) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN) return GQ_ERR_INVALID_ARG;
  if (w_dtype != GQ_BF16 && w_dtype != GQ_FP32) return GQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || !(density >= 0.0 && density <= 1.0)) return GQ_ERR_INVALID_ARG;
  if (steps < 0 || steps > 60 || max_doublings < 0 || max_doublings > 30 || nnz_capacity < 0)
    return GQ_ERR_INVALID_ARG;
  if (!d_W || !d_U || !d_codes || !d_scales || !d_zeros || !d_alpha || !d_row_ptr || !d_loss ||
      !d_ws)
    return GQ_ERR_INVALID_ARG;
  if (nnz_capacity > 0 && (!d_col_idx || !d_values)) return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < ssqr_ws_bytes(m, n)) return GQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(d_U) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(d_row_ptr) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(d_alpha) & 7u) != 0)
    return GQ_ERR_INVALID_ARG;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  QuantArgs a{};
  a.W = d_W; a.wt = w_dtype; a.m = m; a.n = n; a.U = d_U; a.dead = d_dead; a.delta = d_delta;
  a.cfg = gq_quant_cfg{bits, 0, 0, 3, 1.25f, 0, 0};
  a.codes = d_codes; a.scales = d_scales; a.zeros = d_zeros; a.loss = d_loss; a.ws = d_ws;
  a.perm = nullptr;
  SsqrArgs o{};
  o.density = density; o.steps = steps; o.max_doublings = max_doublings; o.alpha = d_alpha;
  o.row_ptr = reinterpret_cast<long long*>(d_row_ptr); o.col_idx = d_col_idx;
  o.values = d_values; o.capacity = nnz_capacity;
  return run_ssqr(a, o, (cudaStream_t)stream);  // synchronizes per doubling round
}

size_t gq_hptq_workspace_size(int64_t m, int64_t n) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN || m * n > (int64_t(1) << 31) - 1) return 0;
  return hptq_ws_bytes(m, n);
}

gq_status gq_hptq_quantize_layer(const void* d_W, gq_dtype w_dtype, int64_t m, int64_t n,
                                 const float* d_U, const uint8_t* d_dead, const double* d_delta,
                                 int bits, double budget, int steps, int max_doublings,
                                 int32_t* d_codes, float* d_scales, double* d_alpha,
                                 int64_t* d_total_bits, double* d_loss, void* d_ws,
                                 size_t ws_bytes, gq_stream_t stream) {
  if (m < 1 || m > kMaxM || n < 1 || n > kMaxN || m * n > (int64_t(1) << 31) - 1)
    return GQ_ERR_INVALID_ARG;
  if (w_dtype != GQ_BF16 && w_dtype != GQ_FP32) return GQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 8 || !(budget > 0.0 && budget < 64.0)) return GQ_ERR_INVALID_ARG;
  if (steps < 0 || steps > 60 || max_doublings < 0 || max_doublings > 30)
    return GQ_ERR_INVALID_ARG;
  if (!d_W || !d_U || !d_codes || !d_scales || !d_alpha || !d_total_bits || !d_loss || !d_ws)
    return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < hptq_ws_bytes(m, n)) return GQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(d_U) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(d_alpha) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(d_total_bits) & 7u) != 0)
    return GQ_ERR_INVALID_ARG;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  QuantArgs a{};
  a.W = d_W; a.wt = w_dtype; a.m = m; a.n = n; a.U = d_U; a.dead = d_dead; a.delta = d_delta;
  a.cfg = gq_quant_cfg{bits, 0, 0, 2, 1.25f, 0, 0};
  a.codes = reinterpret_cast<uint32_t*>(d_codes); a.scales = d_scales; a.zeros = nullptr;
  a.loss = d_loss; a.ws = d_ws; a.perm = nullptr;
  HptqArgs o{};
  o.budget = budget; o.steps = steps; o.max_doublings = max_doublings; o.alpha = d_alpha;
  o.total_bits = reinterpret_cast<long long*>(d_total_bits);
  return run_hptq(a, o, (cudaStream_t)stream);  // synchronizes once per pass
}

gq_status gq_zsic_spacing(const float* d_U, int64_t n, double* d_kappa, gq_stream_t stream) {
  if (n < 1 || n > kMaxN || !d_U || !d_kappa) return GQ_ERR_INVALID_ARG;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  return launch_zsic_spacing(d_U, n, d_kappa, (cudaStream_t)stream) == cudaSuccess ? GQ_OK
                                                                                   : GQ_ERR_CUDA;
}

size_t gq_huffman_workspace_size(int64_t count) {
  if (count < 1 || count > (int64_t(1) << 31) - 1) return 0;
  return huffman_ws_bytes(count);
}

gq_status gq_huffman_encode(const int32_t* d_codes, int64_t count, uint64_t* d_stream,
                            int64_t stream_words, uint8_t* d_lengths, uint64_t* d_codewords,
                            int64_t* d_info, void* d_ws, size_t ws_bytes, gq_stream_t stream) {
  if (count < 1 || count > (int64_t(1) << 31) - 1 || stream_words < 1) return GQ_ERR_INVALID_ARG;
  if (!d_codes || !d_stream || !d_lengths || !d_codewords || !d_info || !d_ws)
    return GQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_stream) & 7u) || (reinterpret_cast<uintptr_t>(d_codewords) & 7u) ||
      (reinterpret_cast<uintptr_t>(d_info) & 7u) || (reinterpret_cast<uintptr_t>(d_codes) & 3u))
    return GQ_ERR_INVALID_ARG;
  if (!aligned256(d_ws) || ws_bytes < huffman_ws_bytes(count)) return GQ_ERR_WORKSPACE;
  gq_status st = ensure_device_setup();
  if (st != GQ_OK) return st;
  auto enqueue = [&](cudaStream_t s) {
    return launch_huffman(d_codes, count, reinterpret_cast<unsigned long long*>(d_stream),
                          stream_words, d_lengths,
                          reinterpret_cast<unsigned long long*>(d_codewords),
                          reinterpret_cast<long long*>(d_info), d_ws, s) == cudaSuccess
               ? GQ_OK : GQ_ERR_CUDA;
  };
  return run_graphed({5, P(d_codes), (uint64_t)count, P(d_stream), (uint64_t)stream_words,
                      P(d_lengths), P(d_codewords), P(d_info), P(d_ws)},
                     (cudaStream_t)stream, enqueue);
}

gq_status gq_debug_wait_test(uint32_t poll_limit, int withhold_arrival) {
  if (withhold_arrival != 0 && withhold_arrival != 1) return GQ_ERR_INVALID_ARG;
  gq::g_wait_polls.store(poll_limit);
  gq::g_wait_withhold.store(withhold_arrival);
  return GQ_OK;
}

gq_status gq_workspace_status(void* d_ws, int* h_ladder_rounds, gq_stream_t stream) {
  if (!d_ws) return GQ_ERR_INVALID_ARG;
  WsHeader h{};
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, d_ws, sizeof(WsHeader), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GQ_ERR_CUDA;
  if (h_ladder_rounds) *h_ladder_rounds = h.ladder_rounds;
  if (h.status != 0) {
    int zero = 0;
    if (cudaMemcpyAsync(d_ws, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
      return GQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GQ_ERR_CUDA;
  }
  return (gq_status)h.status;
}

}  // extern "C"
