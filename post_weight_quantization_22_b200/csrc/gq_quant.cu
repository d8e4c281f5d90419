// The GPTQ / Babai column loop with lazy block updates, code packing and losses.
//
// Sources: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 2.2 (GPTQ's error propagation is the nearest-plane step; back to front it is Babai),
// section 2.3 (no-clipping setting; Theorem 5 bound (1/4) sum s^2 D_jj; the order's role),
// section 3 (HPTQ: one unconstrained integer grid); "WaterSIC", section 2 (ZSIC spacing);
// "RDQ: Residual Distribution Quantization", setup (group-128 asymmetric integer format).
//
// Work layout: the weights are copied once into an fp32 work matrix Wf (rows x n) in the
// processing order (natural, reversed, or a permutation; dead columns zeroed).  Per 128-column
// block: `colloop` runs the column recursion for 32 rows per CTA (8 per warp, in 8-column
// tiles with fp64 tensor-core updates between tiles), keeping the block's part of U in shared
// memory; the tensor-core lazy update (gq_lazy_tc.cu) then applies
// W[:, j+128:] -= E U[j:j+128, j+128:] to the rest of the work matrix.  Grids: per row or per
// group (min-max), clip-free with a per-row ladder, the unconstrained lattice s Z (int32 codes),
// and ZSIC per-column spacing on a per-row grid.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <algorithm>
#include <math.h>

namespace gq {

constexpr int kColWarps = 4;                    // warps per column-loop CTA, 8 rows each
constexpr int kColThreads = 32 * kColWarps;
constexpr int kRowsPerCta = 8 * kColWarps;      // 32 rows per CTA
constexpr int kTiles = kBlock / 8;              // 8-column tiles of a block
constexpr int kUtPitch = 136;                   // floats per row of the transposed U block
// Per-block prepared U for the column loop (see ublk_kernel): the transposed block in fp32
// (128 rows of kUtPitch floats), then 1/U_jj and kappa_j^2 / U_jj^2 in fp64, then the ZSIC
// column factors kappa_j and 1/kappa_j (all 1 for one step per row).  The column loop copies the
// first kUBlkBytes, or all kUBlkBytesZ bytes when the columns have their own spacing.
constexpr uint32_t kUtBytes = (uint32_t)(kBlock * kUtPitch * sizeof(float));
constexpr uint32_t kUBlkBytes = kUtBytes + 2 * kBlock * (uint32_t)sizeof(double);
constexpr uint32_t kUBlkBytesZ = kUtBytes + 4 * kBlock * (uint32_t)sizeof(double);
constexpr int64_t kUBlkDoubles = kUBlkBytesZ / sizeof(double);  // stride between blocks
static_assert(kUBlkBytes % 16 == 0 && kUBlkBytesZ % 16 == 0, "bulk copies move multiples of 16 bytes");
constexpr uint32_t kBulkChunk = 32768;

struct QLayout {
  WsHeader* hdr;
  float* Wf;        // k x n work matrix (compact rows)
  float* Ehi;       // k x ldE scaled errors of every column, tf32 part (processing order)
  float* Elo;       // k x ldE fp32 remainder (E = Ehi + Elo)
  int64_t ldE;
  float* Uhi;       // n x ldu tf32 part of U (columns >= n zero)
  float* Ulo;       // n x ldu fp32 remainder
  int64_t ldu;
  double* Ublk;     // per-block prepared U for the column loop
  uint8_t* codes8;  // m x ldc8 codes in processing order
  int64_t ldc8;
  double* row_s;    // per-row step (group_size 0)
  double* row_z;    // per-row zero point (group_size 0)
  float* alpha;     // per-row ladder factor
  double* row_e2;   // per-row sum of e^2
  double* row_bnd;  // per-row Theorem 5 bound
  double* row_d2;   // per-row ||w0 - q||^2
  int* overflow;    // per-row clip-free overflow flag
  int* rowlist;     // compact row -> original row
  int* counter;
  int* iperm;       // n: processing position of each original column (ordered calls)
  double* kappa;    // n: ZSIC column factors in processing order
  int* codes32;     // m x n int32 codes in processing order (unconstrained lattice only)
  // outlier search (SSQR) only
  double* alpha_d;  // per-row grid factor 2^t of the current pass
  uint8_t* omask;   // m x ldc8: 1 where the entry is an outlier (processing order)
  float* oval;      // m x ldE: the kept value of each outlier
  int* ocount;      // per-row outlier count of the last pass
  double* s_lo;     // per-row search bracket in log2 alpha: lo infeasible (or -8), hi feasible
  double* s_hi;
  double* s_mid;
  int* s_feas;
  size_t bytes;
};

static QLayout q_layout(void* ws, int64_t m, int64_t n, bool unbounded, bool outliers) {
  Carver c(ws);
  QLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.Wf = c.take<float>((size_t)m * n);
  L.ldE = (n + 31) / 32 * 32;  // rows start on 16-byte boundaries for TMA
  L.Ehi = c.take<float>((size_t)m * L.ldE);
  L.Elo = c.take<float>((size_t)m * L.ldE);
  L.ldu = (n + 31) / 32 * 32;
  L.Uhi = c.take<float>((size_t)n * L.ldu);
  L.Ulo = c.take<float>((size_t)n * L.ldu);
  L.Ublk = c.take<double>((size_t)((n + kBlock - 1) / kBlock) * kUBlkDoubles);
  L.ldc8 = (n + 15) / 16 * 16;
  L.codes8 = c.take<uint8_t>((size_t)m * L.ldc8);
  L.row_s = c.take<double>(m);
  L.row_z = c.take<double>(m);
  L.alpha = c.take<float>(m);
  L.row_e2 = c.take<double>(m);
  L.row_bnd = c.take<double>(m);
  L.row_d2 = c.take<double>(m);
  L.overflow = c.take<int>(m);
  L.rowlist = c.take<int>(m);
  L.counter = c.take<int>(4);
  L.iperm = c.take<int>((size_t)n);
  L.kappa = c.take<double>((size_t)n);
  L.codes32 = unbounded ? c.take<int>((size_t)m * n) : nullptr;
  L.alpha_d = nullptr; L.omask = nullptr; L.oval = nullptr; L.ocount = nullptr;
  L.s_lo = nullptr; L.s_hi = nullptr; L.s_mid = nullptr; L.s_feas = nullptr;
  if (outliers) {
    L.alpha_d = c.take<double>(m);
    L.omask = c.take<uint8_t>((size_t)m * L.ldc8);
    L.oval = c.take<float>((size_t)m * L.ldE);
    L.ocount = c.take<int>(m);
    L.s_lo = c.take<double>(m);
    L.s_hi = c.take<double>(m);
    L.s_mid = c.take<double>(m);
    L.s_feas = c.take<int>(m);
  }
  L.bytes = c.off;
  return L;
}

size_t quantize_ws_bytes(int64_t m, int64_t n, const gq_quant_cfg& cfg) {
  return q_layout(nullptr, m, n, cfg.clip == 2, false).bytes;
}

size_t ssqr_ws_bytes(int64_t m, int64_t n) { return q_layout(nullptr, m, n, false, true).bytes; }

// HPTQ: the quantize workspace (unconstrained lattice), then the Huffman statistics' workspace,
// the code table and the info words.
struct HptqLayout {
  QLayout q;
  void* huff_ws;
  uint8_t* lengths;
  unsigned long long* words;
  long long* info;
  uint8_t* zeros;  // m: the per-row zero points the grid kernel writes (all 0 here)
  size_t bytes;
};
static HptqLayout hptq_layout(void* ws, int64_t m, int64_t n) {
  HptqLayout H;
  H.q = q_layout(ws, m, n, true, false);
  Carver c(ws);
  c.off = H.q.bytes;
  c.off = (c.off + 255) / 256 * 256;
  H.huff_ws = ws ? static_cast<char*>(ws) + c.off : nullptr;
  c.off += huffman_ws_bytes(m * n);
  c.off = (c.off + 255) / 256 * 256;
  H.words = c.take<unsigned long long>(4096);
  H.info = c.take<long long>(4);
  H.lengths = c.take<uint8_t>(4096);
  H.zeros = c.take<uint8_t>((size_t)m);
  H.bytes = c.off;
  return H;
}
size_t hptq_ws_bytes(int64_t m, int64_t n) { return hptq_layout(nullptr, m, n).bytes; }

// ------------------------------------------------------------------------------------------
// setup kernels
// ------------------------------------------------------------------------------------------
__global__ void q_reset_kernel(int64_t m, float* alpha, int* overflow, double* loss) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < m) { alpha[i] = 1.f; overflow[i] = 0; }
  if (i < 3) loss[i] = 0.0;
}

// Wf[r'][p] = dead[pi(p)] ? 0 : W[row][pi(p)],  row = rowlist ? rowlist[r'] : r'
template <class TW>
__global__ void q_load_kernel(const TW* W, int64_t n, int64_t k_rows, const int* rowlist,
                              const uint8_t* dead, int reverse, float* Wf) {
  int64_t total = k_rows * n;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t rr = e / n, p = e % n;
    int64_t row = rowlist ? rowlist[rr] : rr;
    int64_t c = reverse ? n - 1 - p : p;
    float v;
    if constexpr (sizeof(TW) == 2) v = __bfloat162float(W[row * n + c]);
    else v = (float)W[row * n + c];
    if (dead && dead[c]) v = 0.f;
    Wf[e] = v;
  }
}

// Ordered calls: Wf[r'][p] = dead[perm[p]] ? 0 : W[row][perm[p]].  One CTA per row; the row
// is staged in shared memory (coalesced reads) and gathered from there.
template <class TW>
__global__ void __launch_bounds__(256) q_load_perm_kernel(const TW* W, int64_t n,
                                                          const int* rowlist,
                                                          const uint8_t* dead, const int* perm,
                                                          float* Wf) {
  extern __shared__ float srow[];
  const int64_t rr = blockIdx.x;
  const int64_t row = rowlist ? rowlist[rr] : rr;
  const TW* wrow = W + row * n;
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
    float v;
    if constexpr (sizeof(TW) == 2) v = __bfloat162float(wrow[c]);
    else v = (float)wrow[c];
    if (dead && dead[c]) v = 0.f;
    srow[c] = v;
  }
  __syncthreads();
  float* out = Wf + rr * n;
  for (int64_t p = threadIdx.x; p < n; p += blockDim.x) out[p] = srow[perm_at(perm, p, n)];
}

// iperm[perm[k]] = k (iperm preset to -1); a repeated or out-of-range entry records
// GQ_ERR_INVALID_ARG.
__global__ void perm_invert_kernel(const int* perm, int64_t n, int* iperm, WsHeader* hdr) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < n;
       k += (int64_t)gridDim.x * blockDim.x) {
    const unsigned p = (unsigned)perm[k];
    if (p >= (unsigned long long)n || atomicExch(&iperm[p], (int)k) != -1)
      record_status(hdr, GQ_ERR_INVALID_ARG);
  }
}

// per-row grid from the (dead-zeroed) row: one warp per row
// clip: 1 min-max grid; 0 clip-free (centred, step widened by the ladder factor alpha);
// 2 unconstrained lattice; 3 outliers (centred, step widened by the fp64 factor alpha_d).
__global__ void q_row_grid_kernel(const float* Wf, int64_t n, int64_t k_rows, const int* rowlist,
                                  int bits, int clip, const float* alpha, const double* alpha_d,
                                  double lattice_alpha, double* row_s, double* row_z,
                                  float* scales, uint8_t* zeros) {
  int64_t rr = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (rr >= k_rows) return;
  const float* w = Wf + rr * n;
  float lo = 0.f, hi = 0.f;  // the range always contains 0
  for (int64_t j = lane; j < n; j += 32) { float v = w[j]; lo = fminf(lo, v); hi = fmaxf(hi, v); }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    int64_t row = rowlist ? rowlist[rr] : rr;
    double dlo = lo, dhi = hi;
    if (dlo == 0.0 && dhi == 0.0) { dlo = -1.0; dhi = 1.0; }
    double maxq = (double)((1 << bits) - 1);
    double s, z;
    if (clip == 1) {
      s = (dhi - dlo) / maxq;
      z = rint(-dlo / s);
    } else if (clip == 2) {  // unconstrained lattice s Z: the min-max step x alpha, zero point 0
      s = ((dhi - dlo) / maxq) * lattice_alpha;
      z = 0.0;
    } else {
      const double al = clip == 3 ? alpha_d[row] : (double)alpha[row];
      s = al * (dhi - dlo) / maxq;
      z = rint(maxq * 0.5 - (dhi + dlo) / (2.0 * s));
    }
    row_s[row] = s;
    row_z[row] = z;
    scales[row] = (float)s;
    zeros[row] = (uint8_t)z;
  }
}

// Round to nearest integer, ties to even, for |x| < 2^51: adding and subtracting 1.5 * 2^52
// leaves no fraction bits, so the fp64 addition itself rounds x (in the default
// round-to-nearest-even mode).  Two fixed-latency adds instead of a conversion instruction on
// the column loop's critical path.  The grid values here are far below 2^51.
__device__ __forceinline__ double rint_small(double x) {
  const double magic = 6755399441055744.0;  // 1.5 * 2^52
  return __dsub_rn(__dadd_rn(x, magic), magic);
}

// tf32 rounding (to nearest, ties away) of an fp32 value, kept in an fp32 container
__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// U -> (Uhi, Ulo) with Uhi = tf32(U), Ulo = U - Uhi; columns n..ldu-1 zero
__global__ void split_u_kernel(const float* U, int64_t n, int64_t ldu, float* Uhi, float* Ulo) {
  const int64_t total = n * ldu;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / ldu, j = e % ldu;
    const float u = j < n ? U[i * n + j] : 0.f;
    const float h = tf32_rna(u);
    Uhi[e] = h;
    Ulo[e] = u - h;
  }
}

// Per-block prepared U, built once per call: the block's 128 x 128 part of U transposed,
// Ut[c][k] = U[j0 + k][j0 + c] for k <= c < width (0 elsewhere), in fp32 (U is fp32, so this
// is exact) with row pitch kUtPitch, then 1/U_jj and 1/U_jj^2 in fp64 (1 past the width).  The
// column loop copies it into shared memory in one go.
// ZSIC ("WaterSIC", section 2: grid spacing proportional to 1/|l_jj|): in the processing order
// the LDL pivot of column j is 1/U_jj^2, so |l_jj| = 1/U_jj and kappa_j = U_jj / geomean(U_kk)
// (normalised to geometric mean 1: the row's steps keep the geometric mean of its step).  One CTA.
__global__ void __launch_bounds__(1024) q_zsic_kernel(const float* U, int64_t n, double* kappa) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) acc += log((double)U[j * n + j]);
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    acc = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (threadIdx.x == 0) red[0] = exp(-acc / (double)n);  // 1 / geometric mean
  }
  __syncthreads();
  const double inv_gm = red[0];
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) kappa[j] = (double)U[j * n + j] * inv_gm;
}

__global__ void ublk_kernel(const float* U, int64_t n, double* Ublk, const double* kappa) {
  const int64_t b = blockIdx.y;
  const int64_t j0 = b * kBlock;
  const int bw = (int)((n - j0) < kBlock ? (n - j0) : kBlock);
  float* ut = reinterpret_cast<float*>(Ublk + b * kUBlkDoubles);
  double* dinv = reinterpret_cast<double*>(reinterpret_cast<char*>(ut) + kUtBytes);
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < kBlock * kUtPitch + kBlock;
       e += gridDim.x * blockDim.x) {
    if (e < kBlock * kUtPitch) {
      const int c = e / kUtPitch, k = e % kUtPitch;
      ut[e] = (c < bw && k <= c) ? U[(j0 + k) * n + j0 + c] : 0.f;
    } else {
      const int jj = e - kBlock * kUtPitch;
      const double d = jj < bw ? (double)U[(j0 + jj) * n + j0 + jj] : 1.0;
      const double k = (kappa && jj < bw) ? kappa[j0 + jj] : 1.0;
      dinv[jj] = 1.0 / d;
      dinv[kBlock + jj] = kappa ? (k * k) / (d * d) : 1.0 / (d * d);
      dinv[2 * kBlock + jj] = k;
      dinv[3 * kBlock + jj] = 1.0 / k;
    }
  }
}

// ------------------------------------------------------------------------------------------
// the column loop of one 128-column block
// ------------------------------------------------------------------------------------------
struct ColArgs {
  const double* Ublk;  // per-block prepared U (kUBlkDoubles each)
  WsHeader* hdr;
  const float* Wf;
  int64_t n;
  int64_t k_rows;
  const int* rowlist;
  int64_t j0;
  int bw;
  const float* U;
  int bits;
  int clip;
  float* Ehi;       // k x ldE, column j0 + c of the block at [row][j0 + c]
  float* Elo;
  int64_t ldE;
  uint8_t* codes8;
  int64_t ldc8;
  int* codes32;  // unconstrained lattice: int32 codes (processing order, row stride n), or null
  float* scales;
  uint8_t* zeros;
  int64_t ngroups;
  const double* row_s;
  const double* row_z;
  double* row_e2;
  double* row_bnd;
  int* overflow;
  uint8_t* omask;  // clip 3: outlier flags (row stride ldc8), kept values (row stride ldE), counts
  float* oval;
  int* ocount;
};

// Thread layout: a warp owns 8 rows; lane (g, t) = (lane / 4, lane % 4) holds row g and, of
// every 8-column tile, columns 2t and 2t + 1: w[tile][p] (p = column 2t + p).  That is the
// accumulator layout of the fp64 mma.sync m16n8k8 for its first 8 rows (the other 8 are zero
// padding: 8 rows a warp keep twice as many warps busy as 16, and the loop is latency-bound).
// Per tile of 8 columns the recursion is sequential only inside the tile (each column needs the
// errors of the earlier ones): the owner's value is shared in the quad, every lane of the quad
// computes the code and error of its row, and a lane updates its own later columns of the tile.
// The tile's 8 error columns then update every later tile of the block at once, one fp64
// tensor-core MMA per tile (the errors already sit in the A-operand layout when the k slots of
// lane t are taken as columns 2t and 2t + 1).  This is GPTQ's lazy batch applied again inside
// the block; the group grid, taken at a group's first column, sees the same error-fed values
// as the column-by-column recursion.  The register array is rotated by one tile after each
// tile so that the body, compiled once, refers to fixed registers (a fully unrolled tile loop
// measured 73 us per block against 33: the code no longer fits the instruction cache).
//
// The recursion runs in fp64: the in-block feedback sums cancel strongly when the grid is
// coarse, and an fp32 recursion flips ~1-3 % of the codes on ill-conditioned layers (measured
// against the fp64 oracle), while fp64 here with fp32 storage of W, E and U between blocks
// reproduces the oracle's codes.
// Z: ZSIC spacing (per-row grid only): column j's step is the row step times kappa_j.
// CM: the grid's clip mode (a compile-time copy of the call's clip: 0 clip-free with the
// ladder's overflow flags, 1 clamped, 2 unconstrained lattice with int32 codes, 3 outliers).
template <int G, bool Z, int CM>
__global__ void __launch_bounds__(kColThreads, 1) colloop_kernel(ColArgs a) {
  static_assert(!Z || G == 0, "per-column spacing takes a per-row grid");
  static_assert(G == 0 || CM == 1, "group grids are clamped");
  constexpr uint32_t kCopy = Z ? kUBlkBytesZ : kUBlkBytes;
  extern __shared__ __align__(16) double q_smem[];
  const float* Ut = reinterpret_cast<const float*>(q_smem);
  const double* invd = reinterpret_cast<const double*>(reinterpret_cast<const char*>(q_smem) + kUtBytes);
  const double* invd2 = invd + kBlock;  // kappa_j^2 / U_jj^2
  const double* kap = invd + 2 * kBlock;
  const double* kinv = invd + 3 * kBlock;
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(q_smem) + kCopy);
  const int tid = threadIdx.x;
  const int bw = a.bw;
  const int64_t n = a.n, j0 = a.j0;
  // the prepared block arrives by bulk async copies while the rows load below
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::fence_barrier_init();
    tc::mbar_arrive_expect_tx(bar, kCopy);
    const char* src = reinterpret_cast<const char*>(a.Ublk + (j0 / kBlock) * kUBlkDoubles);
    char* dst = reinterpret_cast<char*>(q_smem);
    for (uint32_t off = 0; off < kCopy; off += kBulkChunk) {
      const uint32_t len = kCopy - off < kBulkChunk ? kCopy - off : kBulkChunk;
      tc::bulk_copy_g2s(dst + off, src + off, len, bar);
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const unsigned full = 0xffffffffu;
  const int qbase = lane & ~3;
  const int64_t rr = (int64_t)blockIdx.x * kRowsPerCta + warp * 8 + g;
  const bool act = rr < a.k_rows;
  const int64_t row = act ? (a.rowlist ? a.rowlist[rr] : rr) : 0;
  const double maxq = (double)((1 << a.bits) - 1);

  double w[kTiles][2];
#pragma unroll
  for (int k = 0; k < kTiles; ++k) {
    const int col = 8 * k + 2 * t;
    float2 x = make_float2(0.f, 0.f);
    if (act) {
      const float* src = a.Wf + rr * n + j0 + col;
      if (col + 1 < bw && ((j0 + col + rr * n) & 1) == 0) {
        x = *reinterpret_cast<const float2*>(src);
      } else {
        if (col < bw) x.x = src[0];
        if (col + 1 < bw) x.y = src[1];
      }
    }
    w[k][0] = x.x;
    w[k][1] = x.y;
  }
  __syncthreads();  // the barrier's initialisation is visible to every waiting thread
  if (!tc::mbar_wait(bar, 0)) {
    if (tid == 0) record_status(a.hdr, GQ_ERR_TIMEOUT);
    return;  // nothing was computed; the bulk copy has been waited for the full bound
  }
  double s = 1.0, inv_s = 1.0, z = 0.0;
  if (G == 0 && act) { s = a.row_s[row]; z = a.row_z[row]; inv_s = 1.0 / s; }
  double e2 = 0.0, bnd = 0.0;
  int ovf = 0;
  constexpr bool clip = CM == 1;      // clamp to [0, 2^b - 1]
  constexpr bool track = CM == 0;     // clip-free: flag codes outside the range for the ladder
  // outliers ("The Geometry of LLM Quantization", section 3, SSQR): an entry whose code leaves
  // [0, 2^b - 1] keeps its current (error-fed) value in full precision: error 0, nothing fed
  // forward, code 0 in the packed stream
  constexpr bool outl = CM == 3;
  int nout = 0;

#pragma unroll 1
  for (int T = 0; T < kTiles; ++T) {
    if (8 * T >= bw) break;
    if constexpr (G > 0) {
      if ((8 * T) % G == 0) {
        // group grid from the current (error-fed) weights of columns [8T, 8T + G)
        double lo = 0.0, hi = 0.0;
#pragma unroll
        for (int k = 0; k < G / 8 && k < kTiles; ++k)
#pragma unroll
          for (int p = 0; p < 2; ++p)
            if (8 * (T + k) + 2 * t + p < bw) { lo = fmin(lo, w[k][p]); hi = fmax(hi, w[k][p]); }
        lo = fmin(lo, __shfl_xor_sync(full, lo, 1));
        hi = fmax(hi, __shfl_xor_sync(full, hi, 1));
        lo = fmin(lo, __shfl_xor_sync(full, lo, 2));
        hi = fmax(hi, __shfl_xor_sync(full, hi, 2));
        if (lo == 0.0 && hi == 0.0) { lo = -1.0; hi = 1.0; }
        s = (hi - lo) / maxq;
        z = rint(-lo / s);
        inv_s = 1.0 / s;
        if (act && t == 0) {
          const int64_t gi = (j0 + 8 * T) / G;
          a.scales[row * a.ngroups + gi] = (float)s;
          a.zeros[row * a.ngroups + gi] = (uint8_t)z;
        }
      }
    }
    // U entries of this tile's recursion: ut[p][i] = U[8T + i][8T + 2t + p]
    double ut[2][8];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const float* up = Ut + (8 * T + 2 * t + p) * kUtPitch + 8 * T;
      const float4 lo4 = *reinterpret_cast<const float4*>(up);
      const float4 hi4 = *reinterpret_cast<const float4*>(up + 4);
      ut[p][0] = lo4.x; ut[p][1] = lo4.y; ut[p][2] = lo4.z; ut[p][3] = lo4.w;
      ut[p][4] = hi4.x; ut[p][5] = hi4.y; ut[p][6] = hi4.z; ut[p][7] = hi4.w;
    }
    const double cmin = -z, cmax = maxq - z;  // code range in the domain c - z
    double ea[2] = {0.0, 0.0}, ca[2] = {0.0, 0.0};  // this lane's errors / codes (cols 2t, 2t+1)
    double xa[2] = {0.0, 0.0};                      // this lane's values before rounding
    bool oa[2] = {false, false};                    // ... and whether they are outliers
    double d2sum = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int jj = 8 * T + i;
      if (jj < bw) {
        const int town = i >> 1, pown = i & 1;
        const double id = invd[jj];
        d2sum += invd2[jj];
        const double x = __shfl_sync(full, w[0][pown], qbase | town);
        double sj = s, isj = inv_s;
        if constexpr (Z) { sj = s * kap[jj]; isj = inv_s * kinv[jj]; }
        double c = rint_small(x * isj);
        bool out = false;
        if (clip) c = fmin(fmax(c, cmin), cmax);
        else if (track || outl) out = c < cmin || c > cmax;
        if (track && out) ovf = 1;
        out = out && outl;
        nout += out ? 1 : 0;
        const double e = out ? 0.0 : fma(-sj, c, x) * id;  // (x - s_j c) / U_jj
        if (t == town) { ea[pown] = e; ca[pown] = c; xa[pown] = x; oa[pown] = out; }
        e2 = fma(e, e, e2);
#pragma unroll
        for (int p = 0; p < 2; ++p)
          if (2 * t + p > i) w[0][p] = fma(-e, ut[p][i], w[0][p]);
      }
    }
    bnd = fma(s * s, d2sum, bnd);
    // this tile's errors (E = E_hi + E_lo for the lazy update) and codes
    {
      const int col = 8 * T + 2 * t;
      if (act && col < bw) {
        const float f0 = (float)ea[0], f1 = (float)ea[1];
        float2 hi2, lo2;
        hi2.x = tf32_rna(f0); hi2.y = tf32_rna(f1);
        lo2.x = f0 - hi2.x; lo2.y = f1 - hi2.y;
        *reinterpret_cast<float2*>(a.Ehi + rr * a.ldE + j0 + col) = hi2;
        *reinterpret_cast<float2*>(a.Elo + rr * a.ldE + j0 + col) = lo2;
        if constexpr (CM == 2) {  // unconstrained lattice: z = 0, any integer
          int* cp = a.codes32 + row * n + j0 + col;
          cp[0] = (int)ca[0];
          if (col + 1 < bw) cp[1] = (int)ca[1];
        } else {
          uint8_t* cp = a.codes8 + row * a.ldc8 + j0 + col;
          cp[0] = oa[0] ? (uint8_t)0 : (uint8_t)(int)fmin(fmax(ca[0] + z, 0.0), maxq);
          if (col + 1 < bw) cp[1] = oa[1] ? (uint8_t)0 : (uint8_t)(int)fmin(fmax(ca[1] + z, 0.0), maxq);
          if (outl) {
            uint8_t* mp = a.omask + row * a.ldc8 + j0 + col;
            float* vp = a.oval + row * a.ldE + j0 + col;
            mp[0] = oa[0] ? 1 : 0;
            if (oa[0]) vp[0] = (float)xa[0];
            if (col + 1 < bw) {
              mp[1] = oa[1] ? 1 : 0;
              if (oa[1]) vp[1] = (float)xa[1];
            }
          }
        }
      }
    }
    // the later tiles of the block take this tile's errors: w[k] -= E_T U[T rows][tile k]
    const double an[4] = {-ea[0], 0.0, -ea[1], 0.0};
#pragma unroll
    for (int k = 1; k < kTiles; ++k) {
      if (T + k < kTiles && 8 * (T + k) < bw) {
        const float2 bv =
            *reinterpret_cast<const float2*>(Ut + (8 * (T + k) + g) * kUtPitch + 8 * T + 2 * t);
        const double b2[2] = {(double)bv.x, (double)bv.y};
        double c4[4] = {w[k][0], w[k][1], 0.0, 0.0};
        tc::dmma_m16n8k8(c4, an, b2);
        w[k][0] = c4[0]; w[k][1] = c4[1];
      }
    }
    // rotate: tile T + 1 moves to position 0
#pragma unroll
    for (int k = 0; k < kTiles - 1; ++k) { w[k][0] = w[k + 1][0]; w[k][1] = w[k + 1][1]; }
  }
  // per-row overflow flag (all lanes of the warp take part in the shuffles)
  int ovf_q = ovf;
  ovf_q |= __shfl_xor_sync(full, ovf_q, 1);
  ovf_q |= __shfl_xor_sync(full, ovf_q, 2);
  // per-row totals (all lanes of a quad hold the same e2 / bnd)
  if (act && t == 0) {
    if (j0 == 0) { a.row_e2[row] = e2; a.row_bnd[row] = bnd; a.overflow[row] = ovf_q; }
    else { a.row_e2[row] += e2; a.row_bnd[row] += bnd; a.overflow[row] |= ovf_q; }
    if (outl) {  // every lane of the quad counted the row's outliers
      if (j0 == 0) a.ocount[row] = nout;
      else a.ocount[row] += nout;
    }
  }
}

// ------------------------------------------------------------------------------------------
// packing + ||w0 - q||^2 per row (one CTA per original row)
// ------------------------------------------------------------------------------------------
template <class TW>
__global__ void __launch_bounds__(128) pack_kernel(const TW* W, const uint8_t* dead, int64_t n,
                                                   const uint8_t* codes8, int64_t ldc8,
                                                   const int* iperm, const double* kappa,
                                                   const int* codes32, int reverse, int bits,
                                                   int group,
                                                   int64_t ngroups, const float* scales,
                                                   const uint8_t* zeros, const uint8_t* omask,
                                                   const float* oval, int64_t ldE, uint32_t* codes,
                                                   double* row_d2) {
  const int64_t r = blockIdx.x;
  const uint8_t* crow = codes8 + r * ldc8;
  if (!codes32 && iperm) {  // ordered call: gather the codes from a shared-memory copy of the row
    extern __shared__ uint8_t scodes[];
    for (int64_t p = threadIdx.x; p < n; p += blockDim.x) scodes[p] = crow[p];
    __syncthreads();
    crow = scodes;
  }
  // processing position of original column c
  auto pos = [&](int64_t c) -> int64_t {
    return iperm ? perm_at(iperm, c, n) : (reverse ? n - 1 - c : c);
  };
  const int* crow32 = codes32 ? codes32 + r * n : nullptr;
  if (codes32) {  // unconstrained lattice: the output is int32 codes in original column order
    int* out = reinterpret_cast<int*>(codes) + r * n;
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) out[c] = crow32[pos(c)];
  }
  const int64_t nwords = codes32 ? 0 : (n * bits + 31) / 32;
  for (int64_t w = threadIdx.x; w < nwords; w += blockDim.x) {
    uint32_t word = 0u;
    int64_t cf = (32 * w) / bits, cl = (32 * w + 31) / bits;
    if (cl > n - 1) cl = n - 1;
    for (int64_t c = cf; c <= cl; ++c) {
      uint32_t code = crow[pos(c)];
      int64_t pos = (int64_t)bits * c - 32 * w;
      if (pos >= 0) word |= code << pos;
      else word |= code >> (-pos);
    }
    codes[r * nwords + w] = word;
  }
  double acc = 0.0;
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) {
    float w0;
    if constexpr (sizeof(TW) == 2) w0 = __bfloat162float(W[r * n + c]);
    else w0 = (float)W[r * n + c];
    if (dead && dead[c]) w0 = 0.f;
    const int64_t pc = pos(c);
    int64_t g = group ? pc / group : 0;  // groups follow the processing order
    float s = scales[r * ngroups + g], z = (float)zeros[r * ngroups + g];
    float code = codes32 ? (float)crow32[pc] : (float)crow[pc];
    const double sk = kappa ? (double)s * kappa[pc] : (double)s;
    double d = (double)w0 - sk * (double)(code - z);
    if (omask && omask[r * ldc8 + pc]) d = (double)w0 - (double)oval[r * ldE + pc];
    acc += d * d;
  }
  __shared__ double red[4];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) row_d2[r] = red[0] + red[1] + red[2] + red[3];
}

__global__ void __launch_bounds__(1024) q_reduce_kernel(int64_t m, const double* row_e2,
                                                        const double* row_bnd,
                                                        const double* row_d2,
                                                        const double* delta, double* loss) {
  __shared__ double red[3][32];
  double a0 = 0, a1 = 0, a2 = 0;
  for (int64_t i = threadIdx.x; i < m; i += blockDim.x) {
    a0 += row_e2[i]; a1 += row_bnd[i]; a2 += row_d2[i];
  }
  for (int o = 16; o > 0; o >>= 1) {
    a0 += __shfl_xor_sync(0xffffffffu, a0, o);
    a1 += __shfl_xor_sync(0xffffffffu, a1, o);
    a2 += __shfl_xor_sync(0xffffffffu, a2, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = a0; red[1][threadIdx.x >> 5] = a1; red[2][threadIdx.x >> 5] = a2;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    int nw = blockDim.x >> 5;
    a0 = threadIdx.x < nw ? red[0][threadIdx.x] : 0;
    a1 = threadIdx.x < nw ? red[1][threadIdx.x] : 0;
    a2 = threadIdx.x < nw ? red[2][threadIdx.x] : 0;
    for (int o = 16; o > 0; o >>= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, o);
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
      a2 += __shfl_xor_sync(0xffffffffu, a2, o);
    }
    if (threadIdx.x == 0) {
      loss[1] = a0;
      loss[2] = a1 * 0.25;
      loss[0] = delta ? 0.5 * (a0 - (*delta) * a2) : 0.0;
    }
  }
}

// clip-free ladder: rows that overflowed -> rowlist, alpha *= ladder
__global__ void q_ladder_kernel(int64_t m, int* overflow, float* alpha, float ladder, int* rowlist,
                                int* counter) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= m) return;
  if (overflow[i]) {
    int k = atomicAdd(counter, 1);
    rowlist[k] = (int)i;
    alpha[i] *= ladder;
  }
}

// ------------------------------------------------------------------------------------------
// orchestration
// ------------------------------------------------------------------------------------------
#define Q_TRY(x)                                    \
  do {                                              \
    cudaError_t _e = (x);                           \
    if (_e != cudaSuccess) return GQ_ERR_CUDA;      \
  } while (0)

constexpr size_t kColSmem = (size_t)kUBlkBytes + 16;  // + the mbarrier
constexpr size_t kColSmemZ = (size_t)kUBlkBytesZ + 16;

cudaError_t quant_init_attributes() {
  const int smem = (int)kColSmem;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, false, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<16, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<32, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<64, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<128, false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, true, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kColSmemZ))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kColSmemZ))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0, true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kColSmemZ))) return e;
  const int row_smem = 32768 * (int)sizeof(float);  // a staged row of the widest layer
  if ((e = cudaFuncSetAttribute(q_load_perm_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, row_smem))) return e;
  return cudaFuncSetAttribute(q_load_perm_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, row_smem);
}

template <int G, bool Z, int CM>
static cudaError_t launch_colloop(const ColArgs& ca, cudaStream_t s) {
  const size_t smem = Z ? kColSmemZ : kColSmem;
  unsigned grid = (unsigned)((ca.k_rows + kRowsPerCta - 1) / kRowsPerCta);
  colloop_kernel<G, Z, CM><<<grid, kColThreads, smem, s>>>(ca);
  count_launches(1);
  return cudaGetLastError();
}

static cudaError_t colloop_dispatch(int group, int spacing, const ColArgs& ca, cudaStream_t s) {
  if (spacing) {
    if (group != 0) return cudaErrorInvalidValue;
    switch (ca.clip) {
      case 0: return launch_colloop<0, true, 0>(ca, s);
      case 1: return launch_colloop<0, true, 1>(ca, s);
      case 2: return launch_colloop<0, true, 2>(ca, s);
      default: return cudaErrorInvalidValue;
    }
  }
  if (group == 0) {
    switch (ca.clip) {
      case 0: return launch_colloop<0, false, 0>(ca, s);
      case 1: return launch_colloop<0, false, 1>(ca, s);
      case 2: return launch_colloop<0, false, 2>(ca, s);
      case 3: return launch_colloop<0, false, 3>(ca, s);
      default: return cudaErrorInvalidValue;
    }
  }
  if (ca.clip != 1) return cudaErrorInvalidValue;
  switch (group) {
    case 16: return launch_colloop<16, false, 1>(ca, s);
    case 32: return launch_colloop<32, false, 1>(ca, s);
    case 64: return launch_colloop<64, false, 1>(ca, s);
    case 128: return launch_colloop<128, false, 1>(ca, s);
    default: return cudaErrorInvalidValue;
  }
}

// Three streams per call, forked from and joined back into the caller's stream (priority
// high to low): A runs the column loop of each block, the update of the next block's columns
// and, at the end of a super-block, the update of the next super-block; B runs the update of
// the rest of the current super-block after each block; C runs the update of all columns after
// the next super-block once a super-block is done.  One set per host thread and device, kept.
constexpr int kSuperBlocks = 8;  // blocks per super-block (1024 columns)
struct QuantStreams {
  bool ready = false;
  cudaStream_t a = nullptr, b = nullptr, c = nullptr;
  cudaEvent_t fork = nullptr, col[4] = {}, mid[4] = {}, sbdone = nullptr, far[2] = {},
              join[3] = {};
};
thread_local QuantStreams t_quant_streams[128];

static cudaError_t quant_streams(QuantStreams** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
  QuantStreams& q = t_quant_streams[dev];
  if (!q.ready) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest))) return e;
    if ((e = cudaStreamCreateWithPriority(&q.a, cudaStreamNonBlocking, greatest))) return e;
    if ((e = cudaStreamCreateWithPriority(&q.b, cudaStreamNonBlocking, (least + greatest) / 2)))
      return e;
    if ((e = cudaStreamCreateWithPriority(&q.c, cudaStreamNonBlocking, least))) return e;
    cudaEvent_t* evs[] = {&q.fork,   &q.col[0], &q.col[1], &q.col[2],  &q.col[3],  &q.mid[0],
                          &q.mid[1], &q.mid[2], &q.mid[3], &q.sbdone, &q.far[0], &q.far[1],
                          &q.join[0], &q.join[1], &q.join[2]};
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming))) return e;
    q.ready = true;
  }
  *out = &q;
  return cudaSuccess;
}

// Per-call set-up shared by every pass: status cleared, ladder factors 1, U split into tf32
// parts, the per-block prepared U (and the ZSIC factors), the inverse permutation.
static gq_status quant_setup(const QuantArgs& a, const QLayout& L, cudaStream_t s) {
  const int64_t m = a.m, n = a.n;
  const gq_quant_cfg& cfg = a.cfg;
  Q_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s));
  q_reset_kernel<<<(unsigned)((m + 255) / 256), 256, 0, s>>>(m, L.alpha, L.overflow, a.loss);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  {
    const int64_t total = n * L.ldu;
    unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, 148 * 32);
    split_u_kernel<<<grid, 256, 0, s>>>(a.U, n, L.ldu, L.Uhi, L.Ulo);
    count_launches(1);
    Q_TRY(cudaGetLastError());
    if (cfg.spacing) {
      q_zsic_kernel<<<1, 1024, 0, s>>>(a.U, n, L.kappa);
      count_launches(1);
      Q_TRY(cudaGetLastError());
    }
    dim3 g2(16, (unsigned)((n + kBlock - 1) / kBlock));
    ublk_kernel<<<g2, 256, 0, s>>>(a.U, n, L.Ublk, cfg.spacing ? L.kappa : nullptr);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  }
  if (a.perm) {
    Q_TRY(cudaMemsetAsync(L.iperm, 0xff, (size_t)n * sizeof(int), s));
    perm_invert_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, 1024), 256, 0, s>>>(
        a.perm, n, L.iperm, L.hdr);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  }
  return GQ_OK;
}

// One pass of the column loop over k_rows rows (all rows, or the rows listed in rowlist): the
// fp32 work matrix loaded, the per-row grids, then the blocks with their lazy updates.
static gq_status quant_pass(const QuantArgs& a, const QLayout& L, int64_t k_rows,
                            const int* rowlist, cudaStream_t s) {
  const int64_t n = a.n;
  const gq_quant_cfg& cfg = a.cfg;
  const int G = cfg.group_size;
  const int64_t ngroups = G ? (n + G - 1) / G : 1;
  const int nblocks = (int)((n + kBlock - 1) / kBlock);
  if (a.perm) {
    const size_t sm = (size_t)n * sizeof(float);
    if (a.wt == GQ_BF16)
      q_load_perm_kernel<__nv_bfloat16><<<(unsigned)k_rows, 256, sm, s>>>(
          static_cast<const __nv_bfloat16*>(a.W), n, rowlist, a.dead, a.perm, L.Wf);
    else
      q_load_perm_kernel<float><<<(unsigned)k_rows, 256, sm, s>>>(
          static_cast<const float*>(a.W), n, rowlist, a.dead, a.perm, L.Wf);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  } else {
    int64_t total = k_rows * n;
    unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, 148 * 64);
    if (a.wt == GQ_BF16)
      q_load_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(a.W), n, k_rows, rowlist, a.dead, cfg.reverse, L.Wf);
    else
      q_load_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(a.W), n, k_rows,
                                                rowlist, a.dead, cfg.reverse, L.Wf);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  }
  if (G == 0) {
    unsigned grid = (unsigned)((k_rows + 7) / 8);
    q_row_grid_kernel<<<grid, 256, 0, s>>>(L.Wf, n, k_rows, rowlist, cfg.bits, cfg.clip,
                                           L.alpha, L.alpha_d, a.lattice_alpha, L.row_s, L.row_z,
                                           a.scales, a.zeros);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  }
  LazyTcMaps maps;
  Q_TRY(lazy_tc_make_maps(&maps, L.Ehi, L.Elo, k_rows, L.ldE, L.Uhi, L.Ulo, n, L.ldu));
  // Two-level lazy updates (GPTQ's lazy batch, applied twice): the columns are grouped into
  // super-blocks of kSuperBlocks blocks.  After block b (columns [j0, j1)) of super-block S:
  //   A: W[:, next block] -= E_b U[b, next block]         (if the next block is in S)
  //   B: W[:, rest of S]  -= E_b U[b, rest of S]
  // and once S is done:
  //   A: W[:, next super-block]      -= E_S U[S, next super-block]   (depth 1024)
  //   C: W[:, everything after that] -= E_S U[S, ...]               (depth 1024)
  // so the fp32 work matrix beyond the current super-block is read and written once per
  // super-block instead of once per block.  E of every column is kept (no buffer reuse).
  // Waits (two streams never read-modify-write the same columns at once): A's update after
  // block b (which writes block b + 1) waits for B's update after block b - 1 (which writes
  // blocks b + 1 .. the end of S), so the column loop of a block always sees every earlier
  // block's contribution; A's next-super-block update waits for C's update after the previous
  // super-block (both write those columns).
  QuantStreams* qs = nullptr;
  Q_TRY(quant_streams(&qs));
  cudaStream_t sa = qs->a, sb = qs->b, sc = qs->c;
  Q_TRY(cudaEventRecord(qs->fork, s));
  Q_TRY(cudaStreamWaitEvent(sa, qs->fork, 0));
  Q_TRY(cudaStreamWaitEvent(sb, qs->fork, 0));
  Q_TRY(cudaStreamWaitEvent(sc, qs->fork, 0));
  bool far_pending = false;
  int far_idx = 0;
  for (int b = 0; b < nblocks; ++b) {
    const int64_t j0 = (int64_t)b * kBlock;
    const int bw = (int)std::min<int64_t>(kBlock, n - j0);
    const int64_t j1 = j0 + bw;
    const int bi = b % kSuperBlocks;
    const int64_t sb0 = (int64_t)(b - bi) * kBlock;
    const int64_t sb1 = std::min<int64_t>(sb0 + (int64_t)kSuperBlocks * kBlock, n);
    ColArgs ca{};
    ca.Ublk = L.Ublk; ca.hdr = L.hdr;
    ca.Wf = L.Wf; ca.n = n; ca.k_rows = k_rows; ca.rowlist = rowlist; ca.j0 = j0; ca.bw = bw;
    ca.U = a.U; ca.bits = cfg.bits; ca.clip = cfg.clip; ca.Ehi = L.Ehi; ca.Elo = L.Elo;
    ca.ldE = L.ldE;
    ca.codes8 = L.codes8;
    ca.codes32 = L.codes32;
    ca.ldc8 = L.ldc8; ca.scales = a.scales; ca.zeros = a.zeros; ca.ngroups = ngroups;
    ca.row_s = L.row_s; ca.row_z = L.row_z; ca.row_e2 = L.row_e2; ca.row_bnd = L.row_bnd;
    ca.overflow = L.overflow;
    ca.omask = L.omask; ca.oval = L.oval; ca.ocount = L.ocount;
    Q_TRY(colloop_dispatch(G, cfg.spacing, ca, sa));
    if (j1 < sb1) {  // the rest of this super-block takes block b's errors (depth 128)
      const int64_t jn = std::min<int64_t>(j1 + kBlock, sb1);
      if (jn < sb1) {
        Q_TRY(cudaEventRecord(qs->col[b & 3], sa));
        Q_TRY(cudaStreamWaitEvent(sb, qs->col[b & 3], 0));
        Q_TRY(launch_lazy_tc(maps, L.Wf, n, k_rows, j0, bw, jn, sb1, L.hdr, sb));
        Q_TRY(cudaEventRecord(qs->mid[b & 3], sb));
      }
      // B's update after block b - 1 also writes the next block: finish it first
      if (bi >= 1) Q_TRY(cudaStreamWaitEvent(sa, qs->mid[(b - 1) & 3], 0));
      Q_TRY(launch_lazy_tc(maps, L.Wf, n, k_rows, j0, bw, j1, jn, L.hdr, sa));
    } else if (sb1 < n) {  // super-block [sb0, sb1) done: everything after it (depth 1024)
      const int64_t sb2 = std::min<int64_t>(sb1 + (int64_t)kSuperBlocks * kBlock, n);
      const int depth = (int)(sb1 - sb0);
      if (sb2 < n) {
        Q_TRY(cudaEventRecord(qs->sbdone, sa));
        Q_TRY(cudaStreamWaitEvent(sc, qs->sbdone, 0));
      }
      if (far_pending) Q_TRY(cudaStreamWaitEvent(sa, qs->far[(far_idx - 1) & 1], 0));
      Q_TRY(launch_lazy_tc(maps, L.Wf, n, k_rows, sb0, depth, sb1, sb2, L.hdr, sa));
      far_pending = false;
      if (sb2 < n) {
        Q_TRY(launch_lazy_tc(maps, L.Wf, n, k_rows, sb0, depth, sb2, n, L.hdr, sc));
        Q_TRY(cudaEventRecord(qs->far[far_idx & 1], sc));
        far_pending = true;
        ++far_idx;
      }
    }
  }
  Q_TRY(cudaEventRecord(qs->join[1], sb));
  Q_TRY(cudaEventRecord(qs->join[2], sc));
  Q_TRY(cudaStreamWaitEvent(sa, qs->join[1], 0));
  Q_TRY(cudaStreamWaitEvent(sa, qs->join[2], 0));
  Q_TRY(cudaEventRecord(qs->join[0], sa));
  Q_TRY(cudaStreamWaitEvent(s, qs->join[0], 0));
  return GQ_OK;
}

// Packing (codes by original column; an outlier's kept value in the error norm), per-row
// ||w0 - q||^2, and the three loss numbers.
static gq_status quant_finish(const QuantArgs& a, const QLayout& L, cudaStream_t s) {
  const int64_t m = a.m, n = a.n;
  const gq_quant_cfg& cfg = a.cfg;
  const int G = cfg.group_size;
  const int64_t ngroups = G ? (n + G - 1) / G : 1;
  const int* iperm = a.perm ? L.iperm : nullptr;
  const double* kappa = cfg.spacing ? L.kappa : nullptr;
  const size_t pack_smem = (a.perm && !L.codes32) ? (size_t)n : 0;
  if (a.wt == GQ_BF16)
    pack_kernel<__nv_bfloat16><<<(unsigned)m, 128, pack_smem, s>>>(
        static_cast<const __nv_bfloat16*>(a.W), a.dead, n, L.codes8, L.ldc8, iperm, kappa,
        L.codes32, cfg.reverse, cfg.bits, G, ngroups, a.scales, a.zeros, L.omask, L.oval,
        L.ldE, a.codes, L.row_d2);
  else
    pack_kernel<float><<<(unsigned)m, 128, pack_smem, s>>>(
        static_cast<const float*>(a.W), a.dead, n, L.codes8, L.ldc8, iperm, kappa, L.codes32,
        cfg.reverse, cfg.bits, G, ngroups, a.scales, a.zeros, L.omask, L.oval, L.ldE, a.codes,
        L.row_d2);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  q_reduce_kernel<<<1, 1024, 0, s>>>(m, L.row_e2, L.row_bnd, L.row_d2, a.delta, a.loss);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  return GQ_OK;
}

// Writes GQ_ERR_NO_FIT into the status word unless an earlier error is there (synchronizes).
static gq_status record_no_fit(const QLayout& L, cudaStream_t s) {
  int code = GQ_ERR_NO_FIT, cur = 0;
  Q_TRY(cudaMemcpyAsync(&cur, &L.hdr->status, sizeof(int), cudaMemcpyDeviceToHost, s));
  Q_TRY(cudaStreamSynchronize(s));
  if (cur == 0)
    Q_TRY(cudaMemcpyAsync(&L.hdr->status, &code, sizeof(int), cudaMemcpyHostToDevice, s));
  Q_TRY(cudaStreamSynchronize(s));
  return GQ_OK;
}

gq_status run_quantize(const QuantArgs& a, cudaStream_t s) {
  const int64_t m = a.m;
  const gq_quant_cfg& cfg = a.cfg;
  QLayout L = q_layout(a.ws, m, a.n, cfg.clip == 2, false);
  gq_status st = quant_setup(a, L, s);
  if (st != GQ_OK) return st;
  int64_t k_rows = m;
  const int* rowlist = nullptr;
  const int max_rounds = cfg.clip ? 1 : cfg.ladder_max + 1;
  int rounds_run = 0;
  for (int round = 0; round < max_rounds; ++round) {
    rounds_run = round;
    if ((st = quant_pass(a, L, k_rows, rowlist, s)) != GQ_OK) return st;
    if (cfg.clip) break;
    // clip-free: collect rows whose codes left [0, 2^b - 1] and rerun them on a wider step
    Q_TRY(cudaMemsetAsync(L.counter, 0, sizeof(int), s));
    q_ladder_kernel<<<(unsigned)((m + 255) / 256), 256, 0, s>>>(m, L.overflow, L.alpha,
                                                                 cfg.ladder, L.rowlist, L.counter);
    count_launches(1);
    Q_TRY(cudaGetLastError());
    int cnt = 0;
    Q_TRY(cudaMemcpyAsync(&cnt, L.counter, sizeof(int), cudaMemcpyDeviceToHost, s));
    Q_TRY(cudaStreamSynchronize(s));
    if (cnt == 0) break;
    if (round == max_rounds - 1) {
      if ((st = record_no_fit(L, s)) != GQ_OK) return st;
      break;
    }
    k_rows = cnt;
    rowlist = L.rowlist;
  }
  if (!cfg.clip) {
    int rr = rounds_run;
    Q_TRY(cudaMemcpyAsync(&L.hdr->ladder_rounds, &rr, sizeof(int), cudaMemcpyHostToDevice, s));
    Q_TRY(cudaStreamSynchronize(s));
  }
  return quant_finish(a, L, s);
}

// ---------------------------------------------------------------------------------------------
// SSQR ("The Geometry of LLM Quantization", section 3: a few weights are kept in full precision
// as sparse floats, the rest quantized on a low-bit grid, the scale set by a binary search for
// a target outlier density).  Reading: the clip-free centred grid of each row widened by alpha;
// alpha is the smallest factor (finest grid) with at most limit = floor(density n) outliers,
// found in log2 alpha by doubling from 1 until feasible and then a fixed number of bisection
// steps between the last infeasible value (or -8 when 1 is feasible) and the feasible one.
// ---------------------------------------------------------------------------------------------
// 2^x; exact for integer x, the correctly rounded-or-close exp2 otherwise
__device__ __forceinline__ double pow2_real(double x) {
  if (x == floor(x) && fabs(x) < 1000.0) return ldexp(1.0, (int)x);
  return exp2(x);
}

enum SsqrMode {
  kSsqrInit = 0,      // hi = 0 (alpha 1), every row still to be checked
  kSsqrCheck = 1,     // after a pass of the listed / unchecked rows: feasibility, new list
  kSsqrDouble = 2,    // before a doubling pass: infeasible rows lo = hi, hi += 1
  kSsqrMid = 3,       // before a bisection pass: mid = (lo + hi) / 2, alpha = 2^mid
  kSsqrBisect = 4,    // after a bisection pass: feasible -> hi = mid, else lo = mid
  kSsqrFinal = 5      // alpha = 2^hi for the final pass, copied out
};

__global__ void ssqr_state_kernel(int64_t m, int mode, int limit, const int* ocount, double* lo,
                                  double* hi, double* mid, int* feas, double* alpha_d,
                                  int* rowlist, int* counter, double* alpha_out) {
  const int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (r >= m) return;
  switch (mode) {
    case kSsqrInit:
      hi[r] = 0.0;
      lo[r] = -8.0;
      feas[r] = 0;
      alpha_d[r] = 1.0;
      break;
    case kSsqrCheck:
      if (!feas[r]) {
        if (ocount[r] <= limit) {
          feas[r] = 1;
        } else {
          rowlist[atomicAdd(counter, 1)] = (int)r;
        }
      }
      break;
    case kSsqrDouble:
      if (!feas[r]) {
        lo[r] = hi[r];
        hi[r] += 1.0;
        alpha_d[r] = pow2_real(hi[r]);
      }
      break;
    case kSsqrMid:
      mid[r] = 0.5 * (lo[r] + hi[r]);
      alpha_d[r] = pow2_real(mid[r]);
      break;
    case kSsqrBisect:
      if (ocount[r] <= limit) hi[r] = mid[r];
      else lo[r] = mid[r];
      break;
    case kSsqrFinal:
      alpha_d[r] = pow2_real(hi[r]);
      alpha_out[r] = alpha_d[r];
      break;
  }
}

// row_ptr = exclusive scan of the per-row outlier counts (one CTA); a total beyond the caller's
// capacity records GQ_ERR_WORKSPACE (the fill below then writes nothing past the capacity).
__global__ void __launch_bounds__(1024) csr_rowptr_kernel(int64_t m, const int* ocount,
                                                          int64_t capacity, long long* row_ptr,
                                                          WsHeader* hdr) {
  __shared__ long long warp_tot[32];
  __shared__ long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = 0; base < m; base += 1024) {
    const int64_t r = base + threadIdx.x;
    long long v = r < m ? (long long)ocount[r] : 0;
    long long x = v;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      long long t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const long long before = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
    if (r < m) row_ptr[r] = before;
    __syncthreads();
    if (threadIdx.x == 1023) carry = before + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    row_ptr[m] = carry;
    if (carry > capacity) record_status(hdr, GQ_ERR_WORKSPACE);
  }
}

// Column indices (ascending) and kept values of each row's outliers; one CTA of 128 threads per
// row, columns in chunks of 128 with a block-wide prefix of the flags.
__global__ void __launch_bounds__(128) csr_fill_kernel(int64_t n, const uint8_t* omask,
                                                       int64_t ldc8, const float* oval,
                                                       int64_t ldE, const long long* row_ptr,
                                                       int64_t capacity, int* col_idx,
                                                       float* values) {
  __shared__ int warp_cnt[4];
  const int64_t r = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long pos = row_ptr[r];
  for (int64_t c0 = 0; c0 < n; c0 += 128) {
    const int64_t c = c0 + threadIdx.x;
    const bool f = c < n && omask[r * ldc8 + c];
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int off = 0;
    for (int w = 0; w < warp; ++w) off += warp_cnt[w];
    const int total = warp_cnt[0] + warp_cnt[1] + warp_cnt[2] + warp_cnt[3];
    if (f) {
      const long long idx = pos + off + __popc(bal & ((1u << lane) - 1u));
      if (idx < capacity) {
        col_idx[idx] = (int)c;
        values[idx] = oval[r * ldE + c];
      }
    }
    pos += total;
    __syncthreads();
  }
}

gq_status run_ssqr(const QuantArgs& a, const SsqrArgs& o, cudaStream_t s) {
  const int64_t m = a.m, n = a.n;
  QLayout L = q_layout(a.ws, m, n, false, true);
  gq_status st = quant_setup(a, L, s);
  if (st != GQ_OK) return st;
  const int limit = (int)floor(o.density * (double)n + 1e-9);
  const unsigned rgrid = (unsigned)((m + 255) / 256);
  auto state = [&](int mode) -> gq_status {
    ssqr_state_kernel<<<rgrid, 256, 0, s>>>(m, mode, limit, L.ocount, L.s_lo, L.s_hi, L.s_mid,
                                            L.s_feas, L.alpha_d, L.rowlist, L.counter, o.alpha);
    count_launches(1);
    Q_TRY(cudaGetLastError());
    return GQ_OK;
  };
  auto check = [&](int* cnt) -> gq_status {
    Q_TRY(cudaMemsetAsync(L.counter, 0, sizeof(int), s));
    gq_status e = state(kSsqrCheck);
    if (e != GQ_OK) return e;
    Q_TRY(cudaMemcpyAsync(cnt, L.counter, sizeof(int), cudaMemcpyDeviceToHost, s));
    Q_TRY(cudaStreamSynchronize(s));
    return GQ_OK;
  };
  // doubling from alpha = 1 until every row is feasible
  if ((st = state(kSsqrInit)) != GQ_OK) return st;
  if ((st = quant_pass(a, L, m, nullptr, s)) != GQ_OK) return st;
  int cnt = 0;
  if ((st = check(&cnt)) != GQ_OK) return st;
  for (int d = 0; d < o.max_doublings && cnt > 0; ++d) {
    if ((st = state(kSsqrDouble)) != GQ_OK) return st;
    if ((st = quant_pass(a, L, cnt, L.rowlist, s)) != GQ_OK) return st;
    if ((st = check(&cnt)) != GQ_OK) return st;
  }
  if (cnt > 0 && (st = record_no_fit(L, s)) != GQ_OK) return st;
  // bisection in log2 alpha, every row at once
  for (int k = 0; k < o.steps; ++k) {
    if ((st = state(kSsqrMid)) != GQ_OK) return st;
    if ((st = quant_pass(a, L, m, nullptr, s)) != GQ_OK) return st;
    if ((st = state(kSsqrBisect)) != GQ_OK) return st;
  }
  // the result: every row at its feasible alpha, packed, losses, outliers as CSR
  if ((st = state(kSsqrFinal)) != GQ_OK) return st;
  if ((st = quant_pass(a, L, m, nullptr, s)) != GQ_OK) return st;
  if ((st = quant_finish(a, L, s)) != GQ_OK) return st;
  csr_rowptr_kernel<<<1, 1024, 0, s>>>(m, L.ocount, o.capacity, o.row_ptr, L.hdr);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  csr_fill_kernel<<<(unsigned)m, 128, 0, s>>>(n, L.omask, L.ldc8, L.oval, L.ldE, o.row_ptr,
                                             o.capacity, o.col_idx, o.values);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  return GQ_OK;
}

// ---------------------------------------------------------------------------------------------
// HPTQ rate control ("The Geometry of LLM Quantization", section 3, HPTQ: normal and outlier
// weights share one unconstrained integer lattice, and Huffman coding of the integers gives a
// variable bit width that meets a compression budget).  Reading: one factor alpha for the whole
// layer multiplies every row's min-max step; the budget counts the Huffman-coded integers
// alone, in bits per weight; alpha is the smallest factor (finest lattice) whose coded size is
// at most budget x m x n bits, found in log2 alpha as the outlier search does: doubling from 1
// until the layer fits, then a fixed number of bisection steps between the last value that
// did not fit (or -8 when 1 fits) and the one that does.  The host drives the search (alpha
// = 2^t computed on the host, the coded size read back after each pass).
// ---------------------------------------------------------------------------------------------
gq_status run_hptq(const QuantArgs& a0, const HptqArgs& o, cudaStream_t s) {
  const int64_t m = a0.m, n = a0.n, count = m * n;
  HptqLayout H = hptq_layout(a0.ws, m, n);
  const QLayout& L = H.q;
  gq_status st = quant_setup(a0, L, s);
  if (st != GQ_OK) return st;
  QuantArgs a = a0;
  a.zeros = H.zeros;
  const double limit = o.budget * (double)count;
  long long info[4] = {0, 0, 0, 0};
  // one pass at alpha = 2^t: the codes, their coded size; false when it exceeds the budget
  auto fits = [&](double t, bool* ok) -> gq_status {
    a.lattice_alpha = pow(2.0, t);
    gq_status e = quant_pass(a, L, m, nullptr, s);
    if (e != GQ_OK) return e;
    Q_TRY(launch_huffman_stats(L.codes32, count, H.lengths, H.words, H.info, H.huff_ws, s));
    Q_TRY(cudaMemcpyAsync(info, H.info, sizeof(info), cudaMemcpyDeviceToHost, s));
    int hstat = 0, qstat = 0;
    Q_TRY(cudaMemcpyAsync(&hstat, H.huff_ws, sizeof(int), cudaMemcpyDeviceToHost, s));
    Q_TRY(cudaMemcpyAsync(&qstat, &L.hdr->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    Q_TRY(cudaStreamSynchronize(s));
    if (qstat != 0) return GQ_OK;  // reported through the workspace status; the search stops
    if (hstat != 0) {              // more distinct integers than the code table holds
      const int code = hstat;
      Q_TRY(cudaMemcpyAsync(&L.hdr->status, &code, sizeof(int), cudaMemcpyHostToDevice, s));
      Q_TRY(cudaStreamSynchronize(s));
      return GQ_OK;
    }
    *ok = (double)info[2] <= limit;
    return GQ_OK;
  };
  auto failed = [&](bool* bad) -> gq_status {
    int cur = 0;
    Q_TRY(cudaMemcpyAsync(&cur, &L.hdr->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    Q_TRY(cudaStreamSynchronize(s));
    *bad = cur != 0;
    return GQ_OK;
  };
  bool ok = false, bad = false;
  double hi = 0.0, lo = -8.0;
  if ((st = fits(hi, &ok)) != GQ_OK) return st;
  if ((st = failed(&bad)) != GQ_OK || bad) return st;
  for (int d = 0; d < o.max_doublings && !ok; ++d) {
    lo = hi;
    hi += 1.0;
    if ((st = fits(hi, &ok)) != GQ_OK) return st;
    if ((st = failed(&bad)) != GQ_OK || bad) return st;
  }
  if (!ok) return record_no_fit(L, s);
  for (int k = 0; k < o.steps; ++k) {
    const double mid = 0.5 * (lo + hi);
    bool mok = false;
    if ((st = fits(mid, &mok)) != GQ_OK) return st;
    if ((st = failed(&bad)) != GQ_OK || bad) return st;
    if (mok) hi = mid; else lo = mid;
  }
  // the result at the feasible alpha: codes, scales, losses, and its coded size
  if ((st = fits(hi, &ok)) != GQ_OK) return st;
  if ((st = failed(&bad)) != GQ_OK || bad) return st;
  if ((st = quant_finish(a, L, s)) != GQ_OK) return st;
  const double alpha = a.lattice_alpha;
  const long long total = info[2];
  Q_TRY(cudaMemcpyAsync(o.alpha, &alpha, sizeof(double), cudaMemcpyHostToDevice, s));
  Q_TRY(cudaMemcpyAsync(o.total_bits, &total, sizeof(long long), cudaMemcpyHostToDevice, s));
  Q_TRY(cudaStreamSynchronize(s));  // the host values above must outlive the copies
  return GQ_OK;
}

}  // namespace gq

namespace gq {
cudaError_t launch_zsic_spacing(const float* U, int64_t n, double* kappa, cudaStream_t s) {
  q_zsic_kernel<<<1, 1024, 0, s>>>(U, n, kappa);
  count_launches(1);
  return cudaGetLastError();
}
}  // namespace gq
