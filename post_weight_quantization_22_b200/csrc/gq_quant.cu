// The GPTQ / Babai column loop with lazy block updates, code packing and losses.
//
// Sources: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 2.2 (GPTQ's error propagation is the nearest-plane step; back to front it is Babai),
// section 2.3 (no-clipping setting; Theorem 5 bound (1/4) sum s^2 D_jj); "RDQ: Residual
// Distribution Quantization", setup (group-128 asymmetric integer format).
//
// Work layout: the weights are copied once into an fp32 work matrix Wf (rows x n) in the
// processing order (columns reversed for the last-to-first variant, dead columns zeroed).  Per
// 128-column block: `colloop` runs the sequential column recursion for 32 rows per CTA (4
// lanes per row, each lane owning 32 of the block's columns in 4-wide chunks), keeping the
// block's part of U in shared memory; the tensor-core lazy update (gq_lazy_tc.cu) then applies
// W[:, j+128:] -= E U[j:j+128, j+128:] to the rest of the work matrix.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <algorithm>
#include <math.h>

namespace gq {

constexpr int kP = 4;                      // lanes per row in the column loop
constexpr int kVPL = kBlock / kP;          // values per lane (32)
constexpr int kSW = 4 * kP;                // segment width: one 4-column chunk per lane
constexpr int kColThreads = 128;
constexpr int kRowsPerCta = kColThreads / kP;  // 32 rows per CTA
// Per-block prepared U for the column loop (see ublk_kernel): 128 x 128 doubles + 2 x 128.
constexpr int64_t kUBlkDoubles = (int64_t)kBlock * kBlock + 2 * kBlock;
constexpr uint32_t kUBlkBytes = (uint32_t)(kUBlkDoubles * sizeof(double));
constexpr uint32_t kBulkChunk = 32768;

struct QLayout {
  WsHeader* hdr;
  float* Wf;        // k x n work matrix (compact rows)
  float* Ehi[2];    // k x 128 scaled errors of a block, tf32 part (blocks alternate buffers)
  float* Elo[2];    // k x 128 fp32 remainder (E = Ehi + Elo)
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
  size_t bytes;
};

static QLayout q_layout(void* ws, int64_t m, int64_t n) {
  Carver c(ws);
  QLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.Wf = c.take<float>((size_t)m * n);
  for (int i = 0; i < 2; ++i) {
    L.Ehi[i] = c.take<float>((size_t)m * kBlock);
    L.Elo[i] = c.take<float>((size_t)m * kBlock);
  }
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
  L.bytes = c.off;
  return L;
}

size_t quantize_ws_bytes(int64_t m, int64_t n, const gq_quant_cfg&) {
  return q_layout(nullptr, m, n).bytes;
}

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

// per-row grid from the (dead-zeroed) row: one warp per row
__global__ void q_row_grid_kernel(const float* Wf, int64_t n, int64_t k_rows, const int* rowlist,
                                  int bits, int clip, const float* alpha, double* row_s,
                                  double* row_z, float* scales, uint8_t* zeros) {
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
    if (clip) {
      s = (dhi - dlo) / maxq;
      z = rint(-dlo / s);
    } else {
      s = (double)alpha[row] * (dhi - dlo) / maxq;
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

// Per-block prepared U, built once per call: the block's 128 x 128 part of U in fp64 with the
// strict lower triangle and the columns past the block's width zeroed, then 1/U_jj and
// 1/U_jj^2 (1 past the width).  The column loop copies it into shared memory in one go.

__global__ void ublk_kernel(const float* U, int64_t n, double* Ublk) {
  const int64_t b = blockIdx.y;
  const int64_t j0 = b * kBlock;
  const int bw = (int)((n - j0) < kBlock ? (n - j0) : kBlock);
  double* dst = Ublk + b * kUBlkDoubles;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < kBlock * kBlock + kBlock;
       e += gridDim.x * blockDim.x) {
    if (e < kBlock * kBlock) {
      const int jj = e / kBlock, kk = e % kBlock;
      dst[e] = (jj < bw && kk >= jj && kk < bw) ? (double)U[(j0 + jj) * n + j0 + kk] : 0.0;
    } else {
      const int jj = e - kBlock * kBlock;
      const double d = jj < bw ? (double)U[(j0 + jj) * n + j0 + jj] : 1.0;
      dst[kBlock * kBlock + jj] = 1.0 / d;
      dst[kBlock * kBlock + kBlock + jj] = 1.0 / (d * d);
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
  float* Ehi;
  float* Elo;
  uint8_t* codes8;
  int64_t ldc8;
  float* scales;
  uint8_t* zeros;
  int64_t ngroups;
  const double* row_s;
  const double* row_z;
  double* row_e2;
  double* row_bnd;
  int* overflow;
};

// Lane ownership: each row is handled by kP = 4 lanes; the block's 128 columns form 8 segments
// of 16, and in each segment lane t owns the 4-column chunk [16 seg + 4t, 16 seg + 4t + 4).
// Each lane keeps its 8 chunks in registers, v[4c + u] = chunk (seg + c); after a segment the
// array is rotated by one chunk, so the unrolled 16-step body refers to fixed registers and the
// segment loop stays a small runtime loop (a fully unrolled 128-step body does not fit the
// instruction cache).  128-thread CTAs of 32 rows.
//
// The recursion runs in fp64: the in-block feedback sums cancel strongly when the grid is
// coarse, and an fp32 recursion flips ~1-3 % of the codes on ill-conditioned layers (measured
// against the fp64 oracle), while fp64 here with fp32 storage of W, E and U between blocks
// reproduces the oracle's codes.
template <int G>
__global__ void __launch_bounds__(kColThreads, 1) colloop_kernel(ColArgs a) {
  extern __shared__ __align__(16) double q_smem[];
  double* Us = q_smem;                       // [128][128] this block's part of U (fp64, masked)
  double* invd = q_smem + kBlock * kBlock;   // [128]  1/U_jj
  double* invd2 = invd + kBlock;             // [128]  1/U_jj^2
  uint64_t* bar = reinterpret_cast<uint64_t*>(invd2 + kBlock);
  const int tid = threadIdx.x;
  const int bw = a.bw;
  const int64_t n = a.n, j0 = a.j0;
  // the prepared block (kUBlkBytes) arrives by bulk async copies while the rows load below
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::fence_barrier_init();
    tc::mbar_arrive_expect_tx(bar, (uint32_t)kUBlkBytes);
    const char* src = reinterpret_cast<const char*>(a.Ublk + (j0 / kBlock) * kUBlkDoubles);
    char* dst = reinterpret_cast<char*>(q_smem);
    for (uint32_t off = 0; off < kUBlkBytes; off += kBulkChunk) {
      const uint32_t len = kUBlkBytes - off < kBulkChunk ? kUBlkBytes - off : kBulkChunk;
      tc::bulk_copy_g2s(dst + off, src + off, len, bar);
    }
  }
  const int lane = tid & 31, warp = tid >> 5;
  const int t = lane % kP;
  const int64_t rr = (int64_t)blockIdx.x * kRowsPerCta + warp * (32 / kP) + lane / kP;
  const bool active = rr < a.k_rows;
  const int64_t row = active ? (a.rowlist ? a.rowlist[rr] : rr) : 0;
  const double maxq = (double)((1 << a.bits) - 1);

  double v[kVPL];
#pragma unroll
  for (int c = 0; c < kVPL / 4; ++c) {
    int k = kSW * c + 4 * t;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) {
      const float* src = a.Wf + rr * n + j0 + k;
      if (k + 3 < bw && ((j0 + k + rr * n) & 3) == 0) {
        x = *reinterpret_cast<const float4*>(src);
      } else {
        float* dx = &x.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) dx[u] = (k + u < bw) ? src[u] : 0.f;
      }
    }
    v[4 * c + 0] = x.x; v[4 * c + 1] = x.y; v[4 * c + 2] = x.z; v[4 * c + 3] = x.w;
  }
  __syncthreads();  // the barrier's initialisation is visible to every waiting thread
  if (!tc::mbar_wait(bar, 0)) {
    if (tid == 0) record_status(a.hdr, GQ_ERR_TIMEOUT);
    return;  // nothing was computed; the bulk copy has been waited for the full bound
  }
  double s = 1.0, inv_s = 1.0, z = 0.0;
  if (G == 0 && active) { s = a.row_s[row]; z = a.row_z[row]; inv_s = 1.0 / s; }
  double e2 = 0.0, bnd = 0.0;
  int ovf = 0;
  const unsigned full = 0xffffffffu;
  const int gbase = lane & ~(kP - 1);
  float* Ehrow = a.Ehi + rr * kBlock;
  float* Elrow = a.Elo + rr * kBlock;
  uint8_t* crow = a.codes8 + row * a.ldc8 + j0;
  constexpr int kGStep = (G > 0 && G < kSW) ? G : kSW;  // distance between possible group starts

  for (int seg = 0; seg < kBlock / kSW; ++seg) {
    if (kSW * seg >= bw) break;
    float eo[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t cw = 0u;
#pragma unroll
    for (int jl = 0; jl < kSW; ++jl) {
      const int jj = kSW * seg + jl;
      if (jj < bw) {
        if constexpr (G > 0) {
          if (jl % kGStep == 0 && (jj % G) == 0) {
            // group grid from the current (error-fed) weights of columns [jj, jj + G)
            double lo = 0.0, hi = 0.0;
#pragma unroll
            for (int c = 0; c < kVPL / 4; ++c)
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int k = kSW * (seg + c) + 4 * t + u;
                if (k >= jj && k < jj + G && k < bw) { lo = fmin(lo, v[4 * c + u]); hi = fmax(hi, v[4 * c + u]); }
              }
#pragma unroll
            for (int o = kP / 2; o > 0; o >>= 1) {
              lo = fmin(lo, __shfl_xor_sync(full, lo, o));
              hi = fmax(hi, __shfl_xor_sync(full, hi, o));
            }
            if (lo == 0.0 && hi == 0.0) { lo = -1.0; hi = 1.0; }
            s = (hi - lo) / maxq;
            z = rint(-lo / s);
            inv_s = 1.0 / s;
            if (active && t == 0) {
              const int64_t g = (j0 + jj) / G;
              a.scales[row * a.ngroups + g] = (float)s;
              a.zeros[row * a.ngroups + g] = (uint8_t)z;
            }
          }
        }
        const double cmin = -z, cmax = maxq - z;  // code range in the shifted domain c - z
        const int owner = jl / 4, slot = jl % 4;
        const double id = invd[jj];
        const double sd = s * id;
        const double x = __shfl_sync(full, v[slot], gbase + owner);
        const double xi = x * id;
        double c = rint_small(x * inv_s);
        if (a.clip) {
          c = fmin(fmax(c, cmin), cmax);
        } else if (c < cmin || c > cmax) {
          ovf = 1;
        }
        const double e = fma(-c, sd, xi);  // (x - s c) / U_jj
        if (t == owner) {
          eo[slot] = (float)e;
          cw |= (uint32_t)(int)fmin(fmax(c + z, 0.0), maxq) << (8 * slot);
        }
        e2 = fma(e, e, e2);
        bnd = fma(s * s, invd2[jj], bnd);
        const double* urow = Us + jj * kBlock + kSW * seg + 4 * t;
        if (t >= owner) {  // the chunk that holds column jj: only its later columns
          const double2 u01 = *reinterpret_cast<const double2*>(urow);
          const double2 u23 = *reinterpret_cast<const double2*>(urow + 2);
          if (t > owner || 0 > slot) v[0] = fma(-e, u01.x, v[0]);
          if (t > owner || 1 > slot) v[1] = fma(-e, u01.y, v[1]);
          if (t > owner || 2 > slot) v[2] = fma(-e, u23.x, v[2]);
          if (t > owner || 3 > slot) v[3] = fma(-e, u23.y, v[3]);
        }
#pragma unroll
        for (int c2 = 1; c2 < kVPL / 4; ++c2) {
          if (c2 < kBlock / kSW - seg) {
            const double2 u01 = *reinterpret_cast<const double2*>(urow + kSW * c2);
            const double2 u23 = *reinterpret_cast<const double2*>(urow + kSW * c2 + 2);
            v[4 * c2 + 0] = fma(-e, u01.x, v[4 * c2 + 0]);
            v[4 * c2 + 1] = fma(-e, u01.y, v[4 * c2 + 1]);
            v[4 * c2 + 2] = fma(-e, u23.x, v[4 * c2 + 2]);
            v[4 * c2 + 3] = fma(-e, u23.y, v[4 * c2 + 3]);
          }
        }
      }
    }
    // this segment's errors and codes
    if (active) {
      const int k = kSW * seg + 4 * t;
      float4 hi, lo;
      hi.x = tf32_rna(eo[0]); hi.y = tf32_rna(eo[1]); hi.z = tf32_rna(eo[2]); hi.w = tf32_rna(eo[3]);
      lo.x = eo[0] - hi.x; lo.y = eo[1] - hi.y; lo.z = eo[2] - hi.z; lo.w = eo[3] - hi.w;
      *reinterpret_cast<float4*>(Ehrow + k) = hi;
      *reinterpret_cast<float4*>(Elrow + k) = lo;
      if (k + 3 < bw) {
        *reinterpret_cast<uint32_t*>(crow + k) = cw;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (k + u < bw) crow[k + u] = (uint8_t)(cw >> (8 * u));
      }
    }
    // rotate: chunk seg + 1 moves to registers 0..3
#pragma unroll
    for (int i = 0; i < kVPL - 4; ++i) v[i] = v[i + 4];
  }
  // per-row overflow flag (all lanes of the warp take part in the shuffle)
  int ovf_row = ovf;
#pragma unroll
  for (int o = kP / 2; o > 0; o >>= 1) ovf_row |= __shfl_xor_sync(0xffffffffu, ovf_row, o);
  if (!active) return;
  // per-row totals (all lanes of a row hold the same e2 / bnd)
  if (t == 0) {
    if (j0 == 0) { a.row_e2[row] = e2; a.row_bnd[row] = bnd; a.overflow[row] = ovf_row; }
    else { a.row_e2[row] += e2; a.row_bnd[row] += bnd; a.overflow[row] |= ovf_row; }
  }
}

// ------------------------------------------------------------------------------------------
// packing + ||w0 - q||^2 per row (one CTA per original row)
// ------------------------------------------------------------------------------------------
template <class TW>
__global__ void __launch_bounds__(128) pack_kernel(const TW* W, const uint8_t* dead, int64_t n,
                                                   const uint8_t* codes8, int64_t ldc8,
                                                   int reverse, int bits, int group,
                                                   int64_t ngroups, const float* scales,
                                                   const uint8_t* zeros, uint32_t* codes,
                                                   double* row_d2) {
  const int64_t r = blockIdx.x;
  const uint8_t* crow = codes8 + r * ldc8;
  const int64_t nwords = (n * bits + 31) / 32;
  for (int64_t w = threadIdx.x; w < nwords; w += blockDim.x) {
    uint32_t word = 0u;
    int64_t cf = (32 * w) / bits, cl = (32 * w + 31) / bits;
    if (cl > n - 1) cl = n - 1;
    for (int64_t c = cf; c <= cl; ++c) {
      uint32_t code = crow[reverse ? n - 1 - c : c];
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
    int64_t g = group ? c / group : 0;
    float s = scales[r * ngroups + g], z = (float)zeros[r * ngroups + g];
    float code = (float)crow[reverse ? n - 1 - c : c];
    double d = (double)w0 - (double)s * (double)(code - z);
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

cudaError_t quant_init_attributes() {
  const int smem = (int)kColSmem;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  if ((e = cudaFuncSetAttribute(colloop_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) return e;
  return cudaFuncSetAttribute(colloop_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

template <int G>
static cudaError_t launch_colloop(const ColArgs& ca, cudaStream_t s) {
  const size_t smem = kColSmem;
  unsigned grid = (unsigned)((ca.k_rows + kRowsPerCta - 1) / kRowsPerCta);
  colloop_kernel<G><<<grid, kColThreads, smem, s>>>(ca);
  count_launches(1);
  return cudaGetLastError();
}

static cudaError_t colloop_dispatch(int group, const ColArgs& ca, cudaStream_t s) {
  switch (group) {
    case 0: return launch_colloop<0>(ca, s);
    case 16: return launch_colloop<16>(ca, s);
    case 32: return launch_colloop<32>(ca, s);
    case 64: return launch_colloop<64>(ca, s);
    case 128: return launch_colloop<128>(ca, s);
    default: return cudaErrorInvalidValue;
  }
}

// Two streams per call, forked from and joined back into the caller's stream: A (higher
// priority) runs the column loop of each block and the lazy update of the next block's 128
// columns; B runs the lazy update of all later columns, overlapped with the next block's
// column loop (look-ahead of one block).  One set per host thread and device, kept.
struct QuantStreams {
  bool ready = false;
  cudaStream_t a = nullptr, b = nullptr;
  cudaEvent_t fork = nullptr, col[2] = {}, rest[2] = {}, join[2] = {};
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
    if ((e = cudaStreamCreateWithPriority(&q.b, cudaStreamNonBlocking, least))) return e;
    cudaEvent_t* evs[] = {&q.fork, &q.col[0], &q.col[1], &q.rest[0], &q.rest[1], &q.join[0],
                          &q.join[1]};
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming))) return e;
    q.ready = true;
  }
  *out = &q;
  return cudaSuccess;
}

gq_status run_quantize(const QuantArgs& a, cudaStream_t s) {
  const int64_t m = a.m, n = a.n;
  QLayout L = q_layout(a.ws, m, n);
  const gq_quant_cfg& cfg = a.cfg;
  const int G = cfg.group_size;
  const int64_t ngroups = G ? (n + G - 1) / G : 1;
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
    dim3 g2(16, (unsigned)((n + kBlock - 1) / kBlock));
    ublk_kernel<<<g2, 256, 0, s>>>(a.U, n, L.Ublk);
    count_launches(1);
    Q_TRY(cudaGetLastError());
  }
  int64_t k_rows = m;
  const int* rowlist = nullptr;
  const int nblocks = (int)((n + kBlock - 1) / kBlock);
  const int max_rounds = cfg.clip ? 1 : cfg.ladder_max + 1;
  int rounds_run = 0;
  for (int round = 0; round < max_rounds; ++round) {
    rounds_run = round;
    {
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
                                             L.alpha, L.row_s, L.row_z, a.scales, a.zeros);
      count_launches(1);
      Q_TRY(cudaGetLastError());
    }
    LazyTcMaps maps[2];
    for (int i = 0; i < 2; ++i)
      Q_TRY(lazy_tc_make_maps(&maps[i], L.Ehi[i], L.Elo[i], k_rows, L.Uhi, L.Ulo, n, L.ldu));
    // Blocks on stream A; the lazy update after block b is split: the next block's 128 columns
    // on A (the next column loop needs them), all later columns on B.  Block b's errors live in
    // buffer b & 1 until its later-column update is done (the column loop of block b + 2, which
    // reuses the buffer, waits for it through the next-block update of block b + 1).
    QuantStreams* qs = nullptr;
    Q_TRY(quant_streams(&qs));
    cudaStream_t sa = qs->a, sb = qs->b;
    Q_TRY(cudaEventRecord(qs->fork, s));
    Q_TRY(cudaStreamWaitEvent(sa, qs->fork, 0));
    Q_TRY(cudaStreamWaitEvent(sb, qs->fork, 0));
    bool rest_pending = false;
    for (int b = 0; b < nblocks; ++b) {
      const int64_t j0 = (int64_t)b * kBlock;
      const int bw = (int)std::min<int64_t>(kBlock, n - j0);
      ColArgs ca{};
      ca.Ublk = L.Ublk; ca.hdr = L.hdr;
      ca.Wf = L.Wf; ca.n = n; ca.k_rows = k_rows; ca.rowlist = rowlist; ca.j0 = j0; ca.bw = bw;
      ca.U = a.U; ca.bits = cfg.bits; ca.clip = cfg.clip; ca.Ehi = L.Ehi[b & 1];
      ca.Elo = L.Elo[b & 1];
      ca.codes8 = L.codes8;
      ca.ldc8 = L.ldc8; ca.scales = a.scales; ca.zeros = a.zeros; ca.ngroups = ngroups;
      ca.row_s = L.row_s; ca.row_z = L.row_z; ca.row_e2 = L.row_e2; ca.row_bnd = L.row_bnd;
      ca.overflow = L.overflow;
      Q_TRY(colloop_dispatch(G, ca, sa));
      const int64_t j1 = j0 + bw;
      if (j1 >= n) continue;
      const int64_t jn = std::min<int64_t>(j1 + kBlock, n);
      Q_TRY(cudaEventRecord(qs->col[b & 1], sa));
      if (rest_pending) Q_TRY(cudaStreamWaitEvent(sa, qs->rest[(b - 1) & 1], 0));
      Q_TRY(launch_lazy_tc(maps[b & 1], L.Wf, n, k_rows, j0, j1, jn, L.hdr, sa));
      rest_pending = false;
      if (jn < n) {
        Q_TRY(cudaStreamWaitEvent(sb, qs->col[b & 1], 0));
        Q_TRY(launch_lazy_tc(maps[b & 1], L.Wf, n, k_rows, j0, jn, n, L.hdr, sb));
        Q_TRY(cudaEventRecord(qs->rest[b & 1], sb));
        rest_pending = true;
      }
    }
    Q_TRY(cudaEventRecord(qs->join[1], sb));
    Q_TRY(cudaStreamWaitEvent(sa, qs->join[1], 0));
    Q_TRY(cudaEventRecord(qs->join[0], sa));
    Q_TRY(cudaStreamWaitEvent(s, qs->join[0], 0));
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
      int code = GQ_ERR_NO_FIT;
      // first error wins: write only if the status word is still clear
      int cur = 0;
      Q_TRY(cudaMemcpyAsync(&cur, &L.hdr->status, sizeof(int), cudaMemcpyDeviceToHost, s));
      Q_TRY(cudaStreamSynchronize(s));
      if (cur == 0) Q_TRY(cudaMemcpyAsync(&L.hdr->status, &code, sizeof(int),
                                          cudaMemcpyHostToDevice, s));
      Q_TRY(cudaStreamSynchronize(s));
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
  if (a.wt == GQ_BF16)
    pack_kernel<__nv_bfloat16><<<(unsigned)m, 128, 0, s>>>(
        static_cast<const __nv_bfloat16*>(a.W), a.dead, n, L.codes8, L.ldc8, cfg.reverse,
        cfg.bits, G, ngroups, a.scales, a.zeros, a.codes, L.row_d2);
  else
    pack_kernel<float><<<(unsigned)m, 128, 0, s>>>(static_cast<const float*>(a.W), a.dead, n,
                                                   L.codes8, L.ldc8, cfg.reverse, cfg.bits, G,
                                                   ngroups, a.scales, a.zeros, a.codes, L.row_d2);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  q_reduce_kernel<<<1, 1024, 0, s>>>(m, L.row_e2, L.row_bnd, L.row_d2, a.delta, a.loss);
  count_launches(1);
  Q_TRY(cudaGetLastError());
  return GQ_OK;
}

}  // namespace gq
