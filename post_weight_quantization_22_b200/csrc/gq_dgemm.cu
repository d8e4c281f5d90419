// fp64 GEMM on the fp64 tensor cores for the factorisation (blocked Cholesky updates, panel
// triangular solves, triangular-inverse doubling).
//
// The factor must stay fp64-accurate (the codes downstream move when U carries fp32-level
// errors), and sm_100a runs fp64 at the same rate on mma.sync (DMMA) and on DFMA: ~37 TFLOP/s
// on 148 SMs.  DMMA m16n8k8 does 1024 multiply-adds per issue, which leaves the issue slots to
// the operand loads.
//
// CTA: 128 x 64 output tile (64 x 64 where 128-row tiles would leave SMs idle), 8 (4) consumer
// warps of 32 x 32 (2 x 4 m16n8k8 tiles each) and one producer warp whose lane 0 streams
// 16-deep K slices of A and B into a 4-stage shared-memory ring by TMA (no multicast; 128-byte
// swizzle), with full / empty mbarriers (bounded waits).
//
// K-slot permutation: a K slice of 16 is consumed as two k8 MMAs.  The MMA only sums over its 8
// k slots, so any assignment of slots to k indices works if A and B agree.  Lane t of a quad
// takes slots t and t+4 from the 16-byte chunk c = (t + 4 (t & 1)) ^ kk of the slice (k = 2c,
// 2c + 1) in k8 step kk.  With the 128-byte swizzle (chunk ^= row & 7) this makes the A (and
// "NT" B) fragment loads single 16-byte loads without bank conflicts, and the "NN" B fragment
// loads (two 8-byte loads from rows 2c and 2c + 1) conflict-free as well.
//
// Zero structure (triangular operands, ragged K) is applied by selecting 0.0 in registers, so
// whatever memory holds outside the structure (the factor's unused upper triangle) is never
// multiplied.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

namespace gq {

namespace {
constexpr int kBN = 64, kBK = 16, kStages = 4;
constexpr uint32_t kTileB = kBN * kBK * 8;  // 8 KB
constexpr int kCPitch = 72;                 // epilogue tile pitch (doubles)

// Tile shape: kWM consumer warps along M (BM = 32 kWM) x 2 along N, plus the producer warp.
template <int kWM>
struct Shape {
  static constexpr int BM = 32 * kWM;
  static constexpr int CWarps = 2 * kWM;
  static constexpr int Threads = (CWarps + 1) * 32;
  static constexpr uint32_t TileA = BM * kBK * 8;
  static constexpr uint32_t StageBytes = TileA + kTileB;
  static constexpr size_t Smem = kStages * StageBytes + 1024 + 2 * kStages * 8;
  static_assert(BM * kCPitch * 8 <= kStages * StageBytes, "epilogue tile must fit the ring");
};

struct DgemmArgs {
  int M, N, K;
  double alpha;
  int beta_one;
  int ax0, ay0, azx, azy;  // A tensor-map coordinates: x = column (k), y = row (i)
  int bx0, by0, bzx, bzy;  // B: NT x = k, y = j; NN x = j, y = k
  double* C;
  int64_t ldc, strideC;
  int a_lower, b_lower, b_upper, lower_tiles, tri_enum, c_vec;
  WsHeader* hdr;
};

}  // namespace

template <bool kNN, int kWM>
__device__ __forceinline__ void dgemm_body(const CUtensorMap& ma, const CUtensorMap& mb,
                                           const DgemmArgs& g) {
  using S = Shape<kWM>;
  constexpr int kBM = S::BM, kCWarps = S::CWarps;
  constexpr uint32_t kTileA = S::TileA, kStageBytes = S::StageBytes;
  extern __shared__ uint8_t dg_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dg_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;

  int ti, tj;
  if (kBM == 2 * kBN && g.tri_enum) {  // lower-triangular tile list: row r holds 2 (r + 1) tiles
    const int t = blockIdx.x;
    int r = (int)((sqrtf(4.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) <= t) ++r;
    while (r > 0 && r * (r + 1) > t) --r;
    ti = r;
    tj = t - r * (r + 1);
  } else {
    ti = blockIdx.y;
    tj = blockIdx.x;
  }
  const int i0 = ti * kBM, j0 = tj * kBN;
  if (i0 >= g.M || j0 >= g.N) return;
  if (g.lower_tiles && j0 >= i0 + kBM) return;
  const int z = blockIdx.z;

  int k_lo = 0, k_hi = g.K;
  if (g.a_lower) k_hi = min(k_hi, i0 + kBM);
  if (g.b_upper) k_hi = min(k_hi, j0 + kBN);
  if (g.b_lower) k_lo = (j0 / kBK) * kBK;
  const int nk = k_hi > k_lo ? (k_hi - k_lo + kBK - 1) / kBK : 0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kCWarps * 32);
    }
    tc::fence_barrier_init();
  }
  __syncthreads();

  int issued = 0;
  double acc[2][4][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0;

  if (warp == kCWarps) {
    if (lane == 0) {
      tc::prefetch_tmap(&ma);
      tc::prefetch_tmap(&mb);
      const int ax = g.ax0 + z * g.azx, ay = g.ay0 + z * g.azy + i0;
      const int bx = g.bx0 + z * g.bzx, by = g.by0 + z * g.bzy;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % kStages;
        if (kc >= kStages && !tc::mbar_wait(&empty[s], ((kc / kStages) - 1) & 1)) {
          record_status(g.hdr, GQ_ERR_TIMEOUT);
          break;
        }
        uint8_t* st = base + s * kStageBytes;
        const int kb = k_lo + kc * kBK;
        tc::mbar_arrive_expect_tx(&full[s], kStageBytes);
        tc::tma_load_2d(st, &ma, &full[s], ax + kb, ay);
        if (!kNN) {
          tc::tma_load_2d(st + kTileA, &mb, &full[s], bx + kb, by + j0);
        } else {
#pragma unroll
          for (int sub = 0; sub < kBN / 16; ++sub)
            tc::tma_load_2d(st + kTileA + sub * 2048, &mb, &full[s], bx + j0 + sub * 16, by + kb);
        }
        issued = kc + 1;
      }
      // The epilogue reads this C tile: bring it into L2 while the last slices are consumed.
      if (g.beta_one && g.c_vec && j0 + kBN <= g.N) {
        const double* c0p = g.C + (int64_t)z * g.strideC + (int64_t)i0 * g.ldc + j0;
        const int rows = min(kBM, g.M - i0);
        for (int r = 0; r < rows; ++r) tc::bulk_prefetch_l2(c0p + (int64_t)r * g.ldc, kBN * 8);
      }
    }
  } else {
    const int wm = warp >> 1, wn = warp & 1;  // warp grid kWM x 2
    const int gq4 = lane >> 2, t = lane & 3;
    const int rowA = wm * 32 + gq4;   // + mi * 16 (+ 8)
    const int colB = wn * 32 + gq4;   // + nj * 8
    // Slices that need the zero structure applied: kc >= mask_from (ragged K end, a_lower,
    // b_upper) or kc < mask_below (b_lower), for this warp's rows and columns.
    int mask_from = (k_hi - k_lo) / kBK;  // the ragged last slice, if any
    if (g.a_lower) mask_from = min(mask_from, max(0, (i0 + wm * 32 - k_lo - kBK + 1 + kBK) / kBK));
    if (g.b_upper) mask_from = min(mask_from, max(0, (j0 + wn * 32 - k_lo - kBK + 1 + kBK) / kBK));
    const int mask_below = g.b_lower ? (j0 + wn * 32 + 31 - k_lo + kBK - 1) / kBK : 0;
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kStages;
      if (!tc::mbar_wait(&full[s], (kc / kStages) & 1)) {
        if (lane == 0) record_status(g.hdr, GQ_ERR_TIMEOUT);
        break;
      }
      const uint8_t* sA = base + s * kStageBytes;
      const uint8_t* sB = sA + kTileA;
      const bool mask = kc >= mask_from || kc < mask_below;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int c = (t + 4 * (t & 1)) ^ kk;
        double a[2][4], b[4][2];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
          const int r0 = rowA + mi * 16;  // r0 & 7 == gq4
          const double2 v0 =
              *reinterpret_cast<const double2*>(sA + r0 * 128 + ((c ^ gq4) << 4));
          const double2 v1 =
              *reinterpret_cast<const double2*>(sA + (r0 + 8) * 128 + ((c ^ gq4) << 4));
          a[mi][0] = v0.x;
          a[mi][1] = v1.x;
          a[mi][2] = v0.y;
          a[mi][3] = v1.y;
        }
#pragma unroll
        for (int nj = 0; nj < 4; ++nj) {
          const int nl = colB + nj * 8;
          if (!kNN) {
            const double2 v =
                *reinterpret_cast<const double2*>(sB + nl * 128 + ((c ^ gq4) << 4));
            b[nj][0] = v.x;
            b[nj][1] = v.y;
          } else {
            const int sub = nl >> 4, nn = nl & 15;
            const int ka = 2 * c, kb1 = 2 * c + 1;
            const uint8_t* p = sB + sub * 2048 + (nn & 1) * 8;
            b[nj][0] = *reinterpret_cast<const double*>(
                p + ka * 128 + ((((nn >> 1) ^ (ka & 7))) << 4));
            b[nj][1] = *reinterpret_cast<const double*>(
                p + kb1 * 128 + ((((nn >> 1) ^ (kb1 & 7))) << 4));
          }
        }
        if (kk == 1) {
          // The whole slice is in registers: release the stage.  Every lane arrives for its own
          // shared-memory reads, after a proxy fence, so the producer's next TMA write into the
          // stage (async proxy) cannot overtake any lane's fragment loads (generic proxy).  A
          // single arrive per warp after __syncwarp let that write land early under load.
          tc::fence_proxy_async_smem();
          tc::mbar_arrive(&empty[s]);
        }
        if (mask) {
          const int ka = k_lo + kc * kBK + 2 * c, kb1 = ka + 1;
#pragma unroll
          for (int mi = 0; mi < 2; ++mi) {
            const int i = i0 + rowA + mi * 16;
            if (!(ka < k_hi && !(g.a_lower && ka > i))) a[mi][0] = 0.0;
            if (!(ka < k_hi && !(g.a_lower && ka > i + 8))) a[mi][1] = 0.0;
            if (!(kb1 < k_hi && !(g.a_lower && kb1 > i))) a[mi][2] = 0.0;
            if (!(kb1 < k_hi && !(g.a_lower && kb1 > i + 8))) a[mi][3] = 0.0;
          }
#pragma unroll
          for (int nj = 0; nj < 4; ++nj) {
            const int j = j0 + colB + nj * 8;
            if (!(ka < k_hi && !(g.b_upper && ka > j) && !(g.b_lower && ka < j))) b[nj][0] = 0.0;
            if (!(kb1 < k_hi && !(g.b_upper && kb1 > j) && !(g.b_lower && kb1 < j)))
              b[nj][1] = 0.0;
          }
        }
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
          for (int nj = 0; nj < 4; ++nj) tc::dmma_m16n8k8(acc[mi][nj], a[mi], b[nj]);
      }
    }

    // Epilogue through shared memory: once every consumer warp is past its last slice the ring
    // is free; the tile goes there (pitch 72 doubles: the 16-byte stores of a quarter-warp hit
    // distinct banks), then each warp updates whole rows of C with coalesced 16-byte accesses.
    // Fragment c0, c1 sits at (g, 2t .. 2t+1), c2, c3 at (g + 8, 2t .. 2t+1) of its 16 x 8 tile.
    asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32) : "memory");
    double* sC = reinterpret_cast<double*>(base);
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int nj = 0; nj < 4; ++nj)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          *reinterpret_cast<double2*>(sC + (rowA + mi * 16 + h * 8) * kCPitch + wn * 32 + nj * 8 +
                                      2 * t) = make_double2(acc[mi][nj][2 * h],
                                                            acc[mi][nj][2 * h + 1]);
    asm volatile("bar.sync 1, %0;" ::"r"(kCWarps * 32) : "memory");
    double* C = g.C + (int64_t)z * g.strideC;
    const int j = j0 + 2 * lane;
    constexpr int kRows = kBM / kCWarps;  // rows per warp, all loads in flight together
    const bool vec = g.c_vec && j + 1 < g.N;
    double2 cv[kRows];
#pragma unroll
    for (int t = 0; t < kRows; ++t) {
      const int i = i0 + warp + t * kCWarps;
      cv[t] = make_double2(0.0, 0.0);
      if (g.beta_one && i < g.M) {
        const double* crow = C + (int64_t)i * g.ldc;
        if (vec) {
          cv[t] = *reinterpret_cast<const double2*>(crow + j);
        } else {
          if (j < g.N) cv[t].x = crow[j];
          if (j + 1 < g.N) cv[t].y = crow[j + 1];
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kRows; ++t) {
      const int r = warp + t * kCWarps, i = i0 + r;
      if (i < g.M) {
        const double2 a2 = *reinterpret_cast<const double2*>(sC + r * kCPitch + 2 * lane);
        double* crow = C + (int64_t)i * g.ldc;
        const double2 o = make_double2(cv[t].x + g.alpha * a2.x, cv[t].y + g.alpha * a2.y);
        if (vec) {
          *reinterpret_cast<double2*>(crow + j) = o;
        } else {
          if (j < g.N) crow[j] = o.x;
          if (j + 1 < g.N) crow[j + 1] = o.y;
        }
      }
    }
  }

  // Leave no copy in flight: after a timeout the producer waits (bounded) for the last phase of
  // every stage it filled; in the normal path those phases are complete already.
  __syncthreads();
  if (warp == kCWarps && lane == 0) {
    for (int kc = issued > kStages ? issued - kStages : 0; kc < issued; ++kc)
      if (!tc::mbar_wait(&full[kc % kStages], (kc / kStages) & 1)) {
        record_status(g.hdr, GQ_ERR_TIMEOUT);
        break;
      }
  }
}

// Entry points.  The 128-row NT kernel holds 112 registers so that two CTAs share an SM; the NN
// kernels (two 8-byte B loads per fragment, more address registers) get fewer CTAs per SM and no
// spills.
__global__ void __maxnreg__(112) dgemm_nt128_kernel(const __grid_constant__ CUtensorMap ma,
                                                    const __grid_constant__ CUtensorMap mb,
                                                    const DgemmArgs g) {
  dgemm_body<false, 4>(ma, mb, g);
}
__global__ void __launch_bounds__(Shape<4>::Threads, 1)
    dgemm_nn128_kernel(const __grid_constant__ CUtensorMap ma,
                       const __grid_constant__ CUtensorMap mb, const DgemmArgs g) {
  dgemm_body<true, 4>(ma, mb, g);
}
__global__ void __launch_bounds__(Shape<2>::Threads, 3)
    dgemm_nt64_kernel(const __grid_constant__ CUtensorMap ma,
                      const __grid_constant__ CUtensorMap mb, const DgemmArgs g) {
  dgemm_body<false, 2>(ma, mb, g);
}
__global__ void __launch_bounds__(Shape<2>::Threads, 2)
    dgemm_nn64_kernel(const __grid_constant__ CUtensorMap ma,
                      const __grid_constant__ CUtensorMap mb, const DgemmArgs g) {
  dgemm_body<true, 2>(ma, mb, g);
}

cudaError_t dgemm_init_attributes() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(dgemm_nt128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Shape<4>::Smem)))
    return e;
  if ((e = cudaFuncSetAttribute(dgemm_nn128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Shape<4>::Smem)))
    return e;
  if ((e = cudaFuncSetAttribute(dgemm_nt64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Shape<2>::Smem)))
    return e;
  return cudaFuncSetAttribute(dgemm_nn64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)Shape<2>::Smem);
}

static bool operand_ok(const DgemmOperand& o) {
  return o.base && (reinterpret_cast<uintptr_t>(o.base) & 15) == 0 && (o.ld % 2) == 0 &&
         o.ld >= o.cols && o.rows > 0 && o.cols > 0;
}

cudaError_t launch_dgemm(const DgemmCall& c, cudaStream_t s) {
  if (c.M <= 0 || c.N <= 0 || c.batch <= 0) return cudaSuccess;
  if (!operand_ok(c.A) || !operand_ok(c.B)) return cudaErrorInvalidValue;
  // TMA: the innermost coordinate of every box start must be even for 8-byte elements.  The
  // starts are col0 + z * zcol + (multiples of 16), so col0 and zcol must be even.
  if ((c.A.col0 | c.A.zcol | c.B.col0 | c.B.zcol) & 1) return cudaErrorInvalidValue;
  // 128-row tiles when they fill the machine, else 64-row tiles (panel solves and updates).
  const int tn = (c.N + kBN - 1) / kBN;
  const int tm128 = (c.M + 127) / 128;
  const bool tall = (long)tm128 * tn * c.batch >= 148 || (c.lower_tiles && c.M == c.N);
  CUtensorMap ma, mb;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  cudaError_t e = encode_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 8, c.A.base, c.A.rows,
                                 c.A.cols, c.A.ld, kBK, tall ? 128 : 64, sw);
  if (e != cudaSuccess) return e;
  if (!c.b_nmajor)
    e = encode_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 8, c.B.base, c.B.rows, c.B.cols,
                       c.B.ld, kBK, kBN, sw);
  else
    e = encode_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 8, c.B.base, c.B.rows, c.B.cols,
                       c.B.ld, 16, kBK, sw);
  if (e != cudaSuccess) return e;
  DgemmArgs g{};
  g.M = c.M; g.N = c.N; g.K = c.K; g.alpha = c.alpha; g.beta_one = c.beta_one;
  g.ax0 = (int)c.A.col0; g.ay0 = (int)c.A.row0; g.azx = (int)c.A.zcol; g.azy = (int)c.A.zrow;
  g.bx0 = (int)c.B.col0; g.by0 = (int)c.B.row0; g.bzx = (int)c.B.zcol; g.bzy = (int)c.B.zrow;
  g.C = c.C; g.ldc = c.ldc; g.strideC = c.strideC;
  g.a_lower = c.a_lower; g.b_lower = c.b_lower; g.b_upper = c.b_upper;
  g.lower_tiles = c.lower_tiles;
  g.c_vec = ((reinterpret_cast<uintptr_t>(c.C) & 15) == 0 && (c.ldc % 2) == 0 &&
             (c.strideC % 2) == 0) ? 1 : 0;
  g.hdr = c.hdr;
  dim3 grid;
  if (tall && c.lower_tiles && c.M == c.N) {
    g.tri_enum = 1;
    grid = dim3((unsigned)(tm128 * (tm128 + 1)), 1, (unsigned)c.batch);
  } else {
    g.tri_enum = 0;
    const int tm = tall ? tm128 : (c.M + 63) / 64;
    grid = dim3((unsigned)tn, (unsigned)tm, (unsigned)c.batch);
  }
  if (tall) {
    if (c.b_nmajor)
      dgemm_nn128_kernel<<<grid, Shape<4>::Threads, Shape<4>::Smem, s>>>(ma, mb, g);
    else
      dgemm_nt128_kernel<<<grid, Shape<4>::Threads, Shape<4>::Smem, s>>>(ma, mb, g);
  } else {
    if (c.b_nmajor)
      dgemm_nn64_kernel<<<grid, Shape<2>::Threads, Shape<2>::Smem, s>>>(ma, mb, g);
    else
      dgemm_nt64_kernel<<<grid, Shape<2>::Threads, Shape<2>::Smem, s>>>(ma, mb, g);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
