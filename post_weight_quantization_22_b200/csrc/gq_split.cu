// fp64-accurate GEMMs of the factorisation on the int8 tensor cores (exact digit products).
//
// The factor's time is in two families of large products, both of depth K = 512 (one
// super-panel of the split path): the trailing Cholesky updates M[i][j] -= sum_k L[i][k] L[j][k] (lower part) and
// the triangular inverse's block products T[i][j] += sum_k L[i][k] X[k][j].  On sm_100a the fp64
// units cap them at ~37 TFLOP/s; the int8 tensor cores run ~100x faster per product, so each
// fp64 operand is cut into exact int8 pieces (the splitting idea of Ozaki et al., "Error-free
// transformations of matrix multiplication by using fast routines of matrix multiplication and
// its applications", Numer. Algorithms 59 (2012)):
//
//   every operand row r (a row of L, or a column of X) gets a power-of-two scale 2^e_r with
//   |v| 2^-e_r <= 1/2 over its K entries, and v 2^-e_r = sum_{s < S} d_s 2^-7(s+1) with signed
//   7-bit digits d_s in [-64, 64] (round to nearest at every step, so the first S digits carry
//   7S = 42 bits of the row's scale; the remainder below 2^-(7S+1) is dropped).  Then
//     sum_k a_ik b_jk = 2^(e_i + e_j) sum_{p + q <= S - 1} 2^-7(p+q+2) sum_k dA_p,ik dB_q,jk,
//   each inner sum an exact int8 x int8 -> int32 tensor-core product (|sum| < 2^24 for K = 512),
//   grouped by class c = p + q into S int32 accumulators in tensor memory and combined in fp64
//   in the epilogue.  The dropped pairs p + q >= S weigh below 2^-7(S+1) of the kept ones.
//
// With S = 6 (21 digit products per multiply-add) one product carries about 2^-42 of
// |a_i| |b_j| (measured 1.5e-12 relative on a 256-deep update), far inside what the factor needs
// (the codes move only when U carries errors near 1e-6).
//
// Kernels: split_rows_kernel (digits of row-major rows, K contiguous: the panel's rows of L),
// split_cols_kernel (digits of the columns of a row-major block, transposed through shared
// memory: a block row of the inverse), and split_gemm_kernel (tcgen05 kind::i8, 128 x 64 tiles,
// TMA-fed 2-stage ring of 72 KB stages (two 32-deep k-steps each, 64-byte swizzled rows; a
// 4-stage ring of 36 KB one-k-step stages with the 32-byte swizzle measured 12 % slower),
// warp-specialised: a producer warp, an MMA warp and
// eight epilogue warps; a CTA runs a few tiles and hands the accumulator back to the MMA warp
// as soon as the epilogue has read it, so the update of C overlaps the next tile's products).
// For one A digit the products with consecutive B digits are one instruction of N up to 256
// (their B planes sit back to back in shared memory, their classes side by side in TMEM).
// The epilogue warps, two per TMEM lane quadrant, each read 32 columns of all classes, two
// classes per load-and-wait; each thread stages its row's 32 scaled values in shared memory
// and adds them to C with one bulk fp64 reduce-add, done at L2 (C is never loaded into the SM).
#include "gq_internal.cuh"
#include "gq_tc.cuh"

namespace gq {

namespace {
constexpr int kSBM = 128, kSBN = 64;  // output tile
constexpr int kSBK = 64;              // K bytes per stage (two MMA k-steps of 32)
constexpr int kSStages = 2;
constexpr uint32_t kSATile = kSBM * kSBK;                  // 8 KB per digit plane
constexpr uint32_t kSBTile = kSBN * kSBK;                  // 4 KB per digit plane
constexpr uint32_t kSStage = kSplitDigits * (kSATile + kSBTile);  // 72 KB
constexpr int kSEpiWarps = 8;        // two per TMEM lane quadrant, 32 columns each
constexpr int kSEpiPitch = 32 * 8 + 16;  // bytes per staged row of 32 doubles (padded: the
                                         // 16-byte stores of a warp spread over the banks)
constexpr uint32_t kSEpiBytes = kSEpiWarps * 32 * kSEpiPitch;  // each epilogue warp's 32 rows
constexpr size_t kSSmem = kSStages * kSStage + 1024 + 256 + kSEpiBytes;
static_assert(kSSmem <= 227 * 1024, "the stages and the epilogue staging fit one CTA's shared memory");
constexpr int kSThreads = 32 * (2 + kSEpiWarps);  // warp 0 producer, warp 1 MMA, then epilogue
constexpr int kSTilesPerCta = 4;     // tiles per CTA aimed at (CTAs retire regularly, so other
                                     // streams' kernels get SMs)
constexpr uint32_t kSTmemCols = 512; // kSplitDigits x 64 columns, rounded up to a power of two
static_assert(kSplitDigits * kSBN <= (int)kSTmemCols, "class accumulators must fit in TMEM");
static_assert(kSplitDigits % 2 == 0, "the epilogue reads the classes two at a time");
// int8 x int8 -> s32, A and B K-major, M 128, N columns (a multiple of 16, at most 256)
__host__ __device__ constexpr uint32_t split_idesc(uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((uint32_t)(kSBM >> 4) << 24);
}

struct SplitArgs {
  double* C;
  int64_t ldc;
  int M, N;          // output rows and columns
  int nk;            // K chunks of kSBK
  int planeA, planeB;  // rows of one digit plane (plane d starts at row d x plane)
  int a0, b0;        // plane row of output row 0 / output column 0
  const int* ea;     // exponent of each plane row of A, B
  const int* eb;
  double alpha;
  int lower;         // only entries with column <= row
  int tiles, ntn;    // tiles enumerated, column tiles
  int ctas;          // CTAs of the launch; CTA c runs tiles [c tiles / ctas, (c + 1) tiles / ctas)
  WsHeader* hdr;
};

__device__ __forceinline__ double pow2(int e) {  // 2^e for -1022 <= e <= 1023
  return __longlong_as_double((long long)(1023 + e) << 52);
}

// Scale exponent of an operand row from its largest magnitude: |v| 2^-e < 1/2, clamped to
// [-1000, 1000] so that 2^e, 2^-e and the epilogue's products of scales stay normal (entries
// below 2^-1000 keep fewer digits; the factor's entries are nowhere near).
__device__ __forceinline__ int split_exponent(double mx) {
  if (!(mx > 0.0)) return 0;
  const int e = ilogb(mx) + 2;
  return e < -1000 ? -1000 : (e > 1000 ? 1000 : e);
}

// Tile t of the enumeration: row-major over all tiles, or over the tiles that reach the lower
// triangle (row r of 128-row tiles holds min(2 r + 2, ntn) 64-column tiles).
__device__ __forceinline__ void tile_of(const SplitArgs& g, int t, int& bi, int& bj) {
  if (!g.lower) {
    bi = t / g.ntn;
    bj = t - bi * g.ntn;
    return;
  }
  const int rs = (g.ntn - 1) / 2;  // first row whose count is ntn
  const int before = rs * (rs + 1);
  if (t < before) {
    int r = (int)((sqrtf(4.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((r + 1) * (r + 2) <= t) ++r;
    while (r > 0 && r * (r + 1) > t) --r;
    bi = r;
    bj = t - r * (r + 1);
  } else {
    const int u = t - before;
    bi = rs + u / g.ntn;
    bj = u - (u / g.ntn) * g.ntn;
  }
}
}  // namespace

// ---------------------------------------------------------------------------------------------
// digit splits (K = kSplitK values per operand row)
// ---------------------------------------------------------------------------------------------
// Row r of A (rows x kSplitK, leading dimension lda): exponent ex[r] and digit planes
// D[s][r][k] (plane stride plane_rows x kSplitK bytes).  One warp per row; lane l takes the 8
// consecutive values k = 256 g + 8 l .. + 7 of each 256-wide group g.  tri: A is a lower
// triangular block whose diagonal starts at (0, 0); entries k > r count as zero (whatever
// the memory holds there).
constexpr int kRowGroups = kSplitK / 256;
__global__ void __launch_bounds__(256) split_rows_kernel(const double* A, int64_t lda, int rows,
                                                         int64_t plane_rows, int8_t* D, int* ex,
                                                         int tri) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  double v[kRowGroups][8];
#pragma unroll
  for (int g = 0; g < kRowGroups; ++g) {
    const double* src = A + (int64_t)r * lda + 256 * g + 8 * lane;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const double2 x = *reinterpret_cast<const double2*>(src + i);
      const int k = 256 * g + 8 * lane + i;
      v[g][i] = (tri && k > r) ? 0.0 : x.x;
      v[g][i + 1] = (tri && k + 1 > r) ? 0.0 : x.y;
    }
  }
  double mx = 0.0;
#pragma unroll
  for (int g = 0; g < kRowGroups; ++g)
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmax(mx, fabs(v[g][i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const int e = split_exponent(mx);
  if (lane == 0) ex[r] = e;
  const double sc = pow2(-e);
#pragma unroll
  for (int g = 0; g < kRowGroups; ++g) {
    uint64_t packed[kSplitDigits];
#pragma unroll
    for (int s = 0; s < kSplitDigits; ++s) packed[s] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double x = v[g][i] * sc;
#pragma unroll
      for (int s = 0; s < kSplitDigits; ++s) {
        x *= 128.0;
        const double q = rint(x);
        x -= q;
        packed[s] |= (uint64_t)(uint8_t)(int8_t)(int)q << (8 * i);
      }
    }
#pragma unroll
    for (int s = 0; s < kSplitDigits; ++s)
      *reinterpret_cast<uint64_t*>(D + (int64_t)s * plane_rows * kSplitK + (int64_t)r * kSplitK +
                                   256 * g + 8 * lane) = packed[s];
  }
}

// Column j of X (kSplitK rows x cols, leading dimension ldx) as an operand row: exponent ex[j]
// and digit planes D[s][j][k] = digit s of X[k][j] 2^-ex[j].  A CTA takes 32 columns with 512
// threads; thread (ty, tx) = (tid / 32, tid % 32) holds rows kPerTy ty .. + kPerTy - 1 of
// column j0 + tx in registers (read once, coalesced along tx, every load in flight together),
// the column's maximum comes from a shared-memory reduction over ty, and per 8 consecutive rows
// the digits are packed into one 8-byte shared-memory store per plane; the CTA writes the 32
// rows of each plane out with coalesced 8-byte stores.  tri: X is a lower triangular block
// whose diagonal starts at (0, 0); entries with row k < column j count as zero.
constexpr int kColTy = 16;                   // threads down one column
constexpr int kPerTy = kSplitK / kColTy;     // rows per thread
constexpr int kSplitColsThreads = 32 * kColTy;
constexpr int kColPitch = kSplitK + 8;  // bytes per staged row (8-byte stores spread over banks)
constexpr size_t kSplitColsSmem =
    (size_t)kSplitDigits * 32 * kColPitch + (size_t)kColTy * 32 * sizeof(double);
__global__ void __launch_bounds__(kSplitColsThreads) split_cols_kernel(const double* X,
                                                                       int64_t ldx, int cols,
                                                                       int64_t plane_rows,
                                                                       int8_t* D, int* ex,
                                                                       int tri) {
  extern __shared__ __align__(16) uint8_t sc_smem[];
  uint8_t* sD = sc_smem;  // [s][32 columns][kColPitch]
  double* red = reinterpret_cast<double*>(sc_smem + (size_t)kSplitDigits * 32 * kColPitch);
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int j0 = blockIdx.x * 32, j = j0 + tx;
  const bool act = j < cols;
  const double* xcol = X + (int64_t)(kPerTy * ty) * ldx + (act ? j : 0);
  const int kmin = tri ? j : 0;  // rows above kmin of this column count as zero
  double v[kPerTy];
#pragma unroll
  for (int i = 0; i < kPerTy; ++i) {
    const int k = kPerTy * ty + i;
    v[i] = (act && k >= kmin) ? xcol[(int64_t)i * ldx] : 0.0;
  }
  double mx = 0.0;
#pragma unroll
  for (int i = 0; i < kPerTy; ++i) mx = fmax(mx, fabs(v[i]));
  red[ty * 32 + tx] = mx;
  __syncthreads();
  mx = 0.0;
#pragma unroll
  for (int y = 0; y < kColTy; ++y) mx = fmax(mx, red[y * 32 + tx]);
  const int e = split_exponent(mx);
  if (ty == 0 && act) ex[j] = e;
  const double sc = pow2(-e);
#pragma unroll
  for (int g8 = 0; g8 < kPerTy / 8; ++g8) {
    uint64_t packed[kSplitDigits];
#pragma unroll
    for (int s = 0; s < kSplitDigits; ++s) packed[s] = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double x = v[8 * g8 + i] * sc;
#pragma unroll
      for (int s = 0; s < kSplitDigits; ++s) {
        x *= 128.0;
        const double q = rint(x);
        x -= q;
        packed[s] |= (uint64_t)(uint8_t)(int8_t)(int)q << (8 * i);
      }
    }
#pragma unroll
    for (int s = 0; s < kSplitDigits; ++s)
      *reinterpret_cast<uint64_t*>(sD + ((size_t)s * 32 + tx) * kColPitch + kPerTy * ty + 8 * g8) =
          packed[s];
  }
  __syncthreads();
  // plane s, rows j0 .. j0 + 31: kSplitK / 8 words each, written in order by consecutive threads
  constexpr int kWords = kSplitK / 8;
  for (int s = 0; s < kSplitDigits; ++s) {
    for (int idx = threadIdx.x; idx < 32 * kWords; idx += kSplitColsThreads) {
      const int rr = idx / kWords, w = idx % kWords;
      if (j0 + rr < cols)
        *reinterpret_cast<uint64_t*>(D + (int64_t)s * plane_rows * kSplitK +
                                     (int64_t)(j0 + rr) * kSplitK + 8 * w) =
            *reinterpret_cast<const uint64_t*>(sD + ((size_t)s * 32 + rr) * kColPitch + 8 * w);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// C (+)= alpha 2^(ea_i + eb_j) sum_c 2^-7(c+2) acc_c   (tcgen05 kind::i8)
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kSThreads, 1)
    split_gemm_kernel(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mb,
                      const SplitArgs g) {
  extern __shared__ uint8_t sg_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sg_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kSStages * kSStage);
  uint64_t* empty = full + kSStages;
  uint64_t* tfull = empty + kSStages;  // the tile's products are complete
  uint64_t* tempty = tfull + 1;        // the epilogue has read the accumulators (4 warps)
  uint64_t* fin = tempty + 1;          // every product this CTA issued has completed
  uint32_t* tslot = reinterpret_cast<uint32_t*>(fin + 1);
  __shared__ int s_issued;
  __shared__ __align__(16) double s_colscale[kSEpiWarps][32];  // per epilogue warp: 2^eb of its columns
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_begin = (int)((int64_t)blockIdx.x * g.tiles / g.ctas);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * g.tiles / g.ctas);
  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(tfull, 1);
    tc::mbar_init(tempty, kSEpiWarps);
    tc::mbar_init(fin, 1);
    tc::fence_barrier_init();
    tc::prefetch_tmap(&ma);
    tc::prefetch_tmap(&mb);
    s_issued = 0;
  }
  if (warp == 1) tc::tmem_alloc(tslot, kSTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {  // producer
      int it = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        int bi, bj;
        tile_of(g, t, bi, bj);
        for (int kc = 0; kc < g.nk; ++kc, ++it) {
          const int s = it % kSStages;
          if (it >= kSStages && !tc::mbar_wait(&empty[s], ((it / kSStages) - 1) & 1)) {
            record_status(g.hdr, GQ_ERR_TIMEOUT);
            ok = false;
            break;
          }
          uint8_t* st = base + s * kSStage;
          tc::mbar_arrive_expect_tx(&full[s], kSStage);
#pragma unroll
          for (int d = 0; d < kSplitDigits; ++d) {
            tc::tma_load_2d(st + d * kSATile, &ma, &full[s], kc * kSBK,
                            d * g.planeA + g.a0 + bi * kSBM);
            tc::tma_load_2d(st + kSplitDigits * kSATile + d * kSBTile, &mb, &full[s], kc * kSBK,
                            d * g.planeB + g.b0 + bj * kSBN);
          }
        }
      }
      s_issued = it;
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      int it = 0, done = 0;
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        if (done > 0 && !tc::mbar_wait(tempty, (done - 1) & 1)) {
          record_status(g.hdr, GQ_ERR_TIMEOUT);
          break;
        }
        tc::fence_after_sync();
        for (int kc = 0; kc < g.nk; ++kc, ++it) {
          const int s = it % kSStages;
          if (!tc::mbar_wait(&full[s], (it / kSStages) & 1)) {
            record_status(g.hdr, GQ_ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t a0 = tc::smem_u32(base + s * kSStage);
          const uint32_t b0 = a0 + kSplitDigits * kSATile;
          // the stage's descriptors once; an operand at a constant byte offset from the stage
          // is the same descriptor with offset / 16 added to its start-address field (the
          // field holds address / 16 in 14 bits, and no address here reaches 2^18)
          const uint64_t ad0 = tc::sdesc(a0, 16, 512, tc::kLayoutSW64);
          const uint64_t bd0 = tc::sdesc(b0, 16, 512, tc::kLayoutSW64);
          // Digit pairs (p, q) with p + q < S (weight >= 2^-7(S+1)).  For one p the products
          // with q = 0 .. S-1-p go to classes p .. S-1, which sit side by side in TMEM, and the
          // B planes q = 0 .. sit back to back in shared memory (64 rows each, the same swizzle
          // phase), so they are one product A_p [B_0; B_1; ..] with N = 64 (S - p), cut at
          // N = 256: 8 instructions per k-step instead of 21, and each A plane read once.
#pragma unroll
          for (int k = 0; k < kSBK / 32; ++k) {
#pragma unroll
            for (int p = 0; p < kSplitDigits; ++p) {
#pragma unroll
              for (int q0 = 0; p + q0 < kSplitDigits; q0 += 256 / kSBN) {
                const int nq = min(kSplitDigits - p - q0, 256 / kSBN);
                // p = 0 opens every class accumulator of the tile
                const uint32_t acc = (kc == 0 && k == 0 && p == 0) ? 0u : 1u;
                tc::mma_i8(tmem + (p + q0) * kSBN, ad0 + (uint64_t)((p * kSATile + k * 32) >> 4),
                           bd0 + (uint64_t)((q0 * kSBTile + k * 32) >> 4),
                           split_idesc((uint32_t)(nq * kSBN)), acc);
              }
            }
          }
          tc::mma_commit(&empty[s]);
        }
        if (!ok) break;
        tc::mma_commit(tfull);
        ++done;
      }
    }
  } else {  // epilogue: warp w reads TMEM lanes 32 (w % 4) .., columns 32 ((w - 2) / 4) ..
    const int quad = warp & 3, half = (warp - 2) >> 2;
    double* colscale = s_colscale[warp - 2];
    // this thread's staging row (a 32-bit shared-memory address)
    const uint32_t srow = tc::smem_u32(base + kSStages * kSStage + 256) +
                          (uint32_t)(((warp - 2) * 32 + lane) * kSEpiPitch);
    int done = 0;
    for (int t = t_begin; t < t_end; ++t, ++done) {
      int bi, bj;
      tile_of(g, t, bi, bj);
      const int i = bi * kSBM + quad * 32 + lane;
      const int jt = bj * kSBN + half * 32;  // this warp's first column
      double* crow = g.C + (int64_t)i * g.ldc + jt;
      const bool rowok = i < g.M && jt < g.N;
      const bool vec = rowok && jt + 32 <= g.N && (!g.lower || jt + 31 <= i) &&
                       ((reinterpret_cast<uintptr_t>(crow) & 15) == 0);
      // the columns' scales into this warp's slice of shared memory, one load per column (read
      // inside the store loop, they would be reloaded after every store to C: the compiler
      // cannot rule out that C aliases the exponents).  Warp-private: no barrier beyond the
      // warp, so a warp that gives up on a bounded wait strands no other.
      __syncwarp();  // the previous tile's reads of the slice are done
      colscale[lane] = jt + lane < g.N ? pow2(g.eb[g.b0 + jt + lane]) : 0.0;
      __syncwarp();
      if (!tc::mbar_wait(tfull, done & 1)) {
        if (lane == 0) record_status(g.hdr, GQ_ERR_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      double acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = 0.0;
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + half * 32;
      // Classes c and c + 1 weigh 2^-7 apart and every class sum is below 2^23 in magnitude,
      // so 128 acc_c + acc_(c+1) is exact in int32: one conversion to fp64 per pair (the fp64
      // conversions, not the loads, are the slow part of this phase).
#pragma unroll
      for (int c = kSplitDigits - 2; c >= 0; c -= 2) {  // smallest classes first, two per wait
        uint32_t va[32], vb[32];
        tc::tmem_ld32x2(tbase + (c + 1) * kSBN, tbase + c * kSBN, va, vb);
        const double w = pow2(-7 * (c + 3));
#pragma unroll
        for (int j = 0; j < 32; ++j)
          acc[j] = fma((double)((int)vb[j] * 128 + (int)va[j]), w, acc[j]);
      }
      // the accumulators are in registers: the MMA warp may start the next tile
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty);
      if (vec) {
        // The row's 32 scaled values into its staging row, then one bulk reduce-add of 256
        // bytes into C at L2: no load of C into the SM.  si cs acc is exact (a power-of-two
        // scaling of acc), so C + si cs acc rounds once, as fma(si cs, acc, C) would.
        const double si = g.alpha * pow2(g.ea[g.a0 + i]);
        tc::bulk_wait_group_read0();  // the previous tile's reduce has read this staging row
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const double2 cs = *reinterpret_cast<const double2*>(colscale + j);
          tc::st_shared_f64x2(srow + 8 * j, (si * cs.x) * acc[j], (si * cs.y) * acc[j + 1]);
        }
        tc::fence_proxy_async_smem();  // the stores above, visible to the bulk copy
        tc::bulk_reduce_add_f64(crow, srow, 32 * sizeof(double));
        tc::bulk_commit_group();
      } else if (rowok) {
        const double si = g.alpha * pow2(g.ea[g.a0 + i]);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = jt + j;
          if (col < g.N && (!g.lower || col <= i)) crow[j] = fma(si * colscale[j], acc[j], crow[j]);
        }
      }
    }
  }

  // Teardown: no copy or product may be in flight when the CTA leaves.  In the normal path
  // every phase below has completed already; after a timeout the waits are bounded.
  if (warp >= 2) tc::bulk_wait_group0();  // this thread's reduces into C have completed
  __syncthreads();
  if (warp == 0 && lane == 0) {
    const int issued = s_issued;
    for (int kc = issued > kSStages ? issued - kSStages : 0; kc < issued; ++kc)
      if (!tc::mbar_wait(&full[kc % kSStages], (kc / kSStages) & 1)) {
        record_status(g.hdr, GQ_ERR_TIMEOUT);
        break;
      }
  }
  if (warp == 1 && lane == 0) {  // one more commit tracks every product issued before it
    tc::mma_commit(fin);
    if (!tc::mbar_wait(fin, 0)) record_status(g.hdr, GQ_ERR_TIMEOUT);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, kSTmemCols);
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
cudaError_t split_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(split_gemm_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(split_cols_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kSplitColsSmem);
}

cudaError_t launch_split_rows(const double* A, int64_t lda, int rows, SplitOperand op,
                              cudaStream_t s, int tri) {
  if (rows <= 0) return cudaSuccess;
  if ((reinterpret_cast<uintptr_t>(A) & 15) || (lda & 1)) return cudaErrorInvalidValue;
  split_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(A, lda, rows, op.plane_rows,
                                                               op.digits, op.ex, tri);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_split_cols(const double* X, int64_t ldx, int cols, SplitOperand op,
                              cudaStream_t s, int tri) {
  if (cols <= 0) return cudaSuccess;
  split_cols_kernel<<<(unsigned)((cols + 31) / 32), kSplitColsThreads, kSplitColsSmem, s>>>(
      X, ldx, cols, op.plane_rows, op.digits, op.ex, tri);
  count_launches(1);
  return cudaGetLastError();
}

static cudaError_t encode_digits_map(CUtensorMap* map, const int8_t* D, int64_t plane_rows,
                                     uint32_t box_rows) {
  return encode_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D,
                        (int64_t)kSplitDigits * plane_rows, kSplitK, kSplitK, kSBK, box_rows,
                        CU_TENSOR_MAP_SWIZZLE_64B);
}

cudaError_t launch_split_gemm(double* C, int64_t ldc, int M, int N, const SplitOperand& A,
                              int a_row0, const SplitOperand& B, int b_row0, double alpha,
                              int lower, WsHeader* hdr, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  CUtensorMap ma, mb;
  cudaError_t e = encode_digits_map(&ma, A.digits, A.plane_rows, kSBM);
  if (e != cudaSuccess) return e;
  if ((e = encode_digits_map(&mb, B.digits, B.plane_rows, kSBN)) != cudaSuccess) return e;
  SplitArgs g{};
  g.C = C; g.ldc = ldc; g.M = M; g.N = N; g.nk = kSplitK / kSBK;
  g.planeA = (int)A.plane_rows; g.planeB = (int)B.plane_rows; g.a0 = a_row0; g.b0 = b_row0;
  g.ea = A.ex; g.eb = B.ex; g.alpha = alpha; g.lower = lower; g.hdr = hdr;
  const int mt = (M + kSBM - 1) / kSBM;
  g.ntn = (N + kSBN - 1) / kSBN;
  if (lower) {
    const int rs = (g.ntn - 1) / 2;
    g.tiles = mt <= rs ? mt * (mt + 1) : rs * (rs + 1) + (mt - rs) * g.ntn;
  } else {
    g.tiles = mt * g.ntn;
  }
  // whole waves over the SMs (the nearest count of waves of kSTilesPerCta tiles, at least one),
  // the tiles split evenly: no short last wave, and a small product spreads over every SM
  int dev = 0, sms = 148;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const int per_wave = sms * kSTilesPerCta;
  const int waves = std::max(1, (g.tiles + per_wave / 2) / per_wave);
  g.ctas = std::min(g.tiles, sms * waves);
  split_gemm_kernel<<<(unsigned)g.ctas, kSThreads, kSSmem, s>>>(ma, mb, g);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
