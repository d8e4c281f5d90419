// Lazy block update on the tensor cores: W[:, j1:jend] -= E[:, k0:k0+K] U[k0:k0+K, j1:jend] in
// fp32 accuracy.
//
// GPTQ defers the trailing update of the columns after a 128-column block to one rank-128 GEMM
// (the lazy batch); here it runs as tcgen05.mma kind::tf32 with the 3xTF32 split: each fp32
// operand is carried as hi + lo (hi = tf32 rounding, lo = the fp32 remainder), and
// acc += A_hi B_hi + A_hi B_lo + A_lo B_hi, accumulated in fp32 in tensor memory.  The column
// loop writes E as E_hi / E_lo; U is split once per quantize call.
//
// CTA tile 128 (rows) x 128 (columns), K (a block of 128, or a super-block of 1024) in slices of
// 16 (3-deep ring, 32 KB a stage), operands by TMA (no multicast).  Each 256-deep part of K
// accumulates in its own 128-column TMEM accumulator (up to four), and the epilogue adds them in
// fp64: no fp32 accumulation chain is longer than 256 (the codes of ill-conditioned layers
// notice longer ones). A = E columns k0.. (K-major, rows of 16 fp32 =
// 64 B, 64-byte swizzle), B = U rows k0.. (MN-major, 4 runs of 32 columns, 128-byte swizzle
// with 32-byte chunks: the layout the tensor cores require for 32-bit MN-major operands).  Warp 0 lane 0 issues the loads, warp 1
// lane 0 the MMAs; all eight warps read the accumulator (warps w and w + 4 share TMEM lanes
// 32 (w % 4) ..; they take the left and right 64 columns) and subtract it from the fp32 work
// matrix, with their work-matrix loads issued before the accumulator is ready.
#include "gq_internal.cuh"
#include "gq_tc.cuh"

#include <cudaTypedefs.h>
#include <mutex>

namespace gq {

namespace {
constexpr int kLBK = 16;                                  // K per stage
constexpr int kLStages = 3;
constexpr int kLThreads = 256;
constexpr uint32_t kLTile = 128 * kLBK * 4;               // 8 KB per operand tile
constexpr uint32_t kLRun = 32 * kLBK * 4;                 // one 32-column run of a B tile
constexpr uint32_t kLStage = 4 * kLTile;                  // A_hi, A_lo, B_hi, B_lo
constexpr size_t kLSmem = kLStages * kLStage + 1024 + 256;
constexpr uint32_t kLIdesc = tc::idesc_f32acc(2, 2, 0, 1, 128, 128);  // tf32, A K-major, B MN-major
constexpr int kLAccSlices = 16;   // slices of kLBK per TMEM accumulator (depth 256)
constexpr int kLMaxAcc = 4;       // accumulators (512 TMEM columns): K up to 1024 in full parts
}  // namespace

// kDeep = false: K <= 256, one accumulator (128 TMEM columns), two CTAs an SM, the work
// matrix's tile loaded before the accumulator is ready.  kDeep = true: K up to 1024 in up to
// four accumulators (512 columns), one CTA an SM, the tile loaded after.
template <bool kDeep>
__global__ void __launch_bounds__(kLThreads, kDeep ? 1 : 2)
    lazy_tc_kernel(const __grid_constant__ CUtensorMap m_ahi, const __grid_constant__ CUtensorMap m_alo,
                   const __grid_constant__ CUtensorMap m_bhi, const __grid_constant__ CUtensorMap m_blo,
                   float* Wf, int64_t n, int64_t k_rows, int k0, int nk, int j1,
                   WsHeader* hdr) {
  extern __shared__ uint8_t lz_smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(lz_smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kLStages * kLStage);
  uint64_t* empty = full + kLStages;
  uint64_t* accum = empty + kLStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accum + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile_n = blockIdx.x, tile_m = blockIdx.y;

  if (tid == 0) {
    for (int s = 0; s < kLStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    tc::mbar_init(accum, 1);
    tc::fence_barrier_init();
    tc::prefetch_tmap(&m_ahi); tc::prefetch_tmap(&m_alo);
    tc::prefetch_tmap(&m_bhi); tc::prefetch_tmap(&m_blo);
  }
  constexpr uint32_t kCols = kDeep ? 128 * kLMaxAcc : 128;
  if (warp == 1) tc::tmem_alloc(tslot, kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  const int NK = nk;  // slices of kLBK
  const int nacc = kDeep ? min(kLMaxAcc, (NK + kLAccSlices - 1) / kLAccSlices) : 1;

  const int64_t row = (int64_t)tile_m * 128 + (warp & 3) * 32 + lane;
  const int64_t colt = (int64_t)j1 + tile_n * 128;  // first column of this tile
  const int chalf = (warp >> 2) * 64;                // this warp's 64 columns of the tile
  float* wrow = Wf + row * n + colt + chalf;
  const bool vec = ((reinterpret_cast<uintptr_t>(Wf) & 15) == 0) && (n % 4 == 0);
  if (warp == 0 && lane == 0) {
    // producer
    for (int kc = 0; kc < NK; ++kc) {
      const int s = kc % kLStages;
      if (kc >= kLStages && !tc::mbar_wait(&empty[s], ((kc / kLStages) - 1) & 1)) {
        record_status(hdr, GQ_ERR_TIMEOUT);
        break;
      }
      uint8_t* st = base + s * kLStage;
      tc::mbar_arrive_expect_tx(&full[s], kLStage);
      tc::tma_load_2d(st, &m_ahi, &full[s], k0 + kc * kLBK, tile_m * 128);
      tc::tma_load_2d(st + kLTile, &m_alo, &full[s], k0 + kc * kLBK, tile_m * 128);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int x = j1 + tile_n * 128 + g * 32, y = k0 + kc * kLBK;
        tc::tma_load_2d(st + 2 * kLTile + g * kLRun, &m_bhi, &full[s], x, y);
        tc::tma_load_2d(st + 3 * kLTile + g * kLRun, &m_blo, &full[s], x, y);
      }
    }
    // the epilogue's read-modify-write tile: into L2 while the MMAs run
    if (vec && colt + 128 <= n) {
      const int64_t r0 = (int64_t)tile_m * 128;
      const int rows = (int)min((int64_t)128, k_rows - r0);
      for (int r = 0; r < rows; ++r) tc::bulk_prefetch_l2(Wf + (r0 + r) * n + colt, 512);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    for (int kc = 0; kc < NK; ++kc) {
      const int s = kc % kLStages;
      if (!tc::mbar_wait(&full[s], (kc / kLStages) & 1)) {
        record_status(hdr, GQ_ERR_TIMEOUT);
        break;
      }
      tc::fence_after_sync();
      const uint32_t a_hi = tc::smem_u32(base + s * kLStage);
      const uint32_t a_lo = a_hi + kLTile, b_hi = a_hi + 2 * kLTile, b_lo = a_hi + 3 * kLTile;
      const int acc_i = kDeep ? min(kc / kLAccSlices, kLMaxAcc - 1) : 0;
      const bool first = kc == acc_i * kLAccSlices;  // the accumulator's first slice
      const uint32_t tacc = tmem + acc_i * 128;
#pragma unroll
      for (int k = 0; k < kLBK / 8; ++k) {
        const uint64_t dah = tc::sdesc(a_hi + k * 32, 16, 512, tc::kLayoutSW64);
        const uint64_t dal = tc::sdesc(a_lo + k * 32, 16, 512, tc::kLayoutSW64);
        const uint64_t dbh = tc::sdesc(b_hi + k * 1024, kLRun, 512, tc::kLayoutSW128Base32B);
        const uint64_t dbl = tc::sdesc(b_lo + k * 1024, kLRun, 512, tc::kLayoutSW128Base32B);
        tc::mma_tf32(tacc, dah, dbh, kLIdesc, !(first && k == 0));
        tc::mma_tf32(tacc, dah, dbl, kLIdesc, 1);
        tc::mma_tf32(tacc, dal, dbh, kLIdesc, 1);
      }
      tc::mma_commit(&empty[s]);
    }
    tc::mma_commit(accum);
  }
  __syncwarp();

  // Epilogue: TMEM lane = tile row; this warp's two chunks of 32 columns.  Both chunks of the
  // work matrix are loaded before the accumulator is waited for, so the load latency overlaps
  // the MMAs (and the other CTA on the SM).
  const bool full_row = row < k_rows && colt + 128 <= n && vec;
  float4 wv[2][8];
  if (!kDeep && full_row) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[c][i] = *reinterpret_cast<const float4*>(wrow + c * 32 + 4 * i);
  }
  bool ok = tc::mbar_wait(accum, 0);
  if (!ok && lane == 0) record_status(hdr, GQ_ERR_TIMEOUT);
  tc::fence_after_sync();
  if (ok) {
    if constexpr (!kDeep) {  // one accumulator: subtract it from the preloaded tile
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        tc::tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + chalf + cc * 32, v);
        const int64_t col0 = colt + chalf + cc * 32;
        if (full_row) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 w = wv[cc][i];
            w.x -= v[4 * i]; w.y -= v[4 * i + 1]; w.z -= v[4 * i + 2]; w.w -= v[4 * i + 3];
            *reinterpret_cast<float4*>(wrow + cc * 32 + 4 * i) = w;
          }
        } else if (row < k_rows && col0 < n) {
          float* dst = Wf + row * n + col0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < n) dst[i] -= v[i];
        }
      }
    } else {  // the accumulators added in fp64, one fp32 rounding into the work matrix
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        // this chunk of the work matrix is loaded first, so the loads overlap the reads of the
        // accumulators and their fp64 sum
        float4 wc[8];
        if (full_row) {
#pragma unroll
          for (int i = 0; i < 8; ++i) wc[i] = *reinterpret_cast<const float4*>(wrow + cc * 32 + 4 * i);
        }
        double u[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = 0.0;
        for (int ai = 0; ai < nacc; ++ai) {
          float v[32];
          tc::tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + ai * 128 + chalf + cc * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] += (double)v[i];
        }
        const int64_t col0 = colt + chalf + cc * 32;
        if (full_row) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w0 = wc[i];
            float4 w;
            w.x = (float)((double)w0.x - u[4 * i]);
            w.y = (float)((double)w0.y - u[4 * i + 1]);
            w.z = (float)((double)w0.z - u[4 * i + 2]);
            w.w = (float)((double)w0.w - u[4 * i + 3]);
            *reinterpret_cast<float4*>(wrow + cc * 32 + 4 * i) = w;
          }
        } else if (row < k_rows && col0 < n) {
          float* dst = Wf + row * n + col0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < n) dst[i] = (float)((double)dst[i] - u[i]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, kCols);
}

// ---- host side ----
namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

cudaError_t get_encode() {
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (g_encode) return cudaSuccess;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// fp32 row-major matrix (rows x cols, leading dimension ld elements) as a 2-D tensor map with a
// box of 32 columns x box_rows rows, zero fill outside; swizzle as the operand's layout needs.
cudaError_t encode_f32(CUtensorMap* map, const float* p, int64_t rows, int64_t cols, int64_t ld,
                       uint32_t box_rows, CUtensorMapSwizzle swz) {
  return encode_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sizeof(float), p, rows, cols, ld,
                        32, box_rows, swz);
}
}  // namespace

cudaError_t encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, size_t elem_bytes,
                           const void* p, int64_t rows, int64_t cols, int64_t ld,
                           uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dt, 2, const_cast<void*>(p), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t lazy_tc_init_attributes() {
  cudaError_t e = cudaFuncSetAttribute(lazy_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLSmem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(lazy_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kLSmem);
}

cudaError_t lazy_tc_make_maps(LazyTcMaps* maps, const float* Ehi, const float* Elo, int64_t rows,
                              int64_t ldE, const float* Uhi, const float* Ulo, int64_t n,
                              int64_t ldu) {
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  const CUtensorMapSwizzle ka = CU_TENSOR_MAP_SWIZZLE_64B;             // K-major A, 64-byte rows
  const CUtensorMapSwizzle mb = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;    // MN-major 32-bit B
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if ((e = encode_tmap_2d(&maps->ahi, f32, 4, Ehi, rows, n, ldE, kLBK, 128, ka))) return e;
  if ((e = encode_tmap_2d(&maps->alo, f32, 4, Elo, rows, n, ldE, kLBK, 128, ka))) return e;
  if ((e = encode_f32(&maps->bhi, Uhi, n, n, ldu, kLBK, mb))) return e;
  return encode_f32(&maps->blo, Ulo, n, n, ldu, kLBK, mb);
}

cudaError_t launch_lazy_tc(const LazyTcMaps& maps, float* Wf, int64_t n, int64_t k_rows,
                           int64_t k0, int K, int64_t j1, int64_t jend, WsHeader* hdr,
                           cudaStream_t s) {
  if (jend > n) jend = n;
  if (j1 >= jend || k_rows <= 0 || K <= 0) return cudaSuccess;
  if (K % kLBK || k0 % kLBK || k0 + K > n) return cudaErrorInvalidValue;
  dim3 grid((unsigned)((jend - j1 + 127) / 128), (unsigned)((k_rows + 127) / 128));
  if (K <= kLAccSlices * kLBK)
    lazy_tc_kernel<false><<<grid, kLThreads, kLSmem, s>>>(maps.ahi, maps.alo, maps.bhi, maps.blo,
                                                          Wf, n, k_rows, (int)k0, K / kLBK,
                                                          (int)j1, hdr);
  else
    lazy_tc_kernel<true><<<grid, kLThreads, kLSmem, s>>>(maps.ahi, maps.alo, maps.bhi, maps.blo,
                                                         Wf, n, k_rows, (int)k0, K / kLBK,
                                                         (int)j1, hdr);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gq
