// Canonical Huffman coding of integer codes on the device.
//
// Sources: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane Algorithm",
// section 3 (HPTQ: normal and outlier weights share one unconstrained integer grid, and the
// integers are Huffman-coded so that the bit width follows the weight distribution);
// "WaterSIC", section 2 (the ZSIC integers are entropy-coded instead of clipped to a range).
//
// One stream of kernels:
//   range      min / max code (atomics);
//   histogram  counts of the spanned values (at most kHuffMaxSym; per-CTA shared-memory bins,
//              the lanes of a warp holding the same value adding with one atomic);
//   build      one CTA: the used symbols sorted by (count, symbol) with a bitonic sort, the
//              two-queue Huffman merge (ties take the leaf), depths from the root down, then the
//              canonical codewords (consecutive within a length, shifted left at each new
//              length) and the total length;
//   tile sums  the code lengths of each 4096-code tile;
//   scan       exclusive scan of the tile sums (one CTA);
//   zero       the stream words that will receive bits (the total is known now);
//   encode     each CTA scans its tile's lengths in shared memory; each thread assembles its
//              codewords word by word in a register and ORs the words into the stream, MSB
//              first in 64-bit words (stream bit i = bit 63 - i % 64 of word i / 64; a
//              codeword may straddle two words).
// Device-detected failures (more than kHuffMaxSym values spanned, a codeword longer than 63
// bits, a stream too small for the total) are recorded in the workspace status and skip the
// encoding.
#include "gq_internal.cuh"

#include <limits.h>

#include <algorithm>

namespace gq {

constexpr int kHuffMaxSym = 4096;
constexpr int kHuffTile = 4096;     // codes per tile
constexpr int kHuffThreads = 256;   // tile kernels: 16 codes per thread
constexpr int kHuffPer = kHuffTile / kHuffThreads;
constexpr size_t kHuffBuildSmem = (size_t)kHuffMaxSym * 8          // keys, then codewords
                                  + (size_t)2 * kHuffMaxSym * 8      // node weights
                                  + (size_t)2 * kHuffMaxSym * 4      // parents
                                  + (size_t)2 * kHuffMaxSym          // depths
                                  + (size_t)kHuffMaxSym;             // lengths

struct HuffLayout {
  WsHeader* hdr;
  int* state;                       // [0] min code, [1] max code, [2] skip flag
  unsigned long long* hist;         // kHuffMaxSym
  unsigned long long* tile_sum;     // ntiles
  unsigned long long* tile_off;     // ntiles
  size_t bytes;
};

static HuffLayout huff_layout(void* ws, int64_t count) {
  const int64_t ntiles = (count + kHuffTile - 1) / kHuffTile;
  Carver c(ws);
  HuffLayout L;
  L.hdr = c.take<WsHeader>(1);
  L.state = c.take<int>(4);
  L.hist = c.take<unsigned long long>(kHuffMaxSym);
  L.tile_sum = c.take<unsigned long long>((size_t)ntiles);
  L.tile_off = c.take<unsigned long long>((size_t)ntiles);
  L.bytes = c.off;
  return L;
}

size_t huffman_ws_bytes(int64_t count) { return huff_layout(nullptr, count).bytes; }

__global__ void huff_init_kernel(int* state, unsigned long long* hist) {
  for (int i = threadIdx.x; i < kHuffMaxSym; i += blockDim.x) hist[i] = 0ull;
  if (threadIdx.x == 0) { state[0] = INT_MAX; state[1] = INT_MIN; state[2] = 0; }
}

__global__ void huff_range_kernel(const int* codes, int64_t count, int* state) {
  int lo = INT_MAX, hi = INT_MIN;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int v = codes[e];
    lo = min(lo, v);
    hi = max(hi, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&state[0], lo);
    atomicMax(&state[1], hi);
  }
}

constexpr int kHistThreads = 128;
constexpr int kPrivSym = 64;  // spans up to this many values count in lane-private counters
static_assert((kHistThreads / 32) * kPrivSym * 32 * 4 <= kHuffMaxSym * 8, "counters fit the bins");
__global__ void __launch_bounds__(kHistThreads) huff_hist_kernel(const int* codes, int64_t count,
                                                                 const int* state,
                                                                 unsigned long long* hist) {
  __shared__ unsigned long long bins[kHuffMaxSym];
  const int lo = state[0];
  const long long K = (long long)state[1] - lo + 1;
  if (K > kHuffMaxSym) return;  // the same for every CTA; the build kernel reports it
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (K <= kPrivSym) {
    // few values (low-bit codes): every lane counts into its own column of its warp's
    // counters, [warp][symbol][lane] (consecutive lanes in consecutive banks), no atomics
    unsigned* priv = reinterpret_cast<unsigned*>(bins);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < (kHistThreads / 32) * kPrivSym * 32; i += blockDim.x) priv[i] = 0u;
    __syncthreads();
    unsigned* mine = priv + (size_t)warp * kPrivSym * 32 + lane;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count; e += stride)
      mine[(codes[e] - lo) * 32] += 1u;
    __syncthreads();
    if (threadIdx.x < K) {
      unsigned long long c = 0ull;
      for (int w = 0; w < kHistThreads / 32; ++w)
        for (int l = 0; l < 32; ++l) c += priv[((size_t)w * kPrivSym + threadIdx.x) * 32 + l];
      if (c) atomicAdd(&hist[threadIdx.x], c);
    }
    return;
  }
  for (int i = threadIdx.x; i < K; i += blockDim.x) bins[i] = 0ull;
  __syncthreads();
  // the lanes of a warp that hold the same symbol add their count with one atomic
  const int64_t e_end = (count + stride - 1) / stride * stride;  // every lane runs each round
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < e_end; e += stride) {
    const int sym = e < count ? codes[e] - lo : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, sym);
    if (sym >= 0 && (threadIdx.x & 31) == __ffs(peers) - 1)
      atomicAdd(&bins[sym], (unsigned long long)__popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x)
    if (bins[i]) atomicAdd(&hist[i], bins[i]);
}

__global__ void __launch_bounds__(1024) huff_build_kernel(int* state,
                                                          const unsigned long long* hist,
                                                          int64_t stream_words,
                                                          uint8_t* lengths_out,
                                                          unsigned long long* words_out,
                                                          long long* info, WsHeader* hdr) {
  extern __shared__ __align__(16) unsigned long long hb[];
  unsigned long long* keys = hb;                                   // then the codewords
  unsigned long long* wt = keys + kHuffMaxSym;                     // 2 K node weights
  int* parent = reinterpret_cast<int*>(wt + 2 * kHuffMaxSym);      // 2 K
  uint8_t* depth = reinterpret_cast<uint8_t*>(parent + 2 * kHuffMaxSym);  // 2 K
  uint8_t* lens = depth + 2 * kHuffMaxSym;                         // K
  __shared__ int s_nz, s_bad, s_maxlen;
  __shared__ unsigned long long s_total;
  const int tid = threadIdx.x;
  const int lo = state[0];
  const long long K = (long long)state[1] - lo + 1;
  if (tid == 0) { s_nz = 0; s_bad = 0; s_maxlen = 0; s_total = 0ull; }
  for (int i = tid; i < kHuffMaxSym; i += blockDim.x) lengths_out[i] = 0;
  for (int i = tid; i < kHuffMaxSym; i += blockDim.x) words_out[i] = 0ull;
  if (K > kHuffMaxSym) {
    if (tid == 0) {
      record_status(hdr, GQ_ERR_UNSUPPORTED);
      state[2] = 1;
      info[0] = lo; info[1] = K; info[2] = -1; info[3] = 0;
    }
    return;
  }
  __syncthreads();
  // used symbols as (count << 12 | symbol); unused sort last.  Only the spanned symbols are
  // sorted: the next power of two at or above K.
  int KP = 2;
  while (KP < K) KP <<= 1;
  for (int i = tid; i < KP; i += blockDim.x) {
    const unsigned long long c = i < K ? hist[i] : 0ull;
    keys[i] = c ? ((c << 12) | (unsigned long long)i) : ~0ull;
    if (c) atomicAdd(&s_nz, 1);
    lens[i] = 0;
  }
  __syncthreads();
  for (int k = 2; k <= KP; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < KP; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          if ((a > b) == ((i & k) == 0)) { keys[i] = b; keys[ixj] = a; }
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    const int nz = s_nz;
    if (nz == 1) {
      lens[keys[0] & 4095ull] = 1;
    } else {
      for (int i = 0; i < nz; ++i) wt[i] = keys[i] >> 12;
      int q1 = 0, q2 = nz, next = nz;
      for (int m = 0; m < nz - 1; ++m) {
        const int a = (q1 < nz && (q2 >= next || wt[q1] <= wt[q2])) ? q1++ : q2++;
        const int b = (q1 < nz && (q2 >= next || wt[q1] <= wt[q2])) ? q1++ : q2++;
        wt[next] = wt[a] + wt[b];
        parent[a] = next;
        parent[b] = next;
        ++next;
      }
      depth[2 * nz - 2] = 0;
      for (int i = 2 * nz - 3; i >= 0; --i) {  // parents carry larger ids than their children
        const int d = depth[parent[i]] + 1;
        if (d > 63) s_bad = 1;
        depth[i] = (uint8_t)(d > 63 ? 63 : d);
      }
      for (int i = 0; i < nz; ++i) lens[keys[i] & 4095ull] = depth[i];
    }
    // canonical codewords: consecutive within a length, shifted left at each new length
    int bl_count[64] = {};
    int maxlen = 0;
    for (int sym = 0; sym < K; ++sym) {
      const int ln = lens[sym];
      if (ln) { ++bl_count[ln]; maxlen = ln > maxlen ? ln : maxlen; }
    }
    unsigned long long next_code[64];
    unsigned long long code = 0ull;
    for (int ln = 1; ln <= maxlen; ++ln) {
      code = (code + (unsigned long long)bl_count[ln - 1]) << 1;
      next_code[ln] = code;
    }
    for (int sym = 0; sym < K; ++sym) {
      const int ln = lens[sym];
      keys[sym] = ln ? next_code[ln]++ : 0ull;
    }
    s_maxlen = maxlen;
  }
  __syncthreads();
  for (int i = tid; i < K; i += blockDim.x)
    if (lens[i]) atomicAdd(&s_total, hist[i] * (unsigned long long)lens[i]);
  __syncthreads();
  if (tid == 0) {
    const unsigned long long total = s_total;
    const bool fits = total <= 64ull * (unsigned long long)stream_words;
    if (s_bad) record_status(hdr, GQ_ERR_UNSUPPORTED);
    else if (!fits) record_status(hdr, GQ_ERR_WORKSPACE);
    state[2] = (s_bad || !fits) ? 1 : 0;
    info[0] = lo; info[1] = K; info[2] = (long long)total; info[3] = s_maxlen;
  }
  for (int i = tid; i < K; i += blockDim.x) {
    lengths_out[i] = lens[i];
    words_out[i] = keys[i];
  }
}

// Exclusive scan of one value per thread over the block (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v,
                                                                   unsigned long long* warp_sums,
                                                                   unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < nw ? warp_sums[lane] : 0ull;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) warp_sums[lane] = w;  // inclusive totals of the warps
  }
  __syncthreads();
  const unsigned long long before = warp ? warp_sums[warp - 1] : 0ull;
  if (total) *total = warp_sums[nw - 1];
  return before + x - v;
}

__global__ void __launch_bounds__(kHuffThreads) huff_tile_sum_kernel(const int* codes,
                                                                     int64_t count,
                                                                     const int* state,
                                                                     const uint8_t* lengths,
                                                                     unsigned long long* tile_sum) {
  __shared__ uint8_t sl[kHuffMaxSym];
  __shared__ unsigned long long red[kHuffThreads / 32];
  if (state[2]) return;
  const int lo = state[0];
  const int K = state[1] - lo + 1;  // <= kHuffMaxSym once the build has passed
  for (int i = threadIdx.x; i < K; i += blockDim.x) sl[i] = lengths[i];
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * kHuffTile;
  unsigned long long acc = 0ull;
  for (int i = threadIdx.x; i < kHuffTile; i += blockDim.x) {
    const int64_t e = t0 + i;
    if (e < count) acc += sl[codes[e] - lo];
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long s = 0ull;
    for (int w = 0; w < kHuffThreads / 32; ++w) s += red[w];
    tile_sum[blockIdx.x] = s;
  }
}

__global__ void __launch_bounds__(1024) huff_scan_kernel(const int* state,
                                                         const unsigned long long* tile_sum,
                                                         int64_t ntiles,
                                                         unsigned long long* tile_off) {
  __shared__ unsigned long long ws[32];
  if (state[2]) return;
  const int64_t per = (ntiles + blockDim.x - 1) / blockDim.x;
  const int64_t a = threadIdx.x * per;
  const int64_t b = a + per < ntiles ? a + per : ntiles;
  unsigned long long mine = 0ull;
  for (int64_t i = a; i < b; ++i) mine += tile_sum[i];
  unsigned long long run = block_exclusive_scan(mine, ws, nullptr);
  for (int64_t i = a; i < b; ++i) {
    tile_off[i] = run;
    run += tile_sum[i];
  }
}

__global__ void __launch_bounds__(kHuffThreads) huff_encode_kernel(
    const int* codes, int64_t count, const int* state, const uint8_t* lengths,
    const unsigned long long* words, const unsigned long long* tile_off,
    unsigned long long* stream) {
  __shared__ uint8_t sl[kHuffMaxSym];
  __shared__ unsigned long long sw[kHuffMaxSym];
  __shared__ unsigned long long wsum[kHuffThreads / 32];
  if (state[2]) return;
  const int lo = state[0];
  const int K = state[1] - lo + 1;  // <= kHuffMaxSym once the build has passed
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    sl[i] = lengths[i];
    sw[i] = words[i];
  }
  __syncthreads();
  const int64_t e0 = (int64_t)blockIdx.x * kHuffTile + (int64_t)threadIdx.x * kHuffPer;
  int sym[kHuffPer];
  unsigned long long mine = 0ull;
#pragma unroll
  for (int i = 0; i < kHuffPer; ++i) {
    sym[i] = (e0 + i < count) ? codes[e0 + i] - lo : -1;
    if (sym[i] >= 0) mine += sl[sym[i]];
  }
  unsigned long long pos = tile_off[blockIdx.x] + block_exclusive_scan(mine, wsum, nullptr);
  // this thread's codewords are assembled word by word in a register; a word is ORed into the
  // stream when the bits move on (its first and last words may be shared with the neighbours,
  // hence the atomics; the count drops from one per code to about one per word)
  unsigned long long buf = 0ull, bw = pos >> 6;
#pragma unroll
  for (int i = 0; i < kHuffPer; ++i) {
    if (sym[i] < 0) continue;
    const int ln = sl[sym[i]];
    const unsigned long long cw = sw[sym[i]];
    if ((pos >> 6) != bw) {
      if (buf) atomicOr(&stream[bw], buf);
      bw = pos >> 6;
      buf = 0ull;
    }
    const int o = (int)(pos & 63ull);
    if (o + ln <= 64) {
      buf |= cw << (64 - o - ln);
    } else {
      const int h = o + ln - 64;  // bits that spill into the next word
      buf |= cw >> h;
      atomicOr(&stream[bw], buf);
      ++bw;
      buf = cw << (64 - h);
    }
    pos += (unsigned long long)ln;
  }
  if (buf) atomicOr(&stream[bw], buf);
}

// Zero the stream words that will receive bits (the total is known once the code is built).
__global__ void huff_zero_kernel(const int* state, const long long* info, int64_t nwords,
                                 unsigned long long* stream) {
  if (state[2]) return;
  const long long total = info[2];
  int64_t used = (total + 63) / 64;
  if (used > nwords) used = nwords;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < used;
       w += (int64_t)gridDim.x * blockDim.x)
    stream[w] = 0ull;
}

cudaError_t huffman_init_attributes() {
  return cudaFuncSetAttribute(huff_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)kHuffBuildSmem);
}

cudaError_t launch_huffman(const int* codes, int64_t count, unsigned long long* stream_words,
                           int64_t nwords, uint8_t* lengths, unsigned long long* words,
                           long long* info, void* ws, cudaStream_t s) {
  HuffLayout L = huff_layout(ws, count);
  const int64_t ntiles = (count + kHuffTile - 1) / kHuffTile;
  cudaError_t e;
  if ((e = cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s))) return e;
  huff_init_kernel<<<1, 1024, 0, s>>>(L.state, L.hist);
  const unsigned grid = (unsigned)std::min<int64_t>((count + 255) / 256, 148 * 8);
  const unsigned hgrid = (unsigned)std::min<int64_t>((count + kHistThreads - 1) / kHistThreads,
                                                     148 * 16);
  huff_range_kernel<<<grid, 256, 0, s>>>(codes, count, L.state);
  huff_hist_kernel<<<hgrid, kHistThreads, 0, s>>>(codes, count, L.state, L.hist);
  huff_build_kernel<<<1, 1024, kHuffBuildSmem, s>>>(L.state, L.hist, nwords, lengths, words,
                                                    info, L.hdr);
  huff_tile_sum_kernel<<<(unsigned)ntiles, kHuffThreads, 0, s>>>(codes, count, L.state, lengths,
                                                                 L.tile_sum);
  huff_scan_kernel<<<1, 1024, 0, s>>>(L.state, L.tile_sum, ntiles, L.tile_off);
  huff_zero_kernel<<<(unsigned)std::min<int64_t>((nwords + 255) / 256, 148 * 8), 256, 0, s>>>(
      L.state, info, nwords, stream_words);
  huff_encode_kernel<<<(unsigned)ntiles, kHuffThreads, 0, s>>>(codes, count, L.state, lengths,
                                                               words, L.tile_off, stream_words);
  count_launches(8);
  return cudaGetLastError();
}

// The code's statistics alone (range, histogram, build): info[2] = the total bits of the
// Huffman-coded stream, lengths / words the canonical code.  Nothing is encoded.
cudaError_t launch_huffman_stats(const int* codes, int64_t count, uint8_t* lengths,
                                 unsigned long long* words, long long* info, void* ws,
                                 cudaStream_t s) {
  HuffLayout L = huff_layout(ws, count);
  cudaError_t e;
  if ((e = cudaMemsetAsync(L.hdr, 0, sizeof(WsHeader), s))) return e;
  huff_init_kernel<<<1, 1024, 0, s>>>(L.state, L.hist);
  const unsigned grid = (unsigned)std::min<int64_t>((count + 255) / 256, 148 * 8);
  const unsigned hgrid = (unsigned)std::min<int64_t>((count + kHistThreads - 1) / kHistThreads,
                                                     148 * 16);
  huff_range_kernel<<<grid, 256, 0, s>>>(codes, count, L.state);
  huff_hist_kernel<<<hgrid, kHistThreads, 0, s>>>(codes, count, L.state, L.hist);
  // a stream capacity no total reaches (2^63 bits): only the code's own limits are reported
  huff_build_kernel<<<1, 1024, kHuffBuildSmem, s>>>(L.state, L.hist, (int64_t)1 << 57, lengths,
                                                    words, info, L.hdr);
  count_launches(4);
  return cudaGetLastError();
}

}  // namespace gq
