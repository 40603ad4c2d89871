// Device-wide building blocks used by the backward: an exclusive scan with
// functor input/output, a stable LSD radix sort of (key, payload) int32 pairs and
// the segment table of a sorted key array.  No inter-CTA waiting anywhere: every
// step is a separate launch (reduce, scan of block sums, apply).
#pragma once

#include "pkm_internal.cuh"

namespace pkm {
namespace sort {

constexpr int kScanTPB = 512, kScanItems = 8, kScanTile = kScanTPB * kScanItems;
// Radix tiles of 4096 keys and digits of at most 10 bits: each pass reorders its tile in
// shared memory before writing, so the writes leave in runs of the tile's keys per digit
// instead of one scattered word per key.
constexpr int kRadixTile = 4096, kRadixWarps = 8, kRadixMaxBits = 10;

// --------------------------------------------------------------- scan
template <class In>
__global__ void __launch_bounds__(kScanTPB) scan_reduce(In in, int64_t n, int* bsum) {
  const int64_t base = (int64_t)blockIdx.x * kScanTile;
  int s = 0;
  for (int i = threadIdx.x; i < kScanTile; i += kScanTPB) {
    int64_t g = base + i;
    if (g < n) s += in(g);
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ int ws[kScanTPB / 32];
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    int v = threadIdx.x < kScanTPB / 32 ? ws[threadIdx.x] : 0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) bsum[blockIdx.x] = v;
  }
}

// exclusive scan of bsum[0..nb) in place, one CTA of 1024 threads, any nb
__global__ void __launch_bounds__(1024) scan_block_sums(int* bsum, int nb);

// Block-wide exclusive scan of one value per thread; returns the block total too.
__device__ __forceinline__ int block_excl_scan(int v, int* total) {
  __shared__ int wsum[32];
  __shared__ int wtot;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int inc = v;
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int nw = blockDim.x >> 5;
    int x = lane < nw ? wsum[lane] : 0;
    int xi = x;
    for (int o = 1; o < 32; o <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < nw) wsum[lane] = xi - x;
    if (lane == nw - 1) wtot = xi;
  }
  __syncthreads();
  int r = inc - v + wsum[wid];
  *total = wtot;
  __syncthreads();
  return r;
}

template <class In, class Out>
__global__ void __launch_bounds__(kScanTPB) scan_apply(In in, Out out, int64_t n, const int* bsum) {
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanItems;
  int v[kScanItems];
  int s = 0;
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    int64_t g = base + j;
    v[j] = g < n ? in(g) : 0;
    s += v[j];
  }
  int total;
  int run = block_excl_scan(s, &total) + bsum[blockIdx.x];
#pragma unroll
  for (int j = 0; j < kScanItems; ++j) {
    int64_t g = base + j;
    if (g < n) out(g, run, v[j], n);
    run += v[j];
  }
}

template <class In, class Out>
cudaError_t exclusive_scan(In in, Out out, int64_t n, int* bsum, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int nb = (int)((n + kScanTile - 1) / kScanTile);
  scan_reduce<<<nb, kScanTPB, 0, st>>>(in, n, bsum); PKM_COUNT(1);
  scan_block_sums<<<1, 1024, 0, st>>>(bsum, nb); PKM_COUNT(1);
  scan_apply<<<nb, kScanTPB, 0, st>>>(in, out, n, bsum); PKM_COUNT(1);
  return cudaGetLastError();
}

inline int64_t scan_bsum_len(int64_t n) { return (n + kScanTile - 1) / kScanTile + 1; }

// --------------------------------------------------------------- radix sort
struct RadixBuffers {
  int32_t *keysA, *valsA, *keysB, *valsB;
  int* hist;   // >= (1 << kRadixMaxBits) * tiles
  int* bsum;   // >= scan_bsum_len(hist length)
};

inline int64_t radix_tiles(int64_t n) { return (n + kRadixTile - 1) / kRadixTile; }
inline int64_t radix_hist_len(int64_t n) { return (int64_t)(1 << kRadixMaxBits) * radix_tiles(n); }

// Sorts n pairs by key in [0, 2^bits_total) stably.  The first pass reads
// (keys_src, payload = position); later passes ping-pong between A and B.
// Returns the buffers holding the result.  When w_src is given, a float per key rides
// along (w_src[i] with key i) and ends in w_dst; w_tmp (n floats) holds it between passes.
cudaError_t radix_sort(const int32_t* keys_src, int64_t n, int bits_total, const RadixBuffers& b,
                       const int32_t** keys_out, const int32_t** vals_out, cudaStream_t st,
                       const float* w_src = nullptr, float* w_tmp = nullptr,
                       float* w_dst = nullptr);

// Where radix_sort(bits_total) leaves the sorted payloads (*vals_out of that call).
inline const int32_t* radix_sorted_vals(const RadixBuffers& b, int bits_total) {
  if (bits_total < 1) bits_total = 1;
  const int passes = (bits_total + kRadixMaxBits - 1) / kRadixMaxBits;
  return (passes & 1) ? b.valsA : b.valsB;
}

// Segment table of a sorted key array: seg[u] = first position of the u-th
// distinct key, seg[U] = n, *U_out = U, and (when seg_key is not null)
// seg_key[u] = that key.
// When gather_src is not null, gather_dst[i] = gather_src[vals[i]] for every position.
cudaError_t segments(const int32_t* keys, int64_t n, int* seg, int* U_out, int* bsum,
                     cudaStream_t st, int32_t* seg_key = nullptr, const int32_t* vals = nullptr,
                     const float* gather_src = nullptr, float* gather_dst = nullptr);

}  // namespace sort
}  // namespace pkm
