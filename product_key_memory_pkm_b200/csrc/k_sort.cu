// Stable LSD radix sort and segment table (see k_sort.cuh).
#include "k_sort.cuh"

namespace pkm {
namespace sort {

__global__ void __launch_bounds__(1024) scan_block_sums(int* bsum, int nb) {
  int carry = 0;
  for (int base = 0; base < nb; base += 1024) {
    int i = base + threadIdx.x;
    int v = i < nb ? bsum[i] : 0;
    int total;
    int ex = block_excl_scan(v, &total);
    if (i < nb) bsum[i] = ex + carry;
    carry += total;
  }
}

namespace {

__global__ void __launch_bounds__(256) radix_hist(const int32_t* __restrict__ keys, int64_t n,
                                                  int shift, int bins, int* __restrict__ hist,
                                                  int64_t ntiles) {
  __shared__ int h[1 << kRadixMaxBits];
  for (int d = threadIdx.x; d < bins; d += blockDim.x) h[d] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kRadixTile;
  const uint32_t mask = (uint32_t)bins - 1u;
  for (int i = threadIdx.x; i < kRadixTile; i += blockDim.x) {
    int64_t g = base + i;
    if (g < n) atomicAdd(&h[((uint32_t)keys[g] >> shift) & mask], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < bins; d += blockDim.x) hist[(int64_t)d * ntiles + blockIdx.x] = h[d];
}

// One CTA per tile of kRadixTile keys, kRadixWarps warps each owning a contiguous
// quarter.  Per-warp digit counts -> per-warp bases (tile base from the scanned
// histogram plus the counts of earlier warps) -> in-order scatter with
// __match_any_sync ranks.  Stable by construction.
__global__ void __launch_bounds__(kRadixWarps * 32) radix_scatter(
    const int32_t* __restrict__ kin, const int32_t* __restrict__ vin, int32_t* __restrict__ kout,
    int32_t* __restrict__ vout, int64_t n, int shift, int bins, const int* __restrict__ offs,
    int64_t ntiles) {
  extern __shared__ int cnt[];  // [kRadixWarps][bins]
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < kRadixWarps * bins; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  constexpr int kPerWarp = kRadixTile / kRadixWarps;
  const int64_t wbase = (int64_t)blockIdx.x * kRadixTile + (int64_t)wid * kPerWarp;
  const uint32_t mask = (uint32_t)bins - 1u;
  int* wc = cnt + wid * bins;
  for (int c = 0; c < kPerWarp; c += 32) {
    int64_t g = wbase + c + lane;
    if (g < n) atomicAdd(&wc[((uint32_t)kin[g] >> shift) & mask], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < bins; d += blockDim.x) {
    int run = offs[(int64_t)d * ntiles + blockIdx.x];
    for (int w = 0; w < kRadixWarps; ++w) {
      int c = cnt[w * bins + d];
      cnt[w * bins + d] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int c = 0; c < kPerWarp; c += 32) {
    int64_t g = wbase + c + lane;
    const bool valid = g < n;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    if (valid) {
      const int32_t key = kin[g];
      const int32_t val = vin ? vin[g] : (int32_t)g;
      const uint32_t d = ((uint32_t)key >> shift) & mask;
      const unsigned peers = __match_any_sync(vmask, d);
      const int pos = wc[d] + __popc(peers & lt);
      kout[pos] = key;
      vout[pos] = val;
      __syncwarp(vmask);
      if ((peers & lt) == 0) wc[d] += __popc(peers);
    }
    __syncwarp();
  }
}

struct HistIn {
  const int* h;
  __device__ int operator()(int64_t i) const { return h[i]; }
};
struct HistOut {
  int* h;
  __device__ void operator()(int64_t i, int excl, int, int64_t) const { h[i] = excl; }
};

struct FlagIn {
  const int32_t* k;
  __device__ int operator()(int64_t i) const { return (i == 0 || k[i] != k[i - 1]) ? 1 : 0; }
};
struct SegOut {
  int* seg;
  int* U;
  const int32_t* keys;
  int32_t* seg_key;
  const int32_t* vals;
  const float* gsrc;
  float* gdst;
  __device__ void operator()(int64_t i, int excl, int v, int64_t n) const {
    if (gdst) gdst[i] = gsrc[vals[i]];
    if (v) {
      seg[excl] = (int)i;
      if (seg_key) seg_key[excl] = keys[i];
    }
    if (i == n - 1) {
      seg[excl + v] = (int)n;
      *U = excl + v;
    }
  }
};

}  // namespace

cudaError_t radix_sort(const int32_t* keys_src, int64_t n, int bits_total, const RadixBuffers& b,
                       const int32_t** keys_out, const int32_t** vals_out, cudaStream_t st) {
  if (bits_total < 1) bits_total = 1;
  const int passes = (bits_total + kRadixMaxBits - 1) / kRadixMaxBits;
  const int bits = (bits_total + passes - 1) / passes;
  const int bins = 1 << bits;
  const int64_t ntiles = radix_tiles(n);
  const int32_t* kin = keys_src;
  const int32_t* vin = nullptr;
  int32_t* ko = b.keysA;
  int32_t* vo = b.valsA;
  const size_t smem = sizeof(int) * kRadixWarps * bins;
  cudaError_t e = cudaSuccess;
  for (int p = 0; p < passes; ++p) {
    const int shift = p * bits;
    radix_hist<<<(unsigned)ntiles, 256, 0, st>>>(kin, n, shift, bins, b.hist, ntiles); PKM_COUNT(1);
    e = exclusive_scan(HistIn{b.hist}, HistOut{b.hist}, (int64_t)bins * ntiles, b.bsum, st);
    if (e != cudaSuccess) return e;
    radix_scatter<<<(unsigned)ntiles, kRadixWarps * 32, smem, st>>>(kin, vin, ko, vo, n, shift,
                                                                     bins, b.hist, ntiles); PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kin = ko;
    vin = vo;
    if (ko == b.keysA) {
      ko = b.keysB;
      vo = b.valsB;
    } else {
      ko = b.keysA;
      vo = b.valsA;
    }
  }
  *keys_out = kin;
  *vals_out = vin;
  return cudaSuccess;
}

cudaError_t segments(const int32_t* keys, int64_t n, int* seg, int* U_out, int* bsum,
                     cudaStream_t st, int32_t* seg_key, const int32_t* vals,
                     const float* gather_src, float* gather_dst) {
  return exclusive_scan(FlagIn{keys},
                        SegOut{seg, U_out, keys, seg_key, vals, gather_src, gather_dst}, n, bsum,
                        st);
}

}  // namespace sort
}  // namespace pkm
