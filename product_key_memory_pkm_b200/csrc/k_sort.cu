// Stable LSD radix sort and segment table (see k_sort.cuh).
#include <mutex>

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
  const int64_t base = (int64_t)blockIdx.x * kRadixTile;
  const uint32_t mask = (uint32_t)bins - 1u;
  // every key of the thread requested before the first count (keys[j] = position
  // threadIdx.x + 256 j of the tile)
  constexpr int kPer = kRadixTile / 256;
  int32_t kv[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int64_t g = base + threadIdx.x + 256 * j;
    kv[j] = g < n ? keys[g] : -1;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (base + threadIdx.x + 256 * j < n) atomicAdd(&h[((uint32_t)kv[j] >> shift) & mask], 1);
  __syncthreads();
  for (int d = threadIdx.x; d < bins; d += blockDim.x) hist[(int64_t)d * ntiles + blockIdx.x] = h[d];
}

// Shared memory of one radix_scatter CTA: per-warp digit counts, the tile's digit starts,
// each digit's global offset minus its tile start, and the tile's keys, payloads and
// (kW) floats staged in digit order.
inline size_t radix_scatter_smem(int bins, bool with_w) {
  return sizeof(int) * ((size_t)kRadixWarps * bins + 2 * bins) +
         (size_t)kRadixTile * (with_w ? 12 : 8);
}

// One CTA per tile of kRadixTile keys, kRadixWarps warps each owning a contiguous
// 1/kRadixWarps of it, a lane holding 16 of its keys (with their payloads and floats) in
// registers, all loaded up front.  Per-warp digit counts -> per-warp bases within each
// digit and the digit starts within the tile -> the keys placed in the tile's shared-
// memory copy in digit order (__match_any_sync ranks, in order) -> the copy written out
// position by position, each digit's run at its global offset.  Stable by construction.
template <bool kW>
__global__ void __launch_bounds__(kRadixWarps * 32) radix_scatter(
    const int32_t* __restrict__ kin, const int32_t* __restrict__ vin,
    const float* __restrict__ win, int32_t* __restrict__ kout, int32_t* __restrict__ vout,
    float* __restrict__ wout, int64_t n, int shift, int bins, const int* __restrict__ offs,
    int64_t ntiles) {
  constexpr int kPerWarp = kRadixTile / kRadixWarps;
  constexpr int kPerLane = kPerWarp / 32;
  extern __shared__ __align__(16) int rsm[];
  int* cnt = rsm;                          // [kRadixWarps][bins]
  int* dstart = cnt + kRadixWarps * bins;  // [bins]
  int* gofs = dstart + bins;               // [bins]
  int32_t* sk = gofs + bins;               // [kRadixTile]
  int32_t* sv = sk + kRadixTile;           // [kRadixTile]
  float* sw = reinterpret_cast<float*>(sv + kRadixTile);  // [kRadixTile] when kW
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t tbase = (int64_t)blockIdx.x * kRadixTile;
  const int tn = (int)(n - tbase < kRadixTile ? n - tbase : kRadixTile);
  const int w0 = wid * kPerWarp;
  const uint32_t mask = (uint32_t)bins - 1u;
  // key j of this lane: tile position w0 + 32 j + lane
  int32_t key[kPerLane], val[kPerLane];
  float wv[kPerLane];
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    const int i = w0 + 32 * j + lane;
    const bool ok = i < tn;
    key[j] = ok ? kin[tbase + i] : 0;
    val[j] = ok ? (vin ? vin[tbase + i] : (int32_t)(tbase + i)) : 0;
    wv[j] = (kW && ok) ? win[tbase + i] : 0.f;
  }
  for (int e = tid; e < kRadixWarps * bins; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  int* wc = cnt + wid * bins;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j)
    if (w0 + 32 * j + lane < tn) atomicAdd(&wc[((uint32_t)key[j] >> shift) & mask], 1);
  __syncthreads();
  // per digit: the warps' exclusive bases within the digit; the digit's tile total
  for (int d = tid; d < bins; d += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kRadixWarps; ++w) {
      const int c = cnt[w * bins + d];
      cnt[w * bins + d] = run;
      run += c;
    }
    dstart[d] = run;
  }
  __syncthreads();
  // digit starts within the tile: exclusive scan of the totals, thread t owning digits
  // [per * t, per * t + per)
  {
    const int per = (bins + blockDim.x - 1) / blockDim.x;  // <= 4 with 1024 bins
    int v[4] = {0, 0, 0, 0};
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = tid * per + j;
      if (j < per && d < bins) v[j] = dstart[d];
      sum += v[j];
    }
    int total;
    int ex = block_excl_scan(sum, &total);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = tid * per + j;
      if (j < per && d < bins) {
        dstart[d] = ex;
        gofs[d] = offs[(int64_t)d * ntiles + blockIdx.x] - ex;
        ex += v[j];
      }
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    const bool valid = w0 + 32 * j + lane < tn;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    if (valid) {
      const uint32_t d = ((uint32_t)key[j] >> shift) & mask;
      const unsigned peers = __match_any_sync(vmask, d);
      const int lp = dstart[d] + wc[d] + __popc(peers & lt);
      sk[lp] = key[j];
      sv[lp] = val[j];
      if (kW) sw[lp] = wv[j];
      __syncwarp(vmask);
      if ((peers & lt) == 0) wc[d] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
  for (int p = tid; p < tn; p += blockDim.x) {
    const int32_t k = sk[p];
    const int gp = gofs[((uint32_t)k >> shift) & mask] + p;
    kout[gp] = k;
    vout[gp] = sv[p];
    if (kW) wout[gp] = sw[p];
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
                       const int32_t** keys_out, const int32_t** vals_out, cudaStream_t st,
                       const float* w_src, float* w_tmp, float* w_dst) {
  if (bits_total < 1) bits_total = 1;
  const int passes = (bits_total + kRadixMaxBits - 1) / kRadixMaxBits;
  const int bits = (bits_total + passes - 1) / passes;
  const int bins = 1 << bits;
  const int64_t ntiles = radix_tiles(n);
  const bool with_w = w_src != nullptr;
  const int32_t* kin = keys_src;
  const int32_t* vin = nullptr;
  const float* wi = w_src;
  int32_t* ko = b.keysA;
  int32_t* vo = b.valsA;
  const size_t smem = radix_scatter_smem(bins, with_w);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, []() {
    attr_err = cudaFuncSetAttribute(radix_scatter<true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)radix_scatter_smem(1 << kRadixMaxBits, true));
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(radix_scatter<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)radix_scatter_smem(1 << kRadixMaxBits, false));
  });
  cudaError_t e = attr_err;
  if (e != cudaSuccess) return e;
  for (int p = 0; p < passes; ++p) {
    const int shift = p * bits;
    // the floats end in w_dst: the passes before the last alternate so that they do
    float* wo = ((passes - 1 - p) & 1) ? w_tmp : w_dst;
    radix_hist<<<(unsigned)ntiles, 256, 0, st>>>(kin, n, shift, bins, b.hist, ntiles); PKM_COUNT(1);
    e = exclusive_scan(HistIn{b.hist}, HistOut{b.hist}, (int64_t)bins * ntiles, b.bsum, st);
    if (e != cudaSuccess) return e;
    if (with_w)
      radix_scatter<true><<<(unsigned)ntiles, kRadixWarps * 32, smem, st>>>(
          kin, vin, wi, ko, vo, wo, n, shift, bins, b.hist, ntiles);
    else
      radix_scatter<false><<<(unsigned)ntiles, kRadixWarps * 32, smem, st>>>(
          kin, vin, nullptr, ko, vo, nullptr, n, shift, bins, b.hist, ntiles);
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kin = ko;
    vin = vo;
    wi = wo;
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
