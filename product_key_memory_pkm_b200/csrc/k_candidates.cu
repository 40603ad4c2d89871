// F3 pkm_candidate_topk: the k x k Cartesian candidates of one (token, head) and
// the best k of them, then the softmax over the winners ("Large Memory Layers with
// Product Keys", method details: combine the two sub-key sets and keep the k most
// similar keys; "Meta AI 可扩展内存层" 4.3 and 5.3; value row i*|C'| + j from 4.5).
//
// One warp per (token, head).  Lane a holds the a-th best sub-key of the first half
// and walks its row of candidates (a, 0), (a, 1), ... whose sums s1[a] + s2[b] are
// non-increasing in b, so each row is a sorted list.  A k-way merge of the k rows
// takes k steps: each step reduces the heads with one redux.sync max over the
// order key of the fp32 sum, resolves rare exact ties by s1, then s2, then the flat
// row index, emits the winner and advances the winning row.  This visits exactly
// the order (s1+s2 desc, s1 desc, s2 desc, flat asc) over all k*k candidates.
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__global__ void __launch_bounds__(256) candidate_topk_kernel(
    const float* __restrict__ sub_s, const int32_t* __restrict__ sub_i, int32_t* __restrict__ idx,
    float* __restrict__ w_out, int64_t NH, int k, int C2, float scale) {
  grid_dependency_wait();  // the per-half lists come from the previous kernel
  allow_dependent_launch();
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= NH) return;  // warp-uniform
  const float* ss = sub_s + g * 2 * k;
  const int32_t* si = sub_i + g * 2 * k;
  const bool live = lane < k;
  const float s1 = live ? ss[lane] : -INFINITY;
  const float s2 = live ? ss[k + lane] : -INFINITY;
  const int32_t i1 = live ? si[lane] : 0;
  const int32_t j2 = live ? si[k + lane] : 0;

  int ptr = 0;            // this lane's (row a = lane) next column b
  float outS = 0.f;       // lane j ends up holding the j-th winner
  int32_t outIdx = 0;
  for (int step = 0; step < k; ++step) {
    const bool valid = live && ptr < k;
    const int b = valid ? ptr : 0;
    const float s2b = __shfl_sync(kFull, s2, b);
    const int32_t j2b = __shfl_sync(kFull, j2, b);
    const float S = s1 + s2b;
    const uint32_t key = valid ? order_key(S) : 0u;
    const uint32_t m = __reduce_max_sync(kFull, key);
    unsigned cand = __ballot_sync(kFull, valid && key == m);
    if (__popc(cand) > 1) {  // exact fp32 tie of the sums: s1 desc, s2 desc, flat asc
      const bool in = (cand >> lane) & 1u;
      const uint32_t k1 = in ? order_key(s1) : 0u;
      const uint32_t m1 = __reduce_max_sync(kFull, k1);
      cand = __ballot_sync(kFull, in && k1 == m1);
      if (__popc(cand) > 1) {
        const bool in2 = (cand >> lane) & 1u;
        const uint32_t k2 = in2 ? order_key(s2b) : 0u;
        const uint32_t m2 = __reduce_max_sync(kFull, k2);
        cand = __ballot_sync(kFull, in2 && k2 == m2);
        if (__popc(cand) > 1) {
          const bool in3 = (cand >> lane) & 1u;
          const uint32_t f = in3 ? (uint32_t)(i1 * C2 + j2b) : 0xffffffffu;
          const uint32_t mf = __reduce_min_sync(kFull, f);
          cand = __ballot_sync(kFull, in3 && f == mf);
        }
      }
    }
    const int win = __ffs(cand) - 1;
    const float wS = __shfl_sync(kFull, S, win);
    const int32_t wIdx = __shfl_sync(kFull, i1 * C2 + j2b, win);
    if (lane == step) {
      outS = wS;
      outIdx = wIdx;
    }
    if (lane == win) ++ptr;
  }
  // softmax over the k winners of scale * S (winner 0 holds the maximum)
  const float S0 = __shfl_sync(kFull, outS, 0);
  float e = live ? expf(scale * (outS - S0)) : 0.f;
  float sum = e;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
  if (live) {
    idx[g * k + lane] = outIdx;
    w_out[g * k + lane] = e / sum;
  }
}

// The all-k^2 variant (the code snippet of "Meta AI 可扩展内存层" section 10): every one
// of the k*k candidates is kept, a-major (candidate a*k + b pairs the a-th key of the
// first half with the b-th of the second), and the softmax runs over all of them.  One
// warp per (token, head); lanes stride over the candidates.
__global__ void __launch_bounds__(256) candidate_all_kernel(
    const float* __restrict__ sub_s, const int32_t* __restrict__ sub_i, int32_t* __restrict__ idx,
    float* __restrict__ w_out, int64_t NH, int k, int C2, float scale) {
  grid_dependency_wait();  // the per-half lists come from the previous kernel
  allow_dependent_launch();
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= NH) return;  // warp-uniform
  const int kk = k * k;
  const float* s1 = sub_s + g * 2 * k;
  const float* s2 = s1 + k;
  const int32_t* i1 = sub_i + g * 2 * k;
  const int32_t* i2 = i1 + k;
  float mx = -INFINITY;
  for (int c = lane; c < kk; c += 32) mx = fmaxf(mx, scale * (s1[c / k] + s2[c % k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
  float sum = 0.f;
  for (int c = lane; c < kk; c += 32) sum += expf(scale * (s1[c / k] + s2[c % k]) - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
  const float inv = 1.f / sum;
  for (int c = lane; c < kk; c += 32) {
    const int a = c / k, b = c % k;
    idx[g * kk + c] = i1[a] * C2 + i2[b];
    w_out[g * kk + c] = expf(scale * (s1[a] + s2[b]) - mx) * inv;
  }
}

}  // namespace

cudaError_t launch_candidates(const Plan& p, const float* sub_s, const int32_t* sub_i,
                              int32_t* idx, float* w, cudaStream_t st) {
  const int64_t NH = p.N * p.h;
  const int warps = 8;
  const int64_t blocks = (NH + warps - 1) / warps;
  if (p.ksel != p.k) {
    cudaError_t e = launch_dependent(candidate_all_kernel, dim3((unsigned)blocks), dim3(warps * 32),
                                     0, st, sub_s, sub_i, idx, w, NH, p.k, p.C2, p.scale);
    PKM_COUNT(1);
    return e;
  }
  cudaError_t e = launch_dependent(candidate_topk_kernel, dim3((unsigned)blocks), dim3(warps * 32),
                                   0, st, sub_s, sub_i, idx, w, NH, p.k, p.C2, p.scale);
  PKM_COUNT(1);
  return e;
}

}  // namespace pkm
