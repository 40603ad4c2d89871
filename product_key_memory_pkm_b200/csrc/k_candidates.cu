// F3 pkm_candidate_topk: the k x k Cartesian candidates of one (token, head) and
// the best k of them, then the softmax over the winners ("Large Memory Layers with
// Product Keys", method details: combine the two sub-key sets and keep the k most
// similar keys; "Meta AI 可扩展内存层" 4.3 and 5.3; value row i*|C'| + j from 4.5).
//
// One warp per (token, head).  Lane a holds the a-th best sub-key of the first half
// (and, for k > 32, the (a+32)-th as its second row) and walks its row of candidates
// (a, 0), (a, 1), ... whose sums s1[a] + s2[b] are non-increasing in b, so each row is a
// sorted list.  A k-way merge of the k rows takes k steps: each step reduces the rows'
// heads with one redux.sync max over the order key of the fp32 sum, resolves rare exact
// ties by s1, then s2, then the flat row index, emits the winner and advances the
// winning row.  This visits exactly the order (s1+s2 desc, s1 desc, s2 desc, flat asc)
// over all k*k candidates.
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kCandWarps = 8;  // warps per block of the candidate kernels

// Among the rows still in the running (in[r]), keep those whose key equals the warp-wide
// maximum of their keys.  Returns the number of rows left in the warp.
template <int R>
__device__ __forceinline__ int keep_max(bool (&in)[R], const uint32_t (&key)[R]) {
  uint32_t loc = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) loc = in[r] ? max(loc, key[r]) : loc;
  const uint32_t m = __reduce_max_sync(kFull, loc);
  int n = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    in[r] = in[r] && key[r] == m;
    n += __popc(__ballot_sync(kFull, in[r]));
  }
  return n;
}

// R = rows of the k x k grid per lane (1 for k <= 32, 2 for k <= 64).
template <int R>
__global__ void __launch_bounds__(256) candidate_topk_kernel(
    const float* __restrict__ sub_s, const int32_t* __restrict__ sub_i, int32_t* __restrict__ idx,
    float* __restrict__ w_out, int64_t NH, int k, int C2, float scale) {
  grid_dependency_wait();  // the per-half lists come from the previous kernel
  allow_dependent_launch();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  // the winners in order, written by the winning lane of each step
  __shared__ float wS_s[kCandWarps][32 * R];
  __shared__ int32_t wI_s[kCandWarps][32 * R];
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + wid;
  if (g >= NH) return;  // warp-uniform
  const float* ss = sub_s + g * 2 * k;
  const int32_t* si = sub_i + g * 2 * k;
  bool live[R];
  float s1[R], s2[R];
  int32_t i1[R], j2[R];
  int ptr[R];  // row (lane + 32 r)'s next column b
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int a = lane + 32 * r;
    live[r] = a < k;
    s1[r] = live[r] ? ss[a] : -INFINITY;
    s2[r] = live[r] ? ss[k + a] : -INFINITY;
    i1[r] = live[r] ? si[a] : 0;
    j2[r] = live[r] ? si[k + a] : 0;
    ptr[r] = 0;
  }
  for (int step = 0; step < k; ++step) {
    bool in[R];
    float S[R], s2b[R];
    int32_t flat[R];
    uint32_t key[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      in[r] = live[r] && ptr[r] < k;
      const int b = in[r] ? ptr[r] : 0;
      // s2[b] and j2[b] live in lane b & 31, register b >> 5
      float x = __shfl_sync(kFull, s2[0], b & 31);
      int32_t jx = __shfl_sync(kFull, j2[0], b & 31);
      if (R > 1) {
        const float x1 = __shfl_sync(kFull, s2[R - 1], b & 31);
        const int32_t j1 = __shfl_sync(kFull, j2[R - 1], b & 31);
        if (b >= 32) {
          x = x1;
          jx = j1;
        }
      }
      s2b[r] = x;
      S[r] = s1[r] + x;
      flat[r] = i1[r] * C2 + jx;
      key[r] = in[r] ? order_key(S[r]) : 0u;
    }
    if (keep_max<R>(in, key) > 1) {  // exact fp32 tie of the sums: s1 desc, s2 desc, flat asc
      uint32_t k1[R], k2[R], kf[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        k1[r] = order_key(s1[r]);
        k2[r] = order_key(s2b[r]);
        kf[r] = ~(uint32_t)flat[r];  // the smallest flat index has the largest key
      }
      if (keep_max<R>(in, k1) > 1 && keep_max<R>(in, k2) > 1) keep_max<R>(in, kf);
    }
    // the winner: the one row left (flat indices are distinct)
    int wr = 0;
    unsigned bal = __ballot_sync(kFull, in[0]);
    if (R > 1 && !bal) {
      wr = R - 1;
      bal = __ballot_sync(kFull, in[R - 1]);
    }
    const int win = __ffs(bal) - 1;
    if (lane == win) {
      wS_s[wid][step] = wr ? S[R - 1] : S[0];
      wI_s[wid][step] = wr ? flat[R - 1] : flat[0];
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (wr == r) ++ptr[r];
    }
  }
  __syncwarp();
  // lane j, register r: winner j + 32 r
  float outS[R];
  int32_t outIdx[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    outS[r] = live[r] ? wS_s[wid][lane + 32 * r] : 0.f;
    outIdx[r] = live[r] ? wI_s[wid][lane + 32 * r] : 0;
  }
  // softmax over the k winners of scale * S (winner 0 holds the maximum)
  const float S0 = wS_s[wid][0];
  float e[R], sum = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    e[r] = live[r] ? expf(scale * (outS[r] - S0)) : 0.f;
    sum += e[r];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (live[r]) {
      idx[g * k + lane + 32 * r] = outIdx[r];
      w_out[g * k + lane + 32 * r] = e[r] / sum;
    }
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
  const int warps = kCandWarps;
  const int64_t blocks = (NH + warps - 1) / warps;
  if (p.ksel != p.k) {
    cudaError_t e = launch_dependent(candidate_all_kernel, dim3((unsigned)blocks), dim3(warps * 32),
                                     0, st, sub_s, sub_i, idx, w, NH, p.k, p.C2, p.scale);
    PKM_COUNT(1);
    return e;
  }
  cudaError_t e =
      p.k <= 32 ? launch_dependent(candidate_topk_kernel<1>, dim3((unsigned)blocks),
                                   dim3(warps * 32), 0, st, sub_s, sub_i, idx, w, NH, p.k, p.C2,
                                   p.scale)
                : launch_dependent(candidate_topk_kernel<2>, dim3((unsigned)blocks),
                                   dim3(warps * 32), 0, st, sub_s, sub_i, idx, w, NH, p.k, p.C2,
                                   p.scale);
  PKM_COUNT(1);
  return e;
}

}  // namespace pkm
