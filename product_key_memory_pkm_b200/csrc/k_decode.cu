// F1 and F2 for few tokens (decode-shaped calls, N <= 16), on CUDA cores.
//
// With one to a few dozen tokens the tensor-core kernels have one 128-row tile and run
// on as many CTAs as there are output tiles (8 for the query, 2h for the scores), so
// each SM streams megabytes alone.  These kernels spread the same reads over hundreds
// of CTAs instead: the work is two matrix-vector products (Wq: h*dk x d_in; each
// sub-key set: C x dk/2) that must read their matrix once.
//
//   query_small_kernel   one warp per output column o of q: the warp streams row o of
//                        Wq in 16-byte pieces against up to 16 tokens' x held in shared
//                        memory, then applies the BatchNorm epilogue and writes q as
//                        bf16 hi + lo planes (and q-hat), as the tensor-core kernel does.
//   scores_small_kernel  one 8-CTA cluster per (16-token group, head, half): CTA r scores
//                        its 1/8 of the sub-keys against every token of the group and keeps
//                        each token's top-k of its slice; then CTA r merges the 8 sorted
//                        lists of tokens r and r + 8 through distributed shared memory.
//                        Order: (score desc, sub-key index asc), as everywhere.
#include <cooperative_groups.h>

#include "pkm_internal.cuh"

namespace pkm {
namespace {

namespace cg = cooperative_groups;
constexpr unsigned kFull = 0xffffffffu;
constexpr int kTokGroup = 16, kWarps = 8, kSplit = 8;
constexpr int kMaxSlice = 256;  // sub-keys per CTA (a cluster scores up to 8 * 256 per half)

// 16-byte global -> shared copies that stay in flight together (completion waited for
// with cp_async_wait_all before the block barrier).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<unsigned>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------------ F1
__global__ void __launch_bounds__(kWarps * 32) query_small_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wq,
    const float* __restrict__ bn, __nv_bfloat16* __restrict__ q, float* __restrict__ qhat,
    int64_t N, int d_in, int hq, float eps) {
  extern __shared__ __align__(16) __nv_bfloat16 xs[];  // [kTokGroup][d_in]
  allow_dependent_launch();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.y * kTokGroup;
  const int nt = (int)((N - t0 < kTokGroup) ? N - t0 : kTokGroup);
  const int nchunk = d_in / 8;
  for (int i = threadIdx.x; i < nt * nchunk; i += blockDim.x) {
    const int t = i / nchunk, c = i % nchunk;
    cp_async16(reinterpret_cast<uint4*>(xs + (int64_t)t * d_in) + c,
               reinterpret_cast<const uint4*>(x + (t0 + t) * d_in) + c);
  }
  cp_async_wait_all();
  __syncthreads();
  const int o = blockIdx.x * kWarps + wid;
  if (o >= hq) return;
  float acc[kTokGroup];
#pragma unroll
  for (int t = 0; t < kTokGroup; ++t) acc[t] = 0.f;
  const uint4* wr = reinterpret_cast<const uint4*>(Wq + (int64_t)o * d_in);
  constexpr int kAhead = 4;  // row pieces of Wq in flight per lane
  for (int cb = lane; cb < nchunk; cb += 32 * kAhead) {
    uint4 wv[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int c = cb + 32 * u;
      wv[u] = c < nchunk ? wr[c] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      const int c = cb + 32 * u;
      if (c >= nchunk) break;
      float wf[8];
      bf16x8_to_f32(wv[u], wf);
#pragma unroll
      for (int t = 0; t < kTokGroup; ++t) {
        if (t < nt) {
          float xf[8];
          bf16x8_to_f32(reinterpret_cast<const uint4*>(xs + (int64_t)t * d_in)[c], xf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[t] = fmaf(wf[e], xf[e], acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kTokGroup; ++t) {
    if (t < nt) {  // warp-uniform
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) acc[t] += __shfl_xor_sync(kFull, acc[t], s);
    }
  }
  // lane t stores token t's column o
  float mine = 0.f;
#pragma unroll
  for (int t = 0; t < kTokGroup; ++t)
    if (lane == t) mine = acc[t];
  if (lane < nt) {
    // no bn: identity (training-mode BatchNorm follows)
    const float mean = bn ? bn[o] : 0.f, inv = bn ? 1.0f / sqrtf(bn[hq + o] + eps) : 1.f;
    const float gamma = bn ? bn[2 * hq + o] : 1.f, beta = bn ? bn[3 * hq + o] : 0.f;
    const float h = (mine - mean) * inv;
    const float qq = fmaf(gamma, h, beta);
    const __nv_bfloat16 hb = __float2bfloat16_rn(qq);
    const __nv_bfloat16 lb = __float2bfloat16_rn(qq - __bfloat162float(hb));
    const int64_t off = (t0 + lane) * hq + o;
    q[off] = hb;
    q[N * hq + off] = lb;
    if (qhat) qhat[off] = h;
  }
}

// ------------------------------------------------------------------ F2
// (a ranks before b) in (score desc, index asc)
__device__ __forceinline__ bool before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// Shared-memory layout of scores_small_kernel (floats; the sub-key slice in bf16 with a
// 16-byte row pad so that 8 consecutive rows hit distinct banks).
struct SmallLayout {
  int half, per, nrow, KM;
  __host__ __device__ int kc_stride() const { return half + 8; }  // bf16 elements
  __host__ __device__ size_t qs() const { return 0; }
  __host__ __device__ size_t kc() const { return qs() + (size_t)kTokGroup * half * 4; }
  __host__ __device__ size_t sc() const { return kc() + (size_t)per * kc_stride() * 2; }
  __host__ __device__ size_t ls() const { return sc() + (size_t)kTokGroup * per * 4; }
  __host__ __device__ size_t li() const { return ls() + (size_t)kTokGroup * KM * 4; }
  __host__ __device__ size_t ms() const { return li() + (size_t)kTokGroup * KM * 4; }
  __host__ __device__ size_t mi() const { return ms() + (size_t)kTokGroup * kSplit * KM * 4; }
  __host__ __device__ size_t bytes() const { return mi() + (size_t)kTokGroup * kSplit * KM * 4; }
};

template <int KM>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kWarps * 32)
    scores_small_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ sub,
                        float* __restrict__ sub_s, int32_t* __restrict__ sub_i, int64_t N, int h,
                        int dk, int C1, int C2, int k, float lo_scale, bool idw) {
  extern __shared__ __align__(16) unsigned char smraw[];
  grid_dependency_wait();  // q comes from the query kernel
  allow_dependent_launch();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int cl = blockIdx.x / kSplit;  // cluster index: ((g * h + hh) * 2 + s)
  const int s = cl & 1, hh = (cl >> 1) % h, g = (cl >> 1) / h;
  const int half = dk / 2, hq = h * dk;
  const int C = s ? C2 : C1;
  const int per_max = (max(C1, C2) + kSplit - 1) / kSplit;
  const int per = (C + kSplit - 1) / kSplit;
  const int c0 = min(C, rank * per), c1 = min(C, c0 + per);
  const int nct = c1 - c0;
  const int64_t t0 = (int64_t)g * kTokGroup;
  const int nt = (int)((N - t0 < kTokGroup) ? N - t0 : kTokGroup);
  const SmallLayout L{half, per_max, 0, KM};
  float* qs = reinterpret_cast<float*>(smraw + L.qs());
  __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(smraw + L.kc());
  float* sc = reinterpret_cast<float*>(smraw + L.sc());
  float* ls = reinterpret_cast<float*>(smraw + L.ls());
  int* li = reinterpret_cast<int*>(smraw + L.li());
  float* ms = reinterpret_cast<float*>(smraw + L.ms());
  int* mi = reinterpret_cast<int*>(smraw + L.mi());
  const int ks = L.kc_stride();
  // 1. the group's query halves (q = hi + lo_scale * lo) and this CTA's sub-key slice
  const int64_t plane = N * hq;
  const int npc = half / 8;
  const uint4* kg = reinterpret_cast<const uint4*>(
      sub + ((int64_t)hh * (C1 + C2) + (s ? C1 : 0) + c0) * half);
  for (int i = tid; i < nct * npc; i += nthr) {  // the slice: all copies in flight at once
    const int c = i / npc, pc = i % npc;
    cp_async16(kc + (size_t)c * ks + pc * 8, kg + (size_t)c * npc + pc);
  }
  for (int i = tid; i < nt * npc; i += nthr) {  // q = hi + lo_scale * lo, 8 elements a step
    const int t = i / npc, pc = i % npc;
    const int64_t off = (t0 + t) * hq + (int64_t)hh * dk + s * half + pc * 8;
    float hf[8], lf[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(q + off), hf);
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(q + plane + off), lf);
    float4* dst = reinterpret_cast<float4*>(qs + t * half + pc * 8);
    dst[0] = make_float4(hf[0] + lo_scale * lf[0], hf[1] + lo_scale * lf[1],
                         hf[2] + lo_scale * lf[2], hf[3] + lo_scale * lf[3]);
    dst[1] = make_float4(hf[4] + lo_scale * lf[4], hf[5] + lo_scale * lf[5],
                         hf[6] + lo_scale * lf[6], hf[7] + lo_scale * lf[7]);
  }
  cp_async_wait_all();
  for (int i = tid; i < nt * KM; i += nthr) {
    ls[i] = -INFINITY;
    li[i] = 0x7fffffff;
  }
  __syncthreads();
  // 2. scores: one (token, sub-key) dot product per thread and step
  for (int i = tid; i < nt * nct; i += nthr) {
    const int t = i / nct, c = i % nct;
    const __nv_bfloat16* kr = kc + (size_t)c * ks;
    const float* qr = qs + t * half;
    float acc = 0.f, qn = 0.f, cn = 0.f;
    for (int pc = 0; pc < npc; ++pc) {
      float kf[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(kr + pc * 8), kf);
      const float4 a = reinterpret_cast<const float4*>(qr + pc * 8)[0];
      const float4 b = reinterpret_cast<const float4*>(qr + pc * 8)[1];
      const float qf[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(kf[e], qf[e], acc);
      if (idw) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          qn = fmaf(qf[e], qf[e], qn);
          cn = fmaf(kf[e], kf[e], cn);
        }
      }
    }
    // inverse-distance scores: -1/2 log(||q - c||^2 + eps)
    sc[t * per_max + c] = idw ? -0.5f * logf(fmaxf(qn + cn - 2.f * acc, 0.f) + 1e-12f) : acc;
  }
  __syncthreads();
  // 3. each token's top-KM of the slice, best first: every thread places candidates, each
  //    at the number of the slice's candidates that rank before it.
  for (int i = tid; i < nt * nct; i += nthr) {
    const int t = i / nct, c = i % nct;
    const float* st = sc + t * per_max;
    const float v = st[c];
    int r = 0;
    for (int c2 = 0; c2 < nct; ++c2) r += before(st[c2], c0 + c2, v, c0 + c) ? 1 : 0;
    if (r < KM) {
      ls[t * KM + r] = v;
      li[t * KM + r] = c0 + c;
    }
  }
  cluster.sync();
  // 4. CTA r gathers the kSplit sorted lists of the group's tokens t = r, r + kSplit, ...
  //    (at most two per CTA), eight remote elements per thread and step, loads first ...
  const int my_nt = nt > rank ? (nt - rank + kSplit - 1) / kSplit : 0;
  const int n_el = my_nt * kSplit * KM;
  for (int i0 = tid; i0 < n_el; i0 += 8 * nthr) {
    float v[8];
    int x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * nthr;
      if (i < n_el) {
        const int t = rank + (i / (kSplit * KM)) * kSplit, r = (i / KM) % kSplit, j = i % KM;
        v[u] = cluster.map_shared_rank(ls, r)[t * KM + j];
        x[u] = cluster.map_shared_rank(li, r)[t * KM + j];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * nthr;
      if (i < n_el) {
        ms[i] = v[u];
        mi[i] = x[u];
      }
    }
  }
  cluster.sync();  // the lists may be released now
  if (my_nt == 0) return;
  __syncthreads();
  // 5. ... and merges them: every element is placed by merge rank -- its position in its
  //    own list plus, for every other list, how many of that list's elements rank before
  //    it (binary search).
  for (int i = tid; i < n_el; i += nthr) {
    const int lt = i / (kSplit * KM), r = (i / KM) % kSplit, j = i % KM;
    const int t = rank + lt * kSplit;
    const float v = ms[i];
    const int vi = mi[i];
    if (vi == 0x7fffffff) continue;  // padding
    int place = j;
    for (int r2 = 0; r2 < kSplit; ++r2) {
      if (r2 == r) continue;
      const float* lv = ms + (lt * kSplit + r2) * KM;
      const int* lx = mi + (lt * kSplit + r2) * KM;
      int lo = 0, hi = KM;  // first element of list r2 that does not rank before (v, vi)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (before(lv[mid], lx[mid], v, vi)) lo = mid + 1;
        else hi = mid;
      }
      place += lo;
    }
    if (place < k) {
      const int64_t o = (((t0 + t) * h + hh) * 2 + s) * (int64_t)k + place;
      sub_s[o] = v;
      sub_i[o] = vi;
    }
  }
}

}  // namespace

size_t scores_small_smem(const Plan& p, int KM) {
  const SmallLayout L{p.dk / 2, (std::max(p.C1, p.C2) + kSplit - 1) / kSplit, 0, KM};
  return L.bytes();
}

bool small_n_supported(const Plan& p) {
  return !p.fp32 && p.N <= kSmallTokens && p.d_in % 8 == 0 && (p.dk / 2) % 8 == 0 &&
         (std::max(p.C1, p.C2) + kSplit - 1) / kSplit <= kMaxSlice &&
         (size_t)kTokGroup * p.d_in * 2 <= 160 * 1024 &&
         scores_small_smem(p, p.k <= 32 ? 32 : 64) <= 200 * 1024;
}

cudaError_t launch_query_small(const Plan& p, const void* x, const void* Wq, const float* bn,
                               void* q, float* qhat, cudaStream_t st) {
  const size_t smem = (size_t)kTokGroup * p.d_in * 2;
  cudaError_t e;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(query_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  dim3 grid((unsigned)((p.hq + kWarps - 1) / kWarps), (unsigned)((p.N + kTokGroup - 1) / kTokGroup));
  query_small_kernel<<<grid, kWarps * 32, smem, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wq), bn,
      static_cast<__nv_bfloat16*>(q), qhat, p.N, p.d_in, p.hq, p.eps);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_scores_small(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                                int32_t* sub_i, cudaStream_t st) {
  const int groups = (int)((p.N + kTokGroup - 1) / kTokGroup);
  const unsigned grid = (unsigned)(groups * p.h * 2 * kSplit);
  const float lo_scale = p.bf16q ? 0.f : 1.f;
  cudaError_t e;
#define PKM_SS(KMV)                                                                          \
  do {                                                                                       \
    const size_t smem = scores_small_smem(p, KMV);                                           \
    if (smem > 48 * 1024 &&                                                                  \
        (e = cudaFuncSetAttribute(scores_small_kernel<KMV>,                                  \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=  \
            cudaSuccess)                                                                     \
      return e;                                                                              \
    e = launch_dependent(scores_small_kernel<KMV>, dim3(grid), dim3(kWarps * 32), smem, st,  \
                         static_cast<const __nv_bfloat16*>(q),                               \
                         static_cast<const __nv_bfloat16*>(subkeys), sub_s, sub_i, p.N, p.h, \
                         p.dk, p.C1, p.C2, p.k, lo_scale, p.idw);                            \
    if (e != cudaSuccess) return e;                                                         \
  } while (0)
  if (p.k <= 8)
    PKM_SS(8);
  else if (p.k <= 16)
    PKM_SS(16);
  else if (p.k <= 32)
    PKM_SS(32);
  else
    PKM_SS(64);
#undef PKM_SS
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace pkm
