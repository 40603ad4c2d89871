// F4 pkm_gather_bag: y[t] = sum_h sum_j w[t][h][j] * V[idx[t][h][j]]
// ("Meta AI 可扩展内存层" 5.3: only the selected rows of the value matrix are read
// and summed with the softmax weights; heads summed).
//
// HBM-bound random-row gather.  One CTA per token; each thread owns one 16-byte
// column slice of the value width and walks the token's h*k rows, keeping UNROLL
// independent 16-byte loads in flight.  Indices and weights are staged in shared
// memory once per token.  fp32 accumulation in registers, one coalesced store.
#include "pkm_internal.cuh"

namespace pkm {
namespace {

template <typename TV>
struct Vec;  // 16 bytes of values
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kElems = 8;
};
template <>
struct Vec<float> {
  static constexpr int kElems = 4;
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Fast-weight read (kResid): the same bag, and beside y the reconstruction residual
// dy[t] = y[t] - tgt[t] (tgt rows tgt_ld elements apart, fp32 or bf16) for
// t < n_target, 0 after it.
struct Resid {
  const void* tgt;
  int64_t tgt_ld, n_target;
  float* dy;
  bool tgt_bf16;
};

__device__ __forceinline__ float4 load_target4(const Resid& r, int64_t t, int64_t col) {
  if (r.tgt_bf16) {
    const uint2 u = *reinterpret_cast<const uint2*>(
        static_cast<const __nv_bfloat16*>(r.tgt) + t * r.tgt_ld + col);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  }
  return *reinterpret_cast<const float4*>(static_cast<const float*>(r.tgt) + t * r.tgt_ld + col);
}

template <typename TV, int UNROLL, bool kResid = false>
__global__ void __launch_bounds__(256) gather_bag_kernel(const TV* __restrict__ V,
                                                         const int32_t* __restrict__ idx,
                                                         const float* __restrict__ w,
                                                         float* __restrict__ y, int64_t N, int hk,
                                                         int d_v, int64_t K, int* status,
                                                         Resid res = Resid{}) {
  constexpr int E = Vec<TV>::kElems;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem_raw);
  float* s_w = reinterpret_cast<float*>(smem_raw + sizeof(int32_t) * hk);
  const int64_t t = blockIdx.x;
  for (int r = threadIdx.x; r < hk; r += blockDim.x) {
    int32_t row = idx[t * hk + r];
    if (row < 0 || row >= K) {
      set_status(status, kDevIndex);
      row = 0;
    }
    s_idx[r] = row;
    s_w[r] = w[t * hk + r];
  }
  __syncthreads();
  const int nvec = d_v / E;
  for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    int r = 0;
    for (; r + UNROLL <= hk; r += UNROLL) {
      uint4 u[UNROLL];
#pragma unroll
      for (int q = 0; q < UNROLL; ++q)
        u[q] = ld_stream(reinterpret_cast<const uint4*>(V + (int64_t)s_idx[r + q] * d_v) + c);
#pragma unroll
      for (int q = 0; q < UNROLL; ++q) {
        const float wt = s_w[r + q];
        float f[E];
        if constexpr (E == 8) {
          bf16x8_to_f32(u[q], f);
        } else {
          f[0] = __uint_as_float(u[q].x); f[1] = __uint_as_float(u[q].y);
          f[2] = __uint_as_float(u[q].z); f[3] = __uint_as_float(u[q].w);
        }
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(wt, f[e], acc[e]);
      }
    }
    for (; r < hk; ++r) {
      uint4 u = ld_stream(reinterpret_cast<const uint4*>(V + (int64_t)s_idx[r] * d_v) + c);
      const float wt = s_w[r];
      float f[E];
      if constexpr (E == 8) {
        bf16x8_to_f32(u, f);
      } else {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(wt, f[e], acc[e]);
    }
    float4* yo = reinterpret_cast<float4*>(y + t * d_v + (int64_t)c * E);
#pragma unroll
    for (int e = 0; e < E; e += 4) yo[e / 4] = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    if constexpr (kResid) {
      float4* d = reinterpret_cast<float4*>(res.dy + t * d_v + (int64_t)c * E);
      const bool has = t < res.n_target;
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        const float4 tv = has ? load_target4(res, t, (int64_t)c * E + e)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        d[e / 4] = has ? make_float4(acc[e] - tv.x, acc[e + 1] - tv.y, acc[e + 2] - tv.z,
                                     acc[e + 3] - tv.w)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

}  // namespace

cudaError_t launch_gather(const Plan& p, const void* values, const int32_t* idx, const float* w,
                          float* y, cudaStream_t st) {
  const int hk = p.h * p.k;
  const size_t smem = (size_t)hk * 8;
  if (p.vfp32) {
    const int nvec = p.d_v / 4;
    const int threads = min(256, ((nvec + 31) / 32) * 32);
    gather_bag_kernel<float, 8><<<(unsigned)p.N, threads, smem, st>>>(
        static_cast<const float*>(values), idx, w, y, p.N, hk, p.d_v, p.K, p.status); PKM_COUNT(1);
  } else {
    const int nvec = p.d_v / 8;
    const int threads = min(256, ((nvec + 31) / 32) * 32);
    gather_bag_kernel<__nv_bfloat16, 8><<<(unsigned)p.N, threads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(values), idx, w, y, p.N, hk, p.d_v, p.K, p.status); PKM_COUNT(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_resid(const Plan& p, const float* values, const int32_t* idx,
                                const float* w, float* y, const void* tgt, bool tgt_bf16,
                                int64_t tgt_ld, int64_t n_target, float* dy, cudaStream_t st) {
  const int hk = p.h * p.k;
  const size_t smem = (size_t)hk * 8;
  const int nvec = p.d_v / 4;
  const int threads = min(256, ((nvec + 31) / 32) * 32);
  gather_bag_kernel<float, 8, true><<<(unsigned)p.N, threads, smem, st>>>(
      values, idx, w, y, p.N, hk, p.d_v, p.K, p.status,
      Resid{tgt, tgt_ld, n_target, dy, tgt_bf16});
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace pkm
