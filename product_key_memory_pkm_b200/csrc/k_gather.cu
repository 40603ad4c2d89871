// F4 pkm_gather_bag: y[t] = sum_h sum_j w[t][h][j] * V[idx[t][h][j]]
// ("Meta AI 可扩展内存层" 5.3: only the selected rows of the value matrix are read
// and summed with the softmax weights; heads summed).
//
// HBM-bound random-row gather.  One CTA per token; each thread owns one 16-byte
// column slice of the value width and walks the token's h*k rows, keeping UNROLL
// independent 16-byte loads in flight.  Indices and weights are staged in shared
// memory once per token.  fp32 accumulation in registers, one coalesced store.
#include <cooperative_groups.h>

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
  grid_dependency_wait();  // idx and w (and V's last write) come from earlier kernels
  allow_dependent_launch();
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

// Few tokens (decode): one token's h*k rows are split over the S CTAs of a thread-block
// cluster, CTA r taking rows r, r + S, ...; each keeps its partial sums in shared memory
// and, after a cluster barrier, CTA 0 adds the S partials in rank order (reading the
// others' shared memory directly) and stores y.  S times the loads in flight per token
// of the one-CTA-per-token kernel; deterministic.
template <typename TV, int S>
__global__ void __cluster_dims__(S, 1, 1) __launch_bounds__(256)
    gather_bag_split_kernel(const TV* __restrict__ V, const int32_t* __restrict__ idx,
                            const float* __restrict__ w, float* __restrict__ y, int hk, int d_v,
                            int64_t K, int* status) {
  grid_dependency_wait();
  allow_dependent_launch();
  namespace cg = cooperative_groups;
  constexpr int E = Vec<TV>::kElems;
  extern __shared__ __align__(16) float part[];  // [d_v] partial sums of this CTA
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int64_t t = blockIdx.x / S;
  const int nvec = d_v / E;
  for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    int r = rank;
    constexpr int kAhead = 8;  // rows in flight per thread
    for (; r + (kAhead - 1) * S < hk; r += kAhead * S) {
      uint4 u[kAhead];
      float wt[kAhead];
#pragma unroll
      for (int q = 0; q < kAhead; ++q) {
        int32_t row = idx[t * hk + r + q * S];
        if (row < 0 || row >= K) {
          set_status(status, kDevIndex);
          row = 0;
        }
        wt[q] = w[t * hk + r + q * S];
        u[q] = ld_stream(reinterpret_cast<const uint4*>(V + (int64_t)row * d_v) + c);
      }
#pragma unroll
      for (int q = 0; q < kAhead; ++q) {
        float f[E];
        if constexpr (E == 8) {
          bf16x8_to_f32(u[q], f);
        } else {
          f[0] = __uint_as_float(u[q].x); f[1] = __uint_as_float(u[q].y);
          f[2] = __uint_as_float(u[q].z); f[3] = __uint_as_float(u[q].w);
        }
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(wt[q], f[e], acc[e]);
      }
    }
    for (; r < hk; r += S) {
      int32_t row = idx[t * hk + r];
      if (row < 0 || row >= K) {
        set_status(status, kDevIndex);
        row = 0;
      }
      const float wt = w[t * hk + r];
      const uint4 u = ld_stream(reinterpret_cast<const uint4*>(V + (int64_t)row * d_v) + c);
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
#pragma unroll
    for (int e = 0; e < E; ++e) part[c * E + e] = acc[e];
  }
  cluster.sync();
  if (rank == 0) {
    for (int i = threadIdx.x; i < d_v / 4; i += blockDim.x) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < S; ++q) {
        const float4 v = reinterpret_cast<const float4*>(cluster.map_shared_rank(part, q))[i];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      reinterpret_cast<float4*>(y + t * d_v)[i] = s;
    }
  }
  cluster.sync();  // the partials stay readable until CTA 0 has summed them
}

template <typename TV>
cudaError_t launch_gather_split(const Plan& p, const TV* V, const int32_t* idx, const float* w,
                                float* y, cudaStream_t st) {
  constexpr int S = 8;
  const int hk = p.h * p.ksel;
  const int nvec = p.d_v / Vec<TV>::kElems;
  const int threads = min(256, ((nvec + 31) / 32) * 32);
  const size_t smem = (size_t)p.d_v * 4;
  cudaError_t e;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(gather_bag_split_kernel<TV, S>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
          cudaSuccess)
    return e;
  e = launch_dependent(gather_bag_split_kernel<TV, S>, dim3((unsigned)(p.N * S)), dim3(threads),
                       smem, st, V, idx, w, y, hk, p.d_v, p.K, p.status);
  PKM_COUNT(1);
  return e;
}

}  // namespace

cudaError_t launch_gather(const Plan& p, const void* values, const int32_t* idx, const float* w,
                          float* y, cudaStream_t st) {
  const int hk = p.h * p.ksel;
  const size_t smem = (size_t)hk * 8;
  // few tokens: split each token's rows over a cluster of CTAs (d_v*4 bytes of partials)
  if (p.N < (int64_t)p.sm_count && hk >= 16 && (size_t)p.d_v * 4 <= 200 * 1024) {
    if (p.vfp32)
      return launch_gather_split(p, static_cast<const float*>(values), idx, w, y, st);
    return launch_gather_split(p, static_cast<const __nv_bfloat16*>(values), idx, w, y, st);
  }
  if (p.vfp32) {
    const int nvec = p.d_v / 4;
    const int threads = min(256, ((nvec + 31) / 32) * 32);
    PKM_COUNT(1);
    return launch_dependent(gather_bag_kernel<float, 8, false>, dim3((unsigned)p.N), dim3(threads),
                            smem, st, static_cast<const float*>(values), idx, w, y, p.N, hk,
                            p.d_v, p.K, p.status, Resid{});
  } else {
    const int nvec = p.d_v / 8;
    const int threads = min(256, ((nvec + 31) / 32) * 32);
    PKM_COUNT(1);
    return launch_dependent(gather_bag_kernel<__nv_bfloat16, 8, false>, dim3((unsigned)p.N),
                            dim3(threads), smem, st, static_cast<const __nv_bfloat16*>(values), idx,
                            w, y, p.N, hk, p.d_v, p.K, p.status, Resid{});
  }
}

cudaError_t launch_gather_resid(const Plan& p, const float* values, const int32_t* idx,
                                const float* w, float* y, const void* tgt, bool tgt_bf16,
                                int64_t tgt_ld, int64_t n_target, float* dy, cudaStream_t st) {
  const int hk = p.h * p.ksel;
  const size_t smem = (size_t)hk * 8;
  const int nvec = p.d_v / 4;
  const int threads = min(256, ((nvec + 31) / 32) * 32);
  PKM_COUNT(1);
  return launch_dependent(gather_bag_kernel<float, 8, true>, dim3((unsigned)p.N), dim3(threads),
                          smem, st, values, idx, w, y, p.N, hk, p.d_v, p.K, p.status,
                          Resid{tgt, tgt_ld, n_target, dy, tgt_bf16});
}

}  // namespace pkm
