// B3, the value pass of the backward (kept in its own file: profiling records of this
// kernel name the source they were taken from).
//
// One 128-thread CTA per distinct value row r, rows double-buffered in shared memory by
// 1-D bulk async copies; for each selection e of r: dw[e] = dy[t] . V[r] and
// acc += w[e] dy[t]; then dV[r] += acc (or the compact output).  Also the small helpers
// the other backward kernels share.  Included by the backward translation unit only.
#pragma once

#include "pkm_internal.cuh"
#include "tc_common.cuh"

namespace pkm {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

template <typename T>
struct VecT;
template <>
struct VecT<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static void load(const __nv_bfloat16* p, float* f) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    bf16x8_to_f32(u, f);
  }
};
template <>
struct VecT<float> {
  static constexpr int E = 4;
  __device__ static void load(const float* p, float* f) {
    float4 u = *reinterpret_cast<const float4*>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
  }
};

// ------------------------------------------------------------------ B3
// L2 policies: the upstream gradient rows are re-read once per selection and stay
// resident (evict_last); value rows and value-gradient rows stream (evict_first).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ float4 ld_f4_hint(const float* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ uint4 ld_u4_stream(const void* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void st_f4_hint(float* p, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}

template <typename TV>
__device__ __forceinline__ void load_vals(const TV* p, uint64_t pol, float* f);
template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16>(const __nv_bfloat16* p, uint64_t pol,
                                                          float* f) {
  bf16x8_to_f32(ld_u4_stream(p, pol), f);
}
template <>
__device__ __forceinline__ void load_vals<float>(const float* p, uint64_t pol, float* f) {
  uint4 u = ld_u4_stream(p, pol);
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

// One 128-thread CTA per distinct value row r (grid-stride over rows), with the rows
// double-buffered in shared memory: while the CTA works on row u, one thread has
// already issued the 1-D bulk async copies (cp.async.bulk, mbarrier completion, L2
// evict_first) of V[r'] and dV[r'] for its next row u' into the other buffer, so a
// row's bytes are in flight during the previous row's arithmetic without costing
// registers.  Thread j owns 16-byte chunks j, j + 128, ... of the row (CH of them
// per column block).  A row's selections are taken in batches of 64: entry ids and
// weights staged in shared memory; each thread accumulates its chunks of
// sum_e w_e dy[t_e] and a partial dot dy[t_e] . V[r]; partials are reduced over the 4
// warps in a fixed order.  dV[r] is read once and written once (one writer, no
// atomics).  Every mbarrier wait is bounded.
constexpr int kB3Threads = 128, kB3Batch = 64;

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)), "l"(pol)
      : "memory");
}

template <typename TV>
__device__ __forceinline__ void smem_vals(const TV* p, float* f);
template <>
__device__ __forceinline__ void smem_vals<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f);
}
template <>
__device__ __forceinline__ void smem_vals<float>(const float* p, float* f) {
  const float4 u = *reinterpret_cast<const float4*>(p);
  f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}

// ws_sorted[p] = w[ents[p]]: the selection weights in row order, so staging a batch
// needs two independent loads.  A selection's upstream-gradient row is ent_tok[ent] when
// that map is given (entries received from other ranks), else ent / hk (its token).
template <typename TV, int CH>
// resident CTAs per SM the pass is compiled and launched for (a tuning value)
#ifndef PKM_B3_MIN_BLOCKS
#define PKM_B3_MIN_BLOCKS 6
#endif

__global__ void __launch_bounds__(kB3Threads, PKM_B3_MIN_BLOCKS) value_rows_kernel(
    const int* __restrict__ seg, const int* __restrict__ U_ptr, const int32_t* __restrict__ seg_row,
    const int32_t* __restrict__ ents, const TV* __restrict__ V, const float* __restrict__ ws_sorted,
    const float* __restrict__ dy, float* __restrict__ dV, float* __restrict__ dw, int hk, int d_v,
    int64_t K, int* status, float* __restrict__ dVc, int32_t* __restrict__ rows_out,
    int* __restrict__ U_out, const int32_t* __restrict__ ent_tok) {
  constexpr int E = VecT<TV>::E;
  extern __shared__ __align__(16) unsigned char b3_smem[];
  __shared__ int s_t[2][kB3Batch];
  __shared__ int s_e[2][kB3Batch];
  __shared__ float s_w[2][kB3Batch];
  __shared__ float s_part[kB3Threads / 32][kB3Batch];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int U = *U_ptr;
  const int nvec = d_v / E;
  const uint32_t vbytes = (uint32_t)d_v * sizeof(TV), dbytes = dV ? (uint32_t)d_v * 4u : 0u;
  const uint32_t slot_bytes = ((vbytes + 15u) & ~15u) + dbytes;
  const uint64_t pol_keep = policy_evict_last();
  const uint64_t pol_stream = policy_evict_first();
  if (tid == 0) {
    tc::mbar_init(&bar[0], 1);
    tc::mbar_init(&bar[1], 1);
    abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();

  // thread 0: start the copies of row u's V and dV lines into buffer b
  auto issue = [&](int u, int b) {
    const int32_t r = seg_row[u];
    unsigned char* buf = b3_smem + (size_t)b * slot_bytes;
    if (r < 0 || r >= K) {
      set_status(status, kDevIndex);
      tc::mbar_arrive(&bar[b]);  // complete the phase without data
      return;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc::mbar_arrive_expect_tx(&bar[b], vbytes + dbytes);
    bulk_g2s(buf, V + (int64_t)r * d_v, vbytes, &bar[b], pol_stream);
    if (dbytes)
      bulk_g2s(buf + ((vbytes + 15u) & ~15u), dV + (int64_t)r * d_v, dbytes, &bar[b], pol_stream);
  };

  if (U_out && blockIdx.x == 0 && tid == 0) *U_out = U;
  uint32_t phase_bits = 0u;    // bit b: parity of buffer b's next phase
  uint32_t pending_bits = 0u;  // bit b: a copy into buffer b not yet waited for (thread 0)
  if ((int)blockIdx.x < U) {
    if (tid == 0) {
      issue(blockIdx.x, 0);
      pending_bits |= 1u;
    }
    const int q0 = seg[blockIdx.x], q1 = seg[blockIdx.x + 1];
    if (tid < min(kB3Batch, q1 - q0)) {
      const int32_t ent = ents[q0 + tid];
      s_e[0][tid] = ent;
      s_t[0][tid] = ent_tok ? ent_tok[ent] : ent / hk;
      s_w[0][tid] = ws_sorted[q0 + tid];
    }
  }
  int it = 0;
  for (int u = blockIdx.x; u < U; u += gridDim.x, ++it) {
    const int b = it & 1;
    const int un = u + (int)gridDim.x;
    if (tid == 0 && un < U) {
      issue(un, b ^ 1);
      pending_bits |= 2u >> b;  // bit (b ^ 1)
    }
    const int p0 = seg[u], p1 = seg[u + 1];
    const int32_t r = seg_row[u];
    // the next row's first batch: loads in flight while this row is processed
    int nbn = 0;
    int32_t nent = 0;
    float nw = 0.f;
    if (un < U) {
      const int np0 = seg[un];
      nbn = min(kB3Batch, seg[un + 1] - np0);
      if (tid < nbn) {
        nent = ents[np0 + tid];
        nw = ws_sorted[np0 + tid];
      }
    }
    const bool got = tc::mbar_wait(&bar[b], (phase_bits >> b) & 1u, &abort_flag, status);
    phase_bits ^= 1u << b;
    pending_bits &= ~(1u << b);
    __syncthreads();
    if (abort_flag || !got) break;  // uniform: abort_flag is read after the barrier
    if (tid < nbn) {  // publish the next row's batch
      const int64_t tn = ent_tok ? ent_tok[nent] : nent / hk;
      s_e[b ^ 1][tid] = nent;
      s_t[b ^ 1][tid] = (int)tn;
      s_w[b ^ 1][tid] = nw;
    }
    if (r < 0 || r >= K) {  // status already recorded by the issuing thread
      __syncthreads();
      continue;
    }
    const TV* sV = reinterpret_cast<const TV*>(b3_smem + (size_t)b * slot_bytes);
    const float* sD = reinterpret_cast<const float*>(b3_smem + (size_t)b * slot_bytes +
                                                     ((vbytes + 15u) & ~15u));
    // dense table (+=) or compact rows (u-th distinct row, overwritten)
    float* dVr = dV ? dV + (int64_t)r * d_v : (dVc ? dVc + (int64_t)u * d_v : nullptr);
    if (rows_out && tid == 0) rows_out[u] = r;
    for (int cb = 0; cb < nvec; cb += kB3Threads * CH) {
      float v[CH][E], acc[CH][E];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int vec = cb + tid + kB3Threads * c;
        if (vec < nvec) {
          smem_vals<TV>(sV + (int64_t)vec * E, v[c]);
          if (dV) {  // accumulate onto the dense table's row (staged with V)
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4) {
              const float4 a4 = *reinterpret_cast<const float4*>(sD + (int64_t)vec * E + 4 * e4);
              acc[c][4 * e4] = a4.x; acc[c][4 * e4 + 1] = a4.y;
              acc[c][4 * e4 + 2] = a4.z; acc[c][4 * e4 + 3] = a4.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) v[c][e] = acc[c][e] = 0.f;
        }
      }
      for (int pb = p0; pb < p1; pb += kB3Batch) {
        const int nb = min(kB3Batch, p1 - pb);
        if (pb != p0 || cb != 0) {  // the first batch was staged ahead of time
          __syncthreads();          // previous batch's staging fully consumed
          if (tid < nb) {
            const int32_t ent = ents[pb + tid];
            s_e[b][tid] = ent;
            s_t[b][tid] = ent_tok ? ent_tok[ent] : ent / hk;
            s_w[b][tid] = ws_sorted[pb + tid];
          }
          __syncthreads();
        }
        for (int i = 0; i < nb; ++i) {
          const float* dyt = dy + (int64_t)s_t[b][i] * d_v;
          const float wt = s_w[b][i];
          float dot = 0.f;
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const int vec = cb + tid + kB3Threads * c;
            if (vec < nvec) {
#pragma unroll
              for (int e4 = 0; e4 < E / 4; ++e4) {
                const float4 d4 = ld_f4_hint(dyt + (int64_t)vec * E + 4 * e4, pol_keep);
                const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  dot = fmaf(dd[e], v[c][4 * e4 + e], dot);
                  acc[c][4 * e4 + e] = fmaf(wt, dd[e], acc[c][4 * e4 + e]);
                }
              }
            }
          }
          dot = warp_sum(dot);
          if (lane == 0) s_part[wid][i] = dot;
        }
        __syncthreads();
        if (tid < nb) {
          float sdot = 0.f;
#pragma unroll
          for (int ww = 0; ww < kB3Threads / 32; ++ww) sdot += s_part[ww][tid];
          const int32_t ent = s_e[b][tid];
          dw[ent] = (cb == 0) ? sdot : dw[ent] + sdot;
        }
      }
      if (dVr) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const int vec = cb + tid + kB3Threads * c;
          if (vec < nvec) {
#pragma unroll
            for (int e4 = 0; e4 < E / 4; ++e4)
              st_f4_hint(dVr + (int64_t)vec * E + 4 * e4,
                         make_float4(acc[c][4 * e4], acc[c][4 * e4 + 1], acc[c][4 * e4 + 2],
                                     acc[c][4 * e4 + 3]),
                         pol_stream);
          }
        }
      }
    }
    __syncthreads();  // buffer b may be refilled by the next iteration's issue
  }
  // copies still in flight (only after an abort) land before the CTA exits
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      if (!((pending_bits >> b) & 1u)) continue;
      const uint32_t par = (phase_bits >> b) & 1u;
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(&bar[b], par) && clock64() - t0 < tc::kWaitBudgetCycles) {
      }
    }
  }
}

inline size_t value_rows_smem(const Plan& p) {
  const size_t vb = ((size_t)p.d_v * (p.vfp32 ? 4 : 2) + 15) & ~size_t(15);
  return 2 * (vb + (size_t)p.d_v * 4);
}

}  // namespace
}  // namespace pkm
