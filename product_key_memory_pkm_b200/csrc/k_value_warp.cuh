// B3, the value pass of the backward, one warp per distinct value row (kept in its own
// file: profiling records of this kernel name the source they were taken from).
//
// For each distinct selected row r with selections e (sorted by row, stable):
//   dw[e] = dy[t_e] . V[r]      and      dV[r] += sum_e w_e dy[t_e]
// ("Meta AI 可扩展内存层" 6.1 and 9.2: gradients reach only the selected slots; the
// duplicates of a row are combined before its single write, so there are no atomics
// and the result is deterministic).
//
// Every warp is independent: it walks its own rows and keeps `depth` of them in
// flight in its private shared-memory slots.  Lane 0 starts a row's 1-D bulk async
// copies (cp.async.bulk, mbarrier completion, L2 evict_first) of V[r], dV[r] and the
// row's selection ids and weights `depth` rows before the warp works on it, so the
// HBM latency of the row bytes overlaps the arithmetic of the rows before it.  While
// working on a row the warp holds the row's accumulator in registers (lane l owns the
// float4 columns l, l + 32, ...), loads each selection's upstream-gradient row with an
// L2 evict_last policy (those rows are read once per selection), reduces the dot
// product with shuffles and writes dV[r] once.  No block-level barrier is involved.
#pragma once

#include "k_value_rows.cuh"

namespace pkm {
namespace {

constexpr int kVwWarps = 10;   // warps per CTA (one CTA per SM)
constexpr int kVwMeta = 64;    // selection ids / weights staged per row (the rest from L2)
constexpr int kVwMaxDepth = 4;

struct VwSlot {
  int p0, p1, r, u;
};

// Bytes of one slot: staged ids and weights, then V[r] (16-byte padded), then dV[r].
__host__ __device__ inline uint32_t vw_slot_bytes(int d_v, int v_elem_bytes, bool dense) {
  const uint32_t vb = ((uint32_t)d_v * (uint32_t)v_elem_bytes + 15u) & ~15u;
  return 8u * kVwMeta + vb + (dense ? (uint32_t)d_v * 4u : 0u);
}

template <typename TV>
__device__ __forceinline__ float4 vw_v4(const unsigned char* sV, int c);
template <>
__device__ __forceinline__ float4 vw_v4<__nv_bfloat16>(const unsigned char* sV, int c) {
  const uint2 u = *reinterpret_cast<const uint2*>(sV + 8 * c);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 vw_v4<float>(const unsigned char* sV, int c) {
  return *reinterpret_cast<const float4*>(sV + 16 * c);
}

// MAXJ = float4 columns per lane (d_v <= 128 * MAXJ).  Rows of warp gw: gw, gw + GW,
// ... (interleaved) or a contiguous range of about U / GW rows (contiguous != 0).
template <typename TV, int MAXJ>
__global__ void __launch_bounds__(kVwWarps * 32, 1) value_warp_kernel(
    const int* __restrict__ seg, const int* __restrict__ U_ptr, const int32_t* __restrict__ seg_row,
    const int32_t* __restrict__ ents, const TV* __restrict__ V, const float* __restrict__ ws_sorted,
    const float* __restrict__ dy, float* __restrict__ dV, float* __restrict__ dw, int hk, int d_v,
    int64_t K, int* status, float* __restrict__ dVc, int32_t* __restrict__ rows_out,
    int* __restrict__ U_out, const int32_t* __restrict__ ent_tok, int depth, int contiguous) {
  extern __shared__ __align__(128) unsigned char vw_smem[];
  __shared__ __align__(8) uint64_t full[kVwWarps][kVwMaxDepth];
  __shared__ VwSlot hdr[kVwWarps][kVwMaxDepth];
  __shared__ volatile int abort_flag[kVwWarps];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int U = *U_ptr;
  const int nv4 = d_v / 4;
  const bool dense = dV != nullptr;
  const uint32_t vbytes = (uint32_t)d_v * sizeof(TV);
  const uint32_t vpad = (vbytes + 15u) & ~15u;
  const uint32_t dbytes = dense ? (uint32_t)d_v * 4u : 0u;
  const uint32_t slot_bytes = vw_slot_bytes(d_v, (int)sizeof(TV), dense);
  unsigned char* wsm = vw_smem + (size_t)wid * depth * slot_bytes;
  const uint64_t pol_keep = policy_evict_last();
  const uint64_t pol_stream = policy_evict_first();
  if (lane == 0) {
    for (int b = 0; b < depth; ++b) tc::mbar_init(&full[wid][b], 1);
    abort_flag[wid] = 0;
    tc::fence_barrier_init();
  }
  __syncwarp();
  if (U_out && blockIdx.x == 0 && threadIdx.x == 0) *U_out = U;

  const int64_t GW = (int64_t)gridDim.x * kVwWarps;
  const int64_t gw = (int64_t)blockIdx.x * kVwWarps + wid;
  int64_t lo = gw, step = GW, hi = U;
  if (contiguous) {
    lo = gw * U / GW;
    hi = (gw + 1) * U / GW;
    step = 1;
  }
  const int64_t nrows = hi > lo ? (hi - lo + step - 1) / step : 0;

  // lane 0: start the copies of the warp's row n into slot n % depth
  auto issue = [&](int64_t n) {
    const int b = (int)(n % depth);
    const int u = (int)(lo + n * step);
    const int p0 = seg[u], p1 = seg[u + 1];
    const int32_t r = seg_row[u];
    hdr[wid][b] = VwSlot{p0, p1, r, u};
    unsigned char* sl = wsm + (size_t)b * slot_bytes;
    if (r < 0 || r >= K) {
      set_status(status, kDevIndex);
      tc::mbar_arrive(&full[wid][b]);  // complete the phase without data
      return;
    }
    const int a0 = p0 & ~3;
    const int mcnt = min(((p1 + 3) & ~3) - a0, kVwMeta);
    const uint32_t mbytes = 4u * (uint32_t)mcnt;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc::mbar_arrive_expect_tx(&full[wid][b], 2u * mbytes + vbytes + dbytes);
    bulk_g2s(sl, ents + a0, mbytes, &full[wid][b], pol_keep);
    bulk_g2s(sl + 4 * kVwMeta, ws_sorted + a0, mbytes, &full[wid][b], pol_keep);
    bulk_g2s(sl + 8 * kVwMeta, V + (int64_t)r * d_v, vbytes, &full[wid][b], pol_stream);
    if (dense) bulk_g2s(sl + 8 * kVwMeta + vpad, dV + (int64_t)r * d_v, dbytes, &full[wid][b], pol_stream);
  };

  if (lane == 0)
    for (int64_t n = 0; n < depth && n < nrows; ++n) issue(n);
  int64_t issued = nrows < depth ? nrows : (int64_t)depth;
  int64_t n = 0;
  for (; n < nrows; ++n) {
    const int b = (int)(n % depth);
    const uint32_t par = (uint32_t)((n / depth) & 1);
    int got = 1;
    if (lane == 0) got = tc::mbar_wait(&full[wid][b], par, &abort_flag[wid], status) ? 1 : 0;
    if (!__shfl_sync(kFull, got, 0)) break;
    // every lane observes the completed phase itself (acquire): the bulk-copied bytes and
    // the header lane 0 wrote before its arrive are then visible to it
    (void)tc::mbar_try_wait(&full[wid][b], par);
    const VwSlot h = hdr[wid][b];
    const unsigned char* sl = wsm + (size_t)b * slot_bytes;
    if (h.r >= 0 && h.r < K) {
      // staged selections start at p0 & ~3; the first kVwMeta - (p0 & 3) of the row are there
      const int32_t* sE = reinterpret_cast<const int32_t*>(sl) + (h.p0 & 3);
      const float* sW = reinterpret_cast<const float*>(sl + 4 * kVwMeta) + (h.p0 & 3);
      const int mcnt = kVwMeta - (h.p0 & 3);
      const unsigned char* sV = sl + 8 * kVwMeta;
      const float* sD = reinterpret_cast<const float*>(sl + 8 * kVwMeta + vpad);
      float4 acc[MAXJ];
#pragma unroll
      for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        acc[j] = (dense && c < nv4) ? *reinterpret_cast<const float4*>(sD + 4 * c)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      const int nsel = h.p1 - h.p0;
      for (int e = 0; e < nsel; ++e) {
        int32_t ent;
        float wt;
        if (e < mcnt) {
          ent = sE[e];
          wt = sW[e];
        } else {
          ent = ents[h.p0 + e];
          wt = ws_sorted[h.p0 + e];
        }
        const int64_t t = ent_tok ? (int64_t)ent_tok[ent] : (int64_t)(ent / hk);
        const float* dyt = dy + t * d_v;
        float4 d[MAXJ];
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
          const int c = lane + 32 * j;
          if (c < nv4) d[j] = ld_f4_hint(dyt + 4 * c, pol_keep);
        }
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
          const int c = lane + 32 * j;
          if (c < nv4) {
            const float4 v = vw_v4<TV>(sV, c);
            dot = fmaf(d[j].x, v.x, dot);
            dot = fmaf(d[j].y, v.y, dot);
            dot = fmaf(d[j].z, v.z, dot);
            dot = fmaf(d[j].w, v.w, dot);
            acc[j].x = fmaf(wt, d[j].x, acc[j].x);
            acc[j].y = fmaf(wt, d[j].y, acc[j].y);
            acc[j].z = fmaf(wt, d[j].z, acc[j].z);
            acc[j].w = fmaf(wt, d[j].w, acc[j].w);
          }
        }
        dot = warp_sum(dot);
        if (lane == 0) dw[ent] = dot;
      }
      float* dst = dense ? dV + (int64_t)h.r * d_v : (dVc ? dVc + (int64_t)h.u * d_v : nullptr);
      if (dst) {
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
          const int c = lane + 32 * j;
          if (c < nv4) st_f4_hint(dst + 4 * c, acc[j], pol_stream);
        }
      }
      if (rows_out && lane == 0) rows_out[h.u] = h.r;
    }
    __syncwarp();  // every lane is done with slot b before it is refilled
    if (lane == 0 && issued < nrows) {
      issue(issued);
      ++issued;
    }
  }
  // after an abort: the copies of rows n .. issued-1 (one per slot) land before the
  // warp exits, each waited for with a bounded wait
  if (n < nrows && lane == 0) {
    for (int64_t m = n; m < issued; ++m) {
      const int b = (int)(m % depth);
      const uint32_t par = (uint32_t)((m / depth) & 1);
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(&full[wid][b], par) && clock64() - t0 < tc::kWaitBudgetCycles) {
      }
    }
  }
}

}  // namespace
}  // namespace pkm
