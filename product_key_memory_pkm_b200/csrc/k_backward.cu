// Backward of the product-key memory layer with the selected keys held fixed
// (the top-k is piecewise constant; "Meta AI 可扩展内存层" 6.1 and 9.2: only the
// selected slots receive gradient, and the top-k passes gradient only to the
// selected positions).
//
//   B1-B2  sort the N*h*k selections by value row (stable LSD radix), segment table
//   B3     one warp per distinct row r: read V[r] once, for each selection e of r
//          dw[e] = dy[t] . V[r] and acc += w[e] * dy[t]; then dV[r] += acc
//          (duplicates combined before the single write; no atomics)
//   B4     one warp per (t, h): dS = w (dw - sum w dw), g1/g2 = score_scale * dS
//          summed onto the selected sub-keys of each half
//   B5     dq_half = sum_a g[a] C[i_a];  BatchNorm backward dq_pre = dq gamma /
//          sqrt(var + eps); d gamma, d beta by deterministic two-stage reduction
//          dC[i] += sum over (t, a) choosing i of g * q_half[t]  (sorted segments)
//   B7     dx = dq_pre Wq,  dWq += dq_pre^T x
#include <cmath>

#include "k_sort.cuh"
#include "k_value_rows.cuh"
#include "tc_common.cuh"

namespace pkm {
namespace {

// Fast-weight write ("Fast-weight Product Key Memory", section 2.2: the chunk's
// reconstruction loss is descended by sparse gradient steps on the selected value
// rows): for each distinct row r, V[r] <- V[r] - lr * sum_{selections e of r}
// w_e * dy[t_e].  One 256-thread CTA per row (grid-stride), thread j owning float4
// columns j, j + 256, ...; the row's selections are taken in row order (stable
// sort), four at a time so four dy lines are in flight.  One writer per row: no
// atomics, deterministic.  fp32 tables only.
//
// kAdam: the same pass applies lazy Adam instead ("Meta AI 可扩展内存层" section 6.3:
// optimiser state only for rows that received a gradient): with g the row's gradient,
// m <- b1 m + (1 - b1) g, v <- b2 v + (1 - b2) g^2, V <- V - lr (m / bc1) / (sqrt(v / bc2)
// + eps), bc = 1 - beta^step; m and v are fp32 tables shaped like V.
constexpr int kSgdThreads = 256;

struct AdamArgs {
  float* m;
  float* v;
  float b1, b2, eps, inv_bc1, inv_bc2;
};

//
// The segments may carry composite keys (chunk * K + row, sorted once for a whole
// sequence): then `bounds` gives this chunk's segment range [bounds[0], bounds[1]) and
// the row is key - key_base.  Without bounds the range is [0, U) and key_base is 0.
template <bool kAdam>
__global__ void __launch_bounds__(kSgdThreads) rows_step_kernel(
    const int* __restrict__ seg, const int* __restrict__ U_ptr,
    const int32_t* __restrict__ seg_row, const int32_t* __restrict__ ents,
    const float* __restrict__ ws_sorted, const float* __restrict__ dy, float* __restrict__ V,
    float lr, int hk, int d_v, int64_t K, int* status, const int* __restrict__ bounds,
    int64_t key_base, AdamArgs ad) {
  grid_dependency_wait();  // the residual (and the table's last reader) precede this write
  allow_dependent_launch();
  const int u0 = bounds ? bounds[0] : 0;
  const int u1 = bounds ? bounds[1] : *U_ptr;
  const int nvec = d_v / 4;
  for (int u = u0 + blockIdx.x; u < u1; u += gridDim.x) {
    const int64_t r = (int64_t)seg_row[u] - key_base;
    if (r < 0 || r >= K) {
      if (threadIdx.x == 0) set_status(status, kDevIndex);
      continue;
    }
    const int p0 = seg[u], p1 = seg[u + 1];
    float4* Vr = reinterpret_cast<float4*>(V + (int64_t)r * d_v);
    for (int c = threadIdx.x; c < nvec; c += kSgdThreads) {
      const float4 v = Vr[c];
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int q = p0;
      for (; q + 4 <= p1; q += 4) {
        float4 d[4];
        float wt[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          wt[i] = ws_sorted[q + i];
          d[i] = reinterpret_cast<const float4*>(dy + (int64_t)(ents[q + i] / hk) * d_v)[c];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc.x = fmaf(wt[i], d[i].x, acc.x); acc.y = fmaf(wt[i], d[i].y, acc.y);
          acc.z = fmaf(wt[i], d[i].z, acc.z); acc.w = fmaf(wt[i], d[i].w, acc.w);
        }
      }
      for (; q < p1; ++q) {
        const float wt = ws_sorted[q];
        const float4 d = reinterpret_cast<const float4*>(dy + (int64_t)(ents[q] / hk) * d_v)[c];
        acc.x = fmaf(wt, d.x, acc.x); acc.y = fmaf(wt, d.y, acc.y);
        acc.z = fmaf(wt, d.z, acc.z); acc.w = fmaf(wt, d.w, acc.w);
      }
      if constexpr (kAdam) {
        float4* Mr = reinterpret_cast<float4*>(ad.m + r * d_v);
        float4* Sr = reinterpret_cast<float4*>(ad.v + r * d_v);
        float4 m = Mr[c], s = Sr[c];
        const float g[4] = {acc.x, acc.y, acc.z, acc.w};
        float* mm = &m.x;
        float* ss = &s.x;
        float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mm[i] = fmaf(ad.b1, mm[i], (1.f - ad.b1) * g[i]);
          ss[i] = fmaf(ad.b2, ss[i], (1.f - ad.b2) * g[i] * g[i]);
          vv[i] -= lr * (mm[i] * ad.inv_bc1) / (sqrtf(ss[i] * ad.inv_bc2) + ad.eps);
        }
        Mr[c] = m;
        Sr[c] = s;
        Vr[c] = make_float4(vv[0], vv[1], vv[2], vv[3]);
      } else {
        Vr[c] = make_float4(fmaf(-lr, acc.x, v.x), fmaf(-lr, acc.y, v.y),
                            fmaf(-lr, acc.z, v.z), fmaf(-lr, acc.w, v.w));
      }
    }
  }
}


// ------------------------------------------------------------------ B4 (inverse distance)
__global__ void idw_scale_kernel(float* __restrict__ gsub, const float* __restrict__ sub_s,
                                 int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    gsub[i] *= expf(2.f * sub_s[i]);
}

// ------------------------------------------------------------------ B4 (all-k^2 variant)
// Every candidate (a, b) of the k x k grid is selected: dS_ab = scale w_ab (dw_ab -
// sum w dw); the first half's a-th sub-key collects the row sum over b, the second
// half's b-th the column sum over a.  One warp per (token, head).
__global__ void __launch_bounds__(256) softmax_bwd_all_kernel(
    const float* __restrict__ w, const float* __restrict__ dw, float* __restrict__ gsub,
    int64_t NH, int k, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= NH) return;
  const int kk = k * k;
  const float* wg = w + g * kk;
  const float* dg = dw + g * kk;
  float s = 0.f;
  for (int c = lane; c < kk; c += 32) s = fmaf(wg[c], dg[c], s);
  s = warp_sum(s);
  for (int a = lane; a < k; a += 32) {
    float g1 = 0.f, g2 = 0.f;
    for (int j = 0; j < k; ++j) {
      const int ca = a * k + j, cb = j * k + a;
      g1 += scale * wg[ca] * (dg[ca] - s);
      g2 += scale * wg[cb] * (dg[cb] - s);
    }
    gsub[g * 2 * k + a] = g1;
    gsub[g * 2 * k + k + a] = g2;
  }
}

// ------------------------------------------------------------------ B4
// One warp per (token, head); lane j holds winners j and j + 32 (R = 2, for k > 32).
// dS_j = scale w_j (dw_j - sum w dw); the first half's a-th sub-key collects dS_j of the
// winners that use it (and likewise the second half's b-th), summed in winner order.
template <int R>
__global__ void __launch_bounds__(256) softmax_bwd_kernel(
    const float* __restrict__ w, const float* __restrict__ dw, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ sub_i, float* __restrict__ gsub, int64_t NH, int k, int C2,
    float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (g >= NH) return;
  bool live[R];
  float wj[R], dwj[R], dsum[R], g1[R], g2[R];
  int32_t I[R], J[R], ia[R], jb[R];
  float part = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = lane + 32 * r;
    live[r] = j < k;
    wj[r] = live[r] ? w[g * k + j] : 0.f;
    dwj[r] = live[r] ? dw[g * k + j] : 0.f;
    const int32_t ij = live[r] ? idx[g * k + j] : 0;
    I[r] = ij / C2;
    J[r] = ij % C2;
    ia[r] = live[r] ? sub_i[g * 2 * k + j] : -1;
    jb[r] = live[r] ? sub_i[g * 2 * k + k + j] : -1;
    part = fmaf(wj[r], dwj[r], part);
    g1[r] = g2[r] = 0.f;
  }
  const float s = warp_sum(part);
#pragma unroll
  for (int r = 0; r < R; ++r) dsum[r] = scale * wj[r] * (dwj[r] - s);
#pragma unroll
  for (int rs = 0; rs < R; ++rs) {  // winners 32 rs ... 32 rs + 31, in order
    const int n = min(32, k - 32 * rs);
    for (int j = 0; j < n; ++j) {
      const int32_t Ij = __shfl_sync(kFull, I[rs], j);
      const int32_t Jj = __shfl_sync(kFull, J[rs], j);
      const float D = __shfl_sync(kFull, dsum[rs], j);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (ia[r] == Ij) g1[r] += D;
        if (jb[r] == Jj) g2[r] += D;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (live[r]) {
      gsub[g * 2 * k + lane + 32 * r] = g1[r];
      gsub[g * 2 * k + k + lane + 32 * r] = g2[r];
    }
  }
}

// ------------------------------------------------------------------ B5a + B6
// grid (token blocks, h*2); 8 warps, each warp walks tokens; lane owns 16-byte
// chunks of the half (MAXC chunks at most).  Writes dq_pre (fp32) and per-block
// partial sums of dq * qhat and dq for the BatchNorm affine gradients.
constexpr int kDqTokensPerBlock = 64;

template <typename TS, int MAXC, bool kSplit>
__global__ void __launch_bounds__(256) dq_kernel(
    const float* __restrict__ gsub, const int32_t* __restrict__ sub_i, const TS* __restrict__ sub,
    const float* __restrict__ bn, const float* __restrict__ qhat, void* __restrict__ dq_out,
    float* __restrict__ part, int64_t N, int h, int dk, int C1, int C2, int k, float eps,
    const void* __restrict__ q_idw) {
  // q_idw (inverse-distance scores; gsub then holds u = g / ||q - c||^2): subtract
  // q * sum_a u_a, q read from the saved query (bf16 hi + lo planes, or fp32)
  constexpr int E = VecT<TS>::E;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int hs = blockIdx.y, hh = hs >> 1, s = hs & 1;
  const int half = dk / 2, hq = h * dk;
  const int nvec = half / E;
  const TS* Cb = sub + ((int64_t)hh * (C1 + C2) + (s ? C1 : 0)) * half;
  const int col0 = hh * dk + s * half;
  float pg[MAXC][E], pb[MAXC][E];
#pragma unroll
  for (int c = 0; c < MAXC; ++c)
#pragma unroll
    for (int e = 0; e < E; ++e) pg[c][e] = pb[c][e] = 0.f;
  const int64_t tb = (int64_t)blockIdx.x * kDqTokensPerBlock;
  for (int tt = wid; tt < kDqTokensPerBlock; tt += 8) {
    const int64_t t = tb + tt;
    if (t >= N) break;
    const int64_t gb = ((t * h + hh) * 2 + s) * k;
    float acc[MAXC][E];
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
    float usum = 0.f;
    for (int a = 0; a < k; ++a) {
      const float ga = gsub[gb + a];
      usum += ga;
      const int32_t row = sub_i[gb + a];
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int vec = lane + 32 * c;
        if (vec < nvec) {
          float f[E];
          VecT<TS>::load(Cb + (int64_t)row * half + vec * E, f);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[c][e] = fmaf(ga, f[e], acc[c][e]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int vec = lane + 32 * c;
      if (vec < nvec) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int col = col0 + vec * E + e;
          if (q_idw) {
            float qv;
            if constexpr (E == 8) {
              const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q_idw);
              qv = __bfloat162float(qb[t * hq + col]) + __bfloat162float(qb[N * hq + t * hq + col]);
            } else {
              qv = static_cast<const float*>(q_idw)[t * hq + col];
            }
            acc[c][e] = fmaf(-usum, qv, acc[c][e]);
          }
          const float gam = bn[2 * hq + col], var = bn[hq + col];
          const float val = acc[c][e] * gam / sqrtf(var + eps);
          if constexpr (kSplit) {
            // dq_pre as two bf16 planes [2][N][hq]: hi = bf16(v), lo = bf16(v - hi)
            __nv_bfloat16* pl = static_cast<__nv_bfloat16*>(dq_out);
            const __nv_bfloat16 hi = __float2bfloat16_rn(val);
            pl[t * hq + col] = hi;
            pl[N * hq + t * hq + col] = __float2bfloat16_rn(val - __bfloat162float(hi));
          } else {
            static_cast<float*>(dq_out)[t * hq + col] = val;
          }
          if (qhat) pg[c][e] = fmaf(acc[c][e], qhat[t * hq + col], pg[c][e]);
          pb[c][e] += acc[c][e];
        }
      }
    }
  }
  if (!part) return;
  // reduce partials over the 8 warps in a fixed order
  __shared__ float red[8][2][32 * 8];
  for (int c = 0; c < MAXC; ++c) {
    const int vec = lane + 32 * c;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      red[wid][0][lane * E + e] = pg[c][e];
      red[wid][1][lane * E + e] = pb[c][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) {
      float sg = 0.f, sb = 0.f;
      for (int ww = 0; ww < 8; ++ww) {
        sg += red[ww][0][i];
        sb += red[ww][1][i];
      }
      const int v2 = i / E + 32 * c;
      if (v2 < nvec) {
        const int col = col0 + v2 * E + (i % E);
        part[((int64_t)blockIdx.x * 2 + 0) * hq + col] = sg;
        part[((int64_t)blockIdx.x * 2 + 1) * hq + col] = sb;
      }
    }
    __syncthreads();
    (void)vec;
  }
}

// dbn[which][c] += sum over the nblk partial rows, in a fixed order: 32 columns per
// block (lane = column), 32 warps; warp w sums the rows b = w, w + 32, ... in four running
// sums (rows w + 32 (4 m + i) into sum i), then the 32 warp sums are added in warp order.
constexpr int kDbnWarps = 32;
__global__ void __launch_bounds__(kDbnWarps * 32) dbn_reduce_kernel(const float* __restrict__ part,
                                                                    int nblk, int hq,
                                                                    float* __restrict__ dbn) {
  __shared__ float red[kDbnWarps][32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  const bool live = col < 2 * hq;
  const int which = live ? col / hq : 0, c = live ? col % hq : 0;
  float s4[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    for (int b0 = wid; b0 < nblk; b0 += 4 * kDbnWarps) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = b0 + kDbnWarps * i;
        if (b < nblk) s4[i] += part[((int64_t)b * 2 + which) * hq + c];
      }
    }
  }
  red[wid][lane] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  __syncthreads();
  if (wid == 0 && live) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kDbnWarps; ++w) t += red[w][lane];
    dbn[which * hq + c] += t;
  }
}

// ------------------------------------------------------------------ B5b keys
__global__ void subkey_keys_kernel(const int32_t* __restrict__ sub_i, int32_t* __restrict__ keys,
                                   int64_t n, int h, int k, int C1, int C2) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int s = (int)((e / k) % 2);
  const int hh = (int)((e / (2 * k)) % h);
  keys[e] = hh * (C1 + C2) + (s ? C1 : 0) + sub_i[e];
}

// ------------------------------------------------------------------ B5b
template <bool kSplitQ, int MAXC>
__global__ void __launch_bounds__(256) subkey_grad_kernel(
    const int* __restrict__ seg, const int* __restrict__ U_ptr, const int32_t* __restrict__ rows,
    const int32_t* __restrict__ ents, const float* __restrict__ gsub, const void* __restrict__ q,
    float* __restrict__ dsub, int64_t N, int h, int dk, int C1, int C2, int k, int* status,
    float lo_scale, const void* __restrict__ sub_idw) {
  // sub_idw (inverse-distance scores; gsub holds u): subtract c_R * sum u over the segment
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int U = *U_ptr;
  const int half = dk / 2, hq = h * dk;
  constexpr int E = kSplitQ ? 8 : 4;
  const int nvec = half / E;
  const int64_t plane = N * hq;
  const int rows_total = h * (C1 + C2);
  for (int64_t u = warp0; u < U; u += nwarps) {
    const int p0 = seg[u], p1 = seg[u + 1];
    const int32_t R = rows[p0];
    if (R < 0 || R >= rows_total) {
      set_status(status, kDevIndex);
      continue;
    }
    const int hh = R / (C1 + C2);
    const int s = (R % (C1 + C2)) >= C1 ? 1 : 0;
    const int64_t colb = (int64_t)hh * dk + s * half;
    float acc[MAXC][E];
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[c][e] = 0.f;
    float usum = 0.f;
    for (int p = p0; p < p1; ++p) {
      const int32_t ent = ents[p];
      const int64_t t = ent / (2 * h * k);
      const float gv = gsub[ent];
      usum += gv;
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int vec = lane + 32 * c;
        if (vec < nvec) {
          float f[E];
          const int64_t off = t * hq + colb + (int64_t)vec * E;
          if constexpr (kSplitQ) {
            const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
            float lo[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + off), f);
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(qb + plane + off), lo);
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] += lo_scale * lo[e];
          } else {
            float4 u4 = *reinterpret_cast<const float4*>(static_cast<const float*>(q) + off);
            f[0] = u4.x; f[1] = u4.y; f[2] = u4.z; f[3] = u4.w;
          }
#pragma unroll
          for (int e = 0; e < E; ++e) acc[c][e] = fmaf(gv, f[e], acc[c][e]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int vec = lane + 32 * c;
      if (vec < nvec) {
        float* o = dsub + (int64_t)R * half + (int64_t)vec * E;
        if (sub_idw) {
          const int64_t so = (int64_t)R * half + (int64_t)vec * E;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float cv = kSplitQ
                                 ? __bfloat162float(static_cast<const __nv_bfloat16*>(sub_idw)[so + e])
                                 : static_cast<const float*>(sub_idw)[so + e];
            acc[c][e] = fmaf(-usum, cv, acc[c][e]);
          }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] += acc[c][e];
      }
    }
  }
}

inline int bits_for(int64_t maxkey) {
  int b = 1;
  while (b < 31 && ((int64_t)1 << b) <= maxkey) ++b;
  return b;
}

// ------------------------------------------------------------------ workspace
struct Layout {
  size_t keysA, valsA, keysB, valsB, hist, bsum, seg, segrow, wsorted, U, dw, gsub, dq, part,
      G, dspart, bneff, bntot, total;
};

inline size_t up256(size_t v) { return (v + 255) & ~size_t(255); }

Layout layout(const Plan& p) {
  Layout L{};
  // E1 selections (value pass), E2 per-half list entries (sub-key pass)
  const int64_t E1 = p.N * p.h * p.ksel, E2 = 2 * p.N * p.h * p.k;
  const int64_t En = std::max(E1, E2);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t r = o;
    o += up256(bytes);
    return r;
  };
  L.keysA = take(4 * En);
  L.valsA = take(4 * En);
  L.keysB = take(4 * En);
  L.valsB = take(4 * En);
  const int64_t hl = sort::radix_hist_len(En);
  L.hist = take(4 * hl);
  const int64_t bl = std::max(sort::scan_bsum_len(hl), sort::scan_bsum_len(En));
  L.bsum = take(4 * bl);
  L.seg = take(4 * (En + 1));
  L.segrow = take(4 * (En + 1));
  L.wsorted = take(4 * E1);
  L.U = take(4);
  L.dw = take(4 * E1);
  L.gsub = take(4 * E2);
  L.dq = take(4 * p.N * p.hq);
  // BatchNorm partial sums: 64-token blocks (CUDA-core path) or 32-token blocks (fused
  // into the tensor-core dq GEMM)
  const int64_t nblk = std::max((p.N + kDqTokensPerBlock - 1) / kDqTokensPerBlock,
                                subgrad_part_blocks(p.N));
  L.part = take(4 * nblk * 2 * p.hq);
  if (!p.fp32) {  // tensor-core sub-key gradients: dense G planes, split partials
    L.G = take(2 * (size_t)(2 * p.h) * 2 * subgrad_pad_tokens(p.N) * subgrad_pad_keys(p.C1, p.C2));
    L.dspart = take(4 * subgrad_partial_floats(p));
  }
  L.bneff = take(4 * 4 * (size_t)p.hq);  // training-mode BatchNorm: (mean, var, gamma, beta)
  L.bntot = take(4 * 2 * (size_t)p.hq);  // and the column sums (d gamma, d beta)
  L.total = o;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

}  // namespace

size_t backward_workspace_bytes(const Plan& p) { return layout(p).total; }

size_t value_stage_scratch_bytes(const Plan& p) { return layout(p).U + 4; }

struct BwdCtx {
  sort::RadixBuffers rb;
  int* seg;
  int32_t* seg_row;
  float* w_sorted;
  int* U;
  float* dw;
  float* gsub;
  float* dq_pre;
  float* part;
  __nv_bfloat16* G;
  float* dspart;
  float* bneff;
  float* bntot;
};

static BwdCtx bwd_ctx(const Plan& p, void* ws, float* dw_out) {
  const Layout L = layout(p);
  BwdCtx c;
  c.rb = sort::RadixBuffers{at<int32_t>(ws, L.keysA), at<int32_t>(ws, L.valsA),
                            at<int32_t>(ws, L.keysB), at<int32_t>(ws, L.valsB),
                            at<int>(ws, L.hist), at<int>(ws, L.bsum)};
  c.seg = at<int>(ws, L.seg);
  c.seg_row = at<int32_t>(ws, L.segrow);
  c.w_sorted = at<float>(ws, L.wsorted);
  c.U = at<int>(ws, L.U);
  c.dw = dw_out ? dw_out : at<float>(ws, L.dw);
  c.gsub = at<float>(ws, L.gsub);
  c.dq_pre = at<float>(ws, L.dq);
  c.part = at<float>(ws, L.part);
  c.G = at<__nv_bfloat16>(ws, L.G);
  c.dspart = at<float>(ws, L.dspart);
  c.bneff = at<float>(ws, L.bneff);
  c.bntot = at<float>(ws, L.bntot);
  return c;
}

// B1-B2: the selections sorted by value row (stable radix sort), the segment table of
// the distinct rows and the weights in row order, all in the workspace.
// The weights ride through the sort beside their selections (read in entry order, written
// in runs), so no pass gathers them at random; wtmp (E1 floats: the caller's dw, which
// the row pass overwrites, else the workspace's) holds them between passes.
cudaError_t launch_value_sort(const Plan& p, const pkm_saved& s, void* ws, cudaStream_t st,
                              float* wtmp) {
  const int64_t E1 = p.N * p.h * p.ksel;
  BwdCtx c = bwd_ctx(p, ws, wtmp);
  const int32_t *rows_sorted, *ents_sorted;
  cudaError_t e = sort::radix_sort(s.idx, E1, bits_for(p.K - 1), c.rb, &rows_sorted,
                                   &ents_sorted, st, s.w, c.dw, c.w_sorted);
  if (e != cudaSuccess) return e;
  return sort::segments(rows_sorted, E1, c.seg, c.U, c.rb.bsum, st, c.seg_row);
}

// B3: one pass per distinct value row over what launch_value_sort left in the workspace.
cudaError_t launch_value_rows(const Plan& p, const void* values, const float* dy, float* dV,
                              float* dw_out, void* ws, cudaStream_t st, float* dVc,
                              int32_t* rows_out, int* U_out, const int32_t* ent_tok) {
  BwdCtx c = bwd_ctx(p, ws, dw_out);
  const int32_t* ents_sorted = sort::radix_sorted_vals(c.rb, bits_for(p.K - 1));
  const int hk = p.h * p.ksel;
  cudaError_t e;
  const int E = p.vfp32 ? 4 : 8;
  const int nvec = p.d_v / E;
  const int blocks = p.sm_count * PKM_B3_MIN_BLOCKS;
  const size_t smem = value_rows_smem(p);
#define PKM_B3(TV, CHV)                                                                      \
  do {                                                                                       \
    if (smem > 48 * 1024 &&                                                                  \
        (e = cudaFuncSetAttribute(value_rows_kernel<TV, CHV>,                                \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != \
            cudaSuccess)                                                                     \
      return e;                                                                              \
    value_rows_kernel<TV, CHV><<<blocks, kB3Threads, smem, st>>>(                            \
        c.seg, c.U, c.seg_row, ents_sorted, static_cast<const TV*>(values), c.w_sorted, dy,  \
        dV, c.dw, hk, p.d_v, p.K, p.status, dVc, rows_out, U_out, ent_tok);                  \
  } while (0)
  if (p.vfp32) {
    if (nvec <= kB3Threads) PKM_B3(float, 1);
    else PKM_B3(float, 2);
  } else {
    if (nvec <= kB3Threads) PKM_B3(__nv_bfloat16, 1);
    else PKM_B3(__nv_bfloat16, 2);
  }
#undef PKM_B3
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_value_grad(const Plan& p, const void* values, const pkm_saved& s,
                              const float* dy, float* dV, float* dw_out, void* ws,
                              cudaStream_t st, float* dVc, int32_t* rows_out, int* U_out,
                              const int32_t* ent_tok) {
  cudaError_t e = launch_value_sort(p, s, ws, st, dw_out);
  if (e != cudaSuccess) return e;
  return launch_value_rows(p, values, dy, dV, dw_out, ws, st, dVc, rows_out, U_out, ent_tok);
}

cudaError_t launch_value_sgd(const Plan& p, float* values, const pkm_saved& s, const float* dy,
                             float lr, void* ws, cudaStream_t st) {
  const int64_t E1 = p.N * p.h * p.ksel;
  if (fw_chunk_sort_fits(p, p.N)) {  // few selections: one CTA sorts them in shared memory
    cudaError_t e = launch_fw_chunk_sort(p, p.N, s.idx, s.w, ws, st);
    if (e != cudaSuccess) return e;
    return launch_fw_chunk_write(p, p.N, 0, ws, dy, values, lr, st);
  }
  BwdCtx c = bwd_ctx(p, ws, nullptr);
  cudaError_t e;
  const int32_t *rows_sorted, *ents_sorted;
  e = sort::radix_sort(s.idx, E1, bits_for(p.K - 1), c.rb, &rows_sorted, &ents_sorted, st);
  if (e != cudaSuccess) return e;
  e = sort::segments(rows_sorted, E1, c.seg, c.U, c.rb.bsum, st, c.seg_row, ents_sorted, s.w,
                     c.w_sorted);
  if (e != cudaSuccess) return e;
  const int64_t blocks = std::min<int64_t>(E1, (int64_t)p.sm_count * 8);
  rows_step_kernel<false><<<(unsigned)blocks, kSgdThreads, 0, st>>>(
      c.seg, c.U, c.seg_row, ents_sorted, c.w_sorted, dy, values, lr, p.h * p.ksel, p.d_v, p.K,
      p.status, nullptr, 0, AdamArgs{});
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_value_adam(const Plan& p, float* values, float* m, float* v,
                              const pkm_saved& s, const float* dy, float lr, float beta1,
                              float beta2, float eps, int64_t step, void* ws, cudaStream_t st) {
  const int64_t E1 = p.N * p.h * p.ksel;
  BwdCtx c = bwd_ctx(p, ws, nullptr);
  cudaError_t e;
  const int32_t *rows_sorted, *ents_sorted;
  e = sort::radix_sort(s.idx, E1, bits_for(p.K - 1), c.rb, &rows_sorted, &ents_sorted, st);
  if (e != cudaSuccess) return e;
  e = sort::segments(rows_sorted, E1, c.seg, c.U, c.rb.bsum, st, c.seg_row, ents_sorted, s.w,
                     c.w_sorted);
  if (e != cudaSuccess) return e;
  AdamArgs ad{m, v, beta1, beta2, eps,
              (float)(1.0 / (1.0 - std::pow((double)beta1, (double)step))),
              (float)(1.0 / (1.0 - std::pow((double)beta2, (double)step)))};
  const int64_t blocks = std::min<int64_t>(E1, (int64_t)p.sm_count * 8);
  rows_step_kernel<true><<<(unsigned)blocks, kSgdThreads, 0, st>>>(
      c.seg, c.U, c.seg_row, ents_sorted, c.w_sorted, dy, values, lr, p.h * p.ksel, p.d_v, p.K,
      p.status, nullptr, 0, ad);
  PKM_COUNT(1);
  return cudaGetLastError();
}

// Hit monitoring ("Meta AI 可扩展内存层" sections 6.4 and 11.2): one thread per
// selection adds 1 to its slot and to the two sub-keys of its head.  Integer atomics:
// the counts do not depend on the order.
namespace {
__global__ void hit_counts_kernel(const int32_t* __restrict__ idx, int64_t E, int h, int k,
                                  int C1, int C2, int64_t K, int32_t* __restrict__ slot,
                                  int32_t* __restrict__ sub, int* status) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < E;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int32_t r = idx[e];
    if (r < 0 || r >= K) {
      set_status(status, kDevIndex);
      continue;
    }
    if (slot) atomicAdd(slot + r, 1);
    if (sub) {
      const int hh = (int)((e / k) % h);
      int32_t* row = sub + (int64_t)hh * (C1 + C2);
      atomicAdd(row + r / C2, 1);
      atomicAdd(row + C1 + r % C2, 1);
    }
  }
}
}  // namespace

cudaError_t launch_hit_counts(const Plan& p, const int32_t* idx, int32_t* slot, int32_t* sub,
                              cudaStream_t st) {
  const int64_t E = p.N * p.h * p.ksel;
  const int64_t blocks = std::min<int64_t>((E + 255) / 256, (int64_t)p.sm_count * 16);
  hit_counts_kernel<<<(unsigned)blocks, 256, 0, st>>>(idx, E, p.h, p.ksel, p.C1, p.C2, p.K, slot,
                                                      sub, p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

// ---- a whole sequence's writes sorted at once (the selection does not read the table)
namespace {

__global__ void fw_keys_kernel(const int32_t* __restrict__ idx, int64_t E, int hk, int64_t chunk,
                               int64_t K, int32_t* __restrict__ keys, int* status) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int64_t c = (e / hk) / chunk;
  int64_t r = idx[e];
  if (r < 0 || r >= K) {
    set_status(status, kDevIndex);
    r = 0;
  }
  keys[e] = (int32_t)(c * K + r);
}

// bounds[c] = first segment whose key is >= c * K (lower bound), c in [0, nch]
__global__ void fw_bounds_kernel(const int32_t* __restrict__ seg_key, const int* __restrict__ U_ptr,
                                 int nch, int64_t K, int* __restrict__ bounds) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c > nch) return;
  const int U = *U_ptr;
  const int64_t want = (int64_t)c * K;
  int lo = 0, hi = U;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)seg_key[mid] < want) lo = mid + 1;
    else hi = mid;
  }
  bounds[c] = lo;
}

// One CTA per chunk sorts the chunk's selections by value row in shared memory (the
// selections of a chunk are contiguous) and writes the chunk's segment table at a fixed
// stride: seg[u] (position of the u-th distinct row's first selection), seg_row[u],
// seg[U_c] = n_c, U_c; ents[i] (global selection id) and w_sorted[i] in row order.
// Keys are (row << 32 | local selection id), so a bitonic network over unique keys
// gives the stable order (rows ascending, selections of a row in id order).
constexpr int kFwSortThreads = 1024, kFwSortMax = 16384;

__global__ void __launch_bounds__(kFwSortThreads) fw_chunk_sort_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t N, int64_t chunk,
    int hk, int64_t K, int stride, int npow2, int* __restrict__ seg,
    int32_t* __restrict__ seg_row, int32_t* __restrict__ ents, float* __restrict__ w_sorted,
    int* __restrict__ U_out, int* status) {
  extern __shared__ __align__(16) unsigned long long fw_keys[];
  __shared__ int warp_tot[kFwSortThreads / 32];
  const int c = blockIdx.x, tid = threadIdx.x;
  const int64_t t0 = (int64_t)c * chunk;
  const int64_t nt = (N - t0 < chunk) ? N - t0 : chunk;
  const int n = (int)(nt * hk);
  const int64_t e0 = t0 * hk;
  const int64_t base = (int64_t)c * stride;
  for (int i = tid; i < npow2; i += kFwSortThreads) {
    unsigned long long key = ~0ull;
    if (i < n) {
      int64_t r = idx[e0 + i];
      if (r < 0 || r >= K) {
        set_status(status, kDevIndex);
        r = 0;
      }
      key = ((unsigned long long)r << 32) | (unsigned)i;
    }
    fw_keys[i] = key;
  }
  __syncthreads();
  // A stage with distance `half` <= 32 pairs elements inside the 64-element blocks that
  // one warp's 32 consecutive pair indices cover, so between two such stages a warp
  // barrier suffices; a block barrier is needed around stages of larger distance.
  for (int size = 2; size <= npow2; size <<= 1) {
    for (int half = size >> 1; half > 0; half >>= 1) {
      for (int j = tid; j < (npow2 >> 1); j += kFwSortThreads) {
        const int lo = 2 * j - (j & (half - 1));
        const int hi = lo + half;
        const bool up = (lo & size) == 0;
        const unsigned long long a = fw_keys[lo], b = fw_keys[hi];
        if ((a > b) == up) {
          fw_keys[lo] = b;
          fw_keys[hi] = a;
        }
      }
      const int next_half = half == 1 ? size : half >> 1;
      if (half > 32 || next_half > 32)
        __syncthreads();
      else
        __syncwarp();
    }
  }
  __syncthreads();
  // segment starts: block-wide exclusive scan of the start flags over thread-owned runs
  const int per = (n + kFwSortThreads - 1) / kFwSortThreads;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int cnt = 0;
  for (int i = i0; i < i1; ++i)
    cnt += (i == 0 || (fw_keys[i] >> 32) != (fw_keys[i - 1] >> 32)) ? 1 : 0;
  const int lane = tid & 31, wid = tid >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int v = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    warp_tot[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int u = incl - cnt + (wid ? warp_tot[wid - 1] : 0);
  for (int i = i0; i < i1; ++i) {
    const unsigned long long key = fw_keys[i];
    const int32_t row = (int32_t)(key >> 32);
    if (i == 0 || row != (int32_t)(fw_keys[i - 1] >> 32)) {
      seg[base + u] = i;
      seg_row[base + u] = row;
      ++u;
    }
    const int64_t e = e0 + (int64_t)(unsigned)(key & 0xffffffffu);
    ents[base + i] = (int32_t)e;
    w_sorted[base + i] = w[e];
  }
  if (tid == kFwSortThreads - 1) {
    const int U = warp_tot[kFwSortThreads / 32 - 1];
    seg[base + U] = n;
    U_out[c] = U;
  }
}

}  // namespace

bool fw_presort_fits(const Plan& p, int64_t chunk) {
  const int64_t nch = (p.N + chunk - 1) / chunk;
  return nch * p.K < ((int64_t)1 << 31);
}

cudaError_t launch_fw_presort(const Plan& p, int64_t chunk, const int32_t* idx, const float* w,
                              int32_t* keys, int* bounds, void* ws, cudaStream_t st) {
  const int64_t E1 = p.N * p.h * p.ksel;
  const int64_t nch = (p.N + chunk - 1) / chunk;
  BwdCtx c = bwd_ctx(p, ws, nullptr);
  fw_keys_kernel<<<(unsigned)((E1 + 255) / 256), 256, 0, st>>>(idx, E1, p.h * p.ksel, chunk, p.K,
                                                               keys, p.status);
  PKM_COUNT(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int32_t *keys_sorted, *ents_sorted;
  e = sort::radix_sort(keys, E1, bits_for(nch * p.K - 1), c.rb, &keys_sorted, &ents_sorted, st);
  if (e != cudaSuccess) return e;
  e = sort::segments(keys_sorted, E1, c.seg, c.U, c.rb.bsum, st, c.seg_row, ents_sorted, w,
                     c.w_sorted);
  if (e != cudaSuccess) return e;
  fw_bounds_kernel<<<(unsigned)((nch + 1 + 255) / 256), 256, 0, st>>>(c.seg_row, c.U, (int)nch,
                                                                      p.K, bounds);
  PKM_COUNT(1);
  return cudaGetLastError();
}

bool fw_chunk_sort_fits(const Plan& p, int64_t chunk) {
  return std::min<int64_t>(chunk, p.N) * p.h * p.ksel <= kFwSortMax;
}

size_t fw_chunk_sort_bytes(const Plan& p, int64_t chunk) {
  const int64_t nch = (p.N + chunk - 1) / chunk;
  const int64_t stride = std::min<int64_t>(chunk, p.N) * p.h * p.ksel + 1;
  // seg, seg_row, ents, w_sorted at `stride` per chunk, then U per chunk
  return (size_t)(4 * 4 * nch * stride + 4 * nch);
}

cudaError_t launch_fw_chunk_sort(const Plan& p, int64_t chunk, const int32_t* idx, const float* w,
                                 void* buf, cudaStream_t st) {
  const int64_t nch = (p.N + chunk - 1) / chunk;
  const int n_max = (int)(std::min<int64_t>(chunk, p.N) * p.h * p.ksel);
  const int stride = n_max + 1;
  int npow2 = 1;
  while (npow2 < n_max) npow2 <<= 1;
  int* seg = static_cast<int*>(buf);
  int32_t* seg_row = seg + nch * stride;
  int32_t* ents = seg_row + nch * stride;
  float* w_sorted = reinterpret_cast<float*>(ents + nch * stride);
  int* U = reinterpret_cast<int*>(w_sorted + nch * stride);
  const size_t smem = (size_t)npow2 * 8;
  cudaError_t e;
  if (smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(fw_chunk_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  fw_chunk_sort_kernel<<<(unsigned)nch, kFwSortThreads, smem, st>>>(
      idx, w, p.N, chunk, p.h * p.ksel, p.K, stride, npow2, seg, seg_row, ents, w_sorted, U,
      p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_fw_chunk_write(const Plan& p, int64_t chunk, int64_t ci, const void* buf,
                                  const float* dy, float* values, float lr, cudaStream_t st) {
  const int64_t nch = (p.N + chunk - 1) / chunk;
  const int n_max = (int)(std::min<int64_t>(chunk, p.N) * p.h * p.ksel);
  const int64_t stride = n_max + 1;
  const int* seg = static_cast<const int*>(buf);
  const int32_t* seg_row = seg + nch * stride;
  const int32_t* ents = seg_row + nch * stride;
  const float* w_sorted = reinterpret_cast<const float*>(ents + nch * stride);
  const int* U = reinterpret_cast<const int*>(w_sorted + nch * stride);
  const int64_t n_c = std::min<int64_t>(chunk, p.N - ci * chunk) * p.h * p.ksel;
  const int64_t blocks = std::min<int64_t>(n_c, (int64_t)p.sm_count * 8);
  const int64_t o = ci * stride;
  PKM_COUNT(1);
  return launch_dependent(rows_step_kernel<false>, dim3((unsigned)blocks), dim3(kSgdThreads), 0,
                          st, seg + o, U + ci, seg_row + o, ents + o, w_sorted + o, dy, values, lr,
                          p.h * p.ksel, p.d_v, p.K, p.status, (const int*)nullptr, (int64_t)0,
                          AdamArgs{});
}

cudaError_t launch_fw_write(const Plan& p, int64_t chunk, int64_t ci, const int* bounds,
                            const float* dy, float* values, float lr, void* ws, cudaStream_t st) {
  BwdCtx c = bwd_ctx(p, ws, nullptr);
  const int32_t* ents_sorted =
      sort::radix_sorted_vals(c.rb, bits_for(((p.N + chunk - 1) / chunk) * p.K - 1));
  const int64_t n_c = std::min<int64_t>(chunk, p.N - ci * chunk);
  const int64_t blocks = std::min<int64_t>(n_c * p.h * p.ksel, (int64_t)p.sm_count * 8);
  PKM_COUNT(1);
  return launch_dependent(rows_step_kernel<false>, dim3((unsigned)blocks), dim3(kSgdThreads), 0,
                          st, c.seg, c.U, c.seg_row, ents_sorted, c.w_sorted, dy, values, lr,
                          p.h * p.ksel, p.d_v, p.K, p.status, bounds + ci, ci * p.K, AdamArgs{});
}

cudaError_t launch_query_grad(const Plan& p, const void* x, const void* Wq, const float* bn,
                              const void* subkeys, const pkm_saved& s, float* dx, float* dWq,
                              float* dbn, float* dsub, float* dw_out, void* ws, cudaStream_t st) {
  if (!(dx || dWq || dbn || dsub)) return cudaSuccess;
  const int64_t E2 = 2 * p.N * p.h * p.k;
  BwdCtx c = bwd_ctx(p, ws, dw_out);
  sort::RadixBuffers& rb = c.rb;
  int* seg = c.seg;
  int* U = c.U;
  const float* dw = c.dw;
  float* gsub = c.gsub;
  float* dq_pre = c.dq_pre;
  float* part = c.part;
  cudaError_t e;
  const int persist_blocks = p.sm_count * 8;
  // Training-mode BatchNorm: the eval-mode kernels below run with the batch statistics,
  // the d gamma / d beta column sums are always formed, and dq_pre is corrected for the
  // statistics' dependence on every token before the dense query gradients.
  const bool train = p.bn_train && (dx || dWq || dbn);
  if (train) {
    if ((e = cudaMemcpyAsync(c.bneff, s.bn_batch, 2 * sizeof(float) * p.hq,
                             cudaMemcpyDeviceToDevice, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(c.bneff + 2 * p.hq, bn + 2 * p.hq, 2 * sizeof(float) * p.hq,
                             cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
      return e;
    bn = c.bneff;
  }
  float* dbn_acc = train ? c.bntot : dbn;  // where the partial column sums are reduced

  // B5 + B6 run on tensor cores (dense G planes) unless the storage or the scorer needs the
  // CUDA-core path; there, with k winners per head, the G row build also computes the
  // softmax backward (B4)
  const bool tc_subgrad = tc_backward_supported(p) && p.half % 64 == 0 && !p.idw;
  const bool fold_b4 = tc_subgrad && p.ksel == p.k;

  // B4: softmax backward onto the selected sub-keys
  if (!fold_b4) {
    const int64_t NH = p.N * p.h;
    if (p.ksel != p.k)
      softmax_bwd_all_kernel<<<(unsigned)((NH + 7) / 8), 256, 0, st>>>(s.w, dw, gsub, NH, p.k,
                                                                       p.scale);
    else if (p.k <= 32)
      softmax_bwd_kernel<1><<<(unsigned)((NH + 7) / 8), 256, 0, st>>>(s.w, dw, s.idx, s.sub_i,
                                                                       gsub, NH, p.k, p.C2,
                                                                       p.scale);
    else
      softmax_bwd_kernel<2><<<(unsigned)((NH + 7) / 8), 256, 0, st>>>(s.w, dw, s.idx, s.sub_i,
                                                                       gsub, NH, p.k, p.C2,
                                                                       p.scale);
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (p.idw) {  // inverse-distance scores: u = g / (||q - c||^2 + eps) = g exp(2 s)
    const int64_t n = 2 * p.N * p.h * p.k;
    idw_scale_kernel<<<(unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)p.sm_count * 16),
                       256, 0, st>>>(gsub, s.sub_s, n);
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // B5 + B6 on tensor cores: dense G planes, dq = G C, BatchNorm backward, dC = G^T Q
  // (the inverse-distance variant's corrections run on the CUDA-core path)
  if (tc_subgrad) {
    const bool want_dq = dx || dWq || dbn;
    e = launch_subgrad_tc(p, gsub, s.sub_i, subkeys, s.q, bn, dbn_acc ? s.qhat : nullptr,
                          c.G, reinterpret_cast<__nv_bfloat16*>(dq_pre),
                          dbn_acc ? part : nullptr, c.dspart, dsub, want_dq, st,
                          fold_b4 ? s.w : nullptr, fold_b4 ? dw : nullptr,
                          fold_b4 ? s.idx : nullptr);
    if (e != cudaSuccess) return e;
    if (dbn_acc) {
      const int64_t nblk = subgrad_part_blocks(p.N);
      if (train && (e = cudaMemsetAsync(c.bntot, 0, 2 * sizeof(float) * p.hq, st)) != cudaSuccess)
        return e;
      dbn_reduce_kernel<<<(2 * p.hq + 31) / 32, kDbnWarps * 32, 0, st>>>(part, (int)nblk, p.hq, dbn_acc);
      PKM_COUNT(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }

  // B5a + B6: dq_pre and BatchNorm affine partials (CUDA-core path)
  if ((dx || dWq || dbn) && !tc_subgrad) {
    const int64_t nblk = (p.N + kDqTokensPerBlock - 1) / kDqTokensPerBlock;
    dim3 grid((unsigned)nblk, (unsigned)(p.h * 2));
    float* partp = dbn_acc ? part : nullptr;
    const float* qh = dbn_acc ? s.qhat : nullptr;
    const bool split = tc_backward_supported(p);
#define PKM_DQ(TS, MC, SPL)                                                                 \
  dq_kernel<TS, MC, SPL><<<grid, 256, 0, st>>>(gsub, s.sub_i, (const TS*)subkeys, bn, qh, \
                                               dq_pre, partp, p.N, p.h, p.dk, p.C1, p.C2,  \
                                               p.k, p.eps, p.idw ? s.q : nullptr)
    if (p.fp32) {
      if (p.half / 4 <= 32) PKM_DQ(float, 1, false);
      else PKM_DQ(float, 4, false);
    } else if (split) {
      if (p.half / 8 <= 32) PKM_DQ(__nv_bfloat16, 1, true);
      else PKM_DQ(__nv_bfloat16, 4, true);
    } else {
      if (p.half / 8 <= 32) PKM_DQ(__nv_bfloat16, 1, false);
      else PKM_DQ(__nv_bfloat16, 4, false);
    }
#undef PKM_DQ
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dbn_acc) {
      if (train && (e = cudaMemsetAsync(c.bntot, 0, 2 * sizeof(float) * p.hq, st)) != cudaSuccess)
        return e;
      dbn_reduce_kernel<<<(2 * p.hq + 31) / 32, kDbnWarps * 32, 0, st>>>(part, (int)nblk, p.hq, dbn_acc); PKM_COUNT(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if (train) {
    // dq_pre is bf16 hi/lo planes wherever the dense query gradients run on tensor cores
    e = launch_bn_train_correct(p, dq_pre, tc_backward_supported(p), s.qhat, c.bneff, c.bntot,
                                st);
    if (e != cudaSuccess) return e;
    if (dbn) {  // the caller's (d gamma, d beta) += the column sums
      const int64_t nblk = tc_subgrad ? subgrad_part_blocks(p.N)
                                      : (p.N + kDqTokensPerBlock - 1) / kDqTokensPerBlock;
      dbn_reduce_kernel<<<(2 * p.hq + 31) / 32, kDbnWarps * 32, 0, st>>>(part, (int)nblk, p.hq, dbn);
      PKM_COUNT(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }

  // B5b: sub-key gradients by sorted segments (CUDA-core path)
  if (dsub && !tc_subgrad) {
    subkey_keys_kernel<<<(unsigned)((E2 + 255) / 256), 256, 0, st>>>(s.sub_i, rb.keysB, E2, p.h,
                                                                      p.k, p.C1, p.C2); PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int32_t *keys_sorted, *ents2;
    // the key array lives in keysB: sort from there (the first pass writes A)
    e = sort::radix_sort(rb.keysB, E2, bits_for((int64_t)p.h * (p.C1 + p.C2) - 1), rb,
                         &keys_sorted, &ents2, st);
    if (e != cudaSuccess) return e;
    e = sort::segments(keys_sorted, E2, seg, U, rb.bsum, st);
    if (e != cudaSuccess) return e;
    const int E = p.fp32 ? 4 : 8;
    const int nv = p.half / E;
    if (p.fp32) {
      if (nv <= 32) subkey_grad_kernel<false, 1><<<persist_blocks, 256, 0, st>>>(seg, U, keys_sorted, ents2, gsub, s.q, dsub, p.N, p.h, p.dk, p.C1, p.C2, p.k, p.status, p.bf16q ? 0.f : 1.f, p.idw ? subkeys : nullptr);
      else subkey_grad_kernel<false, 4><<<persist_blocks, 256, 0, st>>>(seg, U, keys_sorted, ents2, gsub, s.q, dsub, p.N, p.h, p.dk, p.C1, p.C2, p.k, p.status, p.bf16q ? 0.f : 1.f, p.idw ? subkeys : nullptr); PKM_COUNT(1);
    } else {
      if (nv <= 32) subkey_grad_kernel<true, 1><<<persist_blocks, 256, 0, st>>>(seg, U, keys_sorted, ents2, gsub, s.q, dsub, p.N, p.h, p.dk, p.C1, p.C2, p.k, p.status, p.bf16q ? 0.f : 1.f, p.idw ? subkeys : nullptr);
      else subkey_grad_kernel<true, 4><<<persist_blocks, 256, 0, st>>>(seg, U, keys_sorted, ents2, gsub, s.q, dsub, p.N, p.h, p.dk, p.C1, p.C2, p.k, p.status, p.bf16q ? 0.f : 1.f, p.idw ? subkeys : nullptr); PKM_COUNT(1);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  // B7: dense query gradients
  if (tc_backward_supported(p)) {
    if (dx && (e = launch_dx_tc(p, dq_pre, Wq, dx, st)) != cudaSuccess) return e;
    if (dWq && (e = launch_dwq_tc(p, dq_pre, x, dWq, st)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  if (dx) {
    e = gemm_simt_f32(p.N, p.d_in, p.hq, dq_pre, false, p.hq, 1, Wq, !p.fp32, 1, p.d_in, dx,
                      p.d_in, GemmOut::Store, st);
    if (e != cudaSuccess) return e;
  }
  if (dWq) {
    e = gemm_simt_f32(p.hq, p.d_in, p.N, dq_pre, false, 1, p.hq, x, !p.fp32, 1, p.d_in, dWq,
                      p.d_in, GemmOut::Accumulate, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace pkm

namespace pkm {
cudaError_t launch_backward(const Plan& p, const void* x, const void* Wq, const float* bn,
                            const void* subkeys, const void* values, const pkm_saved& s,
                            const float* dy, float* dx, float* dWq, float* dbn, float* dsub,
                            float* dV, float* dw_out, void* ws, cudaStream_t st) {
  cudaError_t e = launch_value_grad(p, values, s, dy, dV, dw_out, ws, st);
  if (e != cudaSuccess) return e;
  return launch_query_grad(p, x, Wq, bn, subkeys, s, dx, dWq, dbn, dsub, dw_out, ws, st);
}
}  // namespace pkm
