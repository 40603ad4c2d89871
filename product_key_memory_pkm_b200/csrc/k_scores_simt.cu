// F2 on CUDA cores: sub-key scores of each query half against its sub-key set
// and the per-half top-k ("Large Memory Layers with Product Keys", method details:
// q split into q1 and q2, each searched in its own sub-key set; "Meta AI 可扩展内存层"
// 4.3 and 5.2).  Used for fp32 storage and as the reference-grade SIMT path.
//
// One CTA owns 64 tokens of one (head, half) and walks all sub-keys of that half
// in tiles of 64: a 64x64 score tile is computed with fp32 FMAs, staged in shared
// memory, and merged into a per-token sorted list ordered by (score desc, index
// asc).  Sub-keys arrive in increasing index order, so a strict '>' test keeps
// equal scores in index order.
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr int TT = 64, TC = 64, BK = 16, TPB = 256;
constexpr int kQsBytes = BK * (TT + 4) * 4, kCsBytes = BK * (TC + 4) * 4;
constexpr int kTileBytes = kQsBytes + kCsBytes + TT * (TC + 1) * 4;
constexpr int simt_smem_bytes(int KM) { return kTileBytes + KM * TT * 8; }

// lo_scale = 0 drops the lo plane: q rounded to bf16 (single-pass scoring)
template <bool kSplitQ>
__device__ __forceinline__ float load_q(const void* q, int64_t plane, int64_t off,
                                        float lo_scale) {
  if constexpr (kSplitQ) {
    const __nv_bfloat16* b = static_cast<const __nv_bfloat16*>(q);
    return __bfloat162float(b[off]) + lo_scale * __bfloat162float(b[plane + off]);
  } else {
    return static_cast<const float*>(q)[off];
  }
}

// kIdw: inverse-distance scores -1/2 log(||q - c||^2 + eps) ("Fast-weight Product Key
// Memory", section 2.2), ||q - c||^2 = ||q||^2 + ||c||^2 - 2 q.c from the same tiles.
constexpr float kIdwEps = 1e-12f;

template <bool kSplitQ, typename TS, int KM, bool kIdw>
__global__ void __launch_bounds__(TPB) scores_topk_simt(const void* __restrict__ q,
                                                        const TS* __restrict__ sub,
                                                        float* __restrict__ sub_s,
                                                        int32_t* __restrict__ sub_i, int64_t N,
                                                        int h, int dk, int C1, int C2, int k,
                                                        float lo_scale) {
  // shared memory (dynamic: 25 KB of tiles plus KM * 512 bytes of lists)
  extern __shared__ __align__(16) unsigned char simt_smem[];
  auto& Qs = *reinterpret_cast<float(*)[BK][TT + 4]>(simt_smem);
  auto& Cs = *reinterpret_cast<float(*)[BK][TC + 4]>(simt_smem + kQsBytes);
  auto& Ssc = *reinterpret_cast<float(*)[TT][TC + 1]>(simt_smem + kQsBytes + kCsBytes);
  auto& Ls = *reinterpret_cast<float(*)[KM][TT]>(simt_smem + kTileBytes);
  auto& Li = *reinterpret_cast<int(*)[KM][TT]>(simt_smem + kTileBytes + KM * TT * 4);

  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  const int hs = blockIdx.y, hh = hs >> 1, s = hs & 1;
  const int half = dk / 2, hq = h * dk;
  const int C = s ? C2 : C1;
  const TS* Csub = sub + ((int64_t)hh * (C1 + C2) + (s ? C1 : 0)) * half;
  const int64_t qoff = (int64_t)hh * dk + s * half;
  const int64_t plane = N * hq;

  for (int e = tid; e < KM * TT; e += TPB) {
    Ls[e / TT][e % TT] = -INFINITY;
    Li[e / TT][e % TT] = 0x7fffffff;
  }

  for (int c0 = 0; c0 < C; c0 += TC) {
    float acc[4][4], qn[4] = {0.f, 0.f, 0.f, 0.f}, cn[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int d0 = 0; d0 < half; d0 += BK) {
      // tiles: Qs[d][tok], Cs[d][col]; 64*16 = 1024 elements each, 4 per thread
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        int e = tid + it * TPB;
        int r = e / BK, dd = e % BK;
        int64_t t = t0 + r;
        float v = 0.f;
        if (t < N && d0 + dd < half) v = load_q<kSplitQ>(q, plane, t * hq + qoff + d0 + dd, lo_scale);
        Qs[dd][r] = v;
        int c = c0 + r;
        float u = 0.f;
        if (c < C && d0 + dd < half) u = to_f32(Csub[(int64_t)c * half + d0 + dd]);
        Cs[dd][r] = u;
      }
      __syncthreads();
#pragma unroll
      for (int dd = 0; dd < BK; ++dd) {
        float4 a = *reinterpret_cast<const float4*>(&Qs[dd][ty * 4]);
        float4 b = *reinterpret_cast<const float4*>(&Cs[dd][tx * 4]);
        float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        if constexpr (kIdw) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            qn[i] = fmaf(av[i], av[i], qn[i]);
            cn[i] = fmaf(bv[i], bv[i], cn[i]);
          }
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = acc[i][j];
        if constexpr (kIdw) v = -0.5f * logf(fmaxf(qn[i] + cn[j] - 2.f * v, 0.f) + kIdwEps);
        Ssc[ty * 4 + i][tx * 4 + j] = v;
      }
    __syncthreads();
    if (tid < TT) {
      const int r = tid;
      float thr = Ls[KM - 1][r];
      const int cn = min(TC, C - c0);
      for (int c = 0; c < cn; ++c) {
        float v = Ssc[r][c];
        if (v > thr) {
          int pos = KM - 1;
          while (pos > 0 && v > Ls[pos - 1][r]) {
            Ls[pos][r] = Ls[pos - 1][r];
            Li[pos][r] = Li[pos - 1][r];
            --pos;
          }
          Ls[pos][r] = v;
          Li[pos][r] = c0 + c;
          thr = Ls[KM - 1][r];
        }
      }
    }
    __syncthreads();
  }
  // write the first k of each token's list: sub_*[t][hh][s][j]
  for (int e = tid; e < TT * k; e += TPB) {
    int r = e / k, j = e % k;
    int64_t t = t0 + r;
    if (t >= N) continue;
    int64_t o = ((t * h + hh) * 2 + s) * k + j;
    sub_s[o] = Ls[j][r];
    sub_i[o] = Li[j][r];
  }
}

template <bool kSplitQ, typename TS, bool kIdw>
cudaError_t dispatch_km(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                        int32_t* sub_i, cudaStream_t st) {
  dim3 grid((unsigned)((p.N + TT - 1) / TT), (unsigned)(p.h * 2));
  const TS* sub = static_cast<const TS*>(subkeys);
  cudaError_t e = cudaSuccess;
#define PKM_LAUNCH(KMV)                                                                      \
  do {                                                                                       \
    constexpr int smem = simt_smem_bytes(KMV);                                               \
    if (smem > 48 * 1024 &&                                                                  \
        (e = cudaFuncSetAttribute(scores_topk_simt<kSplitQ, TS, KMV, kIdw>,                  \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=     \
            cudaSuccess)                                                                     \
      return e;                                                                              \
    scores_topk_simt<kSplitQ, TS, KMV, kIdw><<<grid, TPB, smem, st>>>(                       \
        q, sub, sub_s, sub_i, p.N, p.h, p.dk, p.C1, p.C2, p.k, p.bf16q ? 0.f : 1.f);         \
  } while (0)
  if (p.k <= 8)
    PKM_LAUNCH(8);
  else if (p.k <= 16)
    PKM_LAUNCH(16);
  else if (p.k <= 32)
    PKM_LAUNCH(32);
  else
    PKM_LAUNCH(64);
#undef PKM_LAUNCH
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scores_simt(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                               int32_t* sub_i, cudaStream_t st) {
  if (p.idw) {
    if (p.fp32) return dispatch_km<false, float, true>(p, subkeys, q, sub_s, sub_i, st);
    return dispatch_km<true, __nv_bfloat16, true>(p, subkeys, q, sub_s, sub_i, st);
  }
  if (p.fp32) return dispatch_km<false, float, false>(p, subkeys, q, sub_s, sub_i, st);
  return dispatch_km<true, __nv_bfloat16, false>(p, subkeys, q, sub_s, sub_i, st);
}

}  // namespace pkm
