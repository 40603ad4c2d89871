// Tensor-core forward GEMMs on the tcgen05 engine (tc_gemm.cuh).
//
// F1 query network: q = BN(x Wq^T), 128 x 256 output tiles, K = d_in.  The epilogue
//   applies the eval-mode BatchNorm and writes q as two bf16 planes (hi = bf16(q),
//   lo = bf16(q - hi)) plus the optional fp32 qhat.
// F2 pkm_subkey_scores: for each (128-token block, head, half) the scores
//   s[c] = q_half . C_half[c] over all c, as hi and lo K-blocks accumulated into one
//   fp32 accumulator (q_hi C + q_lo C), 256 sub-keys per chunk.  The epilogue keeps a
//   running top-k per token in a shared-memory min-heap (root = worst kept key by
//   (score desc, index asc)); sub-keys arrive in increasing index order, so a
//   strict '>' against the root keeps equal scores in index order.  Scores never
//   reach HBM.  ("Large Memory Layers with Product Keys", method details: q split
//   in two, each half searched in its own sub-key set; "Meta AI 可扩展内存层" 4.3-4.4.)
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_gemm.cuh"
#include "tc_launch.cuh"

namespace pkm {

// ------------------------------------------------------------------ host: tensor maps
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

using namespace tc;

// ================================================================== F1 query network
struct QueryProb {
  static constexpr int kAMN = 0, kBMN = 0;
  static constexpr int kStages = 4;
  static constexpr int kEpiSmem = 0;
  struct Params {
    int* status;
    const float* bn;
    __nv_bfloat16* q;  // [2][N][hq]
    float* qhat;       // optional
    int64_t N;
    int hq, m_tiles, n_tiles, nk;
    float eps;
  };
  struct EpiState {};

  __device__ static int num_units(const Params& P) { return P.m_tiles * P.n_tiles; }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.nk; }

  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap*,
                              const CUtensorMap* B, int u, int, int kb, void* sa, void* sb,
                              uint64_t* bar) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    tma_load_2d(sa, A0, kb * kBK, mt * kBM, bar);
    tma_load_2d(sb, B, kb * kBK, nt * kBN, bar);
  }

  __device__ static void epi_begin(const Params&, int, int, unsigned char*, EpiState&) {}
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&) {}

  __device__ static void epi_chunk(const Params& P, int u, int, int row, uint32_t taddr,
                                   unsigned char*, EpiState&) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    const int64_t t = (int64_t)mt * kBM + row;
    const int hq = P.hq;
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int n0 = nt * kBN + piece * 32;
      if (n0 >= hq) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld();
      if (t >= P.N) continue;
      uint32_t hi2[16], lo2[16];
      float qh[32];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float qq[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int n = n0 + j + e;
          const float mean = __ldg(P.bn + n), var = __ldg(P.bn + hq + n);
          const float gamma = __ldg(P.bn + 2 * hq + n), beta = __ldg(P.bn + 3 * hq + n);
          const float h = (__uint_as_float(r[j + e]) - mean) / sqrtf(var + P.eps);
          qh[j + e] = h;
          qq[e] = fmaf(gamma, h, beta);
        }
        const __nv_bfloat162 hb = __floats2bfloat162_rn(qq[0], qq[1]);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(qq[0] - hf.x, qq[1] - hf.y);
        hi2[j / 2] = *reinterpret_cast<const uint32_t*>(&hb);
        lo2[j / 2] = *reinterpret_cast<const uint32_t*>(&lb);
      }
      const int64_t o = t * hq + n0;
      uint4* ph = reinterpret_cast<uint4*>(P.q + o);
      uint4* pl = reinterpret_cast<uint4*>(P.q + P.N * hq + o);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        ph[v] = make_uint4(hi2[4 * v], hi2[4 * v + 1], hi2[4 * v + 2], hi2[4 * v + 3]);
        pl[v] = make_uint4(lo2[4 * v], lo2[4 * v + 1], lo2[4 * v + 2], lo2[4 * v + 3]);
      }
      if (P.qhat) {
        float4* pq = reinterpret_cast<float4*>(P.qhat + o);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          pq[v] = make_float4(qh[4 * v], qh[4 * v + 1], qh[4 * v + 2], qh[4 * v + 3]);
      }
    }
  }
};

// ================================================================== F2 sub-key scores
template <int KM>
struct ScoresProb {
  static constexpr int kAMN = 0, kBMN = 0;
  static constexpr int kStages = 3;
  // heap: KM (score, index) slots per row; staging: one 32-column piece per row
  static constexpr int kEpiSmem = KM * kBM * 8 + 32 * kBM * 4;
  struct Params {
    int* status;
    float* sub_s;
    int32_t* sub_i;
    int64_t N;
    int h, dk, half, C1, C2, k, m_tiles, nkh;  // nkh = half / 64
  };
  struct EpiState {
    float thr;
  };

  __device__ static int num_units(const Params& P) { return P.m_tiles * P.h * 2; }
  __device__ static int num_chunks(const Params& P, int u) {
    const int hs = u / P.m_tiles;
    const int C = (hs & 1) ? P.C2 : P.C1;
    return (C + kBN - 1) / kBN;
  }
  __device__ static int num_kblocks(const Params& P) { return 2 * P.nkh; }

  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap* A1,
                              const CUtensorMap* B, int u, int c, int kb, void* sa, void* sb,
                              uint64_t* bar) {
    const int hs = u / P.m_tiles, mt = u % P.m_tiles;
    const int hh = hs >> 1, s = hs & 1;
    const int plane = kb / P.nkh, kk = kb % P.nkh;
    tma_load_2d(sa, plane ? A1 : A0, hh * P.dk + s * P.half + kk * kBK, mt * kBM, bar);
    tma_load_2d(sb, B, kk * kBK, hh * (P.C1 + P.C2) + s * P.C1 + c * kBN, bar);
  }

  __device__ static float* hs_(unsigned char* sm) { return reinterpret_cast<float*>(sm); }
  __device__ static int* hi_(unsigned char* sm) {
    return reinterpret_cast<int*>(sm + KM * kBM * 4);
  }
  __device__ static float* stage_(unsigned char* sm) {
    return reinterpret_cast<float*>(sm + KM * kBM * 8);
  }

  // worse(a, b): a ranks below b in (score desc, index asc)
  __device__ static bool worse(float sa, int ia, float sb, int ib) {
    return sa < sb || (sa == sb && ia > ib);
  }

  // Replace the root of the `n`-slot heap with (v, col) and restore the heap.
  __device__ static void sift_root(float* hs, int* hi, int row, int n, float v, int col) {
    int pos = 0;
    while (true) {
      const int l = 2 * pos + 1;
      if (l >= n) break;
      int c = l;
      float sc = hs[l * kBM + row];
      int ic = hi[l * kBM + row];
      const int r = l + 1;
      if (r < n) {
        const float sr = hs[r * kBM + row];
        const int ir = hi[r * kBM + row];
        if (worse(sr, ir, sc, ic)) {
          c = r;
          sc = sr;
          ic = ir;
        }
      }
      if (worse(sc, ic, v, col)) {
        hs[pos * kBM + row] = sc;
        hi[pos * kBM + row] = ic;
        pos = c;
      } else {
        break;
      }
    }
    hs[pos * kBM + row] = v;
    hi[pos * kBM + row] = col;
  }

  __device__ static void epi_begin(const Params&, int, int row, unsigned char* sm, EpiState& es) {
    float* hs = hs_(sm);
    int* hi = hi_(sm);
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      hs[j * kBM + row] = -INFINITY;
      hi[j * kBM + row] = 0x7fffffff;
    }
    es.thr = -INFINITY;
  }

  __device__ static void epi_chunk(const Params& P, int u, int c, int row, uint32_t taddr,
                                   unsigned char* sm, EpiState& es) {
    const int hs_idx = u / P.m_tiles;
    const int C = (hs_idx & 1) ? P.C2 : P.C1;
    float* hs = hs_(sm);
    int* hi = hi_(sm);
    float* stg = stage_(sm);
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int col0 = c * kBN + piece * 32;
      if (col0 >= C) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld();
      // candidates of this piece against the threshold at its start
      uint32_t mask = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) mask |= (__uint_as_float(r[j]) > es.thr ? 1u : 0u) << j;
      if (C - col0 < 32) mask &= (1u << (C - col0)) - 1u;
      if (mask) {
#pragma unroll
        for (int j = 0; j < 32; ++j) stg[j * kBM + row] = __uint_as_float(r[j]);
        while (mask) {
          const int j = __ffs(mask) - 1;
          mask &= mask - 1u;
          const float v = stg[j * kBM + row];
          if (v > es.thr) {
            sift_root(hs, hi, row, KM, v, col0 + j);
            es.thr = hs[row];
          }
        }
      }
    }
  }

  __device__ static void epi_end(const Params& P, int u, int row, unsigned char* sm, EpiState&) {
    const int hs_idx = u / P.m_tiles, mt = u % P.m_tiles;
    const int hh = hs_idx >> 1, s = hs_idx & 1;
    const int64_t t = (int64_t)mt * kBM + row;
    float* hs = hs_(sm);
    int* hi = hi_(sm);
    const bool live = t < P.N;
    const int64_t o = ((t * P.h + hh) * 2 + s) * P.k;
    // pop the worst remaining key into the last open position (best-first output)
    for (int n = KM; n > 0; --n) {
      const float rs = hs[row];
      const int ri = hi[row];
      if (live && n - 1 < P.k) {
        P.sub_s[o + n - 1] = rs;
        P.sub_i[o + n - 1] = ri;
      }
      if (n > 1) sift_root(hs, hi, row, n - 1, hs[(n - 1) * kBM + row], hi[(n - 1) * kBM + row]);
    }
  }
};

}  // namespace

bool tc_forward_supported(const Plan& p) {
  return !p.simt && p.half % 64 == 0 && p.hq % 32 == 0 && p.d_in % 8 == 0;
}

cudaError_t launch_query_tc(const Plan& p, const void* x, const void* Wq, const float* bn,
                            void* q, float* qhat, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_2d(&ta, x, p.d_in, p.N, (uint64_t)p.d_in * 2, kBK, kBM) ||
      !make_tmap_bf16_2d(&tb, Wq, p.d_in, p.hq, (uint64_t)p.d_in * 2, kBK, kBN))
    return cudaErrorInvalidValue;
  QueryProb::Params P{};
  P.status = p.status;
  P.bn = bn;
  P.q = static_cast<__nv_bfloat16*>(q);
  P.qhat = qhat;
  P.N = p.N;
  P.hq = p.hq;
  P.m_tiles = (int)((p.N + kBM - 1) / kBM);
  P.n_tiles = (p.hq + kBN - 1) / kBN;
  P.nk = (p.d_in + kBK - 1) / kBK;
  P.eps = p.eps;
  return launch_tc<QueryProb>(ta, ta, tb, P, P.m_tiles * P.n_tiles, p.sm_count, st);
}

cudaError_t launch_scores_tc(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                             int32_t* sub_i, cudaStream_t st) {
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  CUtensorMap thi, tlo, tb;
  if (!make_tmap_bf16_2d(&thi, qb, p.hq, p.N, (uint64_t)p.hq * 2, kBK, kBM) ||
      !make_tmap_bf16_2d(&tlo, qb + p.N * p.hq, p.hq, p.N, (uint64_t)p.hq * 2, kBK, kBM) ||
      !make_tmap_bf16_2d(&tb, subkeys, p.half, (uint64_t)p.h * (p.C1 + p.C2),
                         (uint64_t)p.half * 2, kBK, kBN))
    return cudaErrorInvalidValue;
  const int m_tiles = (int)((p.N + kBM - 1) / kBM);
  const int nunits = m_tiles * p.h * 2;
#define PKM_SC(KMV)                                                                   \
  do {                                                                                \
    typename ScoresProb<KMV>::Params P{p.status, sub_s, sub_i, p.N, p.h, p.dk, p.half, \
                                       p.C1, p.C2, p.k, m_tiles, p.half / kBK};       \
    return launch_tc<ScoresProb<KMV>>(thi, tlo, tb, P, nunits, p.sm_count, st);      \
  } while (0)
  if (p.k <= 8) PKM_SC(8);
  if (p.k <= 16) PKM_SC(16);
  PKM_SC(32);
#undef PKM_SC
}

}  // namespace pkm
