// Query-half and sub-key gradients (B5) and the BatchNorm backward (B6) on tensor cores.
//
// The sub-score gradients of one (head, half) form a sparse matrix G [N x C] with k
// nonzeros per token row (the selected sub-keys; "Meta AI 可扩展内存层" 9.2: gradient
// reaches only the selected positions).  It is written densely as bf16 hi/lo planes
// (zeros elsewhere), and both products become tcgen05 GEMMs:
//
//   dq_half = G C_half                 A = G (K-major, K = sub-keys), B = C_half (MN-major)
//   dC_half = G^T Q_half               A = G^T (MN-major, K = tokens), B = Q_half (MN-major)
//
// dq_half uses G_hi + G_lo against the exact bf16 sub-keys; dC_half uses G_hi Q_hi +
// G_hi Q_lo + G_lo Q_hi (the lo x lo term is below 2^-17 relative).  dC_half is split
// over the token dimension in kSplits parts written to a partial buffer and added in
// a fixed order, so results are deterministic.  Padding: G has Np = N rounded up to 64
// token rows and Cp = max(C1, C2) rounded up to 64 columns, all zero outside the
// selections, so tiles that run past N or C multiply by exact zeros.
#include "tc_gemm.cuh"
#include "tc_launch.cuh"

namespace pkm {
namespace {

using namespace tc;

constexpr int kMNBox = 64;
constexpr int kMNBoxBytes = kMNBox * kBK * 2;
constexpr int kSplits = 2;           // token-dimension split of dC_half
constexpr int kBnTokens = 64;        // tokens per BatchNorm-backward block (partials layout)

// ------------------------------------------------------------------ dense G planes
// One warp per (padded token t, head-half hs): zero the row in both planes, then
// write the k selected entries (distinct within a half, so no accumulation; lanes
// stride over them for k > 32).
constexpr int kGWin = 1024;  // columns of a G row built in shared memory at a time

// One warp per (token row, head-half): the row of both planes is built in shared memory
// window by window (zeros, then the row's selected sub-keys), then written out with
// 16-byte stores, so every byte of the planes is written once.
__global__ void __launch_bounds__(256) g_dense_kernel(const float* __restrict__ gsub,
                                                      const int32_t* __restrict__ sub_i,
                                                      __nv_bfloat16* __restrict__ G, int64_t N,
                                                      int64_t Np, int h, int k, int Cp) {
  __shared__ __align__(16) __nv_bfloat16 srow[8][2][kGWin];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t w = (int64_t)blockIdx.x * 8 + wid;
  const int hs2 = 2 * h;
  if (w >= Np * hs2) return;  // warp-uniform
  const int64_t t = w / hs2;
  const int hs = (int)(w % hs2);
  uint4* hi = reinterpret_cast<uint4*>(G + ((int64_t)(hs * 2 + 0) * Np + t) * Cp);
  uint4* lo = reinterpret_cast<uint4*>(G + ((int64_t)(hs * 2 + 1) * Np + t) * Cp);
  // this lane's selections of the row (k <= 64: two per lane at most)
  int32_t ci[2] = {-1, -1};
  __nv_bfloat16 ch[2], cl[2];
  if (t < N) {
    const int hh = hs >> 1, s = hs & 1;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = lane + 32 * r;
      if (j < k) {
        const int64_t o = ((t * h + hh) * 2 + s) * k + j;
        const float g = gsub[o];
        ci[r] = sub_i[o];
        ch[r] = __float2bfloat16_rn(g);
        cl[r] = __float2bfloat16_rn(g - __bfloat162float(ch[r]));
      }
    }
  }
  uint4* sh = reinterpret_cast<uint4*>(srow[wid][0]);
  uint4* sl = reinterpret_cast<uint4*>(srow[wid][1]);
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int c0 = 0; c0 < Cp; c0 += kGWin) {
    const int wn = min(kGWin, Cp - c0) / 8;  // 16-byte pieces of this window
    for (int c = lane; c < wn; c += 32) {
      sh[c] = z;
      sl[c] = z;
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = ci[r] - c0;
      if (i >= 0 && i < wn * 8) {
        srow[wid][0][i] = ch[r];
        srow[wid][1][i] = cl[r];
      }
    }
    __syncwarp();
    for (int c = lane; c < wn; c += 32) {
      hi[c0 / 8 + c] = sh[c];
      lo[c0 / 8 + c] = sl[c];
    }
    __syncwarp();  // the window's shared memory is reused
  }
}

// The same rows built straight from the selection (k <= 32 * R), one warp per (token,
// head) for both halves: the softmax backward dS_j = scale w_j (dw_j - sum_l w_l dw_l)
// of the head's winners, each added to its sub-key's column of each half in winner order
// (the order the per-half-list sums take), so no per-half gradient list goes through
// memory and the head's selection is read once.
template <int R>
__global__ void __launch_bounds__(256) g_dense_dw_kernel(
    const float* __restrict__ w, const float* __restrict__ dw, const int32_t* __restrict__ idx,
    __nv_bfloat16* __restrict__ G, int64_t N, int64_t Np, int h, int k, int C2, int Cp,
    float scale) {
  __shared__ __align__(16) __nv_bfloat16 srow[8][2][kGWin];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t wi = (int64_t)blockIdx.x * 8 + wid;
  if (wi >= Np * h) return;  // warp-uniform
  const int64_t t = wi / h;
  const int hh = (int)(wi % h);
  int32_t ij[R];
  float D[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    ij[r] = -1;
    D[r] = 0.f;
  }
  if (t < N) {  // warp-uniform
    const int64_t o = (t * h + hh) * k;
    float wj[R], dwj[R], part = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = lane + 32 * r;
      const bool live = j < k;
      wj[r] = live ? w[o + j] : 0.f;
      dwj[r] = live ? dw[o + j] : 0.f;
      ij[r] = live ? idx[o + j] : -1;
      part = fmaf(wj[r], dwj[r], part);
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
#pragma unroll
    for (int r = 0; r < R; ++r) D[r] = scale * wj[r] * (dwj[r] - part);
  }
  uint4* sh = reinterpret_cast<uint4*>(srow[wid][0]);
  uint4* sl = reinterpret_cast<uint4*>(srow[wid][1]);
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int s = 0; s < 2; ++s) {
    const int hs = 2 * hh + s;
    uint4* hi = reinterpret_cast<uint4*>(G + ((int64_t)(hs * 2 + 0) * Np + t) * Cp);
    uint4* lo = reinterpret_cast<uint4*>(G + ((int64_t)(hs * 2 + 1) * Np + t) * Cp);
    int32_t col[R];
#pragma unroll
    for (int r = 0; r < R; ++r) col[r] = ij[r] < 0 ? -1 : (s ? ij[r] % C2 : ij[r] / C2);
    // each entry's column total, summed in winner order; the column's first winner writes it
    float gs[R];
    bool first[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      gs[r] = 0.f;
      first[r] = col[r] >= 0;
    }
#pragma unroll
    for (int rs = 0; rs < R; ++rs) {
      for (int b = 0; b < 32; ++b) {
        const int32_t cb = __shfl_sync(0xffffffffu, col[rs], b);
        const float Db = __shfl_sync(0xffffffffu, D[rs], b);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (col[r] >= 0 && cb == col[r]) {
            gs[r] += Db;
            if (b + 32 * rs < lane + 32 * r) first[r] = false;
          }
        }
      }
    }
    __nv_bfloat16 ch[R], cl[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      ch[r] = __float2bfloat16_rn(gs[r]);
      cl[r] = __float2bfloat16_rn(gs[r] - __bfloat162float(ch[r]));
    }
    for (int c0 = 0; c0 < Cp; c0 += kGWin) {
      const int wn = min(kGWin, Cp - c0) / 8;
      for (int c = lane; c < wn; c += 32) {
        sh[c] = z;
        sl[c] = z;
      }
      __syncwarp();
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int i = col[r] - c0;
        if (first[r] && i >= 0 && i < wn * 8) {
          srow[wid][0][i] = ch[r];
          srow[wid][1][i] = cl[r];
        }
      }
      __syncwarp();
      for (int c = lane; c < wn; c += 32) {
        hi[c0 / 8 + c] = sh[c];
        lo[c0 / 8 + c] = sl[c];
      }
      __syncwarp();  // the window's shared memory is reused
    }
  }
}

__device__ __forceinline__ void store_piece(float* dst, int n0, int n_lim,
                                            const uint32_t (&r)[32]) {
  if (n0 + 32 <= n_lim) {
    float4* p = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      p[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                         __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (n0 + j < n_lim) dst[j] = __uint_as_float(r[j]);
  }
}

// ------------------------------------------------------------------ dq_half = G C_half
// The epilogue also runs the BatchNorm eval backward on its tile: dq_pre = dq gamma /
// sqrt(var + eps) is written straight to the bf16 hi/lo planes the dense query GEMMs
// read, and the per-column partial sums of dq * qhat (d gamma) and dq (d beta) over each
// warp's 32 tokens are written as one partial row per 32-token block (summed in block
// order afterwards).
constexpr int kPartTokens = 32;

struct DqProb {
  static constexpr int kAMN = 0, kBMN = 1;
  // a stage holds one k-block of G_hi, G_lo and C_half (64 KiB); two products per k-block
  static constexpr int kStages = 2;
  // two epilogue sets: with the BatchNorm backward a tile's epilogue takes about as long
  // as its mainloop, so each set gets two units' MMA time to finish one (measured: 3
  // stages with one set was slower)
  static constexpr int kSets = 2;
  static constexpr int kAPlanes = 2, kBPlanes = 1;
  // per epilogue warp: a 4 KiB staging tile (first the warp's 32 x 32 accumulator piece
  // for the BatchNorm partial sums, then the dq_pre hi and lo pieces for the TMA stores)
  // and the tile's 256 BatchNorm scales gamma / sqrt(var + eps)
  static constexpr int kWarpStage = 4096;
  static constexpr int kScaleOff = 4 * kWarpStage;
  static constexpr int kEpiSmem = kScaleOff + 4 * kBN * 4;
  struct Params {
    int* status;
    const float* bn;        // [4][hq]
    const float* qhat;      // [N][hq] or null
    float* part;            // [ceil(N / 32)][2][hq] or null
    float eps;
    int64_t N, Np;
    int h, dk, half, C1, C2, Cp, hq, m_tiles, n_tiles, nkc;  // nkc = Cp / 64
  };
  struct EpiState {};
  __device__ static int num_units(const Params& P) { return 2 * P.h * P.m_tiles * P.n_tiles; }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.nkc; }
  __device__ static int num_pairs(const Params&) { return 2; }
  __device__ static int pair_a(const Params&, int i) { return i; }
  __device__ static int pair_b(const Params&, int) { return 0; }
  __device__ static uint32_t tx_bytes(const Params&) { return 2 * kStageA + kStageB; }
  __device__ static void decode(const Params& P, int u, int& hs, int& mt, int& nt) {
    const int per = P.m_tiles * P.n_tiles;
    hs = u / per;
    mt = (u % per) / P.n_tiles;
    nt = u % P.n_tiles;
  }
  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap*,
                              const CUtensorMap* B, const CUtensorMap*, int u, int, int kk,
                              void* sa, void* sb, uint64_t* bar) {
    int hs, mt, nt;
    decode(P, u, hs, mt, nt);
    const int hh = hs >> 1, s = hs & 1;
    for (int plane = 0; plane < 2; ++plane)
      tma_load_2d(static_cast<unsigned char*>(sa) + plane * kStageA, A0, kk * kBK,
                  (int)((int64_t)(hs * 2 + plane) * P.Np + mt * kBM), bar);
    unsigned char* b = static_cast<unsigned char*>(sb);
#pragma unroll
    for (int j = 0; j < kBN / kMNBox; ++j)
      tma_load_2d(b + j * kMNBoxBytes, B, nt * kBN + j * kMNBox,
                  hh * (P.C1 + P.C2) + s * P.C1 + kk * kBK, bar);
  }
  __device__ static float* scales(unsigned char* sm, int quarter) {
    return reinterpret_cast<float*>(sm + kScaleOff) + quarter * kBN;
  }
  __device__ static void epi_begin(const Params& P, int u, int, unsigned char* sm, EpiState&,
                                   const EpiCtx& cx) {
    int hs, mt, nt;
    decode(P, u, hs, mt, nt);
    const int base = (hs >> 1) * P.dk + (hs & 1) * P.half + nt * kBN;
    float* sc = scales(sm, cx.quarter);
    __syncwarp();  // this warp's reads of the previous tile's scales are done
    for (int j = cx.lane; j < kBN; j += 32) {
      const int n = nt * kBN + j;
      sc[j] = n < P.half ? P.bn[2 * P.hq + base + j] / sqrtf(P.bn[P.hq + base + j] + P.eps)
                         : 0.f;
    }
    __syncwarp();
  }
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&,
                                 const EpiCtx&) {}
  // Per 32 x 32 piece (the warp's 32 tokens, 32 columns): the BatchNorm partial sums
  // d gamma = sum_t dq * qhat and d beta = sum_t dq over the warp's tokens, lane c
  // summing column c from the staged piece in token order, then dq_pre = dq * scale as
  // bf16 hi and lo pieces through TMA stores (out0 maps the [2][N][hq] planes).
  __device__ static void epi_chunk(const Params& P, int u, int, int, uint32_t taddr,
                                   unsigned char* sm, EpiState&, const EpiCtx& cx) {
    int hs, mt, nt;
    decode(P, u, hs, mt, nt);
    const int hh = hs >> 1, s = hs & 1, lane = cx.lane;
    const int64_t y0 = (int64_t)mt * kBM + cx.quarter * 32;  // token of the warp's first row
    const bool row_live = y0 + lane < P.N;
    const float* sc = scales(sm, cx.quarter);
    unsigned char* stg = sm + cx.quarter * kWarpStage;
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int n0 = nt * kBN + piece * 32;
      if (n0 >= P.half) break;  // warp-uniform
      const int col = hh * P.dk + s * P.half + n0;
      // qhat of the piece, lane c on column c (row loads of 128 bytes), requested before the
      // accumulator is read
      float qv[32];
      if (P.part && P.qhat) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          qv[i] = y0 + i < P.N ? P.qhat[(y0 + i) * P.hq + col + lane] : 0.f;
      }
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      // the previous piece's stores have read the staging tile
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      if (P.part) {  // warp-uniform
        // row = lane, 16-byte chunk v at chunk v ^ (lane & 7): the column reads below
        // (row i, the 32 lanes on its 32 columns) touch 32 distinct banks
        float4* sr = reinterpret_cast<float4*>(stg);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          sr[lane * 8 + (v ^ (lane & 7))] =
              row_live ? make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();
        const float* srf = reinterpret_cast<const float*>(stg);
        float sg = 0.f, sb = 0.f;
        if (P.qhat) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float a = srf[i * 32 + ((((lane >> 2) ^ (i & 7))) << 2) + (lane & 3)];
            sg = fmaf(a, qv[i], sg);
            sb += a;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) sb += srf[i * 32 + ((((lane >> 2) ^ (i & 7))) << 2) + (lane & 3)];
        }
        if (y0 < P.N) {
          const int64_t tb = y0 / kPartTokens;
          P.part[(tb * 2 + 0) * P.hq + col + lane] = sg;
          P.part[(tb * 2 + 1) * P.hq + col + lane] = sb;
        }
        __syncwarp();  // the staged piece is read before the planes overwrite it
      }
      uint32_t hi2[16], lo2[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float v0 = __uint_as_float(r[j]) * sc[piece * 32 + j];
        const float v1 = __uint_as_float(r[j + 1]) * sc[piece * 32 + j + 1];
        const __nv_bfloat162 hb = __floats2bfloat162_rn(v0, v1);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
        hi2[j / 2] = *reinterpret_cast<const uint32_t*>(&hb);
        lo2[j / 2] = *reinterpret_cast<const uint32_t*>(&lb);
      }
      // 64-byte swizzle: row chunk v at chunk v ^ ((lane >> 1) & 3)
      uint4* s_hi = reinterpret_cast<uint4*>(stg);
      uint4* s_lo = reinterpret_cast<uint4*>(stg + 2048);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int o = lane * 4 + (v ^ ((lane >> 1) & 3));
        s_hi[o] = make_uint4(hi2[4 * v], hi2[4 * v + 1], hi2[4 * v + 2], hi2[4 * v + 3]);
        s_lo[o] = make_uint4(lo2[4 * v], lo2[4 * v + 1], lo2[4 * v + 2], lo2[4 * v + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(cx.out0, s_hi, col, (int)y0, 0);
        tma_store_3d(cx.out0, s_lo, col, (int)y0, 1);
        bulk_commit();
      }
    }
  }
};

// ------------------------------------------------------------------ dC_half = G^T Q_half
struct DsubProb {
  static constexpr int kAMN = 1, kBMN = 1;
  // a stage holds one 64-token block of G_hi, G_lo, Q_hi and Q_lo (96 KiB) and the
  // k-block issues the two or three products on it, so each plane is read once per tile
  static constexpr int kStages = 2;
  static constexpr int kAPlanes = 2, kBPlanes = 2;
  static constexpr int kEpiSmem = 0;
  struct Params {
    int* status;
    float* part;  // [kSplits][2h][Cp][half]
    int64_t N, Np;
    int h, dk, half, C1, C2, Cp, m_tiles, n_tiles, nkt, kper;  // nkt = Np / 64
    int npass;  // 3: G_hi Q_hi, G_hi Q_lo, G_lo Q_hi; 2: without G_hi Q_lo (q rounded)
  };
  struct EpiState {};
  __device__ static int num_units(const Params& P) {
    return kSplits * 2 * P.h * P.m_tiles * P.n_tiles;
  }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.kper; }
  // npass 3: (G_hi, Q_hi), (G_hi, Q_lo), (G_lo, Q_hi); npass 2: (G_hi, Q_hi), (G_lo, Q_hi)
  __device__ static int num_pairs(const Params& P) { return P.npass; }
  __device__ static int pair_a(const Params& P, int i) { return P.npass == 3 ? (i == 2) : i; }
  __device__ static int pair_b(const Params& P, int i) { return P.npass == 3 ? (i == 1) : 0; }
  __device__ static uint32_t tx_bytes(const Params& P) {
    return 2 * kStageA + (P.npass == 3 ? 2 : 1) * kStageB;
  }
  __device__ static void decode(const Params& P, int u, int& sp, int& hs, int& mt, int& nt) {
    const int per = P.m_tiles * P.n_tiles;
    sp = u / (2 * P.h * per);
    const int r = u % (2 * P.h * per);
    hs = r / per;
    mt = (r % per) / P.n_tiles;
    nt = r % P.n_tiles;
  }
  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap*,
                              const CUtensorMap* B, const CUtensorMap*, int u, int, int kb,
                              void* sa, void* sb, uint64_t* bar) {
    int sp, hs, mt, nt;
    decode(P, u, sp, hs, mt, nt);
    const int hh = hs >> 1, s = hs & 1;
    const int kk = sp * P.kper + kb;  // 64-token block
    // token blocks past the padded range read beyond both tensors: zero fill
    const bool live = kk < P.nkt;
    for (int plane = 0; plane < 2; ++plane) {
      const int gy = live ? (int)((int64_t)(hs * 2 + plane) * P.Np + kk * kBK)
                          : (int)(4 * (int64_t)P.h * P.Np);
      unsigned char* a = static_cast<unsigned char*>(sa) + plane * kStageA;
#pragma unroll
      for (int j = 0; j < kBM / kMNBox; ++j)
        tma_load_2d(a + j * kMNBoxBytes, A0, mt * kBM + j * kMNBox, gy, bar);
    }
    for (int plane = 0; plane < (P.npass == 3 ? 2 : 1); ++plane) {
      const int qy = live ? (int)((int64_t)plane * P.N + kk * kBK) : (int)(2 * P.N);
      unsigned char* b = static_cast<unsigned char*>(sb) + plane * kStageB;
#pragma unroll
      for (int j = 0; j < kBN / kMNBox; ++j)
        tma_load_2d(b + j * kMNBoxBytes, B, hh * P.dk + s * P.half + nt * kBN + j * kMNBox, qy,
                    bar);
    }
  }
  __device__ static void epi_begin(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  __device__ static void epi_chunk(const Params& P, int u, int, int row, uint32_t taddr,
                                   unsigned char*, EpiState&, const EpiCtx&) {
    int sp, hs, mt, nt;
    decode(P, u, sp, hs, mt, nt);
    const int C = (hs & 1) ? P.C2 : P.C1;
    const int c = mt * kBM + row;
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int n0 = nt * kBN + piece * 32;
      if (n0 >= P.half) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      if (c < C)
        store_piece(P.part + (((int64_t)sp * 2 * P.h + hs) * P.Cp + c) * P.half + n0, n0, P.half,
                    r);
    }
  }
};

// dsub[h][row(s, c)][d] += sum over splits, in split order.  One block per dsub row; a
// thread takes 4 consecutive d when vec4 (half % 4 == 0 and dsub 16-byte aligned), else one.
__global__ void __launch_bounds__(128) dsub_reduce_kernel(const float* __restrict__ part,
                                                          float* __restrict__ dsub, int h,
                                                          int C1, int C2, int Cp, int half,
                                                          int vec4) {
  const int rr = blockIdx.x;  // hh * (C1 + C2) + row within the head
  const int hh = rr / (C1 + C2), within = rr - hh * (C1 + C2);
  const int s = within >= C1 ? 1 : 0;
  const int c = within - s * C1;
  const int hs = hh * 2 + s;
  float* drow = dsub + (int64_t)rr * half;
  const float* prow = part + ((int64_t)hs * Cp + c) * half;
  const int64_t split = (int64_t)2 * h * Cp * half;  // floats between splits
  if (vec4) {
    for (int v = threadIdx.x; v < half / 4; v += blockDim.x) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int sp = 0; sp < kSplits; ++sp) {
        const float4 q = reinterpret_cast<const float4*>(prow + sp * split)[v];
        acc.x += q.x; acc.y += q.y; acc.z += q.z; acc.w += q.w;
      }
      float4 o = reinterpret_cast<float4*>(drow)[v];
      o.x += acc.x; o.y += acc.y; o.z += acc.z; o.w += acc.w;
      reinterpret_cast<float4*>(drow)[v] = o;
    }
  } else {
    for (int d = threadIdx.x; d < half; d += blockDim.x) {
      float acc = 0.f;
#pragma unroll
      for (int sp = 0; sp < kSplits; ++sp) acc += prow[sp * split + d];
      drow[d] += acc;
    }
  }
}

}  // namespace

int64_t subgrad_pad_tokens(int64_t N) { return (N + 63) / 64 * 64; }
int subgrad_pad_keys(int C1, int C2) { return ((C1 > C2 ? C1 : C2) + 63) / 64 * 64; }
size_t subgrad_partial_floats(const Plan& p) {
  return (size_t)kSplits * 2 * p.h * subgrad_pad_keys(p.C1, p.C2) * p.half;
}

int64_t subgrad_part_blocks(int64_t N) { return (N + kPartTokens - 1) / kPartTokens; }

cudaError_t launch_subgrad_tc(const Plan& p, const float* gsub, const int32_t* sub_i,
                              const void* subkeys, const void* q_planes, const float* bn,
                              const float* qhat, __nv_bfloat16* G, __nv_bfloat16* dq_planes,
                              float* bn_part, float* dsub_part, float* dsub, bool want_dq,
                              cudaStream_t st, const float* w, const float* dw,
                              const int32_t* idx) {
  const int64_t Np = subgrad_pad_tokens(p.N);
  const int Cp = subgrad_pad_keys(p.C1, p.C2);
  const int hs2 = 2 * p.h;
  cudaError_t e;
  {
    const int64_t warps = Np * hs2;
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    const unsigned hblocks = (unsigned)((Np * p.h + 7) / 8);  // one warp per (token, head)
    if (w && p.k <= 32)  // the softmax backward folded into the row build
      g_dense_dw_kernel<1><<<hblocks, 256, 0, st>>>(w, dw, idx, G, p.N, Np, p.h, p.k, p.C2, Cp,
                                                    p.scale);
    else if (w)
      g_dense_dw_kernel<2><<<hblocks, 256, 0, st>>>(w, dw, idx, G, p.N, Np, p.h, p.k, p.C2, Cp,
                                                    p.scale);
    else
      g_dense_kernel<<<blocks, 256, 0, st>>>(gsub, sub_i, G, p.N, Np, p.h, p.k, Cp);
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (want_dq) {
    CUtensorMap ta, tb;
    if (!make_tmap_bf16_2d(&ta, G, Cp, (uint64_t)hs2 * 2 * Np, (uint64_t)Cp * 2, kBK, kBM) ||
        !make_tmap_bf16_2d(&tb, subkeys, p.half, (uint64_t)p.h * (p.C1 + p.C2),
                           (uint64_t)p.half * 2, kMNBox, kBK))
      return cudaErrorInvalidValue;
    // dq_pre planes [2][N][hq] bf16, stored in 32 x 32 tiles
    CUtensorMap tq;
    {
      const uint64_t dims[3] = {(uint64_t)p.hq, (uint64_t)p.N, 2};
      const uint64_t strides[2] = {(uint64_t)p.hq * 2, (uint64_t)p.N * p.hq * 2};
      const uint32_t box[3] = {32, 32, 1};
      if (!make_tmap_store(&tq, false, 3, dq_planes, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    }
    DqProb::Params P{};
    P.status = p.status;
    P.bn = bn;
    P.qhat = qhat;
    P.part = bn_part;
    P.eps = p.eps;
    P.N = p.N;
    P.Np = Np;
    P.h = p.h;
    P.dk = p.dk;
    P.half = p.half;
    P.C1 = p.C1;
    P.C2 = p.C2;
    P.Cp = Cp;
    P.hq = p.hq;
    P.m_tiles = (int)(Np / kBM + (Np % kBM ? 1 : 0));
    P.n_tiles = (p.half + kBN - 1) / kBN;
    P.nkc = Cp / kBK;
    if ((e = launch_tc<DqProb>(ta, ta, tb, P, hs2 * P.m_tiles * P.n_tiles, p.sm_count, st,
                               nullptr, &tq)) != cudaSuccess)
      return e;
  }
  if (dsub) {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q_planes);
    CUtensorMap ta, tb;
    if (!make_tmap_bf16_2d(&ta, G, Cp, (uint64_t)hs2 * 2 * Np, (uint64_t)Cp * 2, kMNBox, kBK) ||
        !make_tmap_bf16_2d(&tb, qb, p.hq, (uint64_t)2 * p.N, (uint64_t)p.hq * 2, kMNBox, kBK))
      return cudaErrorInvalidValue;
    DsubProb::Params P{};
    P.status = p.status;
    P.part = dsub_part;
    P.N = p.N;
    P.Np = Np;
    P.h = p.h;
    P.dk = p.dk;
    P.half = p.half;
    P.C1 = p.C1;
    P.C2 = p.C2;
    P.Cp = Cp;
    P.m_tiles = (Cp + kBM - 1) / kBM;
    P.n_tiles = (p.half + kBN - 1) / kBN;
    P.nkt = (int)(Np / kBK);
    P.kper = (P.nkt + kSplits - 1) / kSplits;
    P.npass = p.bf16q ? 2 : 3;
    const int units = kSplits * hs2 * P.m_tiles * P.n_tiles;
    if ((e = launch_tc<DsubProb>(ta, ta, tb, P, units, p.sm_count, st)) != cudaSuccess) return e;
    const int vec4 = p.half % 4 == 0 && (reinterpret_cast<uintptr_t>(dsub) & 15u) == 0;
    dsub_reduce_kernel<<<(unsigned)(p.h * (p.C1 + p.C2)), 128, 0, st>>>(
        dsub_part, dsub, p.h, p.C1, p.C2, Cp, p.half, vec4);
    PKM_COUNT(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace pkm
