// Tensor-core forward GEMMs on the tcgen05 engine (tc_gemm.cuh).
//
// F1 query network: q = BN(x Wq^T), 128 x 256 output tiles, K = d_in.  The epilogue
//   applies the eval-mode BatchNorm and writes q as two bf16 planes (hi = bf16(q),
//   lo = bf16(q - hi)) plus the optional fp32 qhat.
// F2 pkm_subkey_scores: for each (128-token block, head, half) the scores
//   s[c] = q_half . C_half[c] over all c, as hi and lo K-blocks accumulated into one
//   fp32 accumulator (q_hi C + q_lo C), 256 sub-keys per chunk.  The epilogue keeps a
//   running top-k per token in a shared-memory tournament tree (root = worst kept key
//   by (score desc, index asc)); sub-keys arrive in increasing index order, so a
//   strict '>' against the root keeps equal scores in index order.  Scores never
//   reach HBM.  ("Large Memory Layers with Product Keys", method details: q split
//   in two, each half searched in its own sub-key set; "Meta AI 可扩展内存层" 4.3-4.4.)
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_gemm.cuh"
#include "tc_launch.cuh"

namespace pkm {

// ------------------------------------------------------------------ host: tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
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
  return encode;
}

bool make_tmap_store(CUtensorMap* map, bool fp32, int rank, const void* base,
                     const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                     CUtensorMapSwizzle swizzle) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tmap_encoder();
  if (!encode || rank < 2 || rank > 3) return false;
  cuuint64_t d[3], str[2];
  cuuint32_t bx[3], estr[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) str[i] = strides_bytes[i];
  CUresult r = encode(map,
                      fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      (cuuint32_t)rank, const_cast<void*>(base), d, str, bx, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tmap_encoder();
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
// The epilogue stages each warp's 32 x 32 piece (32 tokens, 32 columns) in shared memory
// and writes it with TMA tile stores: q_hi and q_lo as one 3-D store each into the
// [2][N][hq] planes, qhat as one 2-D store.  A store covers whole 64- and 128-byte row
// segments; stores of a thread's own row touched 32 cache lines per warp instruction and
// bounded the kernel.
struct QueryProb {
  static constexpr int kAMN = 0, kBMN = 0;
  static constexpr int kStages = 3;
  // two epilogue sets (eight epilogue warps): the BatchNorm, the hi/lo split and three
  // output streams of a tile take about as long as its mainloop, so each set gets two
  // units' MMA time to finish one
  static constexpr int kSets = 2;
  // per set: four 8 KiB warp staging tiles (qhat 4 KiB with 128-byte swizzle, q_hi and
  // q_lo 2 KiB each with 64-byte swizzle), then two buffers of the tile's BatchNorm
  // constants {mean, 1/sqrt(var + eps), gamma, beta} (one float4 per column), written by
  // the set's first warp and published through the set's two mbarriers
  static constexpr int kWarpStage = 8192;
  static constexpr int kConstOff = 4 * kWarpStage;
  static constexpr int kEpiSmem = kConstOff + 2 * kBN * 16;
  struct Params {
    int* status;
    const float* bn;
    int64_t N;
    int hq, m_tiles, n_tiles, nk;
    float eps;
    int has_qhat;  // out1 maps qhat [N][hq] fp32
  };
  struct EpiState {};

  __device__ static int num_units(const Params& P) { return P.m_tiles * P.n_tiles; }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.nk; }

  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap*,
                              const CUtensorMap* B, const CUtensorMap*, int u, int, int kb, void* sa, void* sb,
                              uint64_t* bar) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    tma_load_2d(sa, A0, kb * kBK, mt * kBM, bar);
    tma_load_2d(sb, B, kb * kBK, nt * kBN, bar);
  }

  // constants buffer of the set's seq-th unit
  __device__ static float4* consts(unsigned char* sm, int seq) {
    return reinterpret_cast<float4*>(sm + kConstOff) + (seq & 1) * kBN;
  }

  // The set's first warp fills the unit's constants buffer and publishes it.  Buffer
  // seq & 1 was last read in the epilogue of unit seq - 2, which ended before this warp
  // could start unit seq - 1 (the accumulator of seq - 1 is filled only after every
  // thread of the set released seq - 2).
  __device__ static void epi_begin(const Params& P, int u, int, unsigned char* sm, EpiState&,
                                   const EpiCtx& cx) {
    if (cx.quarter != 0) return;
    const int nt = u % P.n_tiles;
    float4* c = consts(sm, cx.seq);
    for (int j = cx.lane; j < kBN; j += 32) {
      const int n = nt * kBN + j;
      float mean = 0.f, inv = 0.f, gamma = 0.f, beta = 0.f;
      if (n < P.hq && !P.bn) {  // identity: q = x Wq^T (training-mode BatchNorm follows)
        inv = 1.f;
        gamma = 1.f;
      } else if (n < P.hq) {
        mean = P.bn[n];
        inv = 1.0f / sqrtf(P.bn[P.hq + n] + P.eps);
        gamma = P.bn[2 * P.hq + n];
        beta = P.bn[3 * P.hq + n];
      }
      c[j] = make_float4(mean, inv, gamma, beta);
    }
    __syncwarp();
    if (cx.lane == 0) mbar_arrive(&cx.bar[cx.seq & 1]);
  }
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&,
                                 const EpiCtx&) {}

  __device__ static void epi_chunk(const Params& P, int u, int, int, uint32_t taddr,
                                   unsigned char* sm, EpiState&, const EpiCtx& cx) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    const int hq = P.hq, lane = cx.lane;
    int got = 0;
    if (lane == 0)
      got = mbar_wait(&cx.bar[cx.seq & 1], (cx.seq >> 1) & 1, cx.abort, cx.status) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, got, 0)) return;
    const float4* cst = consts(sm, cx.seq);
    unsigned char* stg = sm + cx.quarter * kWarpStage;
    float4* s_qh = reinterpret_cast<float4*>(stg);
    uint4* s_hi = reinterpret_cast<uint4*>(stg + 4096);
    uint4* s_lo = reinterpret_cast<uint4*>(stg + 6144);
    const int y0 = mt * kBM + cx.quarter * 32;  // token of the warp's first row
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int n0 = nt * kBN + piece * 32;
      if (n0 >= hq) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      uint32_t hi2[16], lo2[16];
      float qh[32];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float qq[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float4 c4 = cst[piece * 32 + j + e];  // mean, inv, gamma, beta
          const float h = (__uint_as_float(r[j + e]) - c4.x) * c4.y;
          qh[j + e] = h;
          qq[e] = fmaf(c4.z, h, c4.w);
        }
        const __nv_bfloat162 hb = __floats2bfloat162_rn(qq[0], qq[1]);
        const float2 hf = __bfloat1622float2(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(qq[0] - hf.x, qq[1] - hf.y);
        hi2[j / 2] = *reinterpret_cast<const uint32_t*>(&hb);
        lo2[j / 2] = *reinterpret_cast<const uint32_t*>(&lb);
      }
      // the stores of the previous piece have read the staging tile
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      // row = lane; 16-byte chunk v of the row sits at chunk v ^ (address bits 7..9 of the
      // row) for the 128-byte swizzle, v ^ (bits 7..8) for the 64-byte one
      if (P.has_qhat) {
#pragma unroll
        for (int v = 0; v < 8; ++v)
          s_qh[lane * 8 + (v ^ (lane & 7))] =
              make_float4(qh[4 * v], qh[4 * v + 1], qh[4 * v + 2], qh[4 * v + 3]);
      }
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int o = lane * 4 + (v ^ ((lane >> 1) & 3));
        s_hi[o] = make_uint4(hi2[4 * v], hi2[4 * v + 1], hi2[4 * v + 2], hi2[4 * v + 3]);
        s_lo[o] = make_uint4(lo2[4 * v], lo2[4 * v + 1], lo2[4 * v + 2], lo2[4 * v + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(cx.out0, s_hi, n0, y0, 0);
        tma_store_3d(cx.out0, s_lo, n0, y0, 1);
        if (P.has_qhat) tma_store_2d(cx.out1, s_qh, n0, y0);
        bulk_commit();
      }
    }
  }
};

// ================================================================== F2 sub-key scores
// Per-token running top-KM over one half's sub-keys, one epilogue thread per token.
// The kept keys live in a tournament tree in shared memory: KM leaves and, in every
// internal node, the worst key of its subtree, so the root is the current threshold and
// names the leaf to replace.  A key is one 64-bit word ordered like the ranking: the
// high half is the order key of the score, the low half (kColMask - sub-key index) << 5
// | leaf, so a larger word ranks higher (higher score, then lower index) and the root
// word carries its leaf.  Sub-keys arrive in increasing index order, so a new score
// equal to the threshold ranks below every kept key and a strict '>' test is exact.
//
// Per 32-column piece each thread marks the columns above its threshold; the warp then
// runs a uniform loop whose trip count is the largest number of marked columns of any
// lane.  Every iteration takes the lane's next marked column (its score picked from the
// piece's registers one iteration ahead) and, if it still beats the threshold,
// replaces the root's leaf: the siblings along the leaf-to-root path are loaded together
// and the path is rewritten with running minima.  Lanes without a candidate in an
// iteration do the same work with their stores predicated off, so the loop never
// diverges.
template <int KM>
struct ScoresProb {
  static constexpr int kAMN = 0, kBMN = 0;
  // two epilogue sets (two units in flight, two epilogue warps per SM sub-partition);
  // their trees leave room for two operand stages
  static constexpr int kSets = 2;
  static constexpr int kStages = 2;
  static constexpr int kLog = KM == 32 ? 5 : (KM == 16 ? 4 : 3);
  static constexpr int kNodes = 2 * KM;  // nodes 1 .. 2*KM-1; leaves KM .. 2*KM-1
  static constexpr uint32_t kColMask = (1u << 27) - 1u;
  // tree: kNodes 64-bit keys per row (node 0 is a dump for predicated-off stores)
  static constexpr int kEpiSmem = kNodes * kBM * 8;
  struct Params {
    int* status;
    float* sub_s;
    int32_t* sub_i;
    int64_t N;
    int h, dk, half, C1, C2, k, m_tiles, nkh;  // nkh = half / 64
    int planes;  // 2: q_hi and q_lo K-blocks; 1: q_hi only (q rounded to bf16)
  };
  struct EpiState {
    uint64_t root;  // worst kept key
    float thr;      // its score (-inf while a leaf is still empty)
    bool built;
  };

  __device__ static int num_units(const Params& P) { return P.m_tiles * P.h * 2; }
  __device__ static int num_chunks(const Params& P, int u) {
    const int hs = u / P.m_tiles;
    const int C = (hs & 1) ? P.C2 : P.C1;
    return (C + kBN - 1) / kBN;
  }
  __device__ static int num_kblocks(const Params& P) { return P.planes * P.nkh; }

  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap* A1,
                              const CUtensorMap* B, const CUtensorMap*, int u, int c, int kb, void* sa, void* sb,
                              uint64_t* bar) {
    const int hs = u / P.m_tiles, mt = u % P.m_tiles;
    const int hh = hs >> 1, s = hs & 1;
    const int plane = kb / P.nkh, kk = kb % P.nkh;
    tma_load_2d(sa, plane ? A1 : A0, hh * P.dk + s * P.half + kk * kBK, mt * kBM, bar);
    tma_load_2d(sb, B, kk * kBK, hh * (P.C1 + P.C2) + s * P.C1 + c * kBN, bar);
  }

  __device__ static uint64_t* tree_(unsigned char* sm) { return reinterpret_cast<uint64_t*>(sm); }

  // r[j] for a per-lane column j: a five-level tree of selects on the bits of j
  __device__ static float pick(const uint32_t (&r)[32], int j) {
    float a[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = __uint_as_float((j & 16) ? r[i + 16] : r[i]);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = (j & 8) ? a[i + 8] : a[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = (j & 4) ? a[i + 4] : a[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) a[i] = (j & 2) ? a[i + 2] : a[i];
    return (j & 1) ? a[1] : a[0];
  }

  __device__ static uint64_t make_key(float v, int col, int leaf) {
    return ((uint64_t)order_key(v) << 32) | (((kColMask - (uint32_t)col) << 5) | (uint32_t)leaf);
  }
  // an empty leaf: below every real key (the order key of any score is nonzero)
  __device__ static uint64_t empty_key(int leaf) { return (uint64_t)(uint32_t)leaf; }
  __device__ static float key_score(uint64_t key) {
    const uint32_t b = (uint32_t)(key >> 32);
    const float f = __uint_as_float((b & 0x80000000u) ? (b & 0x7fffffffu) : ~b);
    return b == 0u ? -INFINITY : f;
  }
  __device__ static int key_col(uint64_t key) {
    return (int)(kColMask - (((uint32_t)key >> 5) & kColMask));
  }
  __device__ static uint64_t kmin(uint64_t a, uint64_t b) {
    uint64_t m;
    asm("min.u64 %0, %1, %2;" : "=l"(m) : "l"(a), "l"(b));
    return m;
  }

  __device__ static void epi_begin(const Params&, int, int, unsigned char*, EpiState& es,
                                   const EpiCtx&) {
    es.root = 0;
    es.thr = -INFINITY;
    es.built = false;
  }

  // Build the tree from the first KM columns held in registers (columns col0 + j).
  __device__ static void build(uint64_t* tr, int row, const uint32_t (&r)[32], int col0, int C,
                               EpiState& es) {
    uint64_t nd[kNodes];
#pragma unroll
    for (int j = 0; j < KM; ++j)
      nd[KM + j] = col0 + j < C ? make_key(__uint_as_float(r[j]), col0 + j, j) : empty_key(j);
#pragma unroll
    for (int n = KM - 1; n >= 1; --n) nd[n] = kmin(nd[2 * n], nd[2 * n + 1]);
#pragma unroll
    for (int n = 1; n < kNodes; ++n) tr[n * kBM + row] = nd[n];
    es.root = nd[1];
    es.thr = key_score(nd[1]);
    es.built = true;
  }

  __device__ static void epi_chunk(const Params& P, int u, int c, int row, uint32_t taddr,
                                   unsigned char* sm, EpiState& es, const EpiCtx&) {
    const int hs_idx = u / P.m_tiles;
    const int C = (hs_idx & 1) ? P.C2 : P.C1;
    uint64_t* tr = tree_(sm);
    for (int piece = 0; piece < kBN / 32; ++piece) {
      const int col0 = c * kBN + piece * 32;
      if (col0 >= C) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      uint32_t skip = 0u;  // columns already placed by the build
      if (!es.built) {     // first piece of the unit (uniform across the warp)
        build(tr, row, r, col0, C, es);
        skip = KM >= 32 ? 0xffffffffu : ((1u << KM) - 1u);
      }
      // candidates of this piece against the threshold at its start
      uint32_t mask = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) mask |= (__uint_as_float(r[j]) > es.thr ? 1u : 0u) << j;
      mask &= ~skip;
      if (C - col0 < 32) mask &= (1u << (C - col0)) - 1u;
      const int trips = __reduce_max_sync(0xffffffffu, __popc(mask));
      if (trips == 0) continue;  // warp-uniform
      // Branch-free: every lane runs every trip.  A lane without a candidate (or whose
      // candidate no longer beats its threshold) writes its keys into node 0, which the
      // tree does not use, and keeps its root.
      int j = mask ? __ffs(mask) - 1 : 0;
      float v = pick(r, j);
      v = mask ? v : -INFINITY;
      uint64_t* trow = tr + row;  // node n of this row's tree: trow[n * kBM]
      for (int it = 0; it < trips; ++it) {
        // this trip's candidate (v, j); fetch the next one early
        const int jc = j;
        const float vc = v;
        mask &= mask - 1u;
        j = mask ? __ffs(mask) - 1 : 0;
        v = pick(r, j);
        v = mask ? v : -INFINITY;
        const bool act = vc > es.thr;
        const int leaf = (int)((uint32_t)es.root & (uint32_t)(KM - 1));
        const int node0 = KM + leaf;
        uint64_t sib[kLog];
#pragma unroll
        for (int l = 0; l < kLog; ++l) sib[l] = trow[((node0 >> l) ^ 1) * kBM];
        // the path, leaf to root, with running minima; the root itself lives in registers
        // (it is never a sibling), so its node is not stored
        uint64_t cur = make_key(vc, col0 + jc, leaf);
        const int dump = act ? 1 : 0;  // 0: aim the stores at node 0, which is unused
        trow[(node0 & -dump) * kBM] = cur;
#pragma unroll
        for (int l = 0; l < kLog; ++l) {
          cur = kmin(cur, sib[l]);
          if (l + 1 < kLog) trow[((node0 >> (l + 1)) & -dump) * kBM] = cur;
        }
        es.root = act ? cur : es.root;
        es.thr = act ? key_score(cur) : es.thr;
      }
    }
  }

  __device__ static void epi_end(const Params& P, int u, int row, unsigned char* sm, EpiState&,
                                 const EpiCtx&) {
    const int hs_idx = u / P.m_tiles, mt = u % P.m_tiles;
    const int hh = hs_idx >> 1, s = hs_idx & 1;
    const int64_t t = (int64_t)mt * kBM + row;
    if (t >= P.N) return;
    const uint64_t* tr = tree_(sm);
    uint64_t key[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) key[j] = tr[(KM + j) * kBM + row];
    // bitonic sort, best (largest key) first
#pragma unroll
    for (int size = 2; size <= KM; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
        for (int i = 0; i < KM; ++i) {
          const int jx = i ^ stride;
          if (jx > i) {
            const bool desc = (i & size) == 0;
            const uint64_t a = key[i], b = key[jx];
            const bool swap = desc ? (a < b) : (a > b);
            key[i] = swap ? b : a;
            key[jx] = swap ? a : b;
          }
        }
      }
    }
    const int64_t o = ((t * P.h + hh) * 2 + s) * P.k;
    if ((P.k & 3) == 0 && P.k == KM) {  // whole list, 16-byte stores
#pragma unroll
      for (int j = 0; j < KM; j += 4) {
        *reinterpret_cast<float4*>(P.sub_s + o + j) =
            make_float4(key_score(key[j]), key_score(key[j + 1]), key_score(key[j + 2]),
                        key_score(key[j + 3]));
        *reinterpret_cast<int4*>(P.sub_i + o + j) =
            make_int4(key_col(key[j]), key_col(key[j + 1]), key_col(key[j + 2]),
                      key_col(key[j + 3]));
      }
    } else {
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (j < P.k) {
          P.sub_s[o + j] = key_score(key[j]);
          P.sub_i[o + j] = key_col(key[j]);
        }
      }
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
  // q planes [2][N][hq] bf16 and qhat [N][hq] fp32, stored in 32 x 32 tiles
  CUtensorMap tq, tqh;
  {
    const uint64_t dims[3] = {(uint64_t)p.hq, (uint64_t)p.N, 2};
    const uint64_t strides[2] = {(uint64_t)p.hq * 2, (uint64_t)p.N * p.hq * 2};
    const uint32_t box[3] = {32, 32, 1};
    if (!make_tmap_store(&tq, false, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  if (qhat) {
    const uint64_t dims[2] = {(uint64_t)p.hq, (uint64_t)p.N};
    const uint64_t strides[1] = {(uint64_t)p.hq * 4};
    const uint32_t box[2] = {32, 32};
    if (!make_tmap_store(&tqh, true, 2, qhat, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  QueryProb::Params P{};
  P.status = p.status;
  P.bn = bn;
  P.has_qhat = qhat != nullptr;
  P.N = p.N;
  P.hq = p.hq;
  P.m_tiles = (int)((p.N + kBM - 1) / kBM);
  P.n_tiles = (p.hq + kBN - 1) / kBN;
  P.nk = (p.d_in + kBK - 1) / kBK;
  P.eps = p.eps;
  return launch_tc<QueryProb>(ta, ta, tb, P, P.m_tiles * P.n_tiles, p.sm_count, st, nullptr, &tq,
                             qhat ? &tqh : nullptr);
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
                                       p.C1, p.C2, p.k, m_tiles, p.half / kBK,        \
                                       p.bf16q ? 1 : 2};                             \
    return launch_tc<ScoresProb<KMV>>(thi, tlo, tb, P, nunits, p.sm_count, st);      \
  } while (0)
  if (p.k <= 8) PKM_SC(8);
  if (p.k <= 16) PKM_SC(16);
  PKM_SC(32);
#undef PKM_SC
}

}  // namespace pkm
