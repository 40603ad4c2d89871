// Tensor-core dense query gradients (B7) on the tcgen05 engine.
//
//   dx  [N][d_in]   = dq_pre Wq            A = dq_pre planes, K-major (K = h*dk)
//                                          B = Wq [h*dk][d_in], MN-major
//   dWq [h*dk][d_in] += dq_pre^T x         A = dq_pre planes, MN-major (K = tokens)
//                                          B = x [N][d_in], MN-major
//
// dq_pre arrives as two bf16 planes (hi = bf16(dq_pre), lo = bf16(dq_pre - hi)); the
// hi and lo planes are accumulated as two passes over K into the same fp32 TMEM
// accumulator, so the products carry ~16 significant bits of dq_pre.  x and Wq are
// bf16 inputs, exact in the MMA.  Every output element has one writer
// (deterministic).
#include "tc_gemm.cuh"
#include "tc_launch.cuh"

namespace pkm {
namespace {

using namespace tc;

constexpr int kMNBox = 64;          // MN-major TMA box: 64 x 64 elements
constexpr int kMNBoxBytes = kMNBox * kBK * 2;

__device__ __forceinline__ void store_piece(float* dst, int64_t n0, int64_t n_lim,
                                            const uint32_t (&r)[32], bool accumulate) {
  if (n0 + 32 <= n_lim) {
    float4* p = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      float4 x = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                             __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
      if (accumulate) {
        const float4 o = p[v];
        x.x += o.x; x.y += o.y; x.z += o.z; x.w += o.w;
      }
      p[v] = x;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (n0 + j < n_lim) dst[j] = (accumulate ? dst[j] : 0.f) + __uint_as_float(r[j]);
    }
  }
}

// ------------------------------------------------------------------ dx = dq_pre Wq
struct DxProb {
  static constexpr int kAMN = 0, kBMN = 1;
  // a stage holds one k-block of dq_hi, dq_lo and Wq (64 KiB); two products per k-block
  static constexpr int kStages = 3;
  static constexpr int kAPlanes = 2, kBPlanes = 1;
  // per epilogue warp a 32 x 32 fp32 staging tile for the TMA stores of dx
  static constexpr int kEpiSmem = 4 * 4096;
  struct Params {
    int* status;
    float* dx;
    int64_t N;
    int d_in, hq, m_tiles, n_tiles, nkh;  // nkh = ceil(hq / 64)
    int nw;                               // output columns per tile (64 .. 256)
  };
  __device__ static int mma_n(const Params& P) { return P.nw; }
  struct EpiState {};
  __device__ static int num_units(const Params& P) { return P.m_tiles * P.n_tiles; }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.nkh; }
  __device__ static int num_pairs(const Params&) { return 2; }
  __device__ static int pair_a(const Params&, int i) { return i; }
  __device__ static int pair_b(const Params&, int) { return 0; }
  __device__ static uint32_t tx_bytes(const Params& P) {
    return 2 * kStageA + (P.nw / kMNBox) * kMNBoxBytes;
  }
  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap* A1,
                              const CUtensorMap* B, const CUtensorMap*, int u, int, int kk, void* sa, void* sb,
                              uint64_t* bar) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    tma_load_2d(sa, A0, kk * kBK, mt * kBM, bar);
    tma_load_2d(static_cast<unsigned char*>(sa) + kStageA, A1, kk * kBK, mt * kBM, bar);
    unsigned char* b = static_cast<unsigned char*>(sb);
    for (int j = 0; j < P.nw / kMNBox; ++j)
      tma_load_2d(b + j * kMNBoxBytes, B, nt * P.nw + j * kMNBox, kk * kBK, bar);
  }
  __device__ static void epi_begin(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  // dx pieces leave through the warp's staging tile as TMA stores (out0 maps dx); rows
  // past N and columns past d_in are not written
  __device__ static void epi_chunk(const Params& P, int u, int, int, uint32_t taddr,
                                   unsigned char* sm, EpiState&, const EpiCtx& cx) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    const int y0 = mt * kBM + cx.quarter * 32;
    unsigned char* stg = sm + cx.quarter * 4096;
    for (int piece = 0; piece < P.nw / 32; ++piece) {
      const int n0 = nt * P.nw + piece * 32;
      if (n0 >= P.d_in) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      store_piece_tma(cx.out0, stg, cx.lane, r, n0, y0);
    }
  }
};

// ------------------------------------------------------------------ dWq += dq_pre^T x
struct DwqProb {
  static constexpr int kAMN = 1, kBMN = 1;
  // a stage holds one 64-token block of dq_hi, dq_lo and x (64 KiB); two products per
  // k-block
  static constexpr int kStages = 3;
  static constexpr int kAPlanes = 2, kBPlanes = 1;
  static constexpr int kEpiSmem = 0;
  struct Params {
    int* status;
    float* dWq;
    int64_t N;
    int d_in, hq, m_tiles, n_tiles, nkt;  // nkt = ceil(N / 64)
    int nw;                               // output columns per tile (64 .. 256)
  };
  __device__ static int mma_n(const Params& P) { return P.nw; }
  struct EpiState {};
  __device__ static int num_units(const Params& P) { return P.m_tiles * P.n_tiles; }
  __device__ static int num_chunks(const Params&, int) { return 1; }
  __device__ static int num_kblocks(const Params& P) { return P.nkt; }
  __device__ static int num_pairs(const Params&) { return 2; }
  __device__ static int pair_a(const Params&, int i) { return i; }
  __device__ static int pair_b(const Params&, int) { return 0; }
  __device__ static uint32_t tx_bytes(const Params& P) {
    return 2 * kStageA + (P.nw / kMNBox) * kMNBoxBytes;
  }
  __device__ static void load(const Params& P, const CUtensorMap* A0, const CUtensorMap* A1,
                              const CUtensorMap* B, const CUtensorMap*, int u, int, int kk, void* sa, void* sb,
                              uint64_t* bar) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    unsigned char* a = static_cast<unsigned char*>(sa);
    unsigned char* b = static_cast<unsigned char*>(sb);
#pragma unroll
    for (int j = 0; j < kBM / kMNBox; ++j) {
      tma_load_2d(a + j * kMNBoxBytes, A0, mt * kBM + j * kMNBox, kk * kBK, bar);
      tma_load_2d(a + kStageA + j * kMNBoxBytes, A1, mt * kBM + j * kMNBox, kk * kBK, bar);
    }
    for (int j = 0; j < P.nw / kMNBox; ++j)
      tma_load_2d(b + j * kMNBoxBytes, B, nt * P.nw + j * kMNBox, kk * kBK, bar);
  }
  __device__ static void epi_begin(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  __device__ static void epi_end(const Params&, int, int, unsigned char*, EpiState&, const EpiCtx&) {}
  __device__ static void epi_chunk(const Params& P, int u, int, int row, uint32_t taddr,
                                   unsigned char*, EpiState&, const EpiCtx&) {
    const int mt = u / P.n_tiles, nt = u % P.n_tiles;
    const int o = mt * kBM + row;
    for (int piece = 0; piece < P.nw / 32; ++piece) {
      const int n0 = nt * P.nw + piece * 32;
      if (n0 >= P.d_in) break;  // warp-uniform
      uint32_t r[32];
      tmem_ld32(taddr + (uint32_t)(piece * 32), r);
      tmem_wait_ld(r);
      if (o < P.hq) store_piece(P.dWq + (int64_t)o * P.d_in + n0, n0, P.d_in, r, true);
    }
  }
};

// Output-tile width for `cols` columns over `m_tiles` row tiles: the one of 256, 192 and
// 128 whose round count times width (the per-SM MMA time of the last round) is least;
// ties go to the wider tile (fewer operand bytes per product).
int tile_width(int64_t m_tiles, int cols, int sm_count) {
  int best = kBN;
  int64_t best_cost = -1;
  for (int w : {256, 192, 128}) {
    const int64_t units = m_tiles * ((cols + w - 1) / w);
    const int64_t cost = ((units + sm_count - 1) / sm_count) * w;
    if (best_cost < 0 || cost < best_cost) {
      best = w;
      best_cost = cost;
    }
  }
  return best;
}

}  // namespace

bool tc_backward_supported(const Plan& p) { return !p.simt; }

cudaError_t launch_dx_tc(const Plan& p, const void* dq_planes, const void* Wq, float* dx,
                         cudaStream_t st) {
  const __nv_bfloat16* dq = static_cast<const __nv_bfloat16*>(dq_planes);
  CUtensorMap a0, a1, b;
  if (!make_tmap_bf16_2d(&a0, dq, p.hq, p.N, (uint64_t)p.hq * 2, kBK, kBM) ||
      !make_tmap_bf16_2d(&a1, dq + p.N * p.hq, p.hq, p.N, (uint64_t)p.hq * 2, kBK, kBM) ||
      !make_tmap_bf16_2d(&b, Wq, p.d_in, p.hq, (uint64_t)p.d_in * 2, kMNBox, kBK))
    return cudaErrorInvalidValue;
  DxProb::Params P{};
  P.status = p.status;
  P.dx = dx;
  P.N = p.N;
  P.d_in = p.d_in;
  P.hq = p.hq;
  P.m_tiles = (int)((p.N + kBM - 1) / kBM);
  P.nw = tile_width(P.m_tiles, p.d_in, p.sm_count);
  P.n_tiles = (p.d_in + P.nw - 1) / P.nw;
  P.nkh = (p.hq + kBK - 1) / kBK;
  CUtensorMap tdx;
  {
    const uint64_t dims[2] = {(uint64_t)p.d_in, (uint64_t)p.N};
    const uint64_t strides[1] = {(uint64_t)p.d_in * 4};
    const uint32_t box[2] = {32, 32};
    if (!make_tmap_store(&tdx, true, 2, dx, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  return launch_tc<DxProb>(a0, a1, b, P, P.m_tiles * P.n_tiles, p.sm_count, st, nullptr, &tdx);
}

cudaError_t launch_dwq_tc(const Plan& p, const void* dq_planes, const void* x, float* dWq,
                          cudaStream_t st) {
  const __nv_bfloat16* dq = static_cast<const __nv_bfloat16*>(dq_planes);
  CUtensorMap a0, a1, b;
  if (!make_tmap_bf16_2d(&a0, dq, p.hq, p.N, (uint64_t)p.hq * 2, kMNBox, kBK) ||
      !make_tmap_bf16_2d(&a1, dq + p.N * p.hq, p.hq, p.N, (uint64_t)p.hq * 2, kMNBox, kBK) ||
      !make_tmap_bf16_2d(&b, x, p.d_in, p.N, (uint64_t)p.d_in * 2, kMNBox, kBK))
    return cudaErrorInvalidValue;
  DwqProb::Params P{};
  P.status = p.status;
  P.dWq = dWq;
  P.N = p.N;
  P.d_in = p.d_in;
  P.hq = p.hq;
  P.m_tiles = (p.hq + kBM - 1) / kBM;
  P.nw = tile_width(P.m_tiles, p.d_in, p.sm_count);
  P.n_tiles = (p.d_in + P.nw - 1) / P.nw;
  P.nkt = (int)((p.N + kBK - 1) / kBK);
  return launch_tc<DwqProb>(a0, a1, b, P, P.m_tiles * P.n_tiles, p.sm_count, st);
}

}  // namespace pkm
