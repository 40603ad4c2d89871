// CUDA-core GEMM with fp32 accumulation, used by the fp32-storage path, as the
// query network (F1) of the SIMT path, and for the dense query gradients (B7)
// when the tensor-core kernels are not selected.
//
// C[m][n] = sum_k A(m,k) B(n,k) with arbitrary element strides, so the same kernel
// serves x Wq^T (F1), dq_pre Wq (dx) and dq_pre^T x (dWq).
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr int BM = 128, BN = 128, BK = 16, TPB = 256;

template <typename T>
__device__ __forceinline__ float ld_elem(const T* p, int64_t i) { return to_f32(p[i]); }

// Loads a BMxBK (or BNxBK) operand tile into shared memory as [BK][BM] fp32,
// choosing the thread mapping that walks the contiguous dimension.
template <typename T>
__device__ __forceinline__ void load_tile(float (*S)[BM + 4], const T* P, int64_t rows,
                                          int64_t Kk, int64_t r0, int64_t k0, int64_t sr,
                                          int64_t sk) {
  const int tid = threadIdx.x;
  if (sk == 1) {
#pragma unroll
    for (int it = 0; it < (BM * BK) / TPB; ++it) {
      int e = tid + it * TPB;
      int r = e / BK, kk = e % BK;
      int64_t gr = r0 + r, gk = k0 + kk;
      float v = 0.f;
      if (gr < rows && gk < Kk) v = ld_elem(P, gr * sr + gk);
      S[kk][r] = v;
    }
  } else {
#pragma unroll
    for (int it = 0; it < (BM * BK) / TPB; ++it) {
      int e = tid + it * TPB;
      int kk = e / BM, r = e % BM;
      int64_t gr = r0 + r, gk = k0 + kk;
      float v = 0.f;
      if (gr < rows && gk < Kk) v = ld_elem(P, gr * sr + gk * sk);
      S[kk][r] = v;
    }
  }
}

template <typename TA, typename TB, class Epi>
__global__ void __launch_bounds__(TPB) gemm_simt_kernel(int64_t M, int64_t Nn, int64_t Kk,
                                                        const TA* A, int64_t sam, int64_t sak,
                                                        const TB* B, int64_t sbn, int64_t sbk,
                                                        Epi epi) {
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int64_t m0 = (int64_t)blockIdx.y * BM, n0 = (int64_t)blockIdx.x * BN;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int64_t k0 = 0; k0 < Kk; k0 += BK) {
    load_tile(As, A, M, Kk, m0, k0, sam, sak);
    load_tile(Bs, B, Nn, Kk, n0, k0, sbn, sbk);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[8];
      float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (n < Nn) epi(m, n, acc[i][j]);
    }
  }
}

struct EpiStore {
  float* C;
  int64_t ldc;
  __device__ void operator()(int64_t m, int64_t n, float v) const { C[m * ldc + n] = v; }
};
struct EpiAccum {
  float* C;
  int64_t ldc;
  __device__ void operator()(int64_t m, int64_t n, float v) const { C[m * ldc + n] += v; }
};

// F1 epilogue: eval-mode BatchNorm, then the query in its stored representation.
struct EpiQuery {
  const float* bn;  // [4][hq]
  int hq;
  int64_t N;
  float eps;
  bool split;       // bf16 hi/lo planes (else fp32)
  void* q;
  float* qhat;
  __device__ void operator()(int64_t m, int64_t n, float v) const {
    float qh = v, qq = v;  // no bn: identity (training-mode BatchNorm follows)
    if (bn) {
      const float mean = bn[n], var = bn[hq + n], gamma = bn[2 * hq + n], beta = bn[3 * hq + n];
      qh = (v - mean) / sqrtf(var + eps);
      qq = fmaf(gamma, qh, beta);
    }
    int64_t o = m * hq + n;
    if (split) {
      __nv_bfloat16 hi = __float2bfloat16_rn(qq);
      __nv_bfloat16 lo = __float2bfloat16_rn(qq - __bfloat162float(hi));
      __nv_bfloat16* qb = static_cast<__nv_bfloat16*>(q);
      qb[o] = hi;
      qb[N * hq + o] = lo;
    } else {
      static_cast<float*>(q)[o] = qq;
    }
    if (qhat) qhat[o] = qh;
  }
};

template <class Epi>
cudaError_t run(int64_t M, int64_t Nn, int64_t Kk, const void* A, bool a_bf16, int64_t sam,
                int64_t sak, const void* B, bool b_bf16, int64_t sbn, int64_t sbk, Epi epi,
                cudaStream_t st) {
  dim3 grid((unsigned)((Nn + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  using bf = __nv_bfloat16;
  if (a_bf16 && b_bf16)
    gemm_simt_kernel<bf, bf, Epi><<<grid, TPB, 0, st>>>(M, Nn, Kk, (const bf*)A, sam, sak,
                                                        (const bf*)B, sbn, sbk, epi);
  else if (!a_bf16 && b_bf16)
    gemm_simt_kernel<float, bf, Epi><<<grid, TPB, 0, st>>>(M, Nn, Kk, (const float*)A, sam, sak,
                                                           (const bf*)B, sbn, sbk, epi);
  else if (a_bf16 && !b_bf16)
    gemm_simt_kernel<bf, float, Epi><<<grid, TPB, 0, st>>>(M, Nn, Kk, (const bf*)A, sam, sak,
                                                           (const float*)B, sbn, sbk, epi);
  else
    gemm_simt_kernel<float, float, Epi><<<grid, TPB, 0, st>>>(
        M, Nn, Kk, (const float*)A, sam, sak, (const float*)B, sbn, sbk, epi); PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t gemm_simt_f32(int64_t M, int64_t Nn, int64_t Kk, const void* A, bool a_bf16,
                          int64_t sam, int64_t sak, const void* B, bool b_bf16, int64_t sbn,
                          int64_t sbk, float* C, int64_t ldc, GemmOut mode, cudaStream_t st) {
  if (M == 0 || Nn == 0) return cudaSuccess;
  if (mode == GemmOut::Store)
    return run(M, Nn, Kk, A, a_bf16, sam, sak, B, b_bf16, sbn, sbk, EpiStore{C, ldc}, st);
  return run(M, Nn, Kk, A, a_bf16, sam, sak, B, b_bf16, sbn, sbk, EpiAccum{C, ldc}, st);
}

cudaError_t launch_query_simt(const Plan& p, const void* x, const void* Wq, const float* bn,
                              void* q, float* qhat, cudaStream_t st) {
  const bool bf = !p.fp32;
  EpiQuery epi{bn, p.hq, p.N, p.eps, bf, q, qhat};
  // q[t][o] = sum_i x[t][i] Wq[o][i]
  return run(p.N, p.hq, p.d_in, x, bf, p.d_in, 1, Wq, bf, p.d_in, 1, epi, st);
}

}  // namespace pkm
