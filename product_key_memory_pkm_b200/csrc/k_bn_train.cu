// Training-mode BatchNorm on the query (PKM_F_BN_TRAIN): the statistics are the batch's
// own, per column j of pre = x Wq^T over the call's N tokens.
//
//   forward   the query GEMM runs with an identity BatchNorm and leaves pre in the q-hat
//             buffer; bn_stats_kernel computes each column's mean and biased variance
//             (Welford per thread, Chan's pairwise combination across the CTA's warps in
//             a fixed order); bn_apply_kernel writes q-hat = (pre - mean) / sqrt(var + eps)
//             and q = gamma q-hat + beta in its stored form.
//   backward  the eval-mode kernels run with the batch statistics in place of the running
//             ones, which gives gamma / sqrt(var + eps) * dq; the batch statistics'
//             dependence on every token then subtracts gamma / sqrt(var + eps) *
//             (d beta + q-hat * d gamma) / N (bn_train_correct_kernel).
//   running   running mean and variance move toward the batch's with a momentum, the
//             variance unbiased (N / (N - 1)).
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr int kStatWarps = 32;

__global__ void __launch_bounds__(kStatWarps * 32) bn_stats_kernel(
    const float* __restrict__ pre, int64_t N, int hq, float* __restrict__ bn_batch) {
  __shared__ float s_n[kStatWarps][32], s_mean[kStatWarps][32], s_m2[kStatWarps][32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + lane;
  float n = 0.f, mean = 0.f, m2 = 0.f;
  if (j < hq) {
    for (int64_t t = wid; t < N; t += kStatWarps) {
      const float v = pre[t * hq + j];
      n += 1.f;
      const float d = v - mean;
      mean += d / n;
      m2 = fmaf(d, v - mean, m2);
    }
  }
  s_n[wid][lane] = n;
  s_mean[wid][lane] = mean;
  s_m2[wid][lane] = m2;
  __syncthreads();
  if (wid == 0 && j < hq) {
    float na = s_n[0][lane], ma = s_mean[0][lane], qa = s_m2[0][lane];
    for (int w = 1; w < kStatWarps; ++w) {
      const float nb = s_n[w][lane];
      if (nb == 0.f) continue;
      const float mb = s_mean[w][lane], qb = s_m2[w][lane];
      const float nn = na + nb, d = mb - ma;
      ma += d * (nb / nn);
      qa += qb + d * d * (na * nb / nn);
      na = nn;
    }
    bn_batch[j] = ma;
    bn_batch[hq + j] = qa / na;
  }
}

template <bool kPlanes>
__global__ void bn_apply_kernel(float* __restrict__ qhat, void* __restrict__ q,
                                const float* __restrict__ bn, const float* __restrict__ bn_batch,
                                int64_t N, int hq, float eps) {
  const int64_t n4 = N * hq / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t o = 4 * i;
    const int j0 = (int)(o % hq);
    float4 v = reinterpret_cast<float4*>(qhat)[i];
    float* pv = &v.x;
    float qq[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = j0 + e;
      const float h = (pv[e] - bn_batch[j]) / sqrtf(bn_batch[hq + j] + eps);
      pv[e] = h;
      qq[e] = fmaf(bn[2 * hq + j], h, bn[3 * hq + j]);
    }
    reinterpret_cast<float4*>(qhat)[i] = v;
    if constexpr (kPlanes) {
      __nv_bfloat16* qb = static_cast<__nv_bfloat16*>(q);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat16 hb = __float2bfloat16_rn(qq[e]);
        qb[o + e] = hb;
        qb[N * hq + o + e] = __float2bfloat16_rn(qq[e] - __bfloat162float(hb));
      }
    } else {
      reinterpret_cast<float4*>(q)[i] = make_float4(qq[0], qq[1], qq[2], qq[3]);
    }
  }
}

// dq_pre -= gamma * inv * (dbeta + qhat * dgamma) / N, with tot = (dgamma, dbeta) column sums
template <bool kPlanes>
__global__ void bn_train_correct_kernel(void* __restrict__ dq_pre, const float* __restrict__ qhat,
                                        const float* __restrict__ bn_eff,
                                        const float* __restrict__ tot, int64_t N, int hq,
                                        float eps) {
  const int64_t n = N * hq;
  const float invN = 1.f / (float)N;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < n;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(o % hq);
    const float sc = bn_eff[2 * hq + j] / sqrtf(bn_eff[hq + j] + eps);
    const float corr = sc * (tot[hq + j] + qhat[o] * tot[j]) * invN;
    if constexpr (kPlanes) {
      __nv_bfloat16* p = static_cast<__nv_bfloat16*>(dq_pre);
      const float v = __bfloat162float(p[o]) + __bfloat162float(p[n + o]) - corr;
      const __nv_bfloat16 hb = __float2bfloat16_rn(v);
      p[o] = hb;
      p[n + o] = __float2bfloat16_rn(v - __bfloat162float(hb));
    } else {
      static_cast<float*>(dq_pre)[o] -= corr;
    }
  }
}

__global__ void bn_running_kernel(float* __restrict__ bn, const float* __restrict__ bn_batch,
                                  int hq, float momentum, float unbias) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= hq) return;
  bn[j] = (1.f - momentum) * bn[j] + momentum * bn_batch[j];
  bn[hq + j] = (1.f - momentum) * bn[hq + j] + momentum * bn_batch[hq + j] * unbias;
}

}  // namespace

cudaError_t launch_bn_train_forward(const Plan& p, const float* bn, float* qhat_pre, void* q,
                                    float* bn_batch, cudaStream_t st) {
  bn_stats_kernel<<<(unsigned)((p.hq + 31) / 32), kStatWarps * 32, 0, st>>>(qhat_pre, p.N, p.hq,
                                                                            bn_batch);
  PKM_COUNT(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n4 = p.N * p.hq / 4;
  const unsigned blocks = (unsigned)std::min<int64_t>((n4 + 255) / 256, (int64_t)p.sm_count * 16);
  if (p.fp32)
    bn_apply_kernel<false><<<blocks, 256, 0, st>>>(qhat_pre, q, bn, bn_batch, p.N, p.hq, p.eps);
  else
    bn_apply_kernel<true><<<blocks, 256, 0, st>>>(qhat_pre, q, bn, bn_batch, p.N, p.hq, p.eps);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_bn_train_correct(const Plan& p, void* dq_pre, bool planes, const float* qhat,
                                    const float* bn_eff, const float* tot, cudaStream_t st) {
  const int64_t n = p.N * p.hq;
  const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, (int64_t)p.sm_count * 16);
  if (planes)
    bn_train_correct_kernel<true><<<blocks, 256, 0, st>>>(dq_pre, qhat, bn_eff, tot, p.N, p.hq,
                                                          p.eps);
  else
    bn_train_correct_kernel<false><<<blocks, 256, 0, st>>>(dq_pre, qhat, bn_eff, tot, p.N, p.hq,
                                                           p.eps);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_bn_running(const Plan& p, float* bn, const float* bn_batch, float momentum,
                              cudaStream_t st) {
  const float unbias = (float)((double)p.N / (double)(p.N - 1));
  bn_running_kernel<<<(unsigned)((p.hq + 255) / 256), 256, 0, st>>>(bn, bn_batch, p.hq, momentum,
                                                                    unbias);
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace pkm
