// Internal declarations shared by the library's CUDA translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pkm.h"

namespace pkm {

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Monotone map of a finite fp32 score onto uint32 (larger score -> larger key).
// -0.0 is first folded onto +0.0 so that equal scores give equal keys.
__device__ __forceinline__ uint32_t order_key(float v) {
  v = v + 0.0f;
  uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Status codes written by kernels into the device status word (first error wins).
enum : int { kDevOk = 0, kDevTimeout = 1, kDevIndex = 2 };

__device__ __forceinline__ void set_status(int* st, int code) {
  if (st) atomicCAS(st, kDevOk, code);
}

// Unpack 8 bf16 held in a uint4 into floats.
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// ---------------------------------------------------------------- dependent launches
// A kernel launched with launch_dependent may start while the previous kernel on the
// stream is finishing; before it reads anything that kernel wrote it waits in
// grid_dependency_wait (returns at once when launched the ordinary way).  A producer may
// call allow_dependent_launch once its dependents may begin their prologue; the wait
// still covers all of its memory operations.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- launch counter
// Every kernel launch of the library is counted (host side) for diagnostics.
void count_launches(int n);
#define PKM_COUNT(n) ::pkm::count_launches(n)

// ---------------------------------------------------------------- plan
// Sizes derived once per call from pkm_dims.
struct Plan {
  int64_t N;
  int d_in, h, dk, half, C1, C2, k, d_v, hq;  // hq = h*dk
  int64_t K;                                 // C1*C2
  float eps, scale;
  bool fp32;      // fp32 storage
  bool vfp32;     // fp32 value table (fp32, or bf16 x/Wq/subkeys beside fp32 values)
  bool bf16q;     // scores (and the sub-key gradient) take q rounded to bf16 (hi plane)
  bool bn_train;  // training-mode BatchNorm (batch statistics)
  int ksel;       // selections per head: k, or k*k for the all-k^2 variant
  bool idw;       // inverse-distance sub-key scores
  bool simt;      // CUDA-core kernels for bf16 storage
  int sm_count;
  int* status;    // device status word
};

// ---------------------------------------------------------------- forward launches
cudaError_t launch_query_simt(const Plan& p, const void* x, const void* Wq, const float* bn,
                              void* q, float* qhat, cudaStream_t st);
cudaError_t launch_scores_simt(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                               int32_t* sub_i, cudaStream_t st);
// tcgen05 forward GEMMs (bf16 storage, dk/2 % 64 == 0); the tensor-core scorer keeps
// at most kScoresTcMaxK keys per token and half (larger k runs on CUDA cores)
constexpr int kScoresTcMaxK = 32;
bool tc_forward_supported(const Plan& p);
cudaError_t launch_query_tc(const Plan& p, const void* x, const void* Wq, const float* bn,
                            void* q, float* qhat, cudaStream_t st);
cudaError_t launch_scores_tc(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                             int32_t* sub_i, cudaStream_t st);
// tcgen05 backward GEMMs (bf16 storage); dq_planes = [2][N][hq] bf16 (hi, lo)
bool tc_backward_supported(const Plan& p);
cudaError_t launch_dx_tc(const Plan& p, const void* dq_planes, const void* Wq, float* dx,
                         cudaStream_t st);
cudaError_t launch_dwq_tc(const Plan& p, const void* dq_planes, const void* x, float* dWq,
                          cudaStream_t st);
cudaError_t launch_candidates(const Plan& p, const float* sub_s, const int32_t* sub_i,
                              int32_t* idx, float* w, cudaStream_t st);
// Training-mode BatchNorm: statistics of pre (left in the q-hat buffer by an identity-BN
// query GEMM), then q-hat and q; the backward's correction of dq_pre for the batch
// statistics (tot = column sums (d gamma, d beta)); the running-statistics update.
cudaError_t launch_bn_train_forward(const Plan& p, const float* bn, float* qhat_pre, void* q,
                                    float* bn_batch, cudaStream_t st);
cudaError_t launch_bn_train_correct(const Plan& p, void* dq_pre, bool planes, const float* qhat,
                                    const float* bn_eff, const float* tot, cudaStream_t st);
cudaError_t launch_bn_running(const Plan& p, float* bn, const float* bn_batch, float momentum,
                              cudaStream_t st);
// Few tokens (decode): CUDA-core F1 and F2 spread over many CTAs (bf16 storage).
constexpr int64_t kSmallTokens = 16;
bool small_n_supported(const Plan& p);
cudaError_t launch_query_small(const Plan& p, const void* x, const void* Wq, const float* bn,
                               void* q, float* qhat, cudaStream_t st);
cudaError_t launch_scores_small(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                                int32_t* sub_i, cudaStream_t st);
cudaError_t launch_gather(const Plan& p, const void* values, const int32_t* idx, const float* w,
                          float* y, cudaStream_t st);
// The whole few-token forward as one cooperative kernel (workspace: fused_decode_bytes).
bool fused_decode_supported(const Plan& p);
size_t fused_decode_bytes(const Plan& p);
cudaError_t launch_fused_decode(const Plan& p, int dev, const void* x, const void* Wq,
                                const float* bn, const void* subkeys, const void* values,
                                float* y, const pkm_saved& s, void* ws, cudaStream_t st);

// ---------------------------------------------------------------- backward launches
struct BwdWs;  // workspace layout, defined in k_backward.cu
size_t backward_workspace_bytes(const Plan& p);
// Leading bytes of the backward workspace that the value stage uses when the caller
// supplies dw (the value stage touches nothing beyond them).
size_t value_stage_scratch_bytes(const Plan& p);
// Fast-weight pieces (fp32 tables): the bag plus the residual y - target, and the
// SGD step on the distinct selected rows.
cudaError_t launch_gather_resid(const Plan& p, const float* values, const int32_t* idx,
                                const float* w, float* y, const void* tgt, bool tgt_bf16,
                                int64_t tgt_ld, int64_t n_target, float* dy, cudaStream_t st);
cudaError_t launch_value_sgd(const Plan& p, float* values, const pkm_saved& s, const float* dy,
                             float lr, void* ws, cudaStream_t st);
// Lazy Adam on the distinct selected rows (m, v: fp32 tables like the values).
cudaError_t launch_value_adam(const Plan& p, float* values, float* m, float* v,
                              const pkm_saved& s, const float* dy, float lr, float beta1,
                              float beta2, float eps, int64_t step, void* ws, cudaStream_t st);
// Selection counts: slot[r] += selections of row r, sub[h][C1+C2] += winners per sub-key.
cudaError_t launch_hit_counts(const Plan& p, const int32_t* idx, int32_t* slot, int32_t* sub,
                              cudaStream_t st);
// A whole sequence's chunked writes, sorted once by (chunk, row) when chunk count * K
// fits in 31 bits (fw_presort_fits); then each chunk's write reads its segment range.
bool fw_presort_fits(const Plan& p, int64_t chunk);
cudaError_t launch_fw_presort(const Plan& p, int64_t chunk, const int32_t* idx, const float* w,
                              int32_t* keys, int* bounds, void* ws, cudaStream_t st);
// Per-chunk sorts in shared memory (one CTA per chunk) when a chunk has at most 16384
// selections: one launch for every chunk's segment table; the write of chunk ci then
// reads its own table from `buf` (fw_chunk_sort_bytes bytes).
bool fw_chunk_sort_fits(const Plan& p, int64_t chunk);
size_t fw_chunk_sort_bytes(const Plan& p, int64_t chunk);
cudaError_t launch_fw_chunk_sort(const Plan& p, int64_t chunk, const int32_t* idx, const float* w,
                                 void* buf, cudaStream_t st);
cudaError_t launch_fw_chunk_write(const Plan& p, int64_t chunk, int64_t ci, const void* buf,
                                  const float* dy, float* values, float lr, cudaStream_t st);
cudaError_t launch_fw_write(const Plan& p, int64_t chunk, int64_t ci, const int* bounds,
                            const float* dy, float* values, float lr, void* ws, cudaStream_t st);
// dV (dense table, +=) or, when dVc is given, the compact form: dVc[u] = the gradient of
// the u-th distinct selected row (ascending), rows_out[u] = that row, *U_out = U.
// ent_tok, when given, maps every selection to its upstream-gradient row (else
// selection / (h * ksel)).
cudaError_t launch_value_grad(const Plan& p, const void* values, const pkm_saved& s,
                              const float* dy, float* dV, float* dw_out, void* ws,
                              cudaStream_t st, float* dVc = nullptr, int32_t* rows_out = nullptr,
                              int* U_out = nullptr, const int32_t* ent_tok = nullptr);
// wtmp: E1 floats the sort may use between passes (null: the workspace's dw region)
cudaError_t launch_value_sort(const Plan& p, const pkm_saved& s, void* ws, cudaStream_t st,
                              float* wtmp = nullptr);
cudaError_t launch_value_rows(const Plan& p, const void* values, const float* dy, float* dV,
                              float* dw_out, void* ws, cudaStream_t st, float* dVc = nullptr,
                              int32_t* rows_out = nullptr, int* U_out = nullptr,
                              const int32_t* ent_tok = nullptr);
cudaError_t launch_query_grad(const Plan& p, const void* x, const void* Wq, const float* bn,
                              const void* subkeys, const pkm_saved& s, float* dx, float* dWq,
                              float* dbn, float* dsub, float* dw_out, void* ws, cudaStream_t st);
cudaError_t launch_backward(const Plan& p, const void* x, const void* Wq, const float* bn,
                            const void* subkeys, const void* values, const pkm_saved& s,
                            const float* dy, float* dx, float* dWq, float* dbn, float* dsub,
                            float* dV, float* dw_out, void* ws, cudaStream_t st);

// tcgen05 sub-key / query-half gradients and BatchNorm backward (bf16 storage)
int64_t subgrad_pad_tokens(int64_t N);
// Partial-sum blocks (32 tokens each) of the BatchNorm backward fused into dq = G C.
int64_t subgrad_part_blocks(int64_t N);
int subgrad_pad_keys(int C1, int C2);
size_t subgrad_partial_floats(const Plan& p);
cudaError_t launch_subgrad_tc(const Plan& p, const float* gsub, const int32_t* sub_i,
                              const void* subkeys, const void* q_planes, const float* bn,
                              const float* qhat, __nv_bfloat16* G,
                              __nv_bfloat16* dq_planes, float* bn_part, float* dsub_part,
                              float* dsub, bool want_dq, cudaStream_t st, const float* w = nullptr,
                              const float* dw = nullptr, const int32_t* idx = nullptr);

// ---------------------------------------------------------------- row-sharded table
// Workspace layouts (byte offsets) of the source-side routing and the owner-side index.
struct ShardRouteLayout {
  size_t cnt, tri_off, seg_scan, bsum, total;
};
struct ShardOwnerLayout {
  size_t pre, start, rows, wv, tok, total;
};
ShardRouteLayout shard_route_layout(int64_t N, int G);
ShardOwnerLayout shard_owner_layout(int G, int64_t n_tri);
cudaError_t launch_shard_route(const Plan& p, int G, int64_t R, const int32_t* idx, const float* w,
                               int32_t* counts, int32_t* segpos, pkm_triple* send, int32_t* perm,
                               void* ws, cudaStream_t st);
// Prefix sums and segment starts of the received triples (and, when want_arrays, their
// rows, weights and global segments for the value pass) in the owner workspace.
cudaError_t launch_shard_owner_index(const Plan& p, int G, const int32_t* recv_counts,
                                     int64_t n_tri, int64_t n_seg, const pkm_triple* recv,
                                     int64_t shard_rows, void* ws, bool want_arrays,
                                     cudaStream_t st);
cudaError_t launch_shard_bag(const Plan& p, int G, int64_t n_seg, const pkm_triple* recv,
                             const void* values, int64_t shard_rows, float* partial, void* ws,
                             int64_t n_tri, cudaStream_t st);
cudaError_t launch_shard_combine(const Plan& p, int G, const int32_t* segpos, const float* part,
                                 int64_t n_rows, float* y, cudaStream_t st);
cudaError_t launch_shard_gather_dy(const Plan& p, int G, const int32_t* segpos, const float* dy,
                                   int64_t n_rows, float* out, cudaStream_t st);
cudaError_t launch_shard_scatter_dw(const Plan& p, const int32_t* perm, const float* dw_ret,
                                    float* dw, cudaStream_t st);

// ---------------------------------------------------------------- self-test
cudaError_t launch_wait_timeout_probe(long long budget_cycles, int* status, cudaStream_t st);

// ---------------------------------------------------------------- generic CUDA-core GEMM
// C[m][n] (op)= sum_k A(m,k) * B(n,k), A(m,k) = A[m*sam + k*sak], B(n,k) = B[n*sbn + k*sbk].
enum class GemmOut { Store, Accumulate };
cudaError_t gemm_simt_f32(int64_t M, int64_t Nn, int64_t Kk, const void* A, bool a_bf16,
                          int64_t sam, int64_t sak, const void* B, bool b_bf16, int64_t sbn,
                          int64_t sbk, float* C, int64_t ldc, GemmOut mode, cudaStream_t st);

}  // namespace pkm
