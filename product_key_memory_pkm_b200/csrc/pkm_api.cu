// C ABI entry points: host-side validation, plan, launch sequencing.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "pkm_internal.cuh"

namespace pkm {

// One device status word per device (first error wins; cleared by pkm_check_status).
static __device__ int g_status_word;

static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
int g_sm_count[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

// Per-device set-up with that device current: the status word's device address and
// the SM count.  Returns false if a CUDA call failed.
bool device_setup(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  bool ok = true;
  std::call_once(g_dev_once[dev], [&]() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      ok = false;
      return;
    }
    g_status_ptr[dev] = static_cast<int*>(p);
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 148;
    g_sm_count[dev] = sms;
  });
  if (!ok || !g_status_ptr[dev]) return false;
  *dev_out = dev;
  return true;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pkm_status validate_dims(const pkm_dims* d) {
  if (!d) return PKM_ERR_INVALID_ARG;
  if (d->N < 0 || d->d_in <= 0 || d->h <= 0 || d->dk <= 0 || d->C1 <= 0 || d->C2 <= 0 ||
      d->k <= 0 || d->d_v <= 0)
    return PKM_ERR_INVALID_ARG;
  if (d->k > d->C1 || d->k > d->C2) return PKM_ERR_INVALID_ARG;
  if (!(d->bn_eps > 0.f) || !(d->score_scale > 0.f) || d->bn_eps != d->bn_eps ||
      d->score_scale > 3.0e38f)
    return PKM_ERR_INVALID_ARG;
  if ((int64_t)d->C1 * d->C2 >= ((int64_t)1 << 31)) return PKM_ERR_INVALID_ARG;
  if (d->flags & ~(PKM_F_FP32 | PKM_F_SIMT | PKM_F_VALUES_FP32 | PKM_F_BF16_Q | PKM_F_BN_TRAIN |
                   PKM_F_ALL_K2 | PKM_F_IDW))
    return PKM_ERR_INVALID_ARG;
  if ((d->flags & PKM_F_BF16_Q) && (d->flags & PKM_F_FP32)) return PKM_ERR_INVALID_ARG;
  const bool fp32 = d->flags & PKM_F_FP32;
  if (d->dk % 2) return PKM_ERR_INVALID_ARG;
  if (d->d_in % 8 || d->d_v % 8) return PKM_ERR_INVALID_ARG;
  if (fp32 ? (d->dk % 8) : (d->dk % 32)) return PKM_ERR_INVALID_ARG;
  if (d->k > 64 || d->h > 64) return PKM_ERR_UNSUPPORTED;
  const int half = d->dk / 2;
  if (fp32 ? (half / 4 > 128) : (half / 8 > 128)) return PKM_ERR_UNSUPPORTED;
  const int64_t ksel = (d->flags & PKM_F_ALL_K2) ? (int64_t)d->k * d->k : d->k;
  if (d->N * (int64_t)d->h * ksel * 2 >= ((int64_t)1 << 31)) return PKM_ERR_UNSUPPORTED;
  if ((int64_t)d->h * d->dk > 65536) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

// The shape of a call (everything but the device fields).  make_plan, the workspace
// queries and the fixed-scratch size check all derive their Plan from this one function,
// so a buffer layout computed on the host matches the one the launches use.
Plan shape_plan(const pkm_dims* d) {
  Plan p{};
  p.N = d->N;
  p.d_in = d->d_in;
  p.h = d->h;
  p.dk = d->dk;
  p.half = d->dk / 2;
  p.C1 = d->C1;
  p.C2 = d->C2;
  p.k = d->k;
  p.d_v = d->d_v;
  p.hq = d->h * d->dk;
  p.K = (int64_t)d->C1 * d->C2;
  p.eps = d->bn_eps;
  p.scale = d->score_scale;
  p.fp32 = d->flags & PKM_F_FP32;
  p.vfp32 = p.fp32 || (d->flags & PKM_F_VALUES_FP32);
  p.simt = p.fp32 || (d->flags & PKM_F_SIMT);
  p.bf16q = d->flags & PKM_F_BF16_Q;
  p.bn_train = d->flags & PKM_F_BN_TRAIN;
  p.ksel = (d->flags & PKM_F_ALL_K2) ? d->k * d->k : d->k;
  p.idw = d->flags & PKM_F_IDW;
  return p;
}

Plan make_plan(const pkm_dims* d, int dev) {
  Plan p = shape_plan(d);
  p.sm_count = g_sm_count[dev];
  p.status = g_status_ptr[dev];
  return p;
}

pkm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PKM_OK : PKM_ERR_CUDA; }

#define PKM_TRY(expr)                  \
  do {                                 \
    pkm_status _s = (expr);            \
    if (_s != PKM_OK) return _s;       \
  } while (0)

#define PKM_NEED(ptr)                                                   \
  do {                                                                  \
    if (!(ptr) || !aligned16(ptr)) return PKM_ERR_INVALID_ARG;          \
  } while (0)

#define PKM_OPT(ptr)                                                    \
  do {                                                                  \
    if ((ptr) && !aligned16(ptr)) return PKM_ERR_INVALID_ARG;           \
  } while (0)

pkm_status prepare(const pkm_dims* d, Plan* p) {
  PKM_TRY(validate_dims(d));
  int dev = 0;
  if (!device_setup(&dev)) return PKM_ERR_CUDA;
  *p = make_plan(d, dev);
  return PKM_OK;
}

cudaError_t run_query_gemm(const Plan& p, const void* x, const void* Wq, const float* bn, void* q,
                           float* qhat, cudaStream_t st) {
  if (small_n_supported(p)) return launch_query_small(p, x, Wq, bn, q, qhat, st);
  if (tc_forward_supported(p)) return launch_query_tc(p, x, Wq, bn, q, qhat, st);
  return launch_query_simt(p, x, Wq, bn, q, qhat, st);
}

// F1.  Training-mode BatchNorm: the GEMM without BatchNorm leaves x Wq^T in q-hat, whose
// column statistics then normalise it (bn_batch receives them).
cudaError_t run_query(const Plan& p, const void* x, const void* Wq, const float* bn, void* q,
                      float* qhat, cudaStream_t st, float* bn_batch = nullptr) {
  if (!p.bn_train) return run_query_gemm(p, x, Wq, bn, q, qhat, st);
  cudaError_t e = run_query_gemm(p, x, Wq, nullptr, q, qhat, st);
  if (e != cudaSuccess) return e;
  return launch_bn_train_forward(p, bn, qhat, q, bn_batch, st);
}

cudaError_t run_scores(const Plan& p, const void* subkeys, const void* q, float* sub_s,
                       int32_t* sub_i, cudaStream_t st) {
  if (small_n_supported(p)) return launch_scores_small(p, subkeys, q, sub_s, sub_i, st);
  if (tc_forward_supported(p) && !p.idw && p.k <= kScoresTcMaxK)
    return launch_scores_tc(p, subkeys, q, sub_s, sub_i, st);
  return launch_scores_simt(p, subkeys, q, sub_s, sub_i, st);
}

pkm_status check_bn_train(const pkm_dims* d, const pkm_saved* s) {
  if (!(d->flags & PKM_F_BN_TRAIN)) return PKM_OK;
  if (!s || !s->qhat || !s->bn_batch) return PKM_ERR_INVALID_ARG;
  PKM_NEED(s->qhat); PKM_NEED(s->bn_batch);
  return PKM_OK;
}

pkm_status check_saved_fwd(const pkm_saved* s) {
  if (!s) return PKM_ERR_INVALID_ARG;
  PKM_NEED(s->q);
  PKM_OPT(s->qhat);
  PKM_NEED(s->sub_s);
  PKM_NEED(s->sub_i);
  PKM_NEED(s->idx);
  PKM_NEED(s->w);
  return PKM_OK;
}

pkm_status check_workspace(size_t need, void* ws, size_t bytes) {
  if (need == 0) return PKM_OK;
  if (!ws || bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return PKM_ERR_WORKSPACE;
  return PKM_OK;
}

}  // namespace
}  // namespace pkm

using namespace pkm;

extern "C" {

size_t pkm_saved_bytes(const pkm_dims* d, int field) {
  if (validate_dims(d) != PKM_OK) return 0;
  const int64_t ksel = (d->flags & PKM_F_ALL_K2) ? (int64_t)d->k * d->k : d->k;
  const int64_t N = d->N, hq = (int64_t)d->h * d->dk, sel = N * d->h * ksel;
  const bool fp32 = d->flags & PKM_F_FP32;
  switch (field) {
    case PKM_SAVED_Q: return (size_t)(fp32 ? 4 * N * hq : 2 * 2 * N * hq);
    case PKM_SAVED_QHAT: return (size_t)(4 * N * hq);
    case PKM_SAVED_SUB_S:
    case PKM_SAVED_SUB_I: return (size_t)(4 * 2 * N * d->h * d->k);
    case PKM_SAVED_IDX:
    case PKM_SAVED_W: return (size_t)(4 * sel);
    case PKM_SAVED_BN_BATCH: return (size_t)(4 * 2 * hq);
    default: return 0;
  }
}

size_t pkm_workspace_bytes(const pkm_dims* d, int which) {
  if (validate_dims(d) != PKM_OK) return 0;
  if (which == PKM_FWD) return 0;
  if (which == PKM_FWD_FUSED) return d->N == 0 ? 0 : fused_decode_bytes(shape_plan(d));
  if (which != PKM_BWD || d->N == 0) return 0;
  const Plan p = shape_plan(d);
  return backward_workspace_bytes(p);
}

pkm_status pkm_query(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                     const pkm_saved* saved, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(x); PKM_NEED(Wq); PKM_NEED(bn);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->q); PKM_OPT(saved->qhat);
  PKM_TRY(check_bn_train(d, saved));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(run_query(p, x, Wq, bn, saved->q, saved->qhat, st, saved->bn_batch));
}

pkm_status pkm_subkey_scores(const pkm_dims* d, const void* subkeys, const pkm_saved* saved,
                             void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(subkeys);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->q); PKM_NEED(saved->sub_s); PKM_NEED(saved->sub_i);
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(run_scores(p, subkeys, saved->q, saved->sub_s, saved->sub_i, st));
}

pkm_status pkm_candidate_topk(const pkm_dims* d, const pkm_saved* saved, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->sub_s); PKM_NEED(saved->sub_i); PKM_NEED(saved->idx); PKM_NEED(saved->w);
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_candidates(p, saved->sub_s, saved->sub_i, saved->idx, saved->w, st));
}

pkm_status pkm_gather_bag(const pkm_dims* d, const void* values, const int32_t* idx,
                          const float* w, float* y, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(idx); PKM_NEED(w); PKM_NEED(y);
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_gather(p, values, idx, w, y, st));
}

pkm_status pkm_forward(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                       const void* subkeys, const void* values, float* y,
                       const pkm_saved* saved, void* workspace, size_t workspace_bytes,
                       void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(x); PKM_NEED(Wq); PKM_NEED(bn); PKM_NEED(subkeys); PKM_NEED(values); PKM_NEED(y);
  PKM_TRY(check_saved_fwd(saved));
  PKM_TRY(check_bn_train(d, saved));
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_FWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // few tokens with enough workspace: the whole forward as one kernel
  const size_t fused = fused_decode_bytes(p);
  if (fused && workspace && workspace_bytes >= fused &&
      !(reinterpret_cast<uintptr_t>(workspace) & 255u)) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKM_ERR_CUDA;
    const cudaError_t e = launch_fused_decode(p, dev, x, Wq, bn, subkeys, values, y, *saved,
                                              workspace, st);
    if (e == cudaSuccess) return PKM_OK;
    // the CTAs could not all be resident: run the separate kernels instead
    if (e != cudaErrorCooperativeLaunchTooLarge) return PKM_ERR_CUDA;
    (void)cudaGetLastError();
  }
  PKM_TRY(cuda_status(run_query(p, x, Wq, bn, saved->q, saved->qhat, st, saved->bn_batch)));
  PKM_TRY(cuda_status(run_scores(p, subkeys, saved->q, saved->sub_s, saved->sub_i, st)));
  PKM_TRY(cuda_status(launch_candidates(p, saved->sub_s, saved->sub_i, saved->idx, saved->w, st)));
  return cuda_status(launch_gather(p, values, saved->idx, saved->w, y, st));
}

pkm_status pkm_backward(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                        const void* subkeys, const void* values, const pkm_saved* saved,
                        const float* dy, float* dx, float* dWq, float* dbn, float* dsubkeys,
                        float* dvalues, float* dw_out, void* workspace, size_t workspace_bytes,
                        void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(x); PKM_NEED(Wq); PKM_NEED(bn); PKM_NEED(subkeys); PKM_NEED(values); PKM_NEED(dy);
  PKM_TRY(check_saved_fwd(saved));
  PKM_OPT(dx); PKM_OPT(dWq); PKM_OPT(dbn); PKM_OPT(dsubkeys); PKM_OPT(dvalues); PKM_OPT(dw_out);
  if (dbn && !saved->qhat) return PKM_ERR_INVALID_ARG;
  PKM_TRY(check_bn_train(d, saved));
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_backward(p, x, Wq, bn, subkeys, values, *saved, dy, dx, dWq, dbn,
                                     dsubkeys, dvalues, dw_out, workspace, st));
}

pkm_status pkm_value_sort(const pkm_dims* d, const pkm_saved* saved, void* workspace,
                          size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(launch_value_sort(p, *saved, workspace, static_cast<cudaStream_t>(stream)));
}

pkm_status pkm_value_rows(const pkm_dims* d, const void* values, const float* dy,
                          float* dvalues, float* dw, void* workspace, size_t workspace_bytes,
                          void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(dy); PKM_NEED(dw); PKM_OPT(dvalues);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(launch_value_rows(p, values, dy, dvalues, dw, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

pkm_status pkm_value_grad(const pkm_dims* d, const void* values, const pkm_saved* saved,
                          const float* dy, float* dvalues, float* dw, void* workspace,
                          size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(dy); PKM_NEED(dw); PKM_OPT(dvalues);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_value_grad(p, values, *saved, dy, dvalues, dw, workspace, st));
}

pkm_status pkm_query_grad(const pkm_dims* d, const void* x, const void* Wq, const float* bn,
                          const void* subkeys, const pkm_saved* saved, const float* dw, float* dx,
                          float* dWq, float* dbn, float* dsubkeys, void* workspace,
                          size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(x); PKM_NEED(Wq); PKM_NEED(bn); PKM_NEED(subkeys); PKM_NEED(dw);
  PKM_TRY(check_saved_fwd(saved));
  PKM_OPT(dx); PKM_OPT(dWq); PKM_OPT(dbn); PKM_OPT(dsubkeys);
  if (dbn && !saved->qhat) return PKM_ERR_INVALID_ARG;
  PKM_TRY(check_bn_train(d, saved));
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_query_grad(p, x, Wq, bn, subkeys, *saved, dx, dWq, dbn, dsubkeys,
                                       const_cast<float*>(dw), workspace, st));
}

// ---------------------------------------------------------------- fast weights
}  // extern "C"

namespace pkm {
namespace {

// The selection (query, scores, candidates) does not read the value table, so when the
// (chunk, row) keys of a whole sequence fit in 31 bits the loop selects and sorts every
// chunk's writes in one pass up front and each chunk then only reads (bag + residual)
// and writes (SGD on its rows).  Otherwise each chunk runs the whole sequence of steps.
// How the chunk loop sorts its writes.  The selection (query, scores, candidates) does
// not read the value table, so the whole sequence is selected in one pass up front and
// each chunk's writes are sorted before the loop; each chunk then only reads (bag +
// residual) and writes (SGD on its rows).
//   kChunkSort  a chunk has at most 16384 selections: one CTA per chunk sorts them in
//               shared memory (one launch for all chunks);
//   kPresort    otherwise, while chunks * K fits in 31 bits: one global radix sort of
//               every selection by (chunk, row);
//   kPerChunk   otherwise each chunk runs the whole sequence of steps itself.
enum FwMode { kChunkSort, kPresort, kPerChunk };

Plan fw_shape(const pkm_dims* d) {
  Plan p{};
  p.N = d->N; p.h = d->h; p.k = d->k; p.ksel = d->k; p.K = (int64_t)d->C1 * d->C2;
  return p;
}

bool fw_presort_fits(const pkm_dims* d, int64_t chunk) {
  const int64_t nch = (d->N + chunk - 1) / chunk;
  return nch * ((int64_t)d->C1 * d->C2) < ((int64_t)1 << 31);
}

// The fastest strategy that fits, unless the caller's mode bits ask for another one
// (PKM_FW_SORT_GLOBAL falls back to the per-chunk steps when its keys do not fit).
FwMode fw_mode(const pkm_dims* d, int64_t chunk, uint32_t mode) {
  if (mode & PKM_FW_PER_CHUNK) return kPerChunk;
  const bool presort = fw_presort_fits(d, chunk);
  if (mode & PKM_FW_SORT_GLOBAL) return presort ? kPresort : kPerChunk;
  if (fw_chunk_sort_fits(fw_shape(d), chunk)) return kChunkSort;
  return presort ? kPresort : kPerChunk;
}

// Workspace of the chunk loop (each part 256-byte aligned): the saved forward state and
// the residual of the whole sequence (one chunk's for kPerChunk), then the sort state:
// the per-chunk segment tables (kChunkSort), or the sort keys, per-chunk segment bounds
// and the value stage's sort buffers.
struct FwLayout {
  FwMode mode;
  size_t q, sub_s, sub_i, idx, w, dy, keys, bounds, csort, bwd, total;
};

FwLayout fw_layout(const pkm_dims* d, int64_t chunk, uint32_t mode) {
  FwLayout L{};
  L.mode = fw_mode(d, chunk, mode);
  pkm_dims dc = *d;
  if (L.mode == kPerChunk) dc.N = std::min<int64_t>(chunk, d->N);
  const int64_t nch = (d->N + chunk - 1) / chunk;
  const auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o += up(bytes);
    return r;
  };
  L.q = take(pkm_saved_bytes(&dc, PKM_SAVED_Q));
  L.sub_s = take(pkm_saved_bytes(&dc, PKM_SAVED_SUB_S));
  L.sub_i = take(pkm_saved_bytes(&dc, PKM_SAVED_SUB_I));
  L.idx = take(pkm_saved_bytes(&dc, PKM_SAVED_IDX));
  L.w = take(pkm_saved_bytes(&dc, PKM_SAVED_W));
  L.dy = take((size_t)dc.N * d->d_v * 4);
  L.keys = take(L.mode == kPresort ? (size_t)4 * dc.N * d->h * d->k : 0);
  L.bounds = take(L.mode == kPresort ? (size_t)4 * (nch + 1) : 0);
  L.csort = take(L.mode == kChunkSort ? fw_chunk_sort_bytes(fw_shape(d), chunk) : 0);
  L.bwd = take(L.mode == kChunkSort ? 0 : pkm_workspace_bytes(&dc, PKM_BWD));
  L.total = o;
  return L;
}

pkm_status validate_fw(const pkm_dims* d, int64_t chunk, float lr, uint32_t mode) {
  PKM_TRY(validate_dims(d));
  if (chunk < 1 || !(lr == lr) || lr > 3.0e38f || lr < -3.0e38f) return PKM_ERR_INVALID_ARG;
  if (mode & ~(PKM_FW_LOOKAHEAD | PKM_FW_SORT_GLOBAL | PKM_FW_PER_CHUNK))
    return PKM_ERR_INVALID_ARG;
  if ((mode & PKM_FW_LOOKAHEAD) && d->d_in != d->d_v) return PKM_ERR_INVALID_ARG;
  if (!(d->flags & (PKM_F_FP32 | PKM_F_VALUES_FP32))) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

}  // namespace
}  // namespace pkm

extern "C" {

pkm_status pkm_value_sgd(const pkm_dims* d, float lr, float* values, const pkm_saved* saved,
                         const float* dy, void* workspace, size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_fw(d, 1, lr, 0));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(dy);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_value_sgd(p, values, *saved, dy, lr, workspace, st));
}

size_t pkm_fastweight_workspace_bytes(const pkm_dims* d, int64_t chunk, uint32_t mode) {
  if (validate_dims(d) != PKM_OK || chunk < 1 || d->N == 0) return 0;
  return fw_layout(d, chunk, mode).total;
}

pkm_status pkm_fastweight_chunks(const pkm_dims* d, int64_t chunk, float lr, uint32_t mode,
                                 const void* x, const void* Wq, const float* bn,
                                 const void* subkeys, float* values, const float* targets,
                                 float* y, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  PKM_TRY(validate_fw(d, chunk, lr, mode));
  // the loop's BatchNorm is eval; its writes are sorted per k selections
  if (d->flags & (PKM_F_BN_TRAIN | PKM_F_ALL_K2)) return PKM_ERR_INVALID_ARG;
  if (d->N == 0) return PKM_OK;
  const bool lookahead = mode & PKM_FW_LOOKAHEAD;
  PKM_NEED(x); PKM_NEED(Wq); PKM_NEED(bn); PKM_NEED(subkeys); PKM_NEED(values); PKM_NEED(y);
  if (!lookahead) PKM_NEED(targets);
  const FwLayout L = fw_layout(d, chunk, mode);
  PKM_TRY(check_workspace(L.total, workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  pkm_saved s{};
  s.q = ws + L.q;
  s.qhat = nullptr;
  s.sub_s = reinterpret_cast<float*>(ws + L.sub_s);
  s.sub_i = reinterpret_cast<int32_t*>(ws + L.sub_i);
  s.idx = reinterpret_cast<int32_t*>(ws + L.idx);
  s.w = reinterpret_cast<float*>(ws + L.w);
  float* dy = reinterpret_cast<float*>(ws + L.dy);
  const size_t xsz = p.fp32 ? 4 : 2;
  const char* xb = static_cast<const char*>(x);
  const int hk = d->h * d->k;
  const bool tgt_bf16 = lookahead && !p.fp32;
  // the chunk's residual target: the next input (lookahead) or the caller's targets
  auto target = [&](int64_t c0, int64_t n, const void** tgt, int64_t* ld, int64_t* nt) {
    *tgt = lookahead ? static_cast<const void*>(xb + (c0 + 1) * d->d_in * xsz)
                     : static_cast<const void*>(targets + c0 * d->d_v);
    *ld = lookahead ? d->d_in : d->d_v;
    *nt = lookahead ? std::min<int64_t>(n, d->N - 1 - c0) : n;
  };
  if (L.mode != kPerChunk) {
    PKM_TRY(cuda_status(run_query(p, x, Wq, bn, s.q, nullptr, st)));
    PKM_TRY(cuda_status(run_scores(p, subkeys, s.q, s.sub_s, s.sub_i, st)));
    PKM_TRY(cuda_status(launch_candidates(p, s.sub_s, s.sub_i, s.idx, s.w, st)));
    int* bounds = reinterpret_cast<int*>(ws + L.bounds);
    if (L.mode == kChunkSort)
      PKM_TRY(cuda_status(launch_fw_chunk_sort(p, chunk, s.idx, s.w, ws + L.csort, st)));
    else
      PKM_TRY(cuda_status(launch_fw_presort(p, chunk, s.idx, s.w,
                                            reinterpret_cast<int32_t*>(ws + L.keys), bounds,
                                            ws + L.bwd, st)));
    for (int64_t c0 = 0, ci = 0; c0 < d->N; c0 += chunk, ++ci) {
      Plan pc = p;
      pc.N = std::min<int64_t>(chunk, d->N - c0);
      const void* tgt;
      int64_t ld, nt;
      target(c0, pc.N, &tgt, &ld, &nt);
      PKM_TRY(cuda_status(launch_gather_resid(pc, values, s.idx + c0 * hk, s.w + c0 * hk,
                                              y + c0 * d->d_v, tgt, tgt_bf16, ld, nt,
                                              dy + c0 * d->d_v, st)));
      if (L.mode == kChunkSort)
        PKM_TRY(cuda_status(launch_fw_chunk_write(p, chunk, ci, ws + L.csort, dy, values, lr, st)));
      else
        PKM_TRY(cuda_status(launch_fw_write(p, chunk, ci, bounds, dy, values, lr, ws + L.bwd,
                                            st)));
    }
    return PKM_OK;
  }
  for (int64_t c0 = 0; c0 < d->N; c0 += chunk) {
    Plan pc = p;
    pc.N = std::min<int64_t>(chunk, d->N - c0);
    const void* xc = xb + c0 * d->d_in * xsz;
    // read
    PKM_TRY(cuda_status(run_query(pc, xc, Wq, bn, s.q, nullptr, st)));
    PKM_TRY(cuda_status(run_scores(pc, subkeys, s.q, s.sub_s, s.sub_i, st)));
    PKM_TRY(cuda_status(launch_candidates(pc, s.sub_s, s.sub_i, s.idx, s.w, st)));
    const void* tgt;
    int64_t ld, nt;
    target(c0, pc.N, &tgt, &ld, &nt);
    PKM_TRY(cuda_status(launch_gather_resid(pc, values, s.idx, s.w, y + c0 * d->d_v, tgt,
                                            tgt_bf16, ld, nt, dy, st)));
    // write
    PKM_TRY(cuda_status(launch_value_sgd(pc, values, s, dy, lr, ws + L.bwd, st)));
  }
  return PKM_OK;
}

pkm_status pkm_value_grad_rows(const pkm_dims* d, const void* values, const pkm_saved* saved,
                               const float* dy, float* dw, int32_t* rows_out,
                               float* dvalues_rows, int* num_rows, void* workspace,
                               size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(dy); PKM_OPT(dw);
  PKM_NEED(rows_out); PKM_NEED(dvalues_rows);
  if (!num_rows) return PKM_ERR_INVALID_ARG;
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_value_grad(p, values, *saved, dy, nullptr, dw, workspace, st,
                                       dvalues_rows, rows_out, num_rows));
}

pkm_status pkm_value_adam(const pkm_dims* d, float lr, float beta1, float beta2, float eps,
                          int64_t step, float* values, float* m, float* v,
                          const pkm_saved* saved, const float* dy, void* workspace,
                          size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_fw(d, 1, lr, 0));
  if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps > 0.f) ||
      eps > 3.0e38f || step < 1)
    return PKM_ERR_INVALID_ARG;
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(m); PKM_NEED(v); PKM_NEED(dy);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  PKM_TRY(check_workspace(pkm_workspace_bytes(d, PKM_BWD), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_value_adam(p, values, m, v, *saved, dy, lr, beta1, beta2, eps, step,
                                       workspace, st));
}

pkm_status pkm_hit_counts(const pkm_dims* d, const int32_t* idx, int32_t* slot_hits,
                          int32_t* subkey_hits, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0 || (!slot_hits && !subkey_hits)) return PKM_OK;
  PKM_NEED(idx); PKM_OPT(slot_hits); PKM_OPT(subkey_hits);
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_hit_counts(p, idx, slot_hits, subkey_hits, st));
}

pkm_status pkm_bn_running_update(const pkm_dims* d, float* bn, const float* bn_batch,
                                 float momentum, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N < 2 || !(momentum >= 0.f && momentum <= 1.f)) return PKM_ERR_INVALID_ARG;
  PKM_NEED(bn); PKM_NEED(bn_batch);
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_bn_running(p, bn, bn_batch, momentum, st));
}

unsigned long long pkm_launch_count(void) { return g_launches.load(); }

pkm_status pkm_selftest_wait_timeout(uint32_t budget_cycles, void* stream) {
  if (budget_cycles == 0 || budget_cycles > 100000000u) return PKM_ERR_INVALID_ARG;
  int dev = 0;
  if (!device_setup(&dev)) return PKM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_wait_timeout_probe((long long)budget_cycles, g_status_ptr[dev], st));
}

pkm_status pkm_check_status(void* stream) {
  int dev = 0;
  if (!device_setup(&dev)) return PKM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PKM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, g_status_ptr[dev], sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PKM_ERR_CUDA;
  if (v != kDevOk) {
    int z = 0;
    if (cudaMemcpy(g_status_ptr[dev], &z, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return PKM_ERR_CUDA;
  }
  if (v == kDevTimeout) return PKM_ERR_DEVICE_TIMEOUT;
  if (v == kDevIndex) return PKM_ERR_DEVICE_INDEX;
  return PKM_OK;
}

const char* pkm_status_string(pkm_status s) {
  switch (s) {
    case PKM_OK: return "PKM_OK";
    case PKM_ERR_INVALID_ARG: return "PKM_ERR_INVALID_ARG: invalid argument";
    case PKM_ERR_UNSUPPORTED: return "PKM_ERR_UNSUPPORTED: outside this build's limits";
    case PKM_ERR_WORKSPACE: return "PKM_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case PKM_ERR_CUDA: return "PKM_ERR_CUDA: a CUDA runtime call failed";
    case PKM_ERR_DEVICE_TIMEOUT: return "PKM_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    case PKM_ERR_DEVICE_INDEX: return "PKM_ERR_DEVICE_INDEX: a device index check failed";
  }
  return "PKM_ERR_UNKNOWN";
}

const char* pkm_build_info(void) {
  return "pkm_b200 sm_100a (" __DATE__ ")";
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Value-gradient stage with a fixed scratch array (no allocation anywhere).
//
// The scratch is a file-scope device array: every device that loads this library
// reserves it for the life of the process.  In host code the array's name is only a
// host-side stand-in, so its device address is fetched with cudaGetSymbolAddress,
// once per device, with that device current, and passed to the kernels.
namespace pkm {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void*> g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch on the current device, or nullptr if the lookup failed.
// Only a successful lookup is kept: a failed one is retried by the next call, and its
// non-sticky error is cleared.
void* noalloc_scratch(int dev) {
  void* ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (ptr) return ptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ptr = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
  if (ptr) return ptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
  return ptr;
}

}  // namespace
}  // namespace pkm

extern "C" pkm_status pkm_value_grad_noalloc(const pkm_dims* d, const void* values,
                                             const pkm_saved* saved, const float* dy,
                                             float* dvalues, float* dw, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(values); PKM_NEED(dy); PKM_NEED(dw); PKM_OPT(dvalues);
  if (!saved) return PKM_ERR_INVALID_ARG;
  PKM_NEED(saved->idx); PKM_NEED(saved->w);
  // size check on the host, before any CUDA call; shape_plan is the plan make_plan
  // extends, so the layout checked here is the one the launch uses
  if (value_stage_scratch_bytes(shape_plan(d)) > kNoAllocScratchBytes) return PKM_ERR_WORKSPACE;
  Plan p;
  PKM_TRY(prepare(d, &p));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKM_ERR_UNSUPPORTED;
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return PKM_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(launch_value_grad(p, values, *saved, dy, dvalues, dw, scratch, st));
}

// ------------------------------------------------------------------ row-sharded table
namespace pkm {
namespace {

pkm_status validate_shard(const pkm_dims* d, int32_t G) {
  PKM_TRY(validate_dims(d));
  if (G < 1 || G > PKM_MAX_SHARDS) return PKM_ERR_INVALID_ARG;
  if ((int64_t)G * d->N >= ((int64_t)1 << 31)) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

pkm_status validate_owner(int64_t shard_rows, int64_t n_tri, int64_t n_seg) {
  if (shard_rows < 1 || shard_rows >= ((int64_t)1 << 31)) return PKM_ERR_INVALID_ARG;
  if (n_tri < 0 || n_seg < 0 || n_seg > n_tri || (n_tri > 0 && n_seg == 0))
    return PKM_ERR_INVALID_ARG;
  if (n_tri >= ((int64_t)1 << 30)) return PKM_ERR_UNSUPPORTED;
  return PKM_OK;
}

// The owner's value pass sees every received triple as one selection of its own
// one-head, one-key "token" over the shard's rows.
Plan owner_plan(Plan p, int64_t n_tri, int64_t shard_rows) {
  p.N = n_tri;
  p.h = 1;
  p.k = 1;
  p.ksel = 1;
  p.K = shard_rows;
  return p;
}

size_t owner_bytes(const pkm_dims* d, int32_t G, int64_t n_tri) {
  Plan q{};
  q.d_v = d->d_v;
  q.dk = d->dk;
  q.hq = d->dk;
  q.C1 = d->C1;
  q.C2 = d->C2;
  q.fp32 = d->flags & PKM_F_FP32;
  q = owner_plan(q, n_tri > 0 ? n_tri : 1, 1);
  return shard_owner_layout(G, n_tri).total + value_stage_scratch_bytes(q);
}

}  // namespace
}  // namespace pkm

extern "C" {

size_t pkm_shard_workspace_bytes(const pkm_dims* d, int32_t G, int which, int64_t n_triples) {
  if (validate_shard(d, G) != PKM_OK) return 0;
  if (which == PKM_SHARD_ROUTE) return shard_route_layout(d->N > 0 ? d->N : 1, G).total;
  if (which == PKM_SHARD_OWNER && n_triples >= 0) return owner_bytes(d, G, n_triples);
  return 0;
}

pkm_status pkm_shard_route(const pkm_dims* d, int32_t G, int64_t rows_per_shard,
                           const int32_t* idx, const float* w, int32_t* counts, int32_t* segpos,
                           pkm_triple* send, int32_t* perm, void* workspace,
                           size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_shard(d, G));
  const int64_t K = (int64_t)d->C1 * d->C2;
  // G shards of rows_per_shard rows must cover the table (no overflow for large shards)
  if (rows_per_shard < 1 || (rows_per_shard < K && (K + rows_per_shard - 1) / rows_per_shard > G))
    return PKM_ERR_INVALID_ARG;
  PKM_NEED(counts);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d->N == 0)  // nothing to send: zero counts, so the caller's exchange still runs
    return cuda_status(cudaMemsetAsync(counts, 0, sizeof(int32_t) * 2 * (size_t)G, st));
  PKM_NEED(idx); PKM_NEED(w); PKM_NEED(segpos); PKM_NEED(send); PKM_NEED(perm);
  PKM_TRY(check_workspace(shard_route_layout(d->N, G).total, workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(
      launch_shard_route(p, G, rows_per_shard, idx, w, counts, segpos, send, perm, workspace, st));
}

pkm_status pkm_shard_bag(const pkm_dims* d, int32_t G, int64_t shard_rows,
                         const int32_t* recv_counts, int64_t n_triples, int64_t n_segments,
                         const pkm_triple* recv, const void* values, float* partial,
                         void* workspace, size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_shard(d, G));
  PKM_TRY(validate_owner(shard_rows, n_triples, n_segments));
  if (n_segments == 0) return PKM_OK;
  PKM_NEED(recv_counts); PKM_NEED(recv); PKM_NEED(values); PKM_NEED(partial);
  PKM_TRY(check_workspace(owner_bytes(d, G, n_triples), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_shard_owner_index(p, G, recv_counts, n_triples, n_segments, recv,
                                           shard_rows, workspace, false, st);
  if (e != cudaSuccess) return PKM_ERR_CUDA;
  return cuda_status(launch_shard_bag(p, G, n_segments, recv, values, shard_rows, partial,
                                      workspace, n_triples, st));
}

pkm_status pkm_shard_combine(const pkm_dims* d, int32_t G, const int32_t* segpos,
                             const float* partial_recv, int64_t n_rows, float* y, void* stream) {
  PKM_TRY(validate_shard(d, G));
  if (n_rows < 0) return PKM_ERR_INVALID_ARG;
  if (d->N == 0) return PKM_OK;
  PKM_NEED(segpos); PKM_NEED(y);
  if (n_rows > 0) PKM_NEED(partial_recv);
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(launch_shard_combine(p, G, segpos, partial_recv, n_rows, y,
                                          static_cast<cudaStream_t>(stream)));
}

pkm_status pkm_shard_gather_dy(const pkm_dims* d, int32_t G, const int32_t* segpos,
                               const float* dy, float* dy_send, int64_t n_rows, void* stream) {
  PKM_TRY(validate_shard(d, G));
  if (n_rows < 0) return PKM_ERR_INVALID_ARG;
  if (d->N == 0 || n_rows == 0) return PKM_OK;
  PKM_NEED(segpos); PKM_NEED(dy); PKM_NEED(dy_send);
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(launch_shard_gather_dy(p, G, segpos, dy, n_rows, dy_send,
                                            static_cast<cudaStream_t>(stream)));
}

pkm_status pkm_shard_value_grad(const pkm_dims* d, int32_t G, int64_t shard_rows,
                                const int32_t* recv_counts, int64_t n_triples,
                                int64_t n_segments, const pkm_triple* recv, const void* values,
                                const float* dy_recv, float* dvalues, float* dw_recv,
                                void* workspace, size_t workspace_bytes, void* stream) {
  PKM_TRY(validate_shard(d, G));
  PKM_TRY(validate_owner(shard_rows, n_triples, n_segments));
  if (n_triples == 0) return PKM_OK;
  PKM_NEED(recv_counts); PKM_NEED(recv); PKM_NEED(values); PKM_NEED(dy_recv);
  PKM_NEED(dvalues); PKM_NEED(dw_recv);
  PKM_TRY(check_workspace(owner_bytes(d, G, n_triples), workspace, workspace_bytes));
  Plan p;
  PKM_TRY(prepare(d, &p));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_shard_owner_index(p, G, recv_counts, n_triples, n_segments, recv,
                                           shard_rows, workspace, true, st);
  if (e != cudaSuccess) return PKM_ERR_CUDA;
  const ShardOwnerLayout L = shard_owner_layout(G, n_triples);
  char* base = static_cast<char*>(workspace);
  pkm_saved s{};
  s.idx = reinterpret_cast<int32_t*>(base + L.rows);
  s.w = reinterpret_cast<float*>(base + L.wv);
  const int32_t* tok = reinterpret_cast<const int32_t*>(base + L.tok);
  return cuda_status(launch_value_grad(owner_plan(p, n_triples, shard_rows), values, s, dy_recv,
                                       dvalues, dw_recv, base + L.total, st, nullptr, nullptr,
                                       nullptr, tok));
}

pkm_status pkm_shard_scatter_dw(const pkm_dims* d, const int32_t* perm, const float* dw_ret,
                                float* dw, void* stream) {
  PKM_TRY(validate_dims(d));
  if (d->N == 0) return PKM_OK;
  PKM_NEED(perm); PKM_NEED(dw_ret); PKM_NEED(dw);
  Plan p;
  PKM_TRY(prepare(d, &p));
  return cuda_status(launch_shard_scatter_dw(p, perm, dw_ret, dw, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
