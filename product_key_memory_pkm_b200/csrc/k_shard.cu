// Row-sharded value table ("Meta AI 可扩展内存层", 9.1: the value matrix split by rows of
// the product-key index, every device reading only its own rows, candidate indices and
// partial weighted sums exchanged between devices; 4.5: row i*|C'| + j, so a range of
// leading sub-key indices is a contiguous range of rows).
//
// Shard g of G holds rows [g*R, min((g+1)*R, K)).  The rank that owns a batch of tokens
// (the source) runs F1-F3 itself, then:
//   route_kernel        buckets every selection (t, s) by the shard of its row, stably:
//                       the send buffer holds, per destination g, the selections of
//                       token 0, then token 1, ... as triples (segment, local row, w); a
//                       segment is one token's run of selections bound for g, numbered
//                       from 0 per destination.  perm[pos] = t*hk + s.
//   combine_kernel      y[t] = sum over g (ascending) of the partial row g sent back for
//                       t's segment (segpos[g][t], or nothing when t sent g nothing).
//   gather_dy_kernel    the upstream-gradient row of t once per segment, in segment order.
//   scatter_dw_kernel   dw[perm[pos]] = the returned dL/dw of the triple at pos.
// The owner of a shard receives the triples of every source, concatenated in source order:
//   owner_index_kernel  the received triples as arrays: local row, weight and global
//                       segment (source offset added); segment_start_kernel the first
//                       triple of every segment (binary search: segment ids ascend inside a
//                       source's run).
//   shard_bag_kernel    partial[j] = sum over segment j's triples of w * V[row], fp32
//                       (the segment's triples staged in shared memory, 8 rows in flight).
// and the backward's value pass on its rows reuses the value-row kernel with a per-entry
// token map (the entry's segment selects its upstream-gradient row).
#include <algorithm>

#include "k_sort.cuh"
#include "pkm_internal.cuh"

namespace pkm {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRouteWarps = 8;

// Each selection's shard and its rank among the token's earlier selections bound for the
// same shard.  Counting pass (kScatter = false): cnt[g*N + t] = selections of t for g.
// Scatter pass: the triples and perm at their send positions.
template <bool kScatter>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, int64_t N, int hk, int G,
    int64_t R, int64_t K, int32_t* __restrict__ cnt, const int32_t* __restrict__ tri_off,
    const int32_t* __restrict__ seg_scan, pkm_triple* __restrict__ send,
    int32_t* __restrict__ perm, int* status) {
  __shared__ int run[kRouteWarps][PKM_MAX_SHARDS];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kRouteWarps + wid;
  if (t >= N) return;  // warp-uniform; warps only synchronise among themselves below
  int* rw = run[wid];
  for (int g = lane; g < G; g += 32) rw[g] = 0;
  __syncwarp();
  for (int s0 = 0; s0 < hk; s0 += 32) {
    const int s = s0 + lane;
    const bool live = s < hk;
    int64_t row = live ? idx[t * hk + s] : 0;
    if (live && (row < 0 || row >= K)) {  // both passes route a bad row the same way
      if (!kScatter) set_status(status, kDevIndex);
      row = 0;
    }
    const int g = live ? (int)(row / R) : -1;
    const unsigned peers = __match_any_sync(kFull, g);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int rank = live ? rw[g] + before : 0;
    __syncwarp();
    if (live && before == 0) rw[g] += __popc(peers);  // one writer per shard group
    __syncwarp();
    if (kScatter && live) {
      const int64_t gN = (int64_t)g * N;
      const int64_t pos = (int64_t)tri_off[gN + t] + rank;
      pkm_triple tr;
      tr.seg = seg_scan[gN + t] - seg_scan[gN];
      tr.row = (int32_t)(row - (int64_t)g * R);
      tr.w = w[t * hk + s];
      send[pos] = tr;
      perm[pos] = (int32_t)(t * hk + s);
    }
  }
  if (!kScatter) {
    __syncwarp();
    for (int g = lane; g < G; g += 32) cnt[(int64_t)g * N + t] = rw[g];
  }
}

struct CntIn {
  const int32_t* c;
  __device__ int operator()(int64_t i) const { return c[i]; }
};
struct HasIn {
  const int32_t* c;
  __device__ int operator()(int64_t i) const { return c[i] > 0 ? 1 : 0; }
};
struct OffOut {
  int32_t* o;
  __device__ void operator()(int64_t i, int run, int, int64_t) const { o[i] = run; }
};
struct SegOut {
  int32_t* scan;
  int32_t* segpos;
  __device__ void operator()(int64_t i, int run, int v, int64_t) const {
    scan[i] = run;
    segpos[i] = v ? run : -1;
  }
};

// counts[g] = {selections, segments} bound for shard g
__global__ void route_counts_kernel(const int32_t* __restrict__ cnt,
                                    const int32_t* __restrict__ tri_off,
                                    const int32_t* __restrict__ seg_scan, int64_t N, int G,
                                    int32_t* __restrict__ counts) {
  const int64_t last = (int64_t)G * N - 1;
  const int tri_total = tri_off[last] + cnt[last];
  const int seg_total = seg_scan[last] + (cnt[last] > 0 ? 1 : 0);
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int64_t a = (int64_t)g * N, b = (int64_t)(g + 1) * N;
    counts[2 * g] = (g + 1 < G ? tri_off[b] : tri_total) - tri_off[a];
    counts[2 * g + 1] = (g + 1 < G ? seg_scan[b] : seg_total) - seg_scan[a];
  }
}

// ------------------------------------------------------------------ owner side
// pre[0..G] = exclusive scan of the received triple counts, pre[G+1 .. 2G+1] of the
// segment counts; a total that disagrees with the caller's sizes is an index error.
__global__ void owner_prefix_kernel(const int32_t* __restrict__ recv_counts, int G,
                                    int64_t n_tri, int64_t n_seg, int32_t* __restrict__ pre,
                                    int* status) {
  if (threadIdx.x != 0) return;
  int64_t a = 0, b = 0;
  for (int s = 0; s < G; ++s) {
    pre[s] = (int32_t)(a < n_tri ? a : n_tri);
    pre[G + 1 + s] = (int32_t)(b < n_seg ? b : n_seg);
    const int ct = recv_counts[2 * s], cs = recv_counts[2 * s + 1];
    if (ct < 0 || cs < 0 || cs > ct) set_status(status, kDevIndex);
    a += ct > 0 ? ct : 0;
    b += cs > 0 ? cs : 0;
  }
  pre[G] = (int32_t)(a < n_tri ? a : n_tri);
  pre[2 * G + 1] = (int32_t)(b < n_seg ? b : n_seg);
  if (a != n_tri || b != n_seg) set_status(status, kDevIndex);
}

// last s in [0, G) with pre[s] <= i (pre ascending, pre[0] = 0)
__device__ __forceinline__ int source_of(const int32_t* pre, int G, int64_t i) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Arrays of the received triples for the value pass: local row, weight and the global
// segment (its upstream-gradient row).  Out-of-range entries are recorded and clamped.
__global__ void owner_index_kernel(const pkm_triple* __restrict__ recv,
                                   const int32_t* __restrict__ pre, int G, int64_t n_tri,
                                   int64_t n_seg, int64_t shard_rows, int32_t* __restrict__ rows,
                                   float* __restrict__ wv, int32_t* __restrict__ tok,
                                   int* status) {
  const int32_t* seg_pre = pre + G + 1;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_tri;
       i += (int64_t)gridDim.x * blockDim.x) {
    const pkm_triple tr = recv[i];
    const int s = source_of(pre, G, i);
    int64_t j = (int64_t)seg_pre[s] + tr.seg;
    const int64_t seg_end = seg_pre[s + 1];
    if (tr.seg < 0 || j >= seg_end) {
      set_status(status, kDevIndex);
      j = seg_end > seg_pre[s] ? seg_end - 1 : 0;
    }
    if (j >= n_seg) j = n_seg - 1;
    int32_t r = tr.row;
    if (r < 0 || r >= shard_rows) {
      set_status(status, kDevIndex);
      r = 0;
    }
    rows[i] = r;
    wv[i] = tr.w;
    tok[i] = (int32_t)(j < 0 ? 0 : j);
  }
}

// start[j] = first received triple of global segment j, start[n_seg] = n_tri.  Inside a
// source's run the segment ids ascend, so it is a lower bound there; every start stays
// within [0, n_tri] whatever the input.
__global__ void segment_start_kernel(const pkm_triple* __restrict__ recv,
                                     const int32_t* __restrict__ pre, int G, int64_t n_tri,
                                     int64_t n_seg, int32_t* __restrict__ start) {
  const int32_t* seg_pre = pre + G + 1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j <= n_seg;
       j += (int64_t)gridDim.x * blockDim.x) {
    if (j == n_seg) {
      start[j] = (int32_t)n_tri;
      continue;
    }
    const int s = source_of(seg_pre, G, j);
    const int64_t local = j - seg_pre[s];
    int64_t lo = pre[s], hi = pre[s + 1];
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (recv[mid].seg < local) lo = mid + 1;
      else hi = mid;
    }
    start[j] = (int32_t)lo;
  }
}

// 16 bytes of a value row, streamed (no L1 allocation: every row is read once here)
__device__ __forceinline__ uint4 ld_row16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void to_f32(const uint4& u, __nv_bfloat16, float* f) { bf16x8_to_f32(u, f); }
__device__ __forceinline__ void to_f32(const uint4& u, float, float* f) {
  f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

constexpr int kBagChunk = 256, kBagAhead = 8;

// One CTA per segment.  The segment's triples are staged in shared memory (chunks of
// 256), then thread j accumulates 16-byte column slice j (j + blockDim.x, ...) over them
// with eight rows in flight; fp32 sums in triple order.
template <typename TV>
__global__ void __launch_bounds__(256) shard_bag_kernel(
    const pkm_triple* __restrict__ recv, const int32_t* __restrict__ start, const TV* __restrict__ V,
    int64_t shard_rows, int d_v, float* __restrict__ partial, int* status) {
  constexpr int E = 16 / sizeof(TV);
  __shared__ int32_t s_row[kBagChunk];
  __shared__ float s_w[kBagChunk];
  const int64_t j = blockIdx.x;
  const int i0 = start[j], i1 = start[j + 1];
  const int nvec = d_v / E, tid = threadIdx.x;
  for (int vb = 0; vb < nvec; vb += blockDim.x) {  // uniform over the CTA
    const int vec = vb + tid;
    const bool live = vec < nvec;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int base = i0; base < i1; base += kBagChunk) {
      const int n = min(kBagChunk, i1 - base);
      __syncthreads();  // the previous chunk is consumed
      for (int i = tid; i < n; i += blockDim.x) {
        const pkm_triple tr = recv[base + i];
        const bool ok = tr.row >= 0 && tr.row < shard_rows;
        if (!ok) set_status(status, kDevIndex);
        s_row[i] = ok ? tr.row : 0;
        s_w[i] = ok ? tr.w : 0.f;
      }
      __syncthreads();
      if (!live) continue;
      const TV* col = V + (int64_t)vec * E;
      int i = 0;
      for (; i + kBagAhead <= n; i += kBagAhead) {
        uint4 u[kBagAhead];
#pragma unroll
        for (int q = 0; q < kBagAhead; ++q) u[q] = ld_row16(col + (int64_t)s_row[i + q] * d_v);
#pragma unroll
        for (int q = 0; q < kBagAhead; ++q) {
          float f[E];
          to_f32(u[q], TV(), f);
          const float wq = s_w[i + q];
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(wq, f[e], acc[e]);
        }
      }
      for (; i < n; ++i) {
        float f[E];
        to_f32(ld_row16(col + (int64_t)s_row[i] * d_v), TV(), f);
        const float wq = s_w[i];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(wq, f[e], acc[e]);
      }
    }
    if (live) {
      float4* out = reinterpret_cast<float4*>(partial + j * d_v + (int64_t)vec * E);
#pragma unroll
      for (int e4 = 0; e4 < E / 4; ++e4)
        out[e4] = make_float4(acc[4 * e4], acc[4 * e4 + 1], acc[4 * e4 + 2], acc[4 * e4 + 3]);
    }
  }
}

// ------------------------------------------------------------------ source side
// y[t] = sum over g ascending of partial_recv[segpos[g][t]] (fixed order: deterministic)
__global__ void __launch_bounds__(256) combine_kernel(const int32_t* __restrict__ segpos,
                                                      const float* __restrict__ part, int64_t N,
                                                      int G, int64_t n_rows, int d_v,
                                                      float* __restrict__ y, int* status) {
  const int64_t t = blockIdx.x;
  const int nv = d_v / 4;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < G; ++g) {
      const int32_t p = segpos[(int64_t)g * N + t];
      if (p < 0) continue;
      if (p >= n_rows) {
        if (c == threadIdx.x) set_status(status, kDevIndex);
        continue;
      }
      const float4 v = reinterpret_cast<const float4*>(part + (int64_t)p * d_v)[c];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    reinterpret_cast<float4*>(y + t * d_v)[c] = acc;
  }
}

// dy_send[segpos[g][t]] = dy[t] for every segment of t
__global__ void __launch_bounds__(256) gather_dy_kernel(const int32_t* __restrict__ segpos,
                                                        const float* __restrict__ dy, int64_t N,
                                                        int G, int64_t n_rows, int d_v,
                                                        float* __restrict__ out, int* status) {
  const int64_t t = blockIdx.x;
  const int nv = d_v / 4;
  for (int g = 0; g < G; ++g) {
    const int32_t p = segpos[(int64_t)g * N + t];
    if (p < 0) continue;
    if (p >= n_rows) {
      if (threadIdx.x == 0) set_status(status, kDevIndex);
      continue;
    }
    const float4* src = reinterpret_cast<const float4*>(dy + t * d_v);
    float4* dst = reinterpret_cast<float4*>(out + (int64_t)p * d_v);
    for (int c = threadIdx.x; c < nv; c += blockDim.x) dst[c] = src[c];
  }
}

__global__ void scatter_dw_kernel(const int32_t* __restrict__ perm, const float* __restrict__ dw_ret,
                                  int64_t n, float* __restrict__ dw, int* status) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t p = perm[i];
    if (p < 0 || p >= n) {
      set_status(status, kDevIndex);
      continue;
    }
    dw[p] = dw_ret[i];
  }
}

inline unsigned grid_for(int64_t n, int threads, int sm_count) {
  const int64_t b = (n + threads - 1) / threads;
  return (unsigned)std::max<int64_t>(1, std::min<int64_t>(b, (int64_t)sm_count * 16));
}

inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

// ------------------------------------------------------------------ host launchers
ShardRouteLayout shard_route_layout(int64_t N, int G) {
  ShardRouteLayout L{};
  const int64_t n = (int64_t)G * N;
  size_t o = 0;
  L.cnt = o; o += up256(4 * (size_t)n);
  L.tri_off = o; o += up256(4 * (size_t)n);
  L.seg_scan = o; o += up256(4 * (size_t)n);
  L.bsum = o; o += up256(4 * (size_t)sort::scan_bsum_len(n));
  L.total = o;
  return L;
}

cudaError_t launch_shard_route(const Plan& p, int G, int64_t R, const int32_t* idx, const float* w,
                               int32_t* counts, int32_t* segpos, pkm_triple* send, int32_t* perm,
                               void* ws, cudaStream_t st) {
  const ShardRouteLayout L = shard_route_layout(p.N, G);
  char* base = static_cast<char*>(ws);
  int32_t* cnt = reinterpret_cast<int32_t*>(base + L.cnt);
  int32_t* tri_off = reinterpret_cast<int32_t*>(base + L.tri_off);
  int32_t* seg_scan = reinterpret_cast<int32_t*>(base + L.seg_scan);
  int* bsum = reinterpret_cast<int*>(base + L.bsum);
  const int hk = p.h * p.ksel;
  const unsigned blocks = (unsigned)((p.N + kRouteWarps - 1) / kRouteWarps);
  const int64_t n = (int64_t)G * p.N;
  route_kernel<false><<<blocks, kRouteWarps * 32, 0, st>>>(idx, w, p.N, hk, G, R, p.K, cnt, nullptr,
                                                          nullptr, nullptr, nullptr, p.status);
  PKM_COUNT(1);
  cudaError_t e = sort::exclusive_scan(CntIn{cnt}, OffOut{tri_off}, n, bsum, st);
  if (e != cudaSuccess) return e;
  e = sort::exclusive_scan(HasIn{cnt}, SegOut{seg_scan, segpos}, n, bsum, st);
  if (e != cudaSuccess) return e;
  route_counts_kernel<<<1, 256, 0, st>>>(cnt, tri_off, seg_scan, p.N, G, counts);
  PKM_COUNT(1);
  route_kernel<true><<<blocks, kRouteWarps * 32, 0, st>>>(idx, w, p.N, hk, G, R, p.K, cnt, tri_off,
                                                         seg_scan, send, perm, p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

ShardOwnerLayout shard_owner_layout(int G, int64_t n_tri) {
  ShardOwnerLayout L{};
  size_t o = 0;
  L.pre = o; o += up256(4 * (size_t)(2 * G + 2));
  L.start = o; o += up256(4 * (size_t)(n_tri + 1));
  L.rows = o; o += up256(4 * (size_t)std::max<int64_t>(n_tri, 1));
  L.wv = o; o += up256(4 * (size_t)std::max<int64_t>(n_tri, 1));
  L.tok = o; o += up256(4 * (size_t)std::max<int64_t>(n_tri, 1));
  L.total = o;
  return L;
}

cudaError_t launch_shard_owner_index(const Plan& p, int G, const int32_t* recv_counts,
                                     int64_t n_tri, int64_t n_seg, const pkm_triple* recv,
                                     int64_t shard_rows, void* ws, bool want_arrays,
                                     cudaStream_t st) {
  const ShardOwnerLayout L = shard_owner_layout(G, n_tri);
  char* base = static_cast<char*>(ws);
  int32_t* pre = reinterpret_cast<int32_t*>(base + L.pre);
  owner_prefix_kernel<<<1, 32, 0, st>>>(recv_counts, G, n_tri, n_seg, pre, p.status);
  PKM_COUNT(1);
  segment_start_kernel<<<grid_for(n_seg + 1, 256, p.sm_count), 256, 0, st>>>(
      recv, pre, G, n_tri, n_seg, reinterpret_cast<int32_t*>(base + L.start));
  PKM_COUNT(1);
  if (want_arrays) {
    owner_index_kernel<<<grid_for(n_tri, 256, p.sm_count), 256, 0, st>>>(
        recv, pre, G, n_tri, n_seg, shard_rows, reinterpret_cast<int32_t*>(base + L.rows),
        reinterpret_cast<float*>(base + L.wv), reinterpret_cast<int32_t*>(base + L.tok), p.status);
    PKM_COUNT(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_shard_bag(const Plan& p, int G, int64_t n_seg, const pkm_triple* recv,
                             const void* values, int64_t shard_rows, float* partial, void* ws,
                             int64_t n_tri, cudaStream_t st) {
  const ShardOwnerLayout L = shard_owner_layout(G, n_tri);
  const int32_t* start = reinterpret_cast<const int32_t*>(static_cast<char*>(ws) + L.start);
  const int E = p.vfp32 ? 4 : 8;
  const int nvec = p.d_v / E;
  const int threads = std::min(256, std::max(32, (nvec + 31) / 32 * 32));
  if (p.vfp32)
    shard_bag_kernel<float><<<(unsigned)n_seg, threads, 0, st>>>(
        recv, start, static_cast<const float*>(values), shard_rows, p.d_v, partial, p.status);
  else
    shard_bag_kernel<__nv_bfloat16><<<(unsigned)n_seg, threads, 0, st>>>(
        recv, start, static_cast<const __nv_bfloat16*>(values), shard_rows, p.d_v, partial,
        p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_shard_combine(const Plan& p, int G, const int32_t* segpos, const float* part,
                                 int64_t n_rows, float* y, cudaStream_t st) {
  const int threads = std::min(256, std::max(32, (p.d_v / 4 + 31) / 32 * 32));
  combine_kernel<<<(unsigned)p.N, threads, 0, st>>>(segpos, part, p.N, G, n_rows, p.d_v, y,
                                                    p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_shard_gather_dy(const Plan& p, int G, const int32_t* segpos, const float* dy,
                                   int64_t n_rows, float* out, cudaStream_t st) {
  const int threads = std::min(256, std::max(32, (p.d_v / 4 + 31) / 32 * 32));
  gather_dy_kernel<<<(unsigned)p.N, threads, 0, st>>>(segpos, dy, p.N, G, n_rows, p.d_v, out,
                                                      p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

cudaError_t launch_shard_scatter_dw(const Plan& p, const int32_t* perm, const float* dw_ret,
                                    float* dw, cudaStream_t st) {
  const int64_t n = p.N * p.h * p.ksel;
  scatter_dw_kernel<<<grid_for(n, 256, p.sm_count), 256, 0, st>>>(perm, dw_ret, n, dw, p.status);
  PKM_COUNT(1);
  return cudaGetLastError();
}

}  // namespace pkm
