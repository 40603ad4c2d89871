// The whole forward F1-F4 of a few tokens (decode-shaped calls, N <= 16) in one kernel.
//
// A few-token call moves little (the query weights, the sub-keys and N*h*k value rows)
// but, run as four kernels, pays four launch latencies and four rounds of HBM latency
// in series.  Here one CTA per SM runs the four steps as phases separated by grid-wide
// barriers (cooperative launch, so every CTA is resident; every barrier wait is bounded
// and reports PKM_ERR_DEVICE_TIMEOUT instead of hanging):
//
//   A  q = BN(x Wq^T): one warp per output column (Wq row streamed with all its
//      16-byte pieces in flight), the tokens' x in shared memory; q written as the bf16
//      hi/lo planes (and q-hat) the other entry points use ("Large Memory Layers with
//      Product Keys", method details: the query network).
//   B  sub-key scores: one item per (head, half, block of 64 sub-keys); the block's rows
//      copied into shared memory by asynchronous copies (a CTA's first block at kernel
//      start, since it does not depend on q; the others asked of L2 then), every
//      token's scores against them as eight partial dot products per key (each thread
//      accumulating all tokens), and each token's best k of the block by rank (score
//      desc, index asc) written to the workspace.
//   C  one item per (token, head): each half's block lists merged pairwise in shared
//      memory (log2 of the block count levels, every entry placed by its merge rank),
//      then the top k of the k x k candidate combine, found by ranking only the pairs
//      (a, b) with (a + 1)(b + 1) <= k, and the softmax over the k winners (the same
//      total order as pkm_candidate_topk; method details: top-k in each half, then
//      keep k).
//   D  y = sum over heads and winners of w V[row]: one warp per (token, 16 columns),
//      lane pairs reading the 32-byte pieces of 16 rows at a time, then a shuffle sum in
//      a fixed order ("Meta AI 可扩展内存层" 5.3).
//
// The grid barrier lives in a small array of slots in device memory; every call takes
// the next slot, so calls in flight on different streams do not share one.
#include <algorithm>
#include <atomic>
#include <climits>
#include <mutex>

#include "pkm_internal.cuh"

namespace pkm {

constexpr int kFusedBarSlots = 64;
// per slot: {arrivals, departures, -, -}; word 2 of slot 0 is the poison word a timed-out
// barrier sets, after which every fused call reports the timeout and does nothing
static __device__ unsigned int g_fused_bar[kFusedBarSlots][4];

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kFT = 512, kFW = kFT / 32;
constexpr int kBlkKeys = 64;      // sub-keys per scoring item
constexpr int kMaxTok = 16;       // tokens per call (kSmallTokens)
constexpr int kParts = kFT / kBlkKeys;  // partial dot products per scored key
constexpr int kMaxPairs = 128;    // pairs (a, b) with (a + 1)(b + 1) <= k, k <= 32: at most 119
constexpr int kRowsAhead = 8;     // value rows in flight per lane
constexpr int kAhead = 8;         // Wq pieces in flight per lane
constexpr int kStageAhead = 4;    // list entries in flight per thread
constexpr long long kBarBudget = 100000000LL;  // ~50 ms of SM clock

struct FusedArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* Wq;
  const float* bn;
  const __nv_bfloat16* sub;
  const __nv_bfloat16* V;
  float* y;
  __nv_bfloat16* q;  // [2][N][hq]
  float* qhat;       // [N][hq] or null
  float* sub_s;
  int32_t* sub_i;
  int32_t* idx;
  float* w;
  float* part_s;     // [2h][nblk][N][k]
  int32_t* part_i;
  unsigned int* bar;     // this call's slot
  unsigned int* poison;
  int* status;
  int64_t K;
  int N, d_in, h, dk, half, C1, C2, k, d_v, hq, nb1, nb2, nblk;
  int b_off;  // byte offset of phase B's shared memory; > 0: its first block is copied at start
  float eps, scale, lo_scale;
};

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier number `nth` (1, 2, ...) of this call: the arrivals counter only
// grows within a call, so barrier n is passed once it reaches n * gridDim.x (the arrival
// releases this CTA's writes, the wait acquires everyone's).  Returns false, after
// recording the timeout and setting the poison word, if the budget expired.
__device__ bool grid_sync(const FusedArgs& a, unsigned int nth, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned int target = nth * gridDim.x;
    unsigned int old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.bar) : "memory");
    if (old + 1u < target) {
      const long long t0 = clock64();
      while (ld_acquire(a.bar) < target) {
        if (clock64() - t0 > kBarBudget) {
          set_status(a.status, kDevTimeout);
          atomicExch(a.poison, 1u);
          ok = 0;
          break;
        }
        __nanosleep(20);
      }
    }
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

// After the last barrier: the last CTA to leave returns the slot to zero for its next
// call (no CTA reads the arrivals counter once it has passed the last barrier).
__device__ void grid_leave(const FusedArgs& a) {
  if (threadIdx.x == 0 && atomicAdd(a.bar + 1, 1u) == gridDim.x - 1) {
    atomicExch(a.bar, 0u);
    atomicExch(a.bar + 1, 0u);
  }
}

// (a ranks before b) in (score desc, index asc)
__device__ __forceinline__ bool before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// ---------------------------------------------------------------- A: query network
__device__ __forceinline__ void load_wq(const FusedArgs& a, int o, int cb, int nch, uint4 (&wv)[kAhead]) {
  const uint4* wr = reinterpret_cast<const uint4*>(a.Wq + (int64_t)o * a.d_in);
#pragma unroll
  for (int u = 0; u < kAhead; ++u) {
    const int c = cb + 32 * u;
    wv[u] = c < nch ? __ldg(wr + c) : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int TB>
__device__ void phase_query(const FusedArgs& a, unsigned char* sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sm);
  const int nch = a.d_in / 8;
  const int o0 = blockIdx.x * kFW + warp;
  // the first column's Wq pieces and BatchNorm statistics are in flight while x is staged
  uint4 wv[kAhead];
  float bnv[4] = {0.f, 1.f, 1.f, 0.f};
  if (o0 < a.hq) {
    load_wq(a, o0, lane, nch, wv);
#pragma unroll
    for (int r = 0; r < 4; ++r) bnv[r] = __ldg(a.bn + r * a.hq + o0);
  }
  for (int i = tid; i < a.N * nch; i += kFT) {
    const int t = i / nch, c = i % nch;
    reinterpret_cast<uint4*>(xs + (int64_t)t * a.d_in)[c] =
        __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)t * a.d_in) + c);
  }
  __syncthreads();
  for (int o = o0; o < a.hq; o += gridDim.x * kFW) {
    if (o != o0) {
#pragma unroll
      for (int r = 0; r < 4; ++r) bnv[r] = __ldg(a.bn + r * a.hq + o);
    }
    float acc[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) acc[t] = 0.f;
    for (int cb = lane; cb < nch; cb += 32 * kAhead) {
      if (o != o0 || cb != lane) load_wq(a, o, cb, nch, wv);
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int c = cb + 32 * u;
        if (c >= nch) break;
        float wf[8];
        bf16x8_to_f32(wv[u], wf);
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          if (TB == 1 || t < a.N) {
            float xf[8];
            bf16x8_to_f32(reinterpret_cast<const uint4*>(xs + (int64_t)t * a.d_in)[c], xf);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[t] = fmaf(wf[e], xf[e], acc[t]);
          }
        }
      }
    }
    float mine = 0.f;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      if (TB == 1 || t < a.N) {  // warp-uniform
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) acc[t] += __shfl_xor_sync(kFull, acc[t], s);
        if (lane == t) mine = acc[t];
      }
    }
    if (lane < a.N) {
      const float inv = 1.0f / sqrtf(bnv[1] + a.eps);
      const float hval = (mine - bnv[0]) * inv;
      const float qq = fmaf(bnv[2], hval, bnv[3]);
      const __nv_bfloat16 hb = __float2bfloat16_rn(qq);
      const __nv_bfloat16 lb = __float2bfloat16_rn(qq - __bfloat162float(hb));
      const int64_t off = (int64_t)lane * a.hq + o;
      a.q[off] = hb;
      a.q[(int64_t)a.N * a.hq + off] = lb;
      if (a.qhat) a.qhat[off] = hval;
    }
  }
}

// ---------------------------------------------------------------- B: block scores
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}

// The sub-key rows of scoring item `it`: head, half, first key, number of keys.
struct BlockItem {
  int hh, s, blk, c0, nc;
};

__device__ __forceinline__ BlockItem block_item(const FusedArgs& a, int it) {
  const int per_head = a.nb1 + a.nb2;
  BlockItem b;
  b.hh = it / per_head;
  const int r = it % per_head;
  b.s = r < a.nb1 ? 0 : 1;
  b.blk = b.s ? r - a.nb1 : r;
  b.c0 = b.blk * kBlkKeys;
  b.nc = min(kBlkKeys, (b.s ? a.C2 : a.C1) - b.c0);
  return b;
}

__device__ __forceinline__ const __nv_bfloat16* block_rows(const FusedArgs& a, const BlockItem& b) {
  return a.sub + ((int64_t)b.hh * (a.C1 + a.C2) + b.s * a.C1 + b.c0) * a.half;
}

// Ask L2 for this CTA's scoring blocks while the query network runs.
__device__ void prefetch_blocks(const FusedArgs& a) {
  if (threadIdx.x != 0) return;
  const int items = a.h * (a.nb1 + a.nb2);
  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const BlockItem b = block_item(a, it);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(block_rows(a, b)),
                 "r"((uint32_t)(b.nc * a.half * 2))
                 : "memory");
  }
}

// The block rows of scoring item `it` into the padded rows of kc (asynchronous copies).
__device__ void issue_block_rows(const FusedArgs& a, int it, __nv_bfloat16* kc) {
  const BlockItem b = block_item(a, it);
  const int ks = a.half + 8, npc = a.half / 8;
  const uint4* src = reinterpret_cast<const uint4*>(block_rows(a, b));
  for (int i = threadIdx.x; i < b.nc * npc; i += kFT) {
    const int c = i / npc, pc = i % npc;
    cp_async16(kc + (size_t)c * ks + pc * 8, src + i);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int TB>
__device__ void phase_scores(const FusedArgs& a, unsigned char* sm) {
  const int tid = threadIdx.x;
  const int ks = a.half + 8;  // bf16 row stride (16-byte pad: conflict-free rows)
  const int NT = a.N * kBlkKeys;
  sm += a.b_off;
  __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(sm);
  float* qs = reinterpret_cast<float*>(sm + (size_t)kBlkKeys * ks * 2);
  float* scp = qs + (size_t)a.N * a.half;  // [kParts][N][64]
  float* sc = scp + kParts * (size_t)NT;   // [N][64]
  const int npc = a.half / 8;
  const int items = a.h * (a.nb1 + a.nb2);
  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    const BlockItem b = block_item(a, it);
    // the first block's rows were copied at kernel start when there was room
    if (a.b_off == 0 || it != (int)blockIdx.x) issue_block_rows(a, it, kc);
    // q = hi + lo_scale * lo of this head-half, written by phase A (read through L2)
    for (int i = tid; i < a.N * npc; i += kFT) {
      const int t = i / npc, pc = i % npc;
      const int64_t off = (int64_t)t * a.hq + b.hh * a.dk + b.s * a.half + pc * 8;
      float hf[8], lf[8];
      bf16x8_to_f32(__ldcg(reinterpret_cast<const uint4*>(a.q + off)), hf);
      bf16x8_to_f32(__ldcg(reinterpret_cast<const uint4*>(a.q + (int64_t)a.N * a.hq + off)), lf);
#pragma unroll
      for (int e = 0; e < 8; ++e) qs[t * a.half + pc * 8 + e] = hf[e] + a.lo_scale * lf[e];
    }
    cp_async_wait_all();
    __syncthreads();
    // eight partial dot products per key, each over an eighth of the pieces, every
    // token's at once (a key piece is read once for all tokens); a warp covers 32 keys
    // of one part (conflict-free padded rows, the q pieces broadcast)
    {
      const int p = tid / kBlkKeys, c = tid % kBlkKeys;
      float acc[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[t] = 0.f;
      if (c < b.nc) {
        const __nv_bfloat16* kr = kc + (size_t)c * ks;
        const int pc1 = (p + 1) * npc / kParts;
        for (int pc = p * npc / kParts; pc < pc1; ++pc) {
          float kf[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(kr + pc * 8), kf);
#pragma unroll
          for (int t = 0; t < TB; ++t) {
            if (TB == 1 || t < a.N) {
              const float4* qr = reinterpret_cast<const float4*>(qs + (size_t)t * a.half + pc * 8);
              const float4 q0 = qr[0], q1 = qr[1];
              acc[t] = fmaf(kf[0], q0.x, acc[t]);
              acc[t] = fmaf(kf[1], q0.y, acc[t]);
              acc[t] = fmaf(kf[2], q0.z, acc[t]);
              acc[t] = fmaf(kf[3], q0.w, acc[t]);
              acc[t] = fmaf(kf[4], q1.x, acc[t]);
              acc[t] = fmaf(kf[5], q1.y, acc[t]);
              acc[t] = fmaf(kf[6], q1.z, acc[t]);
              acc[t] = fmaf(kf[7], q1.w, acc[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TB; ++t)
        if (TB == 1 || t < a.N) scp[((size_t)p * a.N + t) * kBlkKeys + c] = acc[t];
    }
    __syncthreads();
    for (int i = tid; i < NT; i += kFT) {
      float v = -INFINITY;
      if ((i % kBlkKeys) < b.nc) {
        v = scp[i];
#pragma unroll
        for (int p = 1; p < kParts; ++p) v += scp[(size_t)p * NT + i];
      }
      sc[i] = v;
    }
    __syncthreads();
    // each token's best k of the block, placed by rank; short blocks padded
    const int hs = b.hh * 2 + b.s;
    for (int i = tid; i < NT; i += kFT) {
      const int t = i / kBlkKeys, c = i % kBlkKeys;
      const int64_t lst = (((int64_t)hs * a.nblk + b.blk) * a.N + t) * a.k;
      if (c < b.nc) {
        const float v = sc[i];
        const float4* row = reinterpret_cast<const float4*>(sc + t * kBlkKeys);
        int rank = 0;
#pragma unroll
        for (int c4 = 0; c4 < kBlkKeys / 4; ++c4) {
          const float4 r4 = row[c4];
          rank += before(r4.x, 4 * c4, v, c) + before(r4.y, 4 * c4 + 1, v, c) +
                  before(r4.z, 4 * c4 + 2, v, c) + before(r4.w, 4 * c4 + 3, v, c);
        }
        if (rank < a.k) {
          a.part_s[lst + rank] = v;
          a.part_i[lst + rank] = b.c0 + c;
        }
      } else if (c < a.k) {
        a.part_s[lst + c] = -INFINITY;
        a.part_i[lst + c] = INT_MAX;
      }
    }
    __syncthreads();  // the next item reuses the shared memory
  }
}

// ---------------------------------------------------------------- C: merge + candidates
// Keeps, in every lane, the better (lower lanes) or the worse (upper lanes) of its entry
// and the one `d` lanes away: the stages d = 16 .. 1 sort a bitonic sequence of 32
// entries into rank order (score desc, index asc).
__device__ __forceinline__ void bitonic_sort32(float& vs, int32_t& vi, int lane) {
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    const float ps = __shfl_xor_sync(kFull, vs, d);
    const int32_t pi = __shfl_xor_sync(kFull, vi, d);
    const bool lower = (lane & d) == 0;
    if (lower == before(ps, pi, vs, vi)) {
      vs = ps;
      vi = pi;
    }
  }
}

// Key of a candidate pair in the combine order (sum desc, first-half score desc,
// second-half score desc, flat index asc) as two unsigned words compared high first.
__device__ __forceinline__ ulonglong2 pair_key(float S, float s1, float s2, int32_t f) {
  ulonglong2 kk;
  kk.x = ((unsigned long long)order_key(S) << 32) | order_key(s1);
  kk.y = ((unsigned long long)order_key(s2) << 32) | (uint32_t)~f;
  return kk;
}

__device__ void phase_select(const FusedArgs& a, unsigned char* sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k, nblk = a.nblk;
  const int plane = 2 * nblk * k;  // one buffer: [half][list][k]
  float* LS = reinterpret_cast<float*>(sm);
  int32_t* LI = reinterpret_cast<int32_t*>(LS + 2 * plane);
  ulonglong2* pk = reinterpret_cast<ulonglong2*>(LI + 2 * plane);  // 16-byte aligned
  float* pS = reinterpret_cast<float*>(pk + kMaxPairs);
  int32_t* pf = reinterpret_cast<int32_t*>(pS + kMaxPairs);
  int* poff = reinterpret_cast<int*>(pf + kMaxPairs);  // [32]
  float* oS = reinterpret_cast<float*>(poff + 32);     // [32]
  int32_t* oI = reinterpret_cast<int32_t*>(oS + 32);   // [32]
  __shared__ int s_np;
  for (int it = blockIdx.x; it < a.N * a.h; it += gridDim.x) {
    const int t = it / a.h, hh = it % a.h;
    // both halves' block lists into shared memory
    const int tot0 = a.nb1 * k, tot = tot0 + a.nb2 * k;
    for (int e0 = tid; e0 < tot; e0 += kStageAhead * kFT) {
      float vs[kStageAhead];
      int32_t vi[kStageAhead];
      int at[kStageAhead];
#pragma unroll
      for (int u = 0; u < kStageAhead; ++u) {
        const int e = e0 + u * kFT;
        at[u] = -1;
        if (e < tot) {
          const int s = e < tot0 ? 0 : 1;
          const int e2 = e - (s ? tot0 : 0);
          const int l = e2 / k, j = e2 % k;
          const int64_t src = ((((int64_t)hh * 2 + s) * nblk + l) * a.N + t) * k + j;
          vs[u] = __ldcg(a.part_s + src);
          vi[u] = __ldcg(a.part_i + src);
          at[u] = (s * nblk + l) * k + j;
        }
      }
#pragma unroll
      for (int u = 0; u < kStageAhead; ++u) {
        if (at[u] >= 0) {
          LS[at[u]] = vs[u];
          LI[at[u]] = vi[u];
        }
      }
    }
    __syncthreads();
    // pairwise merge tree, one warp per pair of lists: lists 2m and 2m+1 become list m
    // (an odd last list moves up as it is).  The better of entry j of the first list and
    // entry 31 - j of the second, over 32 lanes (short lists padded with the lowest
    // entry), is a bitonic sequence holding the top 32 of both; sorting it gives the
    // merged list.
    int n0 = a.nb1, n1 = a.nb2, cur = 0;
    while (n0 > 1 || n1 > 1) {
      const float* cs = LS + cur * plane;
      const int32_t* ci = LI + cur * plane;
      float* ns = LS + (cur ^ 1) * plane;
      int32_t* ni = LI + (cur ^ 1) * plane;
      const int u0 = (n0 + 1) >> 1, units = u0 + ((n1 + 1) >> 1);
      for (int un = warp; un < units; un += kFW) {
        const int s = un < u0 ? 0 : 1;
        const int m = un - (s ? u0 : 0);
        const int n = s ? n1 : n0;
        const int la = (s * nblk + 2 * m) * k;
        float vs = lane < k ? cs[la + lane] : -INFINITY;
        int32_t vi = lane < k ? ci[la + lane] : INT_MAX;
        if (2 * m + 1 < n) {
          const int jb = 31 - lane;
          const float bs = jb < k ? cs[la + k + jb] : -INFINITY;
          const int32_t bi = jb < k ? ci[la + k + jb] : INT_MAX;
          if (before(bs, bi, vs, vi)) {
            vs = bs;
            vi = bi;
          }
          bitonic_sort32(vs, vi, lane);
        }
        if (lane < k) {
          ns[(s * nblk + m) * k + lane] = vs;
          ni[(s * nblk + m) * k + lane] = vi;
        }
      }
      __syncthreads();
      cur ^= 1;
      n0 = (n0 + 1) >> 1;
      n1 = (n1 + 1) >> 1;
    }
    const float* f1s = LS + cur * plane;
    const int32_t* f1i = LI + cur * plane;
    const float* f2s = f1s + nblk * k;
    const int32_t* f2i = f1i + nblk * k;
    // the pairs (a, b) with (a + 1)(b + 1) <= k: every pair before (a, b) in the
    // candidate order has a' <= a and b' <= b, so these hold the top k, and a pair's
    // rank among them is its rank among all k x k.  Row a's pairs start at poff[a].
    if (warp == 0) {
      const int64_t so = ((int64_t)t * a.h + hh) * 2 * k;
      if (lane < k) {  // the per-half lists, as pkm_subkey_scores writes them
        a.sub_s[so + lane] = f1s[lane];
        a.sub_i[so + lane] = f1i[lane];
        a.sub_s[so + k + lane] = f2s[lane];
        a.sub_i[so + k + lane] = f2i[lane];
      }
      const int cnt = lane < k ? k / (lane + 1) : 0;
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      poff[lane] = incl - cnt;
      if (lane == 31) s_np = incl;
    }
    __syncthreads();
    for (int i = tid; i < k * k; i += kFT) {
      const int ra = i / k, rb = i % k;
      if ((ra + 1) * (rb + 1) <= k) {
        const int e = poff[ra] + rb;
        const float s1 = f1s[ra], s2 = f2s[rb];
        const int32_t f = f1i[ra] * a.C2 + f2i[rb];
        pS[e] = s1 + s2;
        pf[e] = f;
        pk[e] = pair_key(s1 + s2, s1, s2, f);
      }
    }
    __syncthreads();
    // rank every pair: four threads per pair, each over every fourth pair
    const int np = s_np;
    for (int base = 0; base < 4 * np; base += kFT) {
      const int i = base + tid;
      const bool on = i < 4 * np;
      const int e = i >> 2, q = i & 3;
      int cnt = 0;
      if (on) {
        const ulonglong2 me = pk[e];
#pragma unroll 4
        for (int g = q; g < np; g += 4) {
          const ulonglong2 o = pk[g];
          cnt += (o.x > me.x || (o.x == me.x && o.y > me.y)) ? 1 : 0;
        }
      }
      cnt += __shfl_xor_sync(kFull, cnt, 1);
      cnt += __shfl_xor_sync(kFull, cnt, 2);
      if (on && q == 0 && cnt < k) {
        oS[cnt] = pS[e];
        oI[cnt] = pf[e];
      }
    }
    __syncthreads();
    if (warp == 1 && lane < k) {  // the bag reads the winners' rows next: ask L2 for them
      const int32_t row = oI[lane];
      if (row >= 0 && row < a.K)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.V + (int64_t)row * a.d_v),
                     "r"((uint32_t)(a.d_v * 2))
                     : "memory");
    }
    if (warp == 0) {
      const bool live = lane < k;
      const float outS = live ? oS[lane] : 0.f;
      const float S0 = oS[0];
      const float ex = live ? expf(a.scale * (outS - S0)) : 0.f;
      float sum = ex;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
      if (live) {
        const int64_t wo = ((int64_t)t * a.h + hh) * k;
        const int32_t row = oI[lane];
        a.idx[wo + lane] = row;
        a.w[wo + lane] = ex / sum;
      }
    }
    __syncthreads();  // the next item reuses the lists
  }
}

// ---------------------------------------------------------------- D: bag
// One warp per (token, 16 columns): lane pairs read the two 16-byte halves of a 32-byte
// piece of a row, 16 rows at a time, every row's index and weight loaded before its data.
__device__ void phase_bag(const FusedArgs& a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int hk = a.h * a.k;
  const int ng = (a.d_v + 15) / 16;
  const int rl = lane >> 1;
  for (int it = warp * gridDim.x + blockIdx.x; it < a.N * ng; it += gridDim.x * kFW) {
    const int t = it / ng, g = it % ng;
    const int col = g * 16 + (lane & 1) * 8;
    const bool valid = col < a.d_v;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int r0 = 0; r0 < hk; r0 += 16 * kRowsAhead) {
      int64_t row[kRowsAhead];
      float wt[kRowsAhead];
#pragma unroll
      for (int u = 0; u < kRowsAhead; ++u) {
        const int r = r0 + u * 16 + rl;
        row[u] = -1;
        wt[u] = 0.f;
        if (r < hk) {
          const int32_t ri = __ldcg(a.idx + (int64_t)t * hk + r);
          wt[u] = __ldcg(a.w + (int64_t)t * hk + r);
          if (ri < 0 || ri >= a.K) set_status(a.status, kDevIndex);
          else row[u] = ri;
        }
      }
      uint4 vv[kRowsAhead];
#pragma unroll
      for (int u = 0; u < kRowsAhead; ++u)
        vv[u] = (valid && row[u] >= 0)
                    ? __ldg(reinterpret_cast<const uint4*>(a.V + row[u] * a.d_v + col))
                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < kRowsAhead; ++u) {
        float f[8];
        bf16x8_to_f32(vv[u], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(wt[u], f[e], acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int o = 2; o < 32; o <<= 1) acc[e] += __shfl_xor_sync(kFull, acc[e], o);
    if (valid && rl == 0) {
      float4* yo = reinterpret_cast<float4*>(a.y + (int64_t)t * a.d_v + col);
      yo[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      yo[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// TB: the token count rounded up to a power of two (loops over tokens unroll to TB).
template <int TB>
__global__ void __launch_bounds__(kFT, 1) decode_fused_kernel(const FusedArgs a) {
  extern __shared__ __align__(16) unsigned char fsm[];
  __shared__ int s_ok;
  if (*reinterpret_cast<volatile unsigned int*>(a.poison) != 0u) {
    if (threadIdx.x == 0) set_status(a.status, kDevTimeout);
    return;
  }
  // phase B's first block does not depend on q: when its shared memory lies past phase
  // A's, its rows come in while the query network runs
  if (a.b_off > 0 && (int)blockIdx.x < a.h * (a.nb1 + a.nb2))
    issue_block_rows(a, blockIdx.x, reinterpret_cast<__nv_bfloat16*>(fsm + a.b_off));
  prefetch_blocks(a);
  phase_query<TB>(a, fsm);
  if (!grid_sync(a, 1, &s_ok)) return;
  phase_scores<TB>(a, fsm);
  if (!grid_sync(a, 2, &s_ok)) return;
  phase_select(a, fsm);
  if (!grid_sync(a, 3, &s_ok)) return;
  grid_leave(a);
  phase_bag(a);
}

int nblk_of(int C) { return (C + kBlkKeys - 1) / kBlkKeys; }

constexpr size_t kFusedSmemMax = 200 * 1024;  // dynamic shared memory the layout may take

// Phase B's shared-memory offset: past phase A's staged tokens when both fit.
size_t fused_b_off(const Plan& p) {
  const size_t qa = ((size_t)p.N * p.d_in * 2 + 127) & ~size_t(127);
  const size_t sb = (size_t)kBlkKeys * (p.half + 8) * 2 + (size_t)p.N * p.half * 4 +
                    (kParts + 1) * (size_t)p.N * kBlkKeys * 4;
  return qa + sb <= kFusedSmemMax ? qa : 0;
}

size_t fused_smem(const Plan& p) {
  const size_t qa = (size_t)p.N * p.d_in * 2;
  const size_t sb = (size_t)kBlkKeys * (p.half + 8) * 2 + (size_t)p.N * p.half * 4 +
                    (kParts + 1) * (size_t)p.N * kBlkKeys * 4;
  const size_t sc = (size_t)2 * 2 * nblk_of(std::max(p.C1, p.C2)) * p.k * 8 + kMaxPairs * 24 +
                    96 * 4;
  return std::max(std::max(qa, fused_b_off(p) + sb), sc);
}

constexpr int kMaxFusedDevices = 64;
using FusedKernel = void (*)(const FusedArgs);
constexpr FusedKernel kFusedKernels[5] = {decode_fused_kernel<1>, decode_fused_kernel<2>,
                                          decode_fused_kernel<4>, decode_fused_kernel<8>,
                                          decode_fused_kernel<16>};
std::atomic<int> g_smem_ready[kMaxFusedDevices][5];
std::atomic<void*> g_bar_ptr[kMaxFusedDevices];
std::atomic<unsigned int> g_bar_epoch{0};
std::mutex g_bar_mu;

unsigned int* bar_base(int dev) {
  void* ptr = g_bar_ptr[dev].load(std::memory_order_acquire);
  if (ptr) return static_cast<unsigned int*>(ptr);
  std::lock_guard<std::mutex> lock(g_bar_mu);
  ptr = g_bar_ptr[dev].load(std::memory_order_relaxed);
  if (ptr) return static_cast<unsigned int*>(ptr);
  if (cudaGetSymbolAddress(&ptr, g_fused_bar) != cudaSuccess || !ptr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  g_bar_ptr[dev].store(ptr, std::memory_order_release);
  return static_cast<unsigned int*>(ptr);
}

}  // namespace

bool fused_decode_supported(const Plan& p) {
  return !p.fp32 && !p.vfp32 && !p.bn_train && !p.idw && p.ksel == p.k && p.N >= 1 &&
         p.N <= kMaxTok && p.k <= 32 && p.half % 8 == 0 && p.half <= 512 && p.d_in % 8 == 0 &&
         (size_t)p.N * p.d_in * 2 <= 160 * 1024 && p.d_v % 8 == 0 &&
         std::max(p.C1, p.C2) <= 64 * kBlkKeys && p.h <= 64;
}

size_t fused_decode_bytes(const Plan& p) {
  if (!fused_decode_supported(p)) return 0;
  const size_t n = (size_t)2 * p.h * nblk_of(std::max(p.C1, p.C2)) * p.N * p.k;
  return ((4 * n + 255) & ~size_t(255)) * 2;
}

// Returns cudaErrorCooperativeLaunchTooLarge when the CTAs cannot all be resident (the
// caller then runs the separate kernels).
cudaError_t launch_fused_decode(const Plan& p, int dev, const void* x, const void* Wq,
                                const float* bn, const void* subkeys, const void* values,
                                float* y, const pkm_saved& s, void* ws, cudaStream_t st) {
  if (dev < 0 || dev >= kMaxFusedDevices) return cudaErrorInvalidDevice;
  unsigned int* bars = bar_base(dev);
  if (!bars) return cudaErrorInvalidDevicePointer;
  const int tb = p.N <= 1 ? 0 : p.N <= 2 ? 1 : p.N <= 4 ? 2 : p.N <= 8 ? 3 : 4;
  const FusedKernel kern = kFusedKernels[tb];
  const size_t smem = fused_smem(p);
  // the shared-memory attribute and the residency check, once per device, instantiation
  // and larger shared-memory size
  std::atomic<int>& ready = g_smem_ready[dev][tb];
  if ((int)smem > ready.load(std::memory_order_acquire)) {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
      return e;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFT, smem)) != cudaSuccess)
      return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    int cur = ready.load(std::memory_order_relaxed);
    while ((int)smem > cur && !ready.compare_exchange_weak(cur, (int)smem)) {
    }
  }
  FusedArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.Wq = static_cast<const __nv_bfloat16*>(Wq);
  a.bn = bn;
  a.sub = static_cast<const __nv_bfloat16*>(subkeys);
  a.V = static_cast<const __nv_bfloat16*>(values);
  a.y = y;
  a.q = static_cast<__nv_bfloat16*>(s.q);
  a.qhat = s.qhat;
  a.sub_s = s.sub_s;
  a.sub_i = s.sub_i;
  a.idx = s.idx;
  a.w = s.w;
  const int nblk = nblk_of(std::max(p.C1, p.C2));
  const size_t n = (size_t)2 * p.h * nblk * p.N * p.k;
  a.part_s = static_cast<float*>(ws);
  a.part_i = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + ((4 * n + 255) & ~size_t(255)));
  const unsigned int slot = g_bar_epoch.fetch_add(1u, std::memory_order_relaxed) % kFusedBarSlots;
  a.bar = bars + 4 * slot;
  a.poison = bars + 2;
  a.status = p.status;
  a.K = p.K;
  a.N = (int)p.N;
  a.d_in = p.d_in;
  a.h = p.h;
  a.dk = p.dk;
  a.half = p.half;
  a.C1 = p.C1;
  a.C2 = p.C2;
  a.k = p.k;
  a.d_v = p.d_v;
  a.hq = p.hq;
  a.nb1 = nblk_of(p.C1);
  a.nb2 = nblk_of(p.C2);
  a.nblk = nblk;
  a.eps = p.eps;
  a.scale = p.scale;
  a.lo_scale = p.bf16q ? 0.f : 1.f;
  a.b_off = (int)fused_b_off(p);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.sm_count);
  cfg.blockDim = dim3(kFT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  PKM_COUNT(1);
  return e;
}

}  // namespace pkm
