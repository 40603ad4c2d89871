// Persistent, warp-specialised tcgen05 GEMM engine for bf16 operands with fp32
// accumulation in TMEM:  D[128 x 256] = A[128 x K] * B[256 x K]^T per chunk.
//
//   warp 0     TMA producer: one lane streams A/B k-blocks (64 wide, 128-byte
//              swizzle) into a ring of smem stages (full/empty mbarriers)
//   warp 1     MMA issuer: allocates 512 TMEM columns (two 256-column fp32
//              accumulators), one lane issues tcgen05.mma K=16 steps, commits each
//              stage back to the producer and each finished chunk to the epilogue
//   warps 2..  epilogue: one or two sets of 128 threads; thread r of a set owns
//              accumulator row r (TMEM lane r), reads 32-column pieces with tcgen05.ld
//              and hands them to the problem's epilogue; releases the accumulator with
//              an mbarrier.  One set alternates between the two accumulators chunk by
//              chunk; with two sets (Prob::kSets = 2) set s owns accumulator s and every
//              other unit, and the MMA issuer interleaves the two units' chunks.
//
// A "unit" is a 128-row block of the output that the problem walks in chunks of
// 256 columns (the scoring problem keeps a running top-k across the chunks of a
// row; the other problems have one chunk per unit).  No TMA multicast is used.
//
// Per problem, optionally: several operand planes per stage with several products per
// k-block (PlanesOf: the hi and lo bf16 planes of an operand read once per k-block
// beside the other operand), a narrower MMA (MmaNOf: 192 or 128 columns, to fill the
// SMs), and two output tensor maps for epilogues that write their pieces with TMA tile
// stores (EpiCtx).
//
// Operand layouts in a stage (both 128-byte swizzled, as TMA writes them):
//   K-major  (Prob::kAMN / kBMN == 0): rows of 64 k-elements (128 B), 8-row groups
//            1024 B apart; one TMA box of 64 x rows.
//   MN-major (== 1): rows of 64 MN-elements (128 B), one row per k, 8-k groups
//            1024 B apart (SBO), 64-wide MN blocks 8 KiB apart (LBO); one 64 x 64 TMA
//            box per MN block.  A K=16 step advances 16 rows = 2 KiB.
#pragma once

#include <type_traits>

#include "tc_common.cuh"

namespace pkm {
namespace tc {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStageA = kBM * kBK * 2;  // 16 KiB
constexpr int kStageB = kBN * kBK * 2;  // 32 KiB
constexpr int kStageBytes = kStageA + kStageB;
constexpr uint32_t kTmemCols = 512;

// What the engine hands every epilogue hook besides the problem's parameters: the two
// output tensor maps (for problems that store tiles through TMA), two mbarriers of
// count 1 private to the epilogue set, the CTA's abort flag and the status word, the
// index of the current unit among the set's units, and the thread's warp quarter
// (TMEM lanes [32 * quarter, 32 * quarter + 32)) and lane.
struct EpiCtx {
  const CUtensorMap* out0;
  const CUtensorMap* out1;
  uint64_t* bar;
  volatile int* abort;
  int* status;
  int seq;
  int quarter, lane;
};

// Epilogue sets of a problem (Prob::kSets, default 1).  With one set, the 128 epilogue
// threads alternate between the two 256-column accumulators chunk by chunk.  With two
// sets, each set of 128 threads owns one accumulator and every other unit of the CTA:
// the MMA issuer interleaves the two units' chunks, so two epilogue warps share each
// SM sub-partition and hide each other's latency.
template <class P, class = void>
struct SetsOf {
  static constexpr int value = 1;
};
template <class P>
struct SetsOf<P, std::void_t<decltype(P::kSets)>> {
  static constexpr int value = P::kSets;
};

// Operand planes of a problem's stage.  By default a stage holds one A tile (128 x 64)
// and one B tile (256 x 64) and a k-block is one product of the two.  A problem with
// kAPlanes / kBPlanes > 1 (e.g. the hi and lo bf16 planes of an fp32 operand) loads all
// planes of a k-block into one stage, A planes first, each 16 KiB, then the B planes, each
// 32 KiB, and issues num_pairs(P) products per k-block: pair i multiplies A plane
// pair_a(P, i) with B plane pair_b(P, i), all into the one accumulator.  tx_bytes(P) is
// what the stage's loads deliver (planes a problem does not need are not loaded).
template <class P, class = void>
struct PlanesOf {
  static constexpr int a = 1, b = 1;
  __device__ static int pairs(const typename P::Params&) { return 1; }
  __device__ static int pair_a(const typename P::Params&, int) { return 0; }
  __device__ static int pair_b(const typename P::Params&, int) { return 0; }
  __device__ static uint32_t tx(const typename P::Params&) { return kStageA + kStageB; }
};
template <class P>
struct PlanesOf<P, std::void_t<decltype(P::kAPlanes)>> {
  static constexpr int a = P::kAPlanes, b = P::kBPlanes;
  __device__ static int pairs(const typename P::Params& p) { return P::num_pairs(p); }
  __device__ static int pair_a(const typename P::Params& p, int i) { return P::pair_a(p, i); }
  __device__ static int pair_b(const typename P::Params& p, int i) { return P::pair_b(p, i); }
  __device__ static uint32_t tx(const typename P::Params& p) { return P::tx_bytes(p); }
};

// MMA width of a problem's chunks: kBN (256) by default; a problem with mma_n(P) runs
// narrower chunks (a multiple of 64 up to 256) so that more units fill the SMs.  Its
// accumulator slots stay 256 columns apart.
template <class P, class = void>
struct MmaNOf {
  __device__ static int get(const typename P::Params&) { return kBN; }
};
template <class P>
struct MmaNOf<P, std::void_t<decltype(&P::mma_n)>> {
  __device__ static int get(const typename P::Params& p) { return P::mma_n(p); }
};

template <class Prob>
constexpr int stage_bytes_of() {
  return PlanesOf<Prob>::a * kStageA + PlanesOf<Prob>::b * kStageB;
}

template <class Prob>
constexpr int threads_of() {
  return 64 + 128 * SetsOf<Prob>::value;
}

template <class Prob>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Prob::kStages * stage_bytes_of<Prob>() +
         (size_t)SetsOf<Prob>::value * Prob::kEpiSmem;
}

// The CTA's chunk schedule, walked identically by the producer, the MMA issuer and each
// epilogue set: rounds of kSets consecutive units of the CTA (unit i of the CTA is
// blockIdx.x + i * gridDim.x); within a round chunk c of every unit of the round, unit
// by unit, before chunk c + 1.  set_chunks(r, s) is the number of chunks of the round's
// s-th unit (0 past the end).
template <class Prob>
struct Schedule {
  static constexpr int S = SetsOf<Prob>::value;
  const typename Prob::Params& P;
  int nunits;
  __device__ int unit(int r, int s) const {
    return (int)blockIdx.x + (r * S + s) * (int)gridDim.x;
  }
  __device__ int set_chunks(int r, int s) const {
    const int u = unit(r, s);
    return u < nunits ? Prob::num_chunks(P, u) : 0;
  }
};

template <class Prob>
__global__ void __launch_bounds__(threads_of<Prob>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                   const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmO0,
                   const __grid_constant__ CUtensorMap tmO1, const typename Prob::Params P) {
  constexpr int S = Prob::kStages;
  constexpr int NS = SetsOf<Prob>::value;
  using PL = PlanesOf<Prob>;
  constexpr int SB = stage_bytes_of<Prob>();
  constexpr int kOffB = PL::a * kStageA;  // first B plane within a stage
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S], empty_bar[S], tfull_bar[2], tempty_bar[2],
      drain_bar, epi_bar[2][2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* epi_smem = smem + (size_t)S * SB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 128);
    }
    mbar_init(&drain_bar, 1);
    for (int b = 0; b < 4; ++b) mbar_init(&epi_bar[b >> 1][b & 1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  int* status = P.status;
  const Schedule<Prob> sch{P, Prob::num_units(P)};
  const int nk = Prob::num_kblocks(P);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;  // stages that received at least one load
      uint32_t parity_mask = 0;  // bit s: full-barrier parity the last load on s completes
      bool ok = true;
      for (int r = 0; ok; ++r) {
        int nc[NS], maxc = 0;
#pragma unroll
        for (int s = 0; s < NS; ++s) {
          nc[s] = sch.set_chunks(r, s);
          maxc = nc[s] > maxc ? nc[s] : maxc;
        }
        if (maxc == 0) break;
        for (int c = 0; c < maxc && ok; ++c) {
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            if (c >= nc[s] || !ok) continue;
            const int u = sch.unit(r, s);
            for (int kb = 0; kb < nk; ++kb) {
              if (!mbar_wait(&empty_bar[stage], phase ^ 1u, &abort_flag, status)) {
                ok = false;
                break;
              }
              unsigned char* sa = smem + (size_t)stage * SB;
              mbar_arrive_expect_tx(&full_bar[stage], PL::tx(P));
              Prob::load(P, &tmA0, &tmA1, &tmB, &tmB1, u, c, kb, sa, sa + kOffB,
                         &full_bar[stage]);
              issued_mask |= 1u << stage;
              parity_mask = (parity_mask & ~(1u << stage)) | (phase << stage);
              if (++stage == S) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
        }
      }
      if (!ok) {
        // drain: the last load issued on each stage must land before the CTA exits
        // (earlier loads on a stage completed before the stage was reused)
        for (int s = 0; s < S; ++s) {
          if (!((issued_mask >> s) & 1u)) continue;
          const uint32_t par = (parity_mask >> s) & 1u;
          const long long t0 = clock64();
          while (!mbar_try_wait(&full_bar[s], par) && clock64() - t0 < kWaitBudgetCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBM, MmaNOf<Prob>::get(P), Prob::kAMN, Prob::kBMN);
      int stage = 0;
      uint32_t phase = 0;
      int alt = 0;                // one set: the accumulator of the next chunk
      uint32_t acc_phase = 0u;    // bit a: parity of accumulator a's next phase
      bool ok = true;
      bool issued = false;
      for (int r = 0; ok; ++r) {
        int nc[NS], maxc = 0;
#pragma unroll
        for (int s = 0; s < NS; ++s) {
          nc[s] = sch.set_chunks(r, s);
          maxc = nc[s] > maxc ? nc[s] : maxc;
        }
        if (maxc == 0) break;
        for (int c = 0; c < maxc && ok; ++c) {
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            if (c >= nc[s] || !ok) continue;
            const int acc = NS == 1 ? alt : s;
            if (!mbar_wait(&tempty_bar[acc], ((acc_phase >> acc) & 1u) ^ 1u, &abort_flag, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t dt = tmem_base + (uint32_t)acc * kBN;
            for (int kb = 0; kb < nk; ++kb) {
              if (!mbar_wait(&full_bar[stage], phase, &abort_flag, status)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t s0 = smem_u32(smem + (size_t)stage * SB);
              const int np = PL::pairs(P);
              for (int pi = 0; pi < np; ++pi) {
                const uint32_t sa = s0 + (uint32_t)PL::pair_a(P, pi) * kStageA;
                const uint32_t sb = s0 + kOffB + (uint32_t)PL::pair_b(P, pi) * kStageB;
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k) {
                  const uint64_t da = Prob::kAMN
                                          ? desc_mnmajor_sw128(sa + 2048u * k, 8192u, 1024u)
                                          : desc_kmajor_sw128(sa) + (uint64_t)(2 * k);
                  const uint64_t db = Prob::kBMN
                                          ? desc_mnmajor_sw128(sb + 2048u * k, 8192u, 1024u)
                                          : desc_kmajor_sw128(sb) + (uint64_t)(2 * k);
                  mma_bf16(dt, da, db, idesc, (kb | k | pi) != 0 ? 1u : 0u);
                }
              }
              issued = true;
              umma_commit(&empty_bar[stage]);
              if (++stage == S) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit(&tfull_bar[acc]);
            acc_phase ^= 1u << acc;
            alt ^= 1;
          }
        }
      }
      if (issued) {
        // all MMAs of this CTA complete before TMEM is released
        umma_commit(&drain_bar);
        const long long t0 = clock64();
        while (!mbar_try_wait(&drain_bar, 0) && clock64() - t0 < kWaitBudgetCycles) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int set = NS == 1 ? 0 : (warp - 2) >> 2;
    const int quarter = warp & 3;            // TMEM lanes [32*quarter, 32*quarter + 32)
    const int row = quarter * 32 + lane;     // accumulator row owned by this thread
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    unsigned char* my_smem = epi_smem + (size_t)set * Prob::kEpiSmem;
    EpiCtx cx{&tmO0, &tmO1, epi_bar[set], &abort_flag, status, 0, quarter, lane};
    int alt = 0;
    uint32_t acc_phase = 0u;  // bit a: parity of accumulator a's next phase
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int nc = sch.set_chunks(r, set);
      if (nc == 0) {
        // past this set's last unit: with one set that is the end; with two sets the
        // round may still have a unit for the other set, and later rounds none for this
        if (NS == 1 || sch.set_chunks(r, 0) == 0) break;
        continue;
      }
      const int u = sch.unit(r, set);
      typename Prob::EpiState es;
      Prob::epi_begin(P, u, row, my_smem, es, cx);
      for (int c = 0; c < nc; ++c) {
        const int acc = NS == 1 ? alt : set;
        // warp-uniform wait: lane 0 waits, the result is broadcast, so the warp reaches
        // the .sync.aligned TMEM loads together or not at all
        int got = 0;
        if (lane == 0)
          got = mbar_wait(&tfull_bar[acc], (acc_phase >> acc) & 1u, &abort_flag, status) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        Prob::epi_chunk(P, u, c, row, tmem_base + lane_addr + (uint32_t)acc * kBN, my_smem, es,
                        cx);
        tc_fence_before();
        mbar_arrive(&tempty_bar[acc]);
        acc_phase ^= 1u << acc;
        alt ^= 1;
      }
      if (!ok) break;
      Prob::epi_end(P, u, row, my_smem, es, cx);
      ++cx.seq;
    }
    // tile stores issued by the epilogue complete before the CTA exits
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace tc
}  // namespace pkm
