// persistent_batched.cu -- greedy drafting of a whole block for a band of 5..128 batch rows in one
// cooperative launch (one CTA per SM): the tensor-core counterpart of the fused small-batch kernels.
//
// Domino review page, section 二: at position i, u = SiLU(W1 . [H_i ; S_{i-1}]) (the H_i part, P_i,
// is computed for every position before the launch), z = L_base[i] + W2 . u, t_i = argmax z (lowest
// index on ties), S_i = GRUCell(embed[t_i], S_{i-1}) in the PyTorch gate form.
//
// Every position runs six phases, separated by bounded grid barriers:
//   A  W2 argmax.  The u band (rows = batch, bf16) arrives by TMA into two L_base ring slots and moves
//      into TMEM as the A operand of tcgen05.mma; W2 tiles (warp 0) and L_base tiles (warp 2) stream
//      by TMA into shared-memory rings; warp 1 issues the MMAs into two 128 x 128 accumulators; warps
//      4..11 add L_base, fold the argmax (u64 keys, atomicMax per row and CTA) and write the logits
//      when asked.  Each CTA owns the vocabulary range of the SM it runs on, as in k_w2_argmax.
//   X  every thread copies a share of the embedding rows of the drafted tokens into a row buffer.
//   B  gate inputs W_ih . x.  Item = (128-row tile of W_ih, K slice): one item per CTA.  Warp 0
//      streams the W_ih tile and the rows' K slice by TMA, warp 1 issues the MMAs into one
//      accumulator (rows = gate rows, columns = batch rows), warps 4..11 stage the item's partial
//      sums in shared memory and one TMA store writes them into the item's own slot of a global
//      buffer -- no atomics.
//   C  the GRU cell: each (row, unit) adds its partial sums in a fixed order (bit-reproducible),
//      applies the gates and writes S_i, its two-term bf16 split (hi, lo) for phase D and, when
//      asked, the states output.  With the embedding projection table phase B is skipped and the
//      cell reads the table's row of the drafted token.
//   D  W_hh . S_i and W1's state block . S_i as one stacked product (3Hs + r rows) against the
//      split state (K = 2Hs: the weights repeated along K), items and partial slots as in phase B.
//   E  u_{i+1} = SiLU(P_{i+1} + the W1 partial sums), rounded to bf16 for phase A.
// The last position runs phase A only.  Before position 0: C0 (the split of S0), D and E.  With
// the embedding projection table phases X and B are skipped.
//
// Teacher forcing (given tokens) runs the recurrence only, for shapes the unit-owned recurrence
// kernel (tf_units.cu) does not take (Hs above 1024): C0, then per update D (W_hh . S, the 3Hs gate
// rows alone) and C (the cell, with the gate inputs precomputed for every given token or read from
// the projection table); the caller computes the activations and logits of all positions
// afterwards in two tensor-core GEMMs.
//
// Roles keep running counters of the stages, tiles and phases they have gone through, so the
// mbarriers are initialised once.  Every mbarrier wait and every grid barrier is bounded: a role
// that gives up raises the CTA's abort flag, waits (bounded) for its copies and MMAs in flight, and
// the kernel reports DOMINO_STATUS_DEVICE_TIMEOUT and leaves the position loop in every CTA.
#include "common.cuh"
#include "gemm_tc.h"
#include "internal.h"
#include "persistent.h"
#include "sm_affinity.cuh"
#include "umma.cuh"

#include <algorithm>
#include <atomic>

namespace domino {
namespace {

constexpr int kThreads = 384;           // 12 warps
constexpr int kEpiWarps = 8;            // warps 4..11
constexpr int kTmemCols = 512;
constexpr uint32_t kBox = 128 * 64 * 2; // one 128 x 64 bf16 box, 128-byte swizzle: 16 KB
// phase A: W2 ring of kStagesA boxes, L_base ring of kSide tiles (two boxes each)
constexpr int kStagesA = 8;
constexpr int kSide = 3;
constexpr uint32_t kSideBytes = 2 * kBox;
// phases B and D: stages of an A box and a B box
constexpr int kStagesG = 7;
constexpr uint32_t kStageG = 2 * kBox;
constexpr uint32_t kRegion = 224 * 1024;
static_assert(kStagesA * kBox + kSide * kSideBytes <= kRegion, "phase A rings");
static_assert(kStagesG * kStageG <= kRegion, "phase B/D ring");
constexpr int kUnit = 16;               // vocabulary columns per work unit
constexpr int kTileUnits = 8;           // units per vocabulary tile (128 columns)
constexpr int kMaxKs = 8;               // K slices of phases B and D
constexpr int kTraceArrive = 256;       // first per-CTA arrival stamp of the optional trace
// then, from kTraceArrive + 128 * G: per CTA, milestones of phases B and D at position 1 --
// [(phase * 8 + k) * G + c], k: 0 start, 1 producer done, 3 MMAs issued,
// 4 accumulator in the epilogue, 5 epilogue done
// Poll limit of the waits for a role's own copies and MMAs at the end of a phase (umma.cuh).
constexpr unsigned long long kDrain = kDrainPolls;
constexpr size_t kMisc = 2048;          // mbarriers, the cross-group argmax, tokens, flags
constexpr size_t kSmem = kRegion + kMisc + 1024;
static_assert(kSmem <= 232448, "shared memory budget");

// mbarrier slots
enum : int {
  kFullA = 0, kEmptyA = 8, kSFull = 16, kSEmpty = 19, kAccFA = 22, kAccEA = 24, kAReady = 26, kUFull = 27,
  kMmaA = 28, kFullB = 29, kEmptyB = 36, kAccB = 43, kMmaB = 44, kFullD = 45, kEmptyD = 52, kAccD = 59, kMmaD = 60,
  kNumBars = 61
};
// misc block: kBarSlots mbarriers, best_s [128] u64, 512 spare bytes, four int flags
constexpr int kBarSlots = 62;
static_assert(kNumBars <= kBarSlots && kBarSlots * 8 + 128 * 8 + 128 * 4 + 16 <= (int)kMisc, "misc block");

struct BArgs {
  const bf16* embed;      // [V][d]
  const float* Xp;        // [V][3Hs] projection table, or null
  const bf16* b_ih;       // [3Hs]
  const bf16* b_hh;       // [3Hs]
  const float* P;         // [B][L][r] W1[:, :d] . H
  const float* S0;        // [B][Hs]
  float* S;               // [2][B][Hs] state ping-pong
  float* states;          // [B][L][Hs] or null
  float* logits;          // [B][L][V] or null
  uint64_t* keys;         // [L][B] argmax keys (zero before the launch)
  bf16* u16;              // [B][r] activations of the current position
  bf16* S_hl;             // [B][2Hs] two-term split of the current state
  bf16* X;                // [B][d] embedding rows of the tokens drafted at the current position
  float* partx;           // [ksx][B][3Hs] phase B partial sums
  float* parth;           // [ksd][B][3Hs + r] phase D partial sums
  uint32_t* claim;        // per-SM work-slot claims, all different from epoch before the launch
  uint32_t epoch;
  unsigned* bar;          // grid barrier counter (zero before the launch)
  int32_t* status;
  int B, L, d, Hs, r, V;
  int ksx, ksd;           // K slices of phases B and D
  unsigned long long limit;
  // teacher forcing: the given tokens [B][L] and, unless the projection table is given, their gate
  // inputs W_ih . embed[y] as rows b * (L - 1) + i of Gx [B * (L - 1)][3Hs]; null in greedy drafting
  const int32_t* tokens;
  const float* Gx;
  unsigned long long* trace;  // optional (globaltimer, ns): [0] CTA 0's start, [e] when CTA 0 passed
  int ntrace;                 // grid barrier e, then its end; [kTraceArrive + (e-1) * G + c] when
                              // CTA c arrived at barrier e.  Entries past ntrace are not written.
};

__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* tmap, uint64_t* bar, int x, int y,
                                                 int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
      : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Generic-proxy global writes (the split state, the activations) become visible to the TMA loads
// that other CTAs issue after the next grid barrier.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Element (row, col) of a region of 128-row x 64-column boxes with the 128-byte swizzle.
__device__ __forceinline__ const uint4* box_at(const uint8_t* base, int row, int col) {
  const int box = col >> 6, chunk = (col & 63) >> 3;
  return reinterpret_cast<const uint4*>(base + box * kBox + row * 128 + ((chunk ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1)
    k_greedy_batched(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWn,
                     const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmWih, const __grid_constant__ CUtensorMap tmWhh,
                     const __grid_constant__ CUtensorMap tmW1s, const __grid_constant__ CUtensorMap tmShl,
                     const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmPx,
                     const __grid_constant__ CUtensorMap tmPh, BArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* side_ring = ring + (size_t)kStagesA * kBox;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kRegion);
  uint64_t* best_s = bars + kBarSlots;                             // [128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(best_s + 128 + 64);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* slot_s = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* flag_s = reinterpret_cast<volatile int*>(tmem_slot + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.B, L = p.L, Hs = p.Hs, r = p.r, V = p.V, G = gridDim.x;
  const int H3 = 3 * Hs, HD = 3 * Hs + r;
  const unsigned long long limit = p.limit;

  if (threadIdx.x == 0) {
    *slot_s = claim_slot(p.claim, p.epoch);
    for (int s = 0; s < kStagesA; ++s) { mbar_init(&bars[kFullA + s], 1); mbar_init(&bars[kEmptyA + s], 1); }
    for (int s = 0; s < kSide; ++s) { mbar_init(&bars[kSFull + s], 1); mbar_init(&bars[kSEmpty + s], kEpiWarps); }
    for (int a = 0; a < 2; ++a) { mbar_init(&bars[kAccFA + a], 1); mbar_init(&bars[kAccEA + a], kEpiWarps); }
    mbar_init(&bars[kAReady], kEpiWarps);
    mbar_init(&bars[kUFull], 1);
    mbar_init(&bars[kMmaA], 1);
    for (int s = 0; s < kStagesG; ++s) {
      mbar_init(&bars[kFullB + s], 1);
      mbar_init(&bars[kEmptyB + s], 1);
      mbar_init(&bars[kFullD + s], 1);
      mbar_init(&bars[kEmptyD + s], 1);
    }
    mbar_init(&bars[kAccB], 1);
    mbar_init(&bars[kMmaB], 1);
    mbar_init(&bars[kAccD], 1);
    mbar_init(&bars[kMmaD], 1);
    *abort_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmWn);
    tma_prefetch_desc(&tmL);
    tma_prefetch_desc(&tmU);
    tma_prefetch_desc(&tmWih);
    tma_prefetch_desc(&tmWhh);
    tma_prefetch_desc(&tmW1s);
    tma_prefetch_desc(&tmShl);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmPx);
    tma_prefetch_desc(&tmPh);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const bool tracer = p.trace && blockIdx.x == 0 && threadIdx.x == 0;
  if (tracer && p.ntrace > 0) p.trace[0] = globaltimer_ns();

  // this CTA's vocabulary range in phase A
  const int nunits = (V + kUnit - 1) / kUnit;
  const int slot = *slot_s;
  const int vu0 = (int)((long long)nunits * slot / G), vu1 = (int)((long long)nunits * (slot + 1) / G);
  const int ntiles = (vu1 - vu0 + kTileUnits - 1) / kTileUnits;
  const int kbA = r / 64;

  // running counters (each meaningful in the threads of the role that uses it)
  uint32_t itA = 0, tA = 0, nA = 0;  // W2 stages, vocabulary tiles, phase-A count
  uint32_t itB = 0, nB = 0;          // phase-B stages, phase-B count
  uint32_t itD = 0, nD = 0;          // phase-D stages, phase-D count
  unsigned epoch = 0;                // grid barriers passed

  // ---- grid barrier over a monotonic counter (the k-th waits for k * G arrivals) ----
  auto grid_sync = [&]() -> bool {
    tmem_fence_before_sync();
    fence_proxy_async_global();
    __syncthreads();
    if (threadIdx.x == 0) {
      ++epoch;
      if (p.trace) {
        const long long k = kTraceArrive + (long long)(epoch - 1) * G + blockIdx.x;
        if (k < p.ntrace) p.trace[k] = globaltimer_ns();
      }
      __threadfence();
      atomicAdd(p.bar, 1u);
      const unsigned target = epoch * (unsigned)G;
      bool ok = *abort_s == 0;
      if (ok) {
        ok = false;
        for (unsigned long long it = 0; it < limit; ++it) {
          if (ld_acquire_gpu(p.bar) >= target) { ok = true; break; }
          if ((it & 31) == 31 && ld_relaxed_gpu(p.status) == DOMINO_STATUS_DEVICE_TIMEOUT) break;
        }
      }
      if (!ok) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
      __threadfence();
      *flag_s = ok ? 1 : 0;
      if (tracer && (int)epoch < p.ntrace) p.trace[epoch] = globaltimer_ns();
    }
    __syncthreads();
    const bool ok = *flag_s != 0;
    fence_proxy_async_global();
    tmem_fence_after_sync();
    __syncthreads();  // nobody rewrites the flag before everyone has read it
    return ok;
  };

  // ---- phase A: W2 argmax of position i ----
  auto phase_a = [&](int i) {
    const uint32_t tA0 = tA;
    const uint32_t aph = nA & 1u;
    // the two side slots that local tiles 1 and 2 will use hold the u band until it is in TMEM
    uint8_t* ubuf0 = side_ring + (size_t)((tA0 + 1) % kSide) * kSideBytes;
    uint8_t* ubuf1 = side_ring + (size_t)((tA0 + 2) % kSide) * kSideBytes;
    if (warp == 0) {
      if (lane == 0) {  // W2 producer
        const uint64_t pol = (i == L - 1) ? l2_policy_evict_first() : l2_policy_evict_last();
        bool ok = true;
        uint32_t it = itA;
        for (int t = 0; t < ntiles && ok; ++t) {
          const int ut = vu0 + t * kTileUnits, w = min(kTileUnits, vu1 - ut);
          const int n0 = ut * kUnit;
          for (int kb = 0; kb < kbA; ++kb, ++it) {
            const int s = it % kStagesA;
            if (!mbar_wait_bounded(&bars[kEmptyA + s], ((it / kStagesA) & 1u) ^ 1u, limit, abort_s)) { ok = false; break; }
            uint8_t* dst = ring + (size_t)s * kBox;
            if (w == kTileUnits) {
              mbar_arrive_expect_tx(&bars[kFullA + s], kBox);
              tma_load_2d_hint(dst, &tmW, &bars[kFullA + s], kb * 64, n0, pol);
            } else {  // a narrow last tile: w boxes of 16 rows, stacked as in a full tile
              mbar_arrive_expect_tx(&bars[kFullA + s], (uint32_t)w * (kUnit * 64 * 2));
              for (int j = 0; j < w; ++j)
                tma_load_2d_hint(dst + j * (kUnit * 128), &tmWn, &bars[kFullA + s], kb * 64, n0 + j * kUnit, pol);
            }
          }
        }
        if (!ok) *abort_s = 1;
        int never = 0;  // no copy in flight past the phase
        for (uint32_t j = (it - itA > (uint32_t)kStagesA ? it - kStagesA : itA); j < it; ++j)
          mbar_wait_bounded(&bars[kFullA + j % kStagesA], (j / kStagesA) & 1u, kDrain, &never);
        itA = it;
      }
    } else if (warp == 2) {
      if (lane == 0) {  // L_base producer (read once: evict-first)
        const uint64_t pol = l2_policy_evict_first();
        int t = 0;
        for (; t < ntiles; ++t) {
          const uint32_t tg = tA0 + t;
          const int sl = tg % kSide;
          if (!mbar_wait_bounded(&bars[kSEmpty + sl], ((tg / kSide) & 1u) ^ 1u, limit, abort_s)) { *abort_s = 1; break; }
          if ((t == 1 || t == 2) && !mbar_wait_bounded(&bars[kAReady], aph, limit, abort_s)) { *abort_s = 1; break; }
          const int ut = vu0 + t * kTileUnits, w = min(kTileUnits, vu1 - ut);
          const int n0 = ut * kUnit, nb = (w * kUnit + 63) / 64;
          mbar_arrive_expect_tx(&bars[kSFull + sl], (uint32_t)nb * kBox);
          for (int bx = 0; bx < nb; ++bx)
            tma_load_3d_hint(side_ring + (size_t)sl * kSideBytes + bx * kBox, &tmL, &bars[kSFull + sl], n0 + bx * 64,
                             i, 0, pol);
        }
        int never = 0;
        for (int j = max(0, t - kSide); j < t; ++j) {
          const uint32_t tg = tA0 + j;
          mbar_wait_bounded(&bars[kSFull + tg % kSide], (tg / kSide) & 1u, kDrain, &never);
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {  // MMA issuer
        bool ok = mbar_wait_bounded(&bars[kAReady], aph, limit, abort_s);
        tmem_fence_after_sync();
        uint32_t it = itA;
        for (int t = 0; t < ntiles && ok; ++t) {
          const uint32_t tg = tA0 + t;
          const int ut = vu0 + t * kTileUnits, w = min(kTileUnits, vu1 - ut);
          const uint32_t a = tg & 1u, accph = (tg >> 1) & 1u;
          if (!mbar_wait_bounded(&bars[kAccEA + a], accph ^ 1u, limit, abort_s)) { ok = false; break; }
          tmem_fence_after_sync();
          const uint32_t d_tmem = tbase + 128 + a * 128;
          const uint32_t idesc = idesc_bf16_f32(128, w * kUnit);
          for (int kb = 0; kb < kbA; ++kb, ++it) {
            const int s = it % kStagesA;
            if (!mbar_wait_bounded(&bars[kFullA + s], (it / kStagesA) & 1u, limit, abort_s)) { ok = false; break; }
            tmem_fence_after_sync();
            const uint32_t b_addr = smem_u32(ring + (size_t)s * kBox);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ta(d_tmem, tbase + (uint32_t)(kb * 32 + k * 8), sw128_desc(b_addr + 32 * k), idesc,
                           (kb | k) != 0);
            umma_commit(&bars[kEmptyA + s]);
          }
          if (!ok) break;
          umma_commit(&bars[kAccFA + a]);
        }
        if (!ok) *abort_s = 1;
        itA = itA + (uint32_t)(ntiles * kbA);  // the W2 producer's count, whatever was issued here
        int never = 0;  // every issued MMA has finished before TMEM is reused
        umma_commit(&bars[kMmaA]);
        mbar_wait_bounded(&bars[kMmaA], aph, kDrain, &never);
      }
    } else if (warp >= 4) {  // epilogue
      const int q = warp & 3, g = (warp - 4) >> 2;
      const int row = q * 32 + lane;
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      {  // u band: one TMA load of 128 rows x r into the two free side slots, then into TMEM
        const int nbox = r / 64;
        if (warp == 4 && lane == 0) {
          mbar_arrive_expect_tx(&bars[kUFull], (uint32_t)nbox * kBox);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d((bx < 2 ? ubuf0 : ubuf1) + (bx & 1) * kBox, &tmU, &bars[kUFull], bx * 64, 0);
        }
        if (!mbar_wait_warp(&bars[kUFull], aph, limit, abort_s)) *abort_s = 1;
        const int half = r / 4;  // 32-bit TMEM words per warp
        uint4 v[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int k0 = g * (r / 2) + 8 * c;
          const uint8_t* ub = (k0 < 128) ? ubuf0 : ubuf1;
          v[c] = 4 * c < half ? *box_at(ub, row, k0 & 127) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (4 * c < half) tmem_st4(tbase + lane_off + (uint32_t)(g * half + 4 * c), v[c]);
        tmem_wait_st();
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kAReady]);
      }
      float best = -INFINITY;
      int idx = -1;
      const bool live = row < B;
      for (int t = 0; t < ntiles; ++t) {
        const uint32_t tg = tA0 + t;
        const int ut = vu0 + t * kTileUnits, w = min(kTileUnits, vu1 - ut);
        const int n0 = ut * kUnit, N = w * kUnit;
        const uint32_t a = tg & 1u, accph = (tg >> 1) & 1u;
        const int sl = tg % kSide;
        if (!mbar_wait_warp(&bars[kAccFA + a], accph, limit, abort_s)) { *abort_s = 1; break; }
        if (!mbar_wait_warp(&bars[kSFull + sl], (tg / kSide) & 1u, limit, abort_s)) { *abort_s = 1; break; }
        tmem_fence_after_sync();
        const int cb = g * 64;
        if (cb < N) {
          const uint8_t* side = side_ring + (size_t)sl * kSideBytes;
          const uint32_t taddr = tbase + lane_off + 128 + a * 128 + (uint32_t)cb;
          const int nc = min(64, N - cb);
          uint32_t rr[4][16];
          tmem_ld16(taddr, rr[0]);
          tmem_ld16(taddr + 16, rr[1]);
          tmem_ld16(taddr + 32, rr[2]);
          tmem_ld16(taddr + 48, rr[3]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (16 * h < nc) {
#pragma unroll
              for (int j = 0; j < 16; ++j) reg_fence(rr[h][j]);
              const int col = cb + 16 * h;
              float l[16], f[8];
              widen(*box_at(side, row, col), f);
#pragma unroll
              for (int j = 0; j < 8; ++j) l[j] = f[j];
              widen(*box_at(side, row, col + 8), f);
#pragma unroll
              for (int j = 0; j < 8; ++j) l[8 + j] = f[j];
              const int nbase = n0 + col;
              float z[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) z[j] = __uint_as_float(rr[h][j]) + l[j];
              float zm[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) zm[j] = (nbase + 16 <= V || nbase + j < V) ? z[j] : -INFINITY;
              float t8[8], t4[4];
#pragma unroll
              for (int j = 0; j < 8; ++j) t8[j] = fmaxf(zm[j], zm[j + 8]);
#pragma unroll
              for (int j = 0; j < 4; ++j) t4[j] = fmaxf(t8[j], t8[j + 4]);
              const float mx = fmaxf(fmaxf(t4[0], t4[2]), fmaxf(t4[1], t4[3]));
              if (mx > best) {  // the lowest column of this group holding its maximum
                int jj = 15;
#pragma unroll
                for (int j = 15; j >= 0; --j)
                  if (zm[j] == mx) jj = j;
                best = mx;
                idx = nbase + jj;
              }
              if (p.logits && live) {
                float* o = p.logits + ((size_t)row * L + i) * V + nbase;
                if (nbase + 16 <= V) {
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    reinterpret_cast<float4*>(o)[j] = make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
                } else {
#pragma unroll
                  for (int j = 0; j < 16; ++j)
                    if (nbase + j < V) o[j] = z[j];
                }
              }
            }
          }
        }
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[kAccEA + a]);
          mbar_arrive(&bars[kSEmpty + sl]);
        }
      }
      const uint64_t key = idx >= 0 ? argmax_key(best, idx) : 0ull;
      if (g == 1) best_s[row] = key;
      asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
      if (g == 0 && live) {
        const uint64_t k = umax64(key, best_s[row]);
        if (k) atomicMax(reinterpret_cast<unsigned long long*>(p.keys + (size_t)i * B + row), (unsigned long long)k);
      }
      if (warp == 4 && lane == 0) {  // no u copy in flight past the phase (a timed-out wait)
        int never = 0;
        mbar_wait_bounded(&bars[kUFull], aph, kDrain, &never);
      }
    }
    tA += (uint32_t)ntiles;
    ++nA;
  };

  // ---- phases B and D: one (row tile, K slice) item per CTA, partial sums to a global slot ----
  // isB: A = W_ih (rows [mt*128, +128), columns = k), B = the embedding rows of the drafted tokens;
  // else A = [W_hh ; W1 state block] (k wraps at Hs), B = the split state S_hl.
  auto phase_g = [&](bool isB, int i) {
    const int ntile = (isB || p.tokens) ? H3 / 128 : HD / 128;
    const int ks = isB ? p.ksx : p.ksd;
    const int KB = isB ? p.d / 64 : 2 * Hs / 64;
    const int item = blockIdx.x;
    const bool has = item < ntile * ks;
    const int mt = has ? item / ks : 0, kq = has ? item % ks : 0;
    const int kb0 = kq * KB / ks, kb1 = (kq + 1) * KB / ks;
    uint64_t* full = &bars[isB ? kFullB : kFullD];
    uint64_t* empty = &bars[isB ? kEmptyB : kEmptyD];
    uint64_t* accb = &bars[isB ? kAccB : kAccD];
    uint64_t* mmab = &bars[isB ? kMmaB : kMmaD];
    const uint32_t it0 = isB ? itB : itD;
    const uint32_t nph = (isB ? nB : nD) & 1u;
    const int nst = has ? kb1 - kb0 : 0;
    const long long det = (p.trace && i == 1) ? kTraceArrive + 128LL * G + (isB ? 0 : 8) * (long long)G : -1;
    auto mark = [&](int k) {
      if (det >= 0 && det + (long long)k * G + blockIdx.x < p.ntrace) p.trace[det + (long long)k * G + blockIdx.x] =
          globaltimer_ns();
    };
    if (threadIdx.x == 0) mark(0);
    if (warp == 0) {
      if (lane == 0 && has) {  // TMA producer: the weight tile (and, in phase D, the split state)
        const uint64_t pol = l2_policy_evict_first();
        // phase B: the W_ih boxes past the ring's depth are requested from memory at once, so that
        // their loads meet L2 when ring slots free up (the first kStagesG go straight to the ring)
        if (isB)
          for (int kb = kb0 + kStagesG; kb < kb1; ++kb) tma_prefetch_l2_hint(&tmWih, kb * 64, mt * 128, pol);
        bool ok = true;
        uint32_t it = it0;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % kStagesG;
          if (!mbar_wait_bounded(&empty[s], ((it / kStagesG) & 1u) ^ 1u, limit, abort_s)) { ok = false; break; }
          uint8_t* st = ring + (size_t)s * kStageG;
          if (isB) {
            mbar_arrive_expect_tx(&full[s], 2 * kBox);
            tma_load_2d_hint(st, &tmWih, &full[s], kb * 64, mt * 128, pol);
            tma_load_2d(st + kBox, &tmX, &full[s], kb * 64, 0);
          } else {
            mbar_arrive_expect_tx(&full[s], 2 * kBox);
            const int kx = (kb * 64) % Hs;
            if (mt * 128 < H3) tma_load_2d(st, &tmWhh, &full[s], kx, mt * 128);
            else tma_load_2d(st, &tmW1s, &full[s], kx, mt * 128 - H3);
            tma_load_2d(st + kBox, &tmShl, &full[s], kb * 64, 0);
          }
        }
        if (!ok) *abort_s = 1;
        mark(1);
        int never = 0;
        for (uint32_t j = (it - it0 > (uint32_t)kStagesG ? it - kStagesG : it0); j < it; ++j)
          mbar_wait_bounded(&full[j % kStagesG], (j / kStagesG) & 1u, kDrain, &never);
      }
    } else if (warp == 1) {
      if (lane == 0 && has) {  // MMA issuer: one 128 x 128 accumulator at TMEM column 0
        const uint32_t idesc = idesc_bf16_f32(128, 128);
        bool ok = true;
        uint32_t it = it0;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % kStagesG;
          if (!mbar_wait_bounded(&full[s], (it / kStagesG) & 1u, limit, abort_s)) { ok = false; break; }
          tmem_fence_after_sync();
          const uint32_t a_addr = smem_u32(ring + (size_t)s * kStageG), b_addr = a_addr + kBox;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tbase, sw128_desc(a_addr + 32 * k), sw128_desc(b_addr + 32 * k), idesc, ((kb - kb0) | k) != 0);
          umma_commit(&empty[s]);
        }
        if (!ok) *abort_s = 1;
        mark(3);
        umma_commit(accb);  // completes when every MMA issued above has finished
        int never = 0;
        umma_commit(mmab);
        mbar_wait_bounded(mmab, nph, kDrain, &never);
      }
    } else if (has) {  // warps 2..11
      if (warp >= 4) {  // epilogue: the item's partial sums -> part[kq][n][tile row], by one TMA store
        const int q = warp & 3, g = (warp - 4) >> 2;
        const int row = q * 32 + lane;
        const bool got = mbar_wait_warp(accb, nph, limit, abort_s);
        if (got) {
          if (warp == 4 && lane == 0) mark(4);
          tmem_fence_after_sync();
          const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(g * 64);
          uint32_t rr[64];
          tmem_ld16(taddr, &rr[0]);
          tmem_ld16(taddr + 16, &rr[16]);
          tmem_ld16(taddr + 32, &rr[32]);
          tmem_ld16(taddr + 48, &rr[48]);
          tmem_wait_ld();
          // the MMAs are done, so the ring is free: stage the tile there as [batch row][gate row]
          // (a warp writes 32 consecutive floats per store: no bank conflict)
          float* stg = reinterpret_cast<float*>(ring);
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            reg_fence(rr[c]);
            stg[(g * 64 + c) * 128 + row] = __uint_as_float(rr[c]);
          }
        } else {
          *abort_s = 1;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
        if (warp == 4 && lane == 0) {
          if (got) {  // rows past B fall outside the tensor and are not written
            asm volatile(
                "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                    isB ? &tmPx : &tmPh),
                "r"(mt * 128), "r"(0), "r"(kq), "r"(smem_u32(ring))
                : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // written before the barrier
          }
          mark(5);
        }
      }
    }
    if (isB) { itB = it0 + (uint32_t)nst; ++nB; } else { itD = it0 + (uint32_t)nst; ++nD; }
  };

  // ---- phase X: the embedding rows of the tokens drafted at position i into the row buffer ----
  auto phase_x = [&](int i) {
    const int q8 = p.d / 8;  // 16-byte chunks per row
    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, gstride = (size_t)G * blockDim.x;
    for (size_t c = gtid; c < (size_t)B * q8; c += gstride) {
      const int b = (int)(c / q8), q = (int)(c % q8);
      const int tok = key_index(p.keys[(size_t)i * B + b]);
      const int tk = (tok >= 0 && tok < V) ? tok : 0;
      reinterpret_cast<uint4*>(p.X)[c] = ldg16(p.embed + (size_t)tk * p.d + (size_t)q * 8);
    }
  };

  // ---- phase C: the GRU cell of position i (i = -1: the split of S0) ----
  auto phase_c = [&](int i) {
    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, gstride = (size_t)G * blockDim.x;
    const float* Sprev = i <= 0 ? p.S0 : p.S + (size_t)((i - 1) & 1) * B * Hs;
    float* Snew = p.S + (size_t)(i & 1) * B * Hs;
    for (size_t t = gtid; t < (size_t)B * Hs; t += gstride) {
      const int b = (int)(t / Hs), j = (int)(t % Hs);
      float hn;
      if (i < 0) {
        hn = p.S0[t];
        if (p.states) p.states[(size_t)b * L * Hs + j] = hn;
      } else {
        const int tok = p.tokens ? p.tokens[(size_t)b * L + i] : key_index(p.keys[(size_t)i * B + b]);
        const bool valid = tok >= 0 && tok < V;
        if (!valid && j == 0) set_status(p.status, DOMINO_STATUS_BAD_TOKEN);
        const int tk = valid ? tok : 0;
        // every load of the element is issued before the first add (independent loads, one L2 round
        // trip); the partial sums are then added in slice order, so the result does not depend on it
        float xs[3][kMaxKs], hs[3][kMaxKs], bi[3], bh[3];
#pragma unroll
        for (int gt = 0; gt < 3; ++gt) {
          const int rw = gt * Hs + j;
#pragma unroll
          for (int kq = 0; kq < kMaxKs; ++kq)
            xs[gt][kq] = p.Xp     ? (kq == 0 ? p.Xp[(size_t)tk * H3 + rw] : 0.f)
                         : p.Gx   ? (kq == 0 ? p.Gx[((size_t)b * (L - 1) + i) * H3 + rw] : 0.f)
                                  : (kq < p.ksx ? p.partx[((size_t)kq * B + b) * H3 + rw] : 0.f);
#pragma unroll
          for (int kd = 0; kd < kMaxKs; ++kd) hs[gt][kd] = kd < p.ksd ? p.parth[((size_t)kd * B + b) * HD + rw] : 0.f;
          bi[gt] = to_f32(p.b_ih[rw]);
          bh[gt] = to_f32(p.b_hh[rw]);
        }
        float gi[3], gh[3];
#pragma unroll
        for (int gt = 0; gt < 3; ++gt) {
          float x = xs[gt][0], h = hs[gt][0];
#pragma unroll
          for (int k = 1; k < kMaxKs; ++k) {
            x += xs[gt][k];  // slices past ks add zeros: the sum is unchanged
            h += hs[gt][k];
          }
          gi[gt] = x + bi[gt];
          gh[gt] = h + bh[gt];
        }
        const float rg = sigmoidf_(gi[0] + gh[0]);
        const float zg = sigmoidf_(gi[1] + gh[1]);
        const float ng = tanhf(gi[2] + rg * gh[2]);
        hn = (1.f - zg) * ng + zg * Sprev[t];
        Snew[t] = hn;
        if (p.states && i + 1 < L) p.states[((size_t)b * L + i + 1) * Hs + j] = hn;
      }
      const bf16 hi = __float2bfloat16_rn(hn);
      p.S_hl[(size_t)b * 2 * Hs + j] = hi;
      p.S_hl[(size_t)b * 2 * Hs + Hs + j] = __float2bfloat16_rn(hn - __bfloat162float(hi));
    }
  };

  // ---- phase E: activations of position pos ----
  auto phase_e = [&](int pos) {
    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x, gstride = (size_t)G * blockDim.x;
    for (size_t t = gtid; t < (size_t)B * r; t += gstride) {
      const int b = (int)(t / r), k = (int)(t % r);
      float hs[kMaxKs];
#pragma unroll
      for (int kd = 0; kd < kMaxKs; ++kd) hs[kd] = kd < p.ksd ? p.parth[((size_t)kd * B + b) * HD + H3 + k] : 0.f;
      float a = p.P[((size_t)b * L + pos) * r + k];
#pragma unroll
      for (int kd = 0; kd < kMaxKs; ++kd) a += hs[kd];
      p.u16[(size_t)b * r + k] = __float2bfloat16_rn(siluf_(a));
    }
  };

  bool ok = true;
  if (p.tokens) {  // teacher forcing: the recurrence over the given tokens
    phase_c(-1);
    for (int i = 0; i + 1 < L; ++i) {
      if (!(ok = grid_sync())) break;
      phase_g(false, i);
      if (!(ok = grid_sync())) break;
      phase_c(i);
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
    if (threadIdx.x == 0 && *abort_s) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
    if (tracer && (int)epoch + 1 < p.ntrace) p.trace[epoch + 1] = globaltimer_ns();
    return;
  }
  phase_c(-1);
  ok = grid_sync();
  if (ok) { phase_g(false, 0); ok = grid_sync(); }
  if (ok) { phase_e(0); ok = grid_sync(); }
  for (int i = 0; i < L && ok; ++i) {
    phase_a(i);
    if (i == L - 1) break;
    ok = grid_sync();
    if (ok && !p.Xp) { phase_x(i); ok = grid_sync(); }
    if (ok && !p.Xp) { phase_g(true, i); ok = grid_sync(); }
    if (ok) { phase_c(i); ok = grid_sync(); }
    if (ok) { phase_g(false, i); ok = grid_sync(); }
    if (ok) { phase_e(i + 1); ok = grid_sync(); }
  }

  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0 && *abort_s) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
  if (tracer && (int)epoch + 1 < p.ntrace) p.trace[epoch + 1] = globaltimer_ns();
}

int g_fit_cache[64];  // per device: 0 unknown, 1 fits, -1 does not

bool cooperative_fits() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (g_fit_cache[dev] != 0) return g_fit_cache[dev] > 0;
  int per_sm = 0;
  bool fits = cudaFuncSetAttribute(k_greedy_batched, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem) ==
                  cudaSuccess &&
              cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_greedy_batched, kThreads, kSmem) ==
                  cudaSuccess &&
              per_sm >= 1;
  cudaGetLastError();
  g_fit_cache[dev] = fits ? 1 : -1;
  return fits;
}

int ks_for(int ntile, int KB, int G) {
  int ks = std::max(1, std::min(kMaxKs, G / std::max(1, ntile)));
  return std::min(ks, std::max(1, KB / 2));
}

}  // namespace

size_t batched_partial_floats(const Shape& s) {
  if (s.dtype != DOMINO_DTYPE_BF16 || s.B <= 4 || s.B > 128) return 0;
  return (size_t)kMaxKs * s.B * (3 * (size_t)s.Hs) + (size_t)kMaxKs * s.B * (3 * (size_t)s.Hs + s.r);
}

bool batched_shape_ok(const Shape& s) {
  if (s.dtype != DOMINO_DTYPE_BF16 || s.B <= 4 || s.B > 128) return false;
  if (s.r < 64 || s.r > 256 || s.r % 64 != 0 || s.d % 64 != 0 || s.Hs % 128 != 0 || (3 * s.Hs + s.r) % 128 != 0)
    return false;
  if (s.V < 16 || s.V % 8 != 0 || s.L < 1) return false;
  const int G = sm_count();
  if (G < (3 * s.Hs + s.r) / 128 || G < 1) return false;  // one item per CTA in phases B and D
  return cooperative_fits();
}

bool use_greedy_batched(const Shape& s, const domino_weights_t& w, const void* base_logits) {
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!batched_shape_ok(s)) return false;
  if (!a16(w.W2) || !a16(w.W_ih) || !a16(w.W_hh) || !a16(w.W1) || !a16(w.embed) || !a16(base_logits)) return false;
  return !w.embed_proj || a16(w.embed_proj);
}

const char* batched_plan() {
  return "k_greedy_batched: one cooperative launch, one CTA per SM, per position a tcgen05 W2 argmax, tcgen05 "
         "W_ih and stacked W_hh|W1 products with fixed-slot partial sums, and the GRU cell, separated by bounded "
         "grid barriers";
}

namespace {
cudaError_t launch_batched(const Shape& s, const domino_weights_t& w, const void* base_logits, const float* S0,
                           float* logits_out, float* states_out, const int32_t* tokens, const float* Gx,
                           const Workspace& ws, int32_t* status, uint64_t spin, cudaStream_t st);
}  // namespace

cudaError_t launch_greedy_batched(const Shape& s, const domino_weights_t& w, const void* base_logits,
                                  const float* S0, float* logits_out, float* states_out, const Workspace& ws,
                                  int32_t* status, uint64_t spin, cudaStream_t st) {
  return launch_batched(s, w, base_logits, S0, logits_out, states_out, nullptr, nullptr, ws, status, spin, st);
}

cudaError_t launch_tf_batched(const Shape& s, const domino_weights_t& w, const void* base_logits, const float* S0,
                              const int32_t* tokens, const float* Gx, float* states, const Workspace& ws,
                              int32_t* status, uint64_t spin, cudaStream_t st) {
  if (!tokens || !states || (!Gx && !w.embed_proj && s.L > 1)) return cudaErrorInvalidValue;
  return launch_batched(s, w, base_logits, S0, nullptr, states, tokens, w.embed_proj ? nullptr : Gx, ws, status,
                        spin, st);
}

namespace {
cudaError_t launch_batched(const Shape& s, const domino_weights_t& w, const void* base_logits, const float* S0,
                           float* logits_out, float* states_out, const int32_t* tokens, const float* Gx,
                           const Workspace& ws, int32_t* status, uint64_t spin, cudaStream_t st) {
  using bf = __nv_bfloat16;
  const int G = sm_count();
  cudaError_t e = ensure_sm_rank(st);
  if (e != cudaSuccess) return e;
  CUtensorMap tW, tWn, tL, tU, tWih, tWhh, tW1s, tShl, tX, tPx, tPh;
  const bf* W1s = (const bf*)w.W1 + s.d;
  // base logits [B][L][V] as a 3-D tensor (v, position, row): one 128-row box per position
  bool okm = tmap_bf16_tiles(&tW, w.W2, (uint64_t)s.V, (uint64_t)s.r, 128) &&
             tmap_bf16_tiles(&tWn, w.W2, (uint64_t)s.V, (uint64_t)s.r, kUnit) &&
             tmap_bf16_tiles(&tU, ws.u16, (uint64_t)s.B, (uint64_t)s.r, 128) &&
             tmap_bf16_tiles(&tWih, w.W_ih, 3 * (uint64_t)s.Hs, (uint64_t)s.d, 128) &&
             tmap_bf16_tiles(&tWhh, w.W_hh, 3 * (uint64_t)s.Hs, (uint64_t)s.Hs, 128) &&
             tmap_bf16_tiles(&tW1s, W1s, (uint64_t)s.r, (uint64_t)s.Hs, 128, (uint64_t)(s.d + s.Hs)) &&
             tmap_bf16_tiles(&tShl, ws.S_hl, (uint64_t)s.B, 2 * (uint64_t)s.Hs, 128) &&
             tmap_bf16_tiles(&tX, ws.X, (uint64_t)s.B, (uint64_t)s.d, 128) &&
             tmap_f32_3d(&tPx, ws.part, 3 * (uint64_t)s.Hs, (uint64_t)s.B, kMaxKs, 128, 128) &&
             tmap_f32_3d(&tPh, ws.part + (size_t)kMaxKs * s.B * 3 * s.Hs, 3 * (uint64_t)s.Hs + s.r, (uint64_t)s.B,
                         kMaxKs, 128, 128) &&
             tmap_bf16_3d(&tL, base_logits, (uint64_t)s.V, (uint64_t)s.L, (uint64_t)s.B, 128);
  if (!okm) return cudaErrorInvalidValue;
  BArgs a{};
  a.embed = (const bf*)w.embed; a.Xp = w.embed_proj; a.b_ih = (const bf*)w.b_ih; a.b_hh = (const bf*)w.b_hh;
  a.P = ws.P; a.S0 = S0; a.S = ws.S; a.states = states_out; a.logits = logits_out; a.keys = ws.keys;
  a.u16 = ws.u16; a.S_hl = ws.S_hl; a.X = ws.X; a.partx = ws.part;
  a.parth = ws.part + (size_t)kMaxKs * s.B * 3 * s.Hs;
  a.claim = ws.claim; a.bar = ws.sync; a.status = status;
  a.B = s.B; a.L = s.L; a.d = s.d; a.Hs = s.Hs; a.r = s.r; a.V = s.V;
  a.ksx = ks_for(3 * s.Hs / 128, s.d / 64, G);
  a.ksd = tokens ? ks_for(3 * s.Hs / 128, 2 * s.Hs / 64, G) : ks_for((3 * s.Hs + s.r) / 128, 2 * s.Hs / 64, G);
  a.tokens = tokens;
  a.Gx = Gx;
  // greedy drafting claims against words zeroed just before; teacher forcing against the words its
  // logits GEMM (epoch 1) will claim after it, so it takes epoch 2
  a.epoch = tokens ? 2u : 1u;
  a.limit = spin;
  debug_trace(&a.trace, &a.ntrace);
  void* params[] = {&tW, &tWn, &tL, &tU, &tWih, &tWhh, &tW1s, &tShl, &tX, &tPx, &tPh, &a};
  e = cudaLaunchCooperativeKernel((const void*)k_greedy_batched, dim3(G), dim3(kThreads), params, kSmem, st);
  return note_launch(e);
}
}  // namespace

}  // namespace domino
