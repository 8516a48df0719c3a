// w2_argmax.cu -- the greedy step's W2 product with the L_base residual and the vocabulary argmax
// fused, for a band of up to 128 batch rows (the large-batch path of greedy drafting):
//
//   z[b][v] = L_base[b][v] + sum_k u[b][k] W2[v][k],   keys[b] = max(keys[b], key(argmax_v z[b][v]))
//
// (Domino review page, section 二: L_final = L_base + W2 . SiLU(W1 . [H_i ; S_{i-1}]); greedy
// drafting takes its argmax, lowest index on ties.)
//
// One CTA per SM owns one contiguous range of the vocabulary -- 16-column units, balanced to within
// one unit -- and walks it in tiles of up to 128 columns (the last tile of a range may be narrower:
// its MMA and loads shrink to its width).  The range is chosen by the SM the CTA runs on
// (sm_affinity.cuh), so that at every position of the block the same SM reads the same W2 rows and
// finds them in the L2 of its own die.  Roles:
//   - the activation band u [128 x r] sits in TMEM as the A operand of tcgen05.mma for the whole
//     launch (lane = batch row; 32-bit column c holds k = 2c and 2c + 1), so shared memory holds only
//     the streamed operands.  It arrives by one TMA load into two L_base ring slots that have not
//     been filled yet, and each epilogue thread moves its row from there into its TMEM lane (one
//     16-byte shared-memory read per chunk, where loading it from global memory row by row took
//     one L2 request per row and chunk: 4.6 us for 128 rows against the MMAs' 15);
//   - warp 0 streams W2 tiles (K-major, 128-byte swizzle) through a ring of kStages k-block stages
//     with an L2 evict-last policy: W2 (77.8 MB at V = 151936) is re-read at every position of the
//     block and should stay in B200's 126 MB L2 while the operands streamed beside it pass through.
//     The block's last position reads W2 for the last time in the call and marks it evict-first
//     instead, so that W2 does not hold L2 through the work that follows the draft (the target
//     model's verification pass). Measured on a B200: loads with no hint take as long as evict-last
//     ones (about 22 us per launch at B = 128), and a cp.async producer (two warps of 16-byte copies
//     into the same swizzled ring) took 32 us, so the stream stays one TMA thread;
//   - warp 2 streams the L_base tile of each vocabulary tile (128 batch rows x the tile's columns,
//     read once: evict-first) into a ring of kSide buffers, as far ahead as the ring allows;
//   - warp 1 issues the MMAs (one thread) into two 128 x 128 fp32 accumulators in TMEM;
//   - warps 4..11 run the epilogue: two warps per TMEM lane quadrant, each on half of the columns,
//     add L_base and fold the argmax; the halves meet in shared memory and each CTA publishes one
//     atomicMax per row.
// W2 and L_base are inputs that no kernel of the call writes, so both producers start before the
// wait on the previous grid (programmatic dependent launch); only the epilogue warps, which read u
// and write keys and logits, wait.  Every mbarrier wait is bounded; a role that gives up raises a
// CTA-wide abort flag, the producers wait for their copies in flight, the MMA issuer for its MMAs,
// TMEM is freed and DOMINO_STATUS_DEVICE_TIMEOUT is reported.
#include "common.cuh"
#include "gemm_tc.h"
#include "launch.cuh"
#include "sm_affinity.cuh"
#include "umma.cuh"

#include <algorithm>
#include <atomic>

namespace domino {

namespace {

constexpr int kW2Threads = 384;         // 12 warps: roles above (warp 3 idle)
constexpr int kStages = 8;              // W2 ring: k-blocks of 128 rows x 64 k
constexpr int kSide = 3;                // L_base ring: tiles of 128 rows x 128 columns
constexpr uint32_t kStageBytes = 128 * 64 * 2;
constexpr uint32_t kBoxBytes = 128 * 64 * 2;  // one L_base box: 128 rows x 64 columns
constexpr uint32_t kSideBytes = 2 * kBoxBytes;
constexpr int kUnit = 16;               // columns per work unit (the MMA's N granularity)
constexpr int kTileUnits = 8;           // units per full tile (128 columns)
constexpr int kEpiWarps = 8;
constexpr int kTmemCols = 512;          // A: [0, 128); accumulators: [128, 256), [256, 384)
constexpr size_t kRingBytes = (size_t)kStages * kStageBytes + (size_t)kSide * kSideBytes;
constexpr size_t kMiscBytes = 1280;     // mbarriers, TMEM slot, flags, the cross-group argmax
constexpr size_t kSmemBytes = kRingBytes + kMiscBytes + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");
// The u band (128 rows x r <= 256, bf16: at most four 128 x 64 boxes) is staged through L_base ring
// slots 1 and 2 before their first L_base tile.
static_assert(kSide >= 3 && 2 * kSideBytes >= 4 * kBoxBytes, "u band staging space");

struct W2Args {
  uint64_t* keys;      // [M] argmax keys (atomicMax)
  float* out;          // optional z: out[m * ldo + v]
  long long ldo;
  int M, V, r;
  int last;            // the call's last read of W2: evict-first instead of evict-last
  uint32_t* claim;     // work-slot claim words (one per SM, zero before the call's first launch), or null
  uint32_t epoch;      // nonzero, distinct for every launch that shares the claim words
  int32_t* status;
  unsigned long long limit;
  unsigned long long* trace;  // [gridDim.x][16] globaltimer stamps (ns), or null -- slots:
  // 0 start, 1 end, 2 first W2 stage issued, 3 first L_base tile issued, 4 u band in TMEM (MMA side),
  // 5 first MMA issued, 6 first accumulator in the epilogue, 7 epilogue done, 8 last MMA committed,
  // 9 last W2 stage issued, 10 last L_base tile issued, 11 tiles, 15 wait on the previous grid done
};

__device__ __forceinline__ void tstamp(unsigned long long* trace, int k, unsigned long long v) {
  if (trace) trace[blockIdx.x * 16 + k] = v;
}

// L_base element (row, col) of a side buffer: boxes of 128 rows x 64 columns, 128-byte swizzle.
__device__ __forceinline__ const uint4* side_at(const uint8_t* side, int row, int col) {
  const int box = col >> 6, chunk = (col & 63) >> 3;
  return reinterpret_cast<const uint4*>(side + box * kBoxBytes + row * 128 + ((chunk ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kW2Threads, 1)
    k_w2_argmax(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmWn,
                const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmU, W2Args p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* side_ring = ring + (size_t)kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(side_ring + (size_t)kSide * kSideBytes);
  uint64_t* empty = full + kStages;
  uint64_t* sfull = empty + kStages;
  uint64_t* sempty = sfull + kSide;
  uint64_t* accf = sempty + kSide;
  uint64_t* acce = accf + 2;
  uint64_t* a_ready = acce + 2;
  uint64_t* mma_done = a_ready + 1;
  uint64_t* u_full = mma_done + 1;
  uint64_t* best_s = u_full + 1;  // [128] the second column group's best key per row
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(best_s + 128);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* slot_s = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) *slot_s = claim_slot(p.claim, p.epoch);
  __syncthreads();
  const int G = gridDim.x, c = *slot_s;  // this CTA's vocabulary range (by the SM it runs on)
  const int nunits = (p.V + kUnit - 1) / kUnit;
  const int u0 = (int)((long long)nunits * c / G), u1 = (int)((long long)nunits * (c + 1) / G);
  const int ntiles = (u1 - u0 + kTileUnits - 1) / kTileUnits;
  const int kblocks = p.r / 64;
  const unsigned long long limit = p.limit;
  if (threadIdx.x == 0) tstamp(p.trace, 0, globaltimer_ns());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < kSide; ++s) { mbar_init(&sfull[s], 1); mbar_init(&sempty[s], kEpiWarps); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], kEpiWarps); }
    mbar_init(a_ready, kEpiWarps);
    mbar_init(mma_done, 1);
    mbar_init(u_full, 1);
    *abort_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmWn);
    tma_prefetch_desc(&tmL);
    tma_prefetch_desc(&tmU);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();  // the next kernel may be scheduled; it waits for this grid

  if (warp == 0) {
    if (lane == 0) {  // ---- W2 producer (no wait on the previous grid: W2 is a weight) ----
      const uint64_t pol = p.last ? l2_policy_evict_first() : l2_policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int t = 0; t < ntiles && ok; ++t) {
        const int ut = u0 + t * kTileUnits, w = min(kTileUnits, u1 - ut);
        const int n0 = ut * kUnit;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_bounded(&empty[s], ((it / kStages) & 1u) ^ 1u, limit, abort_s)) { ok = false; break; }
          uint8_t* dst = ring + (size_t)s * kStageBytes;
          if (w == kTileUnits) {
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            tma_load_2d_hint(dst, &tmW, &full[s], kb * 64, n0, pol);
          } else {  // a narrow last tile: w boxes of 16 rows, stacked as in a full tile
            mbar_arrive_expect_tx(&full[s], (uint32_t)w * (kUnit * 64 * 2));
            for (int j = 0; j < w; ++j)
              tma_load_2d_hint(dst + j * (kUnit * 128), &tmWn, &full[s], kb * 64, n0 + j * kUnit, pol);
          }
          if (it == 0) tstamp(p.trace, 2, globaltimer_ns());
        }
      }
      tstamp(p.trace, 9, globaltimer_ns());
      if (!ok) *abort_s = 1;
      int never = 0;  // no copy may be in flight when the CTA exits
      for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0u); j < it; ++j)
        mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1u, kDrainPolls, &never);
    }
  } else if (warp == 2) {
    if (lane == 0) {  // ---- L_base producer (an input of the call: no wait either) ----
      const uint64_t pol = l2_policy_evict_first();
      int t = 0;
      for (; t < ntiles; ++t) {
        const int sl = t % kSide;
        if (!mbar_wait_bounded(&sempty[sl], ((t / kSide) & 1) ^ 1, limit, abort_s)) { *abort_s = 1; break; }
        // slots 1 and 2 hold the u band until the epilogue has moved it into TMEM
        if ((t == 1 || t == 2) && !mbar_wait_bounded(a_ready, 0u, limit, abort_s)) { *abort_s = 1; break; }
        const int ut = u0 + t * kTileUnits, w = min(kTileUnits, u1 - ut);
        const int n0 = ut * kUnit, nb = (w * kUnit + 63) / 64;
        mbar_arrive_expect_tx(&sfull[sl], (uint32_t)nb * kBoxBytes);
        for (int bx = 0; bx < nb; ++bx)
          tma_load_2d_hint(side_ring + (size_t)sl * kSideBytes + bx * kBoxBytes, &tmL, &sfull[sl], n0 + bx * 64, 0,
                           pol);
        if (t == 0) tstamp(p.trace, 3, globaltimer_ns());
      }
      tstamp(p.trace, 10, globaltimer_ns());
      int never = 0;
      for (int j = max(0, t - kSide); j < t; ++j) mbar_wait_bounded(&sfull[j % kSide], (j / kSide) & 1, kDrainPolls, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      bool ok = mbar_wait_bounded(a_ready, 0u, limit, abort_s);
      tstamp(p.trace, 4, globaltimer_ns());
      tmem_fence_after_sync();
      uint32_t it = 0;
      for (int t = 0; t < ntiles && ok; ++t) {
        const int ut = u0 + t * kTileUnits, w = min(kTileUnits, u1 - ut);
        const uint32_t a = t & 1, aph = (t >> 1) & 1;
        if (!mbar_wait_bounded(&acce[a], aph ^ 1u, limit, abort_s)) { ok = false; break; }
        tmem_fence_after_sync();
        const uint32_t d_tmem = tbase + 128 + a * 128;
        const uint32_t idesc = idesc_bf16_f32(128, w * kUnit);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_bounded(&full[s], (it / kStages) & 1u, limit, abort_s)) { ok = false; break; }
          tmem_fence_after_sync();
          const uint32_t b_addr = smem_u32(ring + (size_t)s * kStageBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ta(d_tmem, tbase + (uint32_t)(kb * 32 + k * 8), sw128_desc(b_addr + 32 * k), idesc,
                         (kb | k) != 0);
          umma_commit(&empty[s]);
          if (it == 0) tstamp(p.trace, 5, globaltimer_ns());
        }
        if (!ok) break;
        umma_commit(&accf[a]);
      }
      tstamp(p.trace, 8, globaltimer_ns());
      tstamp(p.trace, 11, (unsigned long long)ntiles);
      if (!ok) *abort_s = 1;
      int never = 0;  // TMEM may be freed only once every issued MMA has finished
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0u, kDrainPolls, &never);
    }
  } else if (warp >= 4) {  // ---- epilogue ----
    const int q = warp & 3, g = (warp - 4) >> 2;
    const int row = q * 32 + lane;          // batch row within the band = TMEM lane
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    pdl_wait();  // u comes from the previous kernel; keys and logits may be read by earlier ones
    if (warp == 4 && lane == 0) tstamp(p.trace, 15, globaltimer_ns());
    {  // u band into TMEM columns [0, r/2): one TMA load of 128 rows x r into ring slots 1 and 2
      // (rows past M read as zeros), then each thread moves its row (= TMEM lane) out of the
      // swizzled boxes, the two warps of a lane quadrant half of the columns each
      uint8_t* ubuf = side_ring + kSideBytes;
      const int nbox = p.r / 64;
      if (warp == 4 && lane == 0) {
        mbar_arrive_expect_tx(u_full, (uint32_t)nbox * kBoxBytes);
        for (int bx = 0; bx < nbox; ++bx) tma_load_2d(ubuf + bx * kBoxBytes, &tmU, u_full, bx * 64, 0);
      }
      if (!mbar_wait_warp(u_full, 0u, limit, abort_s)) *abort_s = 1;
      const int half = p.r / 4;  // 32-bit words per warp: a multiple of 16 (r is a multiple of 64)
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int k0 = g * (p.r / 2) + 8 * i;  // first of the chunk's 8 k values
        v[i] = 4 * i < half ? *side_at(ubuf, row, k0) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (4 * i < half) tmem_st4(tbase + lane_off + (uint32_t)(g * half + 4 * i), v[i]);
      tmem_wait_st();
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(a_ready);
    }
    float best = -INFINITY;
    int idx = -1;
    const bool live = row < p.M;
    for (int t = 0; t < ntiles; ++t) {
      const int ut = u0 + t * kTileUnits, w = min(kTileUnits, u1 - ut);
      const int n0 = ut * kUnit, N = w * kUnit;
      const uint32_t a = t & 1, aph = (t >> 1) & 1;
      const int sl = t % kSide;
      if (!mbar_wait_warp(&accf[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      if (t == 0 && warp == 4 && lane == 0) tstamp(p.trace, 6, globaltimer_ns());
      if (!mbar_wait_warp(&sfull[sl], (t / kSide) & 1, limit, abort_s)) { *abort_s = 1; break; }
      tmem_fence_after_sync();
      const int cb = g * 64;
      if (cb < N) {
        const uint8_t* side = side_ring + (size_t)sl * kSideBytes;
        const uint32_t taddr = tbase + lane_off + 128 + a * 128 + (uint32_t)cb;
        const int nc = min(64, N - cb);  // a multiple of 16
        uint32_t r[4][16];  // all 64 columns of the group (columns past N hold stale sums, unused)
        tmem_ld16(taddr, r[0]);
        tmem_ld16(taddr + 16, r[1]);
        tmem_ld16(taddr + 32, r[2]);
        tmem_ld16(taddr + 48, r[3]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if (16 * h < nc) {
#pragma unroll
            for (int j = 0; j < 16; ++j) reg_fence(r[h][j]);
            const int col = cb + 16 * h;  // column within the tile
            float l[16], f[8];
            widen(*side_at(side, row, col), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) l[j] = f[j];
            widen(*side_at(side, row, col + 8), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) l[8 + j] = f[j];
            const int nbase = n0 + col;
            float z[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) z[j] = __uint_as_float(r[h][j]) + l[j];
            float zm[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) zm[j] = (nbase + 16 <= p.V || nbase + j < p.V) ? z[j] : -INFINITY;
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
            if (p.out && live) {
              float* o = p.out + (size_t)row * p.ldo + nbase;
              if (nbase + 16 <= p.V) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  reinterpret_cast<float4*>(o)[j] = make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  if (nbase + j < p.V) o[j] = z[j];
              }
            }
          }
        }
      }
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acce[a]);
        mbar_arrive(&sempty[sl]);
      }
    }
    if (warp == 4 && lane == 0) tstamp(p.trace, 7, globaltimer_ns());
    // the two column groups of a row meet in shared memory; one atomicMax per row and CTA
    const uint64_t key = idx >= 0 ? argmax_key(best, idx) : 0ull;
    if (g == 1) best_s[row] = key;
    asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
    if (g == 0 && live) {
      const uint64_t k = umax64(key, best_s[row]);
      if (k) atomicMax(reinterpret_cast<unsigned long long*>(p.keys + row), (unsigned long long)k);
    }
  }

  if (warp == 4 && lane == 0) {  // no u copy may be in flight when the CTA exits (a timed-out wait)
    int never = 0;
    mbar_wait_bounded(u_full, 0u, kDrainPolls, &never);
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
  if (threadIdx.x == 0) {
    if (*abort_s && p.status) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
    tstamp(p.trace, 1, globaltimer_ns());
  }
}

cudaError_t set_smem_w2_once() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_w2_argmax, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace

bool w2_argmax_supported(int M, int V, int r, const void* U, const void* W2, const void* Lb, long long ldl) {
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  return M >= 1 && M <= 128 && V >= kUnit && r >= 64 && r <= 256 && r % 64 == 0 && a16(U) && a16(W2) && a16(Lb) &&
         (ldl * 2) % 16 == 0;
}

cudaError_t w2_argmax(const bf16* U, const bf16* W2, int M, int V, int r, const bf16* Lb, long long ldl,
                      uint64_t* keys, float* out, long long ldo, bool last, uint32_t* claim, uint32_t epoch,
                      int32_t* status, uint64_t limit, cudaStream_t st) {
  if (!w2_argmax_supported(M, V, r, U, W2, Lb, ldl)) return cudaErrorInvalidValue;
  if (claim) {
    cudaError_t e = ensure_sm_rank(st);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tw, twn, tl, tu;
  if (!tmap_bf16_tiles(&tw, W2, (uint64_t)V, (uint64_t)r, 128) || !tmap_bf16_tiles(&twn, W2, (uint64_t)V, (uint64_t)r, kUnit) ||
      !tmap_bf16_tiles(&tl, Lb, (uint64_t)M, (uint64_t)V, 128, (uint64_t)ldl) ||
      !tmap_bf16_tiles(&tu, U, (uint64_t)M, (uint64_t)r, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem_w2_once();
  if (e != cudaSuccess) return e;
  const int nunits = (V + kUnit - 1) / kUnit;
  const int grid = std::max(1, std::min(sm_count(), nunits));
  W2Args a{keys, out, ldo, M, V, r, last ? 1 : 0, grid == sm_count() ? claim : nullptr, epoch, status,
           (unsigned long long)limit, nullptr};
  int ntrace = 0;
  debug_trace(&a.trace, &ntrace);
  if (a.trace && ntrace < grid * 16) a.trace = nullptr;
  return note_launch(launch_pdl(k_w2_argmax, dim3(grid), dim3(kW2Threads), kSmemBytes, st, tw, twn, tl, tu, a));
}

}  // namespace domino
