// tf_units.cu -- the teacher-forced GRU recurrence for 5..128 batch rows in one cooperative launch
// in which every CTA owns eight state units, so that an update needs no partial sums in global
// memory and no grid barrier.
//
// Domino review page, section 二 ("Teacher Forcing"): with the tokens y given, every state follows
// from the previous one, S_i = GRUCell(embed[y_i], S_{i-1}), in the PyTorch gate form
//   r = sigmoid(W_ir x + b_ir + W_hr S + b_hr),  z = sigmoid(W_iz x + b_iz + W_hz S + b_hz),
//   n = tanh(W_in x + b_in + r * (W_hn S + b_hn)),  S' = (1 - z) * n + z * S.
// The input halves W_ih . embed[y_i] are computed for every given token before the launch (or read
// from the embedding projection table), so an update is the hidden half plus the cell.
//
// CTA c owns units [8c, 8c + 8); their 24 rows of W_hh (gates r, z, n) stay in shared memory for the
// whole call, and each row's state of these units stays in the registers of one epilogue thread.
// Per update:
//   warp 0      streams the split state S_hl = [hi | lo] of every row (bf16, K = 2Hs) by TMA;
//   warp 1      issues tcgen05.mma: D[row][gate row] += S_hl[row][k] . W_hh[gate row][k mod Hs];
//   warps 4..7  read the accumulator (TMEM lane = batch row), apply the cell to the CTA's units and
//               write the states output and the new split state for every CTA's next update.
// The split state is double-buffered (update i reads buffer i & 1 and writes the other).  Instead of
// a grid barrier, every CTA counts its writes of the state on one ready counter, and only the
// producer thread waits (bounded) for the count before loading; the other roles wait on their
// mbarriers as usual.  A CTA writes a buffer only after it has read the other one whole, which
// needs every CTA's previous cell, which came after that CTA's last read of the buffer being
// written: no write can overtake a read.
//
// Small batches fill the 128-row A tile with K: at B <= 32 (64) a tile carries four (two) K chunks
// of the state, one per row group of 32 (64) rows, and the B operand stacks the matching W_hh chunks
// along N.  Row group g times column group g is the wanted product; the other blocks of the
// accumulator are discarded, and the epilogue adds the groups' blocks in group order, so the result
// does not depend on timing.
//
// Every mbarrier wait and every counter wait is bounded: a role that gives up raises the CTA's abort
// flag, waits (bounded) for its copies and MMAs in flight, and the kernel reports
// DOMINO_STATUS_DEVICE_TIMEOUT.
#include "common.cuh"
#include "gemm_tc.h"
#include "internal.h"
#include "persistent.h"
#include "umma.cuh"

namespace domino {
namespace {

constexpr int kTfThreads = 256;           // warp 0 TMA, warp 1 MMA and TMEM, warps 4..7 epilogue
constexpr int kTfUnits = 8;               // state units per CTA
constexpr int kTfStages = 8;
constexpr uint32_t kTfStage = 128 * 128;  // one 128-row x 64-column bf16 tile, 128-byte swizzle
constexpr uint32_t kTfChunk = 32 * 128;   // the CTA's W_hh rows of one 64-column chunk: 32 (24 used)
constexpr int kTfMaxHs = 1024;
constexpr int kTfRedStride = 25;          // floats per row of the group-sum buffer (odd: no bank conflicts)
constexpr size_t kTfRing = (size_t)kTfStages * kTfStage;
constexpr size_t kTfW = (size_t)(kTfMaxHs / 64) * kTfChunk;
constexpr size_t kTfRed = (size_t)128 * kTfRedStride * 4;
constexpr size_t kTfMisc = 256;
constexpr size_t kTfSmem = kTfRing + kTfW + kTfRed + kTfMisc + 1024;
static_assert(kTfSmem <= 232448, "shared memory budget");
constexpr uint32_t kTfTmemCols = 128;
constexpr unsigned long long kTfDrain = kDrainPolls;

// mbarrier slots
enum : int { kTFull = 0, kTEmpty = kTfStages, kTW = 2 * kTfStages, kTAcc, kTMma, kTBars };
static_assert((kTBars + 1) * 8 + 16 <= (int)kTfMisc, "misc block");

struct TfArgs {
  const float* S0;        // [B][Hs]
  const int32_t* tokens;  // [B][L]
  const float* Gx;        // [B * (L - 1)][3Hs] W_ih . embed[y_i] (row b * (L - 1) + i), or null
  const float* Xp;        // [V][3Hs] projection table (when Gx is null)
  const bf16* b_ih;       // [3Hs]
  const bf16* b_hh;       // [3Hs]
  float* states;          // [B][L][Hs]
  bf16* S_hl;             // [2][B][2Hs] split state, double-buffered
  unsigned* ready;        // the CTAs' state writes, counted (zero before the launch)
  int32_t* status;
  int B, L, Hs, V;
  int chunks3d;           // the split-state map is tmap_bf16_chunks (one box per A tile), else 2-D
  unsigned long long limit;
  unsigned long long* trace;  // optional (globaltimer, ns): [0] CTA 0's start, [1] its set-up issued,
  int ntrace;                 // [i + 2] its update i done, [L + 1] its end; from kTfTraceMarks, per
                              // CTA c the milestones k of update 1 at [kTfTraceMarks + k * G + c]
                              // (k: 0 start, 1 copies issued, 2 copies landed, 3 MMAs issued, 4
                              // accumulator in the epilogue, 5 cell done and counted).  Entries past
                              // ntrace are not written.
};
constexpr int kTfTraceMarks = 128;  // past CTA 0's stamps (L + 2 <= 66 entries)

__device__ __forceinline__ unsigned tf_ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int tf_ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void tf_fence_proxy_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* tmap, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// NU consecutive fp32 values (aligned to their size) into v[0 .. NU).
template <int NU>
__device__ __forceinline__ void load_units(const float* p, float (&v)[8]) {
  if constexpr (NU == 2) {
    const float2 a = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = a.x; v[1] = a.y;
  } else {
#pragma unroll
    for (int k = 0; k < NU / 4; ++k) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(p) + k);
      v[4 * k] = a.x; v[4 * k + 1] = a.y; v[4 * k + 2] = a.z; v[4 * k + 3] = a.w;
    }
  }
}

// The new state of NU units of one row: the states output and the two-term bf16 split (hi, lo).
template <int NU>
__device__ __forceinline__ void put_units(const float (&s)[8], float* out, bf16* hi, bf16* lo) {
  uint32_t h[NU / 2], l[NU / 2];
#pragma unroll
  for (int k = 0; k < NU / 2; ++k) {
    const __nv_bfloat162 ph = __floats2bfloat162_rn(s[2 * k], s[2 * k + 1]);
    const float2 fh = __bfloat1622float2(ph);
    const __nv_bfloat162 pl = __floats2bfloat162_rn(s[2 * k] - fh.x, s[2 * k + 1] - fh.y);
    h[k] = *reinterpret_cast<const uint32_t*>(&ph);
    l[k] = *reinterpret_cast<const uint32_t*>(&pl);
  }
  if constexpr (NU == 2) {
    *reinterpret_cast<float2*>(out) = make_float2(s[0], s[1]);
    *reinterpret_cast<uint32_t*>(hi) = h[0];
    *reinterpret_cast<uint32_t*>(lo) = l[0];
  } else if constexpr (NU == 4) {
    *reinterpret_cast<float4*>(out) = make_float4(s[0], s[1], s[2], s[3]);
    *reinterpret_cast<uint2*>(hi) = make_uint2(h[0], h[1]);
    *reinterpret_cast<uint2*>(lo) = make_uint2(l[0], l[1]);
  } else {
    reinterpret_cast<float4*>(out)[0] = make_float4(s[0], s[1], s[2], s[3]);
    reinterpret_cast<float4*>(out)[1] = make_float4(s[4], s[5], s[6], s[7]);
    *reinterpret_cast<uint4*>(hi) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(lo) = make_uint4(l[0], l[1], l[2], l[3]);
  }
}

// GR: row groups of an A tile (1, 2 or 4; 128 / GR >= B).  The cell of a row is shared by GR
// epilogue threads, 8 / GR units each.  chunks3d: the split state arrives as one 3-D box per A tile
// (tmap_bf16_chunks) instead of GR 2-D boxes.
template <int GR>
__global__ void __launch_bounds__(kTfThreads, 1)
    k_tf_units(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmW, TfArgs p) {
  constexpr int Rg = 128 / GR;  // rows of a row group
  constexpr int NU = 8 / GR;    // units of an epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* wbuf = ring + kTfRing;
  float* red = reinterpret_cast<float*>(wbuf + kTfW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + kTfRed);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kTBars);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.B, L = p.L, Hs = p.Hs, H3 = 3 * Hs, G = gridDim.x;
  const int j0 = blockIdx.x * kTfUnits;
  const int KH = Hs / 64;             // 64-column chunks of a W_hh row
  const int nst = 2 * KH / GR;        // A tiles per update
  const unsigned long long limit = p.limit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTfStages; ++s) { mbar_init(&bars[kTFull + s], 1); mbar_init(&bars[kTEmpty + s], 1); }
    mbar_init(&bars[kTW], 1);
    mbar_init(&bars[kTAcc], 1);
    mbar_init(&bars[kTMma], 1);
    *abort_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmS);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTfTmemCols);
    tmem_relinquish();
  }
  // the fourth 8-row group of every W_hh chunk is not loaded: zeroes (its columns are discarded)
  for (int t = threadIdx.x; t < KH * 64; t += kTfThreads)
    reinterpret_cast<uint4*>(wbuf + (size_t)(t >> 6) * kTfChunk + 3 * 1024)[t & 63] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const bool tracer = p.trace && blockIdx.x == 0 && threadIdx.x == 0;
  if (tracer && p.ntrace > 0) p.trace[0] = globaltimer_ns();

  if (warp == 0 && lane == 0) {  // the CTA's W_hh rows, once: gate g's eight rows at 1 KB g of each chunk
    mbar_arrive_expect_tx(&bars[kTW], 3u * (uint32_t)KH * 1024u);
    for (int kc = 0; kc < KH; ++kc)
#pragma unroll
      for (int g = 0; g < 3; ++g) tma_load_2d(wbuf + (size_t)kc * kTfChunk + g * 1024, &tmW, &bars[kTW], kc * 64, g * Hs + j0);
  }

  // epilogue identity: accumulator row m = 32q + lane (TMEM lane quadrant q); the cell of batch row
  // b = m / GR, units [u0, u0 + NU) of the CTA's eight
  const int q = warp - 4, m = q * 32 + lane;
  const int b = m / GR, u0 = (m % GR) * NU;
  const bool cell = warp >= 4 && b < B;
  float s[8], bi[3][8], bh[3][8];
  if (cell) {
    load_units<NU>(p.S0 + (size_t)b * Hs + j0 + u0, s);
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
      for (int u = 0; u < NU; ++u) {
        bi[g][u] = to_f32(p.b_ih[(size_t)g * Hs + j0 + u0 + u]);
        bh[g][u] = to_f32(p.b_hh[(size_t)g * Hs + j0 + u0 + u]);
      }
    put_units<NU>(s, p.states + (size_t)b * L * Hs + j0 + u0, p.S_hl + (size_t)b * 2 * Hs + j0 + u0,
                  p.S_hl + (size_t)b * 2 * Hs + Hs + j0 + u0);
  }

  // The CTA's units of the new state are written (epilogue warps): count them on the ready counter.
  // The writers fence towards the async proxy (the readers load by TMA), the epilogue warps meet,
  // and one thread publishes with release semantics.
  auto signal_written = [&]() {
    tf_fence_proxy_global();
    asm volatile("bar.sync 2, %0;" ::"r"(128) : "memory");
    if (warp == 4 && lane == 0) {
      __threadfence();
      atomicAdd(p.ready, 1u);
    }
  };
  // Producer: the state holds the writes of update i - 1 (the set-up counts as update -1) once every
  // CTA has counted i + 1 writes.
  auto wait_ready = [&](unsigned target) -> bool {
    for (unsigned long long it = 0; it < limit; ++it) {
      if (tf_ld_acquire(p.ready) >= target) return true;
      if ((it & 31) == 31 && (*abort_s || tf_ld_relaxed(p.status) == DOMINO_STATUS_DEVICE_TIMEOUT)) break;
    }
    set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
    return false;
  };
  if (warp >= 4) signal_written();

  if (tracer && 1 < p.ntrace) p.trace[1] = globaltimer_ns();
  uint32_t it0 = 0;  // A tiles gone through the ring before this update
  for (int i = 0; i + 1 < L; ++i) {
    const int rb = (i & 1) * B;  // first row of the buffer this update reads
    auto mark = [&](int k) {
      const long long e = kTfTraceMarks + (long long)k * G + blockIdx.x;
      if (p.trace && i == 1 && e < p.ntrace) p.trace[e] = globaltimer_ns();
    };
    if (threadIdx.x == 0) mark(0);
    if (warp == 0) {
      if (lane == 0) {  // TMA producer: the split state, GR K chunks per A tile
        // the whole state first, then one proxy fence (a fence between copies would wait for the
        // ones in flight)
        bool good = wait_ready((unsigned)G * (unsigned)(i + 1));
        tf_fence_proxy_global();
        uint32_t it = it0;
        for (int t = 0; t < nst && good; ++t, ++it) {
          const int st = it % kTfStages;
          if (!mbar_wait_bounded(&bars[kTEmpty + st], ((it / kTfStages) & 1u) ^ 1u, limit, abort_s)) {
            good = false;
            break;
          }
          uint8_t* dst = ring + (size_t)st * kTfStage;
          mbar_arrive_expect_tx(&bars[kTFull + st], kTfStage);
          if (p.chunks3d) {
            tma_load_3d(dst, &tmS, &bars[kTFull + st], 0, rb, t * GR);
          } else {
#pragma unroll
            for (int g = 0; g < GR; ++g)
              tma_load_2d(dst + (size_t)g * Rg * 128, &tmS, &bars[kTFull + st], (t * GR + g) * 64, rb);
          }
        }
        if (!good) *abort_s = 1;
        mark(1);
        int never = 0;  // the copies of this update have landed before the role moves on
        for (uint32_t j = (it - it0 > (uint32_t)kTfStages ? it - kTfStages : it0); j < it; ++j)
          mbar_wait_bounded(&bars[kTFull + j % kTfStages], (j / kTfStages) & 1u, kTfDrain, &never);
        mark(2);
      }
    } else if (warp == 1) {
      if (lane == 0) {  // MMA issuer: one 128 x (32 GR) accumulator at TMEM column 0
        bool good = i > 0 || mbar_wait_bounded(&bars[kTW], 0u, limit, abort_s);
        constexpr uint32_t idesc = idesc_bf16_f32(128, 32 * GR);
        uint32_t it = it0;
        for (int t = 0; t < nst && good; ++t, ++it) {
          const int st = it % kTfStages;
          if (!mbar_wait_bounded(&bars[kTFull + st], (it / kTfStages) & 1u, limit, abort_s)) {
            good = false;
            break;
          }
          tmem_fence_after_sync();
          const uint32_t a_addr = smem_u32(ring + (size_t)st * kTfStage);
          const uint32_t b_addr = smem_u32(wbuf + (size_t)((t * GR) % KH) * kTfChunk);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tbase, sw128_desc(a_addr + 32 * k), sw128_desc(b_addr + 32 * k), idesc, (t | k) != 0);
          umma_commit(&bars[kTEmpty + st]);
        }
        if (!good) *abort_s = 1;
        mark(3);
        umma_commit(&bars[kTAcc]);  // completes when every MMA issued above has finished
        int never = 0;
        umma_commit(&bars[kTMma]);
        mbar_wait_bounded(&bars[kTMma], (uint32_t)i & 1u, kTfDrain, &never);
      }
    } else if (warp >= 4) {
      // this update's gate inputs do not depend on the state: loaded before the accumulator is ready
      float x[3][8];
      if (cell) {
        const int tok = p.tokens[(size_t)b * L + i];
        const bool valid = tok >= 0 && tok < p.V;
        if (!valid && blockIdx.x == 0 && u0 == 0) set_status(p.status, DOMINO_STATUS_BAD_TOKEN);
        const float* src = p.Gx ? p.Gx + ((size_t)b * (L - 1) + i) * H3 : p.Xp + (size_t)(valid ? tok : 0) * H3;
#pragma unroll
        for (int g = 0; g < 3; ++g) load_units<NU>(src + (size_t)g * Hs + j0 + u0, x[g]);
      }
      const bool got = mbar_wait_warp(&bars[kTAcc], (uint32_t)i & 1u, limit, abort_s);
      if (!got) *abort_s = 1;
      if (warp == 4 && lane == 0) mark(4);
      tmem_fence_after_sync();
      uint32_t v[32];
      const int grp = m / Rg;  // the row group of this lane's accumulator row: its column block
      const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * 32);
      tmem_ld16(taddr, &v[0]);
      tmem_ld16(taddr + 16, &v[16]);
      tmem_wait_ld();
      float h[3][8];
      if constexpr (GR > 1) {  // the row groups' blocks through shared memory, added in group order
#pragma unroll
        for (int c = 0; c < 24; ++c) red[m * kTfRedStride + c] = __uint_as_float(v[c]);
        asm volatile("bar.sync 1, %0;" ::"r"(128) : "memory");
        if (cell) {
#pragma unroll
          for (int g = 0; g < 3; ++g)
#pragma unroll
            for (int u = 0; u < NU; ++u) {
              float a = red[b * kTfRedStride + g * 8 + u0 + u];
#pragma unroll
              for (int r = 1; r < GR; ++r) a += red[(r * Rg + b) * kTfRedStride + g * 8 + u0 + u];
              h[g][u] = a;
            }
        }
      } else {
#pragma unroll
        for (int g = 0; g < 3; ++g)
#pragma unroll
          for (int u = 0; u < 8; ++u) h[g][u] = __uint_as_float(v[g * 8 + u]);
      }
      if (cell && got) {
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const float gi0 = x[0][u] + bi[0][u], gi1 = x[1][u] + bi[1][u], gi2 = x[2][u] + bi[2][u];
          const float gh0 = h[0][u] + bh[0][u], gh1 = h[1][u] + bh[1][u], gh2 = h[2][u] + bh[2][u];
          const float rg = sigmoidf_(gi0 + gh0);
          const float zg = sigmoidf_(gi1 + gh1);
          const float ng = tanhf(gi2 + rg * gh2);
          s[u] = (1.f - zg) * ng + zg * s[u];
        }
        bf16* hl = p.S_hl + ((size_t)(B - rb) + b) * 2 * Hs;  // the other buffer
        put_units<NU>(s, p.states + ((size_t)b * L + i + 1) * Hs + j0 + u0, hl + j0 + u0, hl + Hs + j0 + u0);
      }
      signal_written();
      if (warp == 4 && lane == 0) mark(5);
    }
    it0 += (uint32_t)nst;
    // the next update's MMAs overwrite the accumulator the epilogue has just read
    tmem_fence_before_sync();
    const bool stop = __syncthreads_or(*abort_s != 0);
    tmem_fence_after_sync();
    if (tracer && i + 2 < p.ntrace) p.trace[i + 2] = globaltimer_ns();
    if (stop) break;
  }

  if (warp == 0 && lane == 0) {  // the W_hh copies have landed (a call with no update never waited)
    int never = 0;
    mbar_wait_bounded(&bars[kTW], 0u, kTfDrain, &never);
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (warp == 1) tmem_dealloc(tbase, kTfTmemCols);
  if (threadIdx.x == 0 && *abort_s) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
  if (tracer && L + 1 < p.ntrace) p.trace[L + 1] = globaltimer_ns();
}

int g_tf_fit[64];  // per device: 0 unknown, 1 fits, -1 does not

template <int GR>
bool tf_fits_one() {
  int per_sm = 0;
  return cudaFuncSetAttribute(k_tf_units<GR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTfSmem) ==
             cudaSuccess &&
         cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_tf_units<GR>, kTfThreads, kTfSmem) == cudaSuccess &&
         per_sm >= 1;
}

bool tf_units_fits() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (g_tf_fit[dev] != 0) return g_tf_fit[dev] > 0;
  const bool fits = tf_fits_one<1>() && tf_fits_one<2>() && tf_fits_one<4>();
  cudaGetLastError();
  g_tf_fit[dev] = fits ? 1 : -1;
  return fits;
}

// Row groups of an A tile: as many as the batch leaves room for, dividing the W_hh chunk count.
int tf_groups(const Shape& s) {
  int gr = s.B <= 32 ? 4 : s.B <= 64 ? 2 : 1;
  while (gr > 1 && (s.Hs / 64) % gr != 0) gr /= 2;
  return gr;
}

}  // namespace

bool tf_units_ok(const Shape& s) {
  if (s.dtype != DOMINO_DTYPE_BF16 || s.B < 1 || s.B > 128 || s.L < 1) return false;
  if (s.Hs % 64 != 0 || s.Hs > kTfMaxHs || s.Hs / kTfUnits > sm_count()) return false;
  return tf_units_fits();
}

const char* tf_units_plan() {
  return "k_tf_units: one cooperative launch, each CTA owning eight state units with their W_hh rows in shared "
         "memory, per update a tcgen05 product of the split state and the cell; the next update's loads wait on "
         "a counter of the CTAs' state writes";
}

cudaError_t launch_tf_units(const Shape& s, const domino_weights_t& w, const float* S0, const int32_t* tokens,
                            const float* Gx, float* states, const Workspace& ws, int32_t* status, uint64_t spin,
                            cudaStream_t st) {
  if (!tokens || !states || (!Gx && !w.embed_proj && s.L > 1)) return cudaErrorInvalidValue;
  const int gr = tf_groups(s);
  // the two split-state buffers are rows [0, B) and [B, 2B) of ws.S_hl (B * L rows of 2Hs)
  const uint64_t rows = s.L > 1 ? 2 * (uint64_t)s.B : (uint64_t)s.B;
  CUtensorMap tS, tW;
  const bool c3 = tmap_bf16_chunks(&tS, ws.S_hl, rows, 2 * (uint64_t)s.Hs, (uint32_t)(128 / gr), (uint32_t)gr);
  if ((!c3 && !tmap_bf16_tiles(&tS, ws.S_hl, rows, 2 * (uint64_t)s.Hs, (uint32_t)(128 / gr))) ||
      !tmap_bf16_tiles(&tW, w.W_hh, 3 * (uint64_t)s.Hs, (uint64_t)s.Hs, 8))
    return cudaErrorInvalidValue;
  TfArgs a{};
  a.S0 = S0;
  a.tokens = tokens;
  a.Gx = w.embed_proj ? nullptr : Gx;
  a.Xp = w.embed_proj;
  a.b_ih = (const bf16*)w.b_ih;
  a.b_hh = (const bf16*)w.b_hh;
  a.states = states;
  a.S_hl = ws.S_hl;
  a.ready = ws.sync;
  a.status = status;
  a.B = s.B; a.L = s.L; a.Hs = s.Hs; a.V = s.V;
  a.chunks3d = c3 ? 1 : 0;
  a.limit = spin;
  debug_trace(&a.trace, &a.ntrace);
  void* params[] = {&tS, &tW, &a};
  const void* kern = gr == 4 ? (const void*)k_tf_units<4> : gr == 2 ? (const void*)k_tf_units<2>
                                                                    : (const void*)k_tf_units<1>;
  const cudaError_t e = cudaLaunchCooperativeKernel(kern, dim3(s.Hs / kTfUnits), dim3(kTfThreads), params, kTfSmem, st);
  return note_launch(e);
}

}  // namespace domino
