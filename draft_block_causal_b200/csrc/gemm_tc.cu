// gemm_tc.cu -- persistent tcgen05 GEMM with fused epilogues (bf16 x bf16 -> fp32 in TMEM).
//
//   D[m][n] = sum_k A[m][k] * B[n][k]      A: [M x K], B: [N x K], both bf16, K-major
//
// One CTA per SM walks output tiles of 128 x BN.  Warp roles:
//   warp 0, one thread : TMA producer -- 128x64 A tile + BNx64 B tile per k-block into a ring of
//                        S shared-memory stages (128-byte swizzle), signalled on full[s]; with a
//                        resident A (K <= 256, one 128-row band) only B streams, two k-blocks a stage
//   warp 1, one thread : MMA issuer   -- four tcgen05.mma (K = 16) per k-block into one of two TMEM
//                        accumulators; tcgen05.commit frees the stage (empty[s]) and, after the
//                        last k-block, publishes the accumulator (acc_full[a])
//   warps 2 ..         : epilogue     -- 4 or 8 warps (EpiWarps); warp w reads TMEM lanes
//                        32*(w%4).. (output rows) and, with 8 warps, half of the columns; then the
//                        epilogue functor; acc_empty[a]
// Split-K: when the output has too few tiles to occupy the SMs, each tile's K range is cut into
// ksplit pieces computed by the ksplit CTAs of one thread-block cluster (one tile per cluster, one
// piece per CTA).  Each CTA stores its partial of every 16-column unit of the tile straight into the
// shared memory of the cluster CTA that owns the unit (st.shared::cluster); after one cluster
// barrier each owner adds the ksplit pieces in piece order (fixed, so results do not depend on
// scheduling) and runs the epilogue functor.  An earlier cluster barrier, arrived at start and
// awaited before the first remote store, guarantees that every CTA of the cluster is running.
// Launches use programmatic stream serialization: a CTA triggers its dependents after set-up and
// waits on the previous grid before touching produced memory; the producer prefetches weight tiles
// into L2 before that wait.  A persistent launch with one CTA per SM may take its work slots by the
// SM it runs on (claim_slot), so that each tile keeps the same SM at every launch.
// Every mbarrier wait is bounded.  A role that gives up raises a CTA-wide abort flag; the others
// stop at their next wait, the producer waits for its copies still in flight, TMEM is freed and
// DOMINO_STATUS_DEVICE_TIMEOUT is reported.
//
// Uses in this library (the Domino head equation, review page section 二):
//   - the W2 product of greedy drafting, batch-major with L_base and the argmax in the epilogue
//     (EpiArgmaxT), and of teacher forcing with L_base added (EpiLogitsRow / EpiLogits);
//   - the GRU products on the tensor cores: W_ih . embedding rows and W_hh . state (EpiStore,
//     transposed), W_hh stacked with W1's state block giving gh and the next activations
//     (EpiGruU), the activations alone (EpiSiluU), and the H-projection W1[:, :d] . H (EpiStore);
//   - the input projection of the embedding table (embed . W_ih^T, EpiStore).
#include "common.cuh"
#include "gemm_tc.h"
#include "launch.cuh"
#include "sm_affinity.cuh"
#include "umma.cuh"

#include <atomic>
#include <mutex>
#include <type_traits>

namespace domino {

namespace {

constexpr int kBM = 128, kBK = 64;
// Warps 0 and 1 produce and issue; 4 * kGroups epilogue warps follow (two warps per TMEM lane
// quadrant, each on half of the tile's columns, for the argmax epilogue whose per-tile work is the
// longest; one per quadrant otherwise).
// An epilogue may state its group count (kGroups); otherwise the side-tile epilogues take two.
template <class Epi, class = void> struct GroupsOf {
  static constexpr int value = Epi::kSide ? 2 : 1;
};
template <class Epi> struct GroupsOf<Epi, std::void_t<decltype(Epi::kGroups)>> {
  static constexpr int value = Epi::kGroups;
};
// An epilogue whose apply() is warp-cooperative (every lane of a warp calls it with the same column
// group) states kWarpCoop; the split-K reduction, which hands units to threads individually, never
// takes it.
template <class Epi, class = void> struct WarpCoop {
  static constexpr bool value = false;
};
template <class Epi> struct WarpCoop<Epi, std::void_t<decltype(Epi::kWarpCoop)>> {
  static constexpr bool value = Epi::kWarpCoop;
};
// Static shared memory an epilogue declares (kStaticSmem), which the stage ring must leave room for.
template <class Epi, class = void> struct StaticSmemOf {
  static constexpr size_t value = 0;
};
template <class Epi> struct StaticSmemOf<Epi, std::void_t<decltype(Epi::kStaticSmem)>> {
  static constexpr size_t value = Epi::kStaticSmem;
};
template <class Epi> struct EpiWarps {
  static constexpr int kGroups = GroupsOf<Epi>::value;
  static constexpr int kThreads = 64 + 128 * kGroups;
};
constexpr uint32_t kABytes = kBM * kBK * 2;

// ---- epilogues ----
// Each epilogue thread owns one output row m of every tile it sees.  apply(state, m, n0, v, N)
// receives 16 consecutive columns n0.. of row m; finish(state, m) runs once after the thread's
// last tile (launches that use it keep a single 128-row band of M, so m is fixed per thread).
struct NoState {};
// Side tile: an epilogue with kSide = true receives, per output tile, a 128 x BN bf16 tile of a third
// operand (rows m, columns n) that the epilogue warps TMA-load one tile ahead into shared memory,
// as BN/64 boxes of 128 x 64 with 128-byte swizzling.  side_bf16() reads element (row, col) of it.
__device__ __forceinline__ const uint4* side_chunk(const uint8_t* side, int row, int col) {
  const int box = col >> 6, chunk = (col & 63) >> 3;
  return reinterpret_cast<const uint4*>(side + box * 16384 + row * 128 + ((chunk ^ (row & 7)) << 4));
}
struct EpiStore {  // out[m * ldo + n] = D, or out[n * ldo + m] = D when trans
  static constexpr bool kSide = false;
  static constexpr bool kARes = false;
  using State = NoState;
  float* out;
  int M;
  long long ldo;
  int trans;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m >= M) return;
    if (trans) {  // lanes hold consecutive m: each store instruction is coalesced across the warp
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (n0 + j < N) out[(size_t)(n0 + j) * ldo + m] = v[j];
      return;
    }
    float* o = out + (size_t)m * ldo + n0;
    if (n0 + 16 <= N && ((reinterpret_cast<uintptr_t>(o) & 15u) == 0)) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<float4*>(o)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (n0 + j < N) o[j] = v[j];
    }
  }
};
// Output element conversion of the logits epilogues (fp32, or bf16 rounded to nearest even).
__device__ __forceinline__ void put(float* p, float v) { *p = v; }
__device__ __forceinline__ void put(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename OutT>
struct EpiLogitsT {  // logits[n][m] = D + Lb[n][m]   (m = vocabulary row, n = (row, position))
  static constexpr bool kSide = false;
  static constexpr bool kARes = false;
  using State = NoState;
  const bf16* Lb;
  OutT* logits;
  int M;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m >= M) return;
    // all loads before any store: the compiler cannot assume that logits and Lb do not alias,
    // and interleaving them would serialise one memory round trip per column
    float l[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) l[j] = (n0 + j < N) ? __bfloat162float(__ldg(Lb + (size_t)(n0 + j) * M + m)) : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (n0 + j < N) put(logits + (size_t)(n0 + j) * M + m, v[j] + l[j]);
  }
};

// Teacher-forced logits, row-major: m = row (b, i) < M, n = vocabulary column < N:
//   logits[m * ld + n] = D + Lb[m * ld + n]
// Each thread owns 16 consecutive columns of one row (n0 is a multiple of 16; rows are 16-byte
// aligned since V % 8 == 0).  Full groups are written through a per-warp staging buffer: the warp's
// 32 rows x 16 columns go to shared memory (16-byte chunks XOR-swizzled so that neither side has
// bank conflicts) and come back so that each store instruction writes whole 64-byte (fp32) or
// 32-byte (bf16) row segments -- 8 or 16 rows per instruction instead of 32 scattered 16-byte
// pieces.  Every lane of the warp calls apply with the same n0.  L_base arrives as the side tile
// (rows m, columns n of the output tile, by TMA one tile ahead), so the epilogue issues no loads.
template <typename OutT>
struct EpiLogitsRowT {
  static constexpr bool kSide = true;
  static constexpr bool kARes = false;
  static constexpr int kGroups = 2;  // the epilogue is the longest phase of a tile: two warps per lane quadrant
  static constexpr bool kWarpCoop = true;
  static constexpr size_t kStaticSmem = 8 * 32 * 16 * 4;  // the staging buffers below
  using State = NoState;
  const bf16* Lb;
  OutT* logits;
  int M;
  long long ld;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t* side,
                                        int row, int c0) const {
    const int lane = threadIdx.x & 31;
    if (n0 + 16 <= N) {  // warp-uniform
      // per epilogue warp: 32 rows x 16 values (fp32: 64 B a row, four 16-byte chunks)
      __shared__ __align__(16) uint32_t stage[8][32 * 16];
      uint32_t* sw = stage[((threadIdx.x >> 5) - 2) & 7];
      float z[16];
      if (m < M) {
        float a[8], b[8];
        widen(*side_chunk(side, row, c0), a);
        widen(*side_chunk(side, row, c0 + 8), b);
#pragma unroll
        for (int j = 0; j < 8; ++j) { z[j] = v[j] + a[j]; z[8 + j] = v[8 + j] + b[j]; }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0.f;
      }
      const int mbase = m - lane;  // the row of lane 0 (the warp's rows are consecutive)
      if constexpr (std::is_same<OutT, float>::value) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(sw + lane * 16 + ((j ^ ((lane >> 1) & 3)) << 2)) =
              make_uint4(__float_as_uint(z[4 * j]), __float_as_uint(z[4 * j + 1]), __float_as_uint(z[4 * j + 2]),
                         __float_as_uint(z[4 * j + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // 8 rows a round, 4 lanes (16 bytes each) a row
          const int r = 8 * i + (lane >> 2), c = lane & 3;
          const uint4 x = *reinterpret_cast<const uint4*>(sw + r * 16 + ((c ^ ((r >> 1) & 3)) << 2));
          if (mbase + r < M) *reinterpret_cast<uint4*>(logits + (size_t)(mbase + r) * ld + n0 + 4 * c) = x;
        }
      } else {  // bf16: 32 B a row, two 16-byte chunks
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const __nv_bfloat162 pr = __floats2bfloat162_rn(z[2 * q], z[2 * q + 1]);
          w[q] = *reinterpret_cast<const uint32_t*>(&pr);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
          *reinterpret_cast<uint4*>(sw + lane * 8 + ((j ^ ((lane >> 2) & 1)) << 2)) =
              make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // 16 rows a round, 2 lanes a row
          const int r = 16 * i + (lane >> 1), c = lane & 1;
          const uint4 x = *reinterpret_cast<const uint4*>(sw + r * 8 + ((c ^ ((r >> 2) & 1)) << 2));
          if (mbase + r < M) *reinterpret_cast<uint4*>(logits + (size_t)(mbase + r) * ld + n0 + 8 * c) = x;
        }
      }
      __syncwarp();  // the buffer is reused by the warp's next group
      return;
    }
    if (m >= M) return;
    const bf16* lr = Lb + (size_t)m * ld + n0;
    OutT* o = logits + (size_t)m * ld + n0;
    float l[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) l[j] = (n0 + j < N) ? __bfloat162float(lr[j]) : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (n0 + j < N) put(o + j, v[j] + l[j]);
  }
};

// Greedy step, batch-major: m = batch row b (< M), n = vocabulary row v.
//   z = D + Lb[b][v] (Lb row stride ldl); per 16-column group the maximum (a tree of 15 max
//   operations) is compared with the running best, and only a group that beats it (strict >, so
//   the earliest group wins ties) is searched for the lowest column holding its maximum -- after
//   the first groups that is rare, so the common cost is an add and a max per element.
//   finish: keys[b] = max(keys[b], key(best)).  When out is set, z is also stored to
//   out[b * ldo + v].
template <bool ARES>
struct EpiArgmaxT {
  static constexpr bool kSide = true;  // the L_base tile [128 rows b x BN columns v]
  static constexpr bool kARes = ARES;  // the activation band is loaded once per CTA
  struct State {
    float best;
    int idx;
  };
  uint64_t* keys;
  int M;
  float* out;
  long long ldo;
  __device__ __forceinline__ void init(State& s) const { s.best = -INFINITY; s.idx = -1; }
  __device__ __forceinline__ void apply(State& s, int m, int n0, const float (&v)[16], int N, const uint8_t* side,
                                        int row, int c0) const {
    if (m >= M) return;
    float l[16];
    float a[8];
    widen(*side_chunk(side, row, c0), a);
#pragma unroll
    for (int j = 0; j < 8; ++j) l[j] = a[j];
    widen(*side_chunk(side, row, c0 + 8), a);
#pragma unroll
    for (int j = 0; j < 8; ++j) l[8 + j] = a[j];
    float z[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) z[j] = v[j] + l[j];
    float zm[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) zm[j] = (n0 + 16 <= N || n0 + j < N) ? z[j] : -INFINITY;  // ragged last tile
    float t8[8], t4[4];
#pragma unroll
    for (int j = 0; j < 8; ++j) t8[j] = fmaxf(zm[j], zm[j + 8]);
#pragma unroll
    for (int j = 0; j < 4; ++j) t4[j] = fmaxf(t8[j], t8[j + 4]);
    const float mx = fmaxf(fmaxf(t4[0], t4[2]), fmaxf(t4[1], t4[3]));
    if (mx > s.best) {  // the lowest column of this group holding its maximum
      int jj = 15;
#pragma unroll
      for (int j = 15; j >= 0; --j)
        if (zm[j] == mx) jj = j;
      s.best = mx;
      s.idx = n0 + jj;
    }
    if (out) {
      if (n0 + 16 <= N) {
        float4* o = reinterpret_cast<float4*>(out + (size_t)m * ldo + n0);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
      } else {
        for (int j = 0; j < 16 && n0 + j < N; ++j) out[(size_t)m * ldo + n0 + j] = z[j];
      }
    }
  }
  __device__ __forceinline__ void finish(State& s, int m) const {
    if (m < M && s.idx >= 0)
      atomicMax(reinterpret_cast<unsigned long long*>(keys + m), (unsigned long long)argmax_key(s.best, s.idx));
  }
};

// Stacked GRU / activation product: rows m < M1 are W_hh rows, gh: out[n * ldo + m] = D; rows
// m >= M1 are W1 state-block rows k = m - M1: u16[n * r + k] = bf16(SiLU(P[n * ldp + k] + D)).
struct EpiGruU {
  static constexpr bool kSide = false;
  static constexpr bool kARes = false;
  using State = NoState;
  float* out;
  long long ldo;
  int M1;
  const float* P;
  long long ldp;
  bf16* u16;
  int r;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m < M1) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (n0 + j < N) out[(size_t)(n0 + j) * ldo + m] = v[j];
    } else if (m < M1 + r) {
      const int k = m - M1;
      float pv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) pv[j] = (n0 + j < N) ? P[(size_t)(n0 + j) * ldp + k] : 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (n0 + j < N) u16[(size_t)(n0 + j) * r + k] = __float2bfloat16_rn(siluf_(pv[j] + v[j]));
    }
  }
};

// u[n][m] = SiLU(P[n * ldp + m] + D) as bf16 (and fp32 when uf is set): m = rank index (M = r), n = row.
struct EpiSiluU {
  static constexpr bool kSide = false;
  static constexpr bool kARes = false;
  using State = NoState;
  const float* P;
  long long ldp;
  bf16* u16;
  float* uf;
  int M;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m >= M) return;
    float pv[16];  // all loads before any store (see EpiLogits)
#pragma unroll
    for (int j = 0; j < 16; ++j) pv[j] = (n0 + j < N) ? __ldg(P + (size_t)(n0 + j) * ldp + m) : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int n = n0 + j;
      if (n < N) {
        const float u = siluf_(pv[j] + v[j]);
        u16[(size_t)n * M + m] = __float2bfloat16_rn(u);
        if (uf) uf[(size_t)n * M + m] = u;
      }
    }
  }
};

// Profiling stamps (trace != null): slot k of CTA b at trace[b * kTraceSlots + k].  Slots: 0/1
// globaltimer at start/end; 2 clock at start, 3 setup done, 4 first stage ready (MMA), 5 last
// accumulator committed (MMA), 6 first accumulator received (epilogue), 7 epilogue work done, 8
// cluster barrier passed, 9 split reduction done, 10 end, 11 last load issued (producer), 12 items,
// 13 first item's epilogue done, 14 first item's accumulator committed (MMA), 15 globaltimer when
// the producer's wait for the previous grid returned.
constexpr int kTraceSlots = 16;
__device__ __forceinline__ void stamp(unsigned long long* trace, int k, unsigned long long v) {
  if (trace) trace[blockIdx.x * kTraceSlots + k] = v;
}
__device__ __forceinline__ unsigned long long clk() { return (unsigned long long)clock64(); }

// Split-K exchange.  The tile's kBM x BN outputs are kUnits = kBM * BN / 16 units of 16 columns of
// one row (unit u = group * kBM + row); cluster CTA o owns units [o*kUnits/ks, (o+1)*kUnits/ks).
// Every CTA stores its partial of each unit into the owner's receive buffer, slot
// (piece * nmax + local index), 64 bytes per slot with the float4 index XOR-ed by bits 1..2 of the
// local index (eight consecutive slots on distinct banks).
__device__ __forceinline__ int unit_owner(int u, int ks, int units) { return (u * ks + ks - 1) / units; }
__device__ __forceinline__ int unit_first(int o, int ks, int units) { return o * units / ks; }
__device__ __forceinline__ uint32_t slot_offset(int slot, int li, int j) {
  return (uint32_t)((slot * 4 + (j ^ ((li >> 1) & 3))) * 16);
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
// shared::cta address -> the same offset in the shared memory of cluster CTA `rank`
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Shared memory (from a 1024-aligned base): [resident A][stage ring][1024 B: mbarriers, TMEM slot]
// [two side tiles][split-K receive buffer], plus 1024 bytes of slack for the alignment.  With a
// resident A (K <= 256, one 128-row band of M) each stage carries two k-blocks of B; otherwise one
// k-block of A and B.
template <int BN, bool SIDE, bool ARES, bool SPLIT = false, size_t STATIC = 0> struct Cfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr int kKBS = ARES ? 2 : 1;
  static constexpr uint32_t kStage = ARES ? kKBS * kBBytes : kABytes + kBBytes;
  static constexpr size_t kAResBytes = ARES ? 4 * (size_t)kABytes : 0;
  static constexpr size_t kSideBytes = SIDE ? (size_t)kBM * BN * 2 : 0;  // one side tile
  static constexpr int kUnits = kBM * BN / 16;
  // ks * ceil(kUnits / ks) slots of 64 bytes, for any ks <= 8
  static constexpr size_t kRecvBytes = SPLIT ? (size_t)(kUnits + 8) * 64 : 0;
  // 227 KB per CTA, less the epilogue's static shared memory (STATIC)
  static constexpr size_t kBudget = 232448 - STATIC - 2048 - 2 * kSideBytes - kAResBytes - kRecvBytes;
  static constexpr int kStagesFit = (int)(kBudget / kStage);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kTmemCols = (2 * BN) <= 32 ? 32 : ((2 * BN) <= 64 ? 64 : ((2 * BN) <= 128 ? 128 : ((2 * BN) <= 256 ? 256 : 512)));
  static constexpr size_t kSmem = kAResBytes + (size_t)kStages * kStage + 2048 + 2 * kSideBytes + kRecvBytes;
  static_assert(kStages >= 2, "shared memory too small for the pipeline");
};

template <int BN, class Epi, bool SPLIT>
__global__ void __launch_bounds__(EpiWarps<Epi>::kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
              const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmS, int M, int N, int K,
              Epi epi, int32_t* status, unsigned long long limit, int a_kwrap, int a_split, int ksplit,
              int a_stream, int indep, uint32_t* __restrict__ claim, uint32_t epoch,
              unsigned long long* __restrict__ trace, int mfirst) {
  static_assert(!SPLIT || (!Epi::kSide && !Epi::kARes), "split-K needs a plain epilogue");
  using C = Cfg<BN, Epi::kSide, Epi::kARes, SPLIT, StaticSmemOf<Epi>::value>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ares = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* smem = ares + C::kAResBytes;  // stage ring
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStage);
  uint64_t* empty = full + S;
  uint64_t* accf = empty + S;
  uint64_t* acce = accf + 2;
  uint64_t* mma_done = acce + 2;
  uint64_t* sidef = mma_done + 1;  // [2] side tile landed
  uint64_t* sidee = sidef + 2;     // [2] side buffer read by all four epilogue warps
  uint64_t* a_full = sidee + 2;    // resident A landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_full + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* slot_s = reinterpret_cast<volatile int*>(tmem_slot + 2);
  // after the barriers (1024 bytes) and the two side tiles: the split-K receive buffer
  uint8_t* const recv_buf = smem + (size_t)S * C::kStage + 1024 + 2 * C::kSideBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool waited_first = false;  // this thread has passed the first split-K cluster barrier
  if (threadIdx.x == 0) {
    stamp(trace, 0, globaltimer_ns());
    stamp(trace, 2, clk());
  }
  // split-K: first cluster barrier, arrived now and awaited just before the first remote store,
  // so that every CTA of the cluster is known to be running when its peers write to it
  if constexpr (SPLIT) cluster_arrive_relaxed();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 4 * EpiWarps<Epi>::kGroups); }
    mbar_init(mma_done, 1);
    mbar_init(&sidef[0], 1);
    mbar_init(&sidef[1], 1);
    mbar_init(&sidee[0], 4 * EpiWarps<Epi>::kGroups);
    mbar_init(&sidee[1], 4 * EpiWarps<Epi>::kGroups);
    mbar_init(a_full, 1);
    *abort_s = 0;
    *slot_s = claim_slot(claim, epoch);
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    if (a_split) tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB);
    if constexpr (Epi::kSide) tma_prefetch_desc(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const int slot = *slot_s;  // this CTA's first work item (blockIdx.x unless SM-affine)
  if (threadIdx.x == 0) {
    stamp(trace, 3, clk());
    pdl_trigger();  // the next kernel on the stream may be scheduled (it waits for this grid to finish)
  }

  const int m_tiles = (M + kBM - 1) / kBM, n_tiles = (N + BN - 1) / BN, kblocks = K / kBK;
  const int tiles = m_tiles * n_tiles;
  // output tile -> (first row, first column): N-tiles within an M band (default), or the M bands of
  // one N tile in turn (mfirst: CTAs that run at the same time then share each B tile through L2)
  auto tile_m0 = [&](int tile) { return (mfirst ? tile % m_tiles : tile / n_tiles) * kBM; };
  auto tile_n0 = [&](int tile) { return (mfirst ? tile / m_tiles : tile % n_tiles) * BN; };
  // item t: output tile t / ksplit, K piece t % ksplit.  With ksplit > 1 the grid has one CTA per
  // item and the CTAs of a tile form one cluster (piece = rank in the cluster).
  const int items = tiles * ksplit;

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer ----
      uint32_t it = 0;
      bool ok = true;
      const uint64_t pol_first = l2_policy_evict_first();
      // While the previous kernel may still run: bring this CTA's first items' tiles of the
      // operands no earlier kernel writes (indep: bit 0 A, bit 1 B) into L2.
      if (indep) {
        int boxes = 0;
        for (int t = slot; t < items && boxes < 64; t += gridDim.x) {
          const int tile = t / ksplit, piece = t - tile * ksplit;
          const int m0 = tile_m0(tile), n0 = tile_n0(tile);
          const int kb0 = piece * kblocks / ksplit, kb1 = (piece + 1) * kblocks / ksplit;
          const bool second = a_split && m0 >= a_split;
          for (int kb = kb0; kb < kb1; ++kb, ++boxes) {
            if ((indep & 1) && !Epi::kARes) {
              const CUtensorMap* pa = second ? &tmA2 : &tmA;
              const int px = a_kwrap ? (kb * kBK) % a_kwrap : kb * kBK, py = second ? m0 - a_split : m0;
              if (a_stream)  // the same eviction priority as the load that will use it
                tma_prefetch_l2_hint(pa, px, py, pol_first);
              else
                tma_prefetch_l2(pa, px, py);
            }
            if (indep & 2) tma_prefetch_l2(&tmB, kb * kBK, n0);
          }
        }
      }
      pdl_wait();
      stamp(trace, 15, globaltimer_ns());
      if constexpr (Epi::kARes) {  // A once: all of K for the single 128-row band
        mbar_arrive_expect_tx(a_full, (uint32_t)kblocks * kABytes);
        for (int kb = 0; kb < kblocks; ++kb) tma_load_2d(ares + kb * kABytes, &tmA, a_full, kb * kBK, 0);
      }
      for (int t = slot; t < items && ok; t += gridDim.x) {
        const int tile = t / ksplit, piece = t - tile * ksplit;
        const int m0 = tile_m0(tile), n0 = tile_n0(tile);
        const int kb0 = piece * kblocks / ksplit, kb1 = (piece + 1) * kblocks / ksplit;
        // rows at and past a_split come from the second A operand
        const bool second = a_split && m0 >= a_split;
        const CUtensorMap* ta = second ? &tmA2 : &tmA;
        const int ay = second ? m0 - a_split : m0;
        if constexpr (Epi::kSide || Epi::kARes) {
          // streamed operands two tiles ahead into L2, so that the stage and side loads of that tile
          // meet L2 latency rather than HBM latency
          const int ta2i = t + 2 * (int)gridDim.x;
          if (ta2i < items) {
            const int tile2 = ta2i / ksplit;
            const int m2 = tile_m0(tile2), n2 = tile_n0(tile2);
            if constexpr (Epi::kARes)
              for (int kb = 0; kb < kblocks; ++kb) tma_prefetch_l2(&tmB, kb * kBK, n2);
            if constexpr (Epi::kSide)  // normal priority: the lines must survive until the side load
              for (int bx = 0; bx < BN / 64; ++bx) tma_prefetch_l2(&tmS, n2 + bx * 64, m2);
          }
        }
        for (int kb = kb0; kb < kb1; kb += C::kKBS, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_s)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], C::kStage);
          uint8_t* st = smem + s * C::kStage;
          if constexpr (Epi::kARes) {
            for (int j = 0; j < C::kKBS; ++j) tma_load_2d(st + j * C::kBBytes, &tmB, &full[s], (kb + j) * kBK, n0);
          } else {
            // with a_kwrap, A's k coordinate wraps (A repeated along K, e.g. W [W | W]); an A read
            // once per call (a_stream) is evicted first so that it does not displace re-read weights
            const int ax = a_kwrap ? (kb * kBK) % a_kwrap : kb * kBK;
            if (a_stream)
              tma_load_2d_hint(st, ta, &full[s], ax, ay, pol_first);
            else
              tma_load_2d(st, ta, &full[s], ax, ay);
            tma_load_2d(st + kABytes, &tmB, &full[s], kb * kBK, n0);
          }
        }
      }
      stamp(trace, 11, clk());
      if (!ok) *abort_s = 1;
      // no copy may be in flight when the CTA exits: wait for the last S issued stages (and A)
      int never = 0;
      for (uint32_t j = (it > (uint32_t)S ? it - S : 0u); j < it; ++j)
        mbar_wait_bounded(&full[j % S], (j / S) & 1u, kDrainPolls, &never);
      if constexpr (Epi::kARes) mbar_wait_bounded(a_full, 0u, kDrainPolls, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      const uint32_t idesc = idesc_bf16_f32(kBM, BN);
      uint32_t it = 0, acc_it = 0;
      bool ok = true;
      if constexpr (Epi::kARes) ok = mbar_wait_bounded(a_full, 0u, limit, abort_s);
      for (int t = slot; t < items && ok; t += gridDim.x, ++acc_it) {
        const uint32_t a = acc_it & 1u, aph = (acc_it >> 1) & 1u;
        if (!mbar_wait_bounded(&acce[a], aph ^ 1u, limit, abort_s)) { ok = false; break; }
        tmem_fence_after_sync();
        const uint32_t d_tmem = tbase + a * BN;
        const int piece = t % ksplit;
        const int kb0 = piece * kblocks / ksplit, kb1 = (piece + 1) * kblocks / ksplit;
        for (int kb = kb0; kb < kb1; kb += C::kKBS, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait_bounded(&full[s], ph, limit, abort_s)) { ok = false; break; }
          if (it == 0) stamp(trace, 4, clk());
          tmem_fence_after_sync();
          const uint32_t st_addr = smem_u32(smem + s * C::kStage);
#pragma unroll
          for (int j = 0; j < C::kKBS; ++j) {
            const uint32_t a_addr = Epi::kARes ? smem_u32(ares + (kb + j) * kABytes) : st_addr;
            const uint32_t b_addr = Epi::kARes ? st_addr + j * C::kBBytes : st_addr + kABytes;
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_bf16(d_tmem, sw128_desc(a_addr + 32 * k), sw128_desc(b_addr + 32 * k), idesc,
                        ((kb - kb0 + j) | k) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&accf[a]);
        if (acc_it == 0) stamp(trace, 14, clk());
        stamp(trace, 5, clk());
      }
      if (!ok) *abort_s = 1;
      // TMEM may only be freed once every issued MMA has finished
      int never = 0;
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0u, kDrainPolls, &never);
    }
  } else {  // ---- epilogue: warps 2 .. 2 + 4 * kGroups - 1 ----
    pdl_wait();
    const int q = warp & 3;  // TMEM lane quadrant this warp may read
    constexpr int G = EpiWarps<Epi>::kGroups, CW = BN / G;  // columns per epilogue group
    const int cb = ((warp - 2) >> 2) * CW;                   // this warp's first column
    uint32_t acc_it = 0;
    typename Epi::State est;
    epi.init(est);
    int m_last = -1;
    uint8_t* side_base = smem + (size_t)S * C::kStage + 1024;  // after the ring and barriers; 1024-aligned
    const bool side_issuer = (warp == 2 && lane == 0);
    // side tile of this CTA's j-th output tile t into buffer j & 1: BN/64 boxes of 128 x 64.  The
    // buffer was last read by tile j - 2; wait (bounded) until all four warps released it.
    auto side_load = [&](uint32_t j, int t) -> bool {
      if constexpr (Epi::kSide) {
        if (!mbar_wait_bounded(&sidee[j & 1u], ((j >> 1) & 1u) ^ 1u, limit, abort_s)) return false;
        const int m0 = tile_m0(t), n0 = tile_n0(t);
        mbar_arrive_expect_tx(&sidef[j & 1u], (uint32_t)C::kSideBytes);
        // the side operand (base logits) is read once: evict it first so that B stays in L2
        const uint64_t pol = l2_policy_evict_first();
        for (int bx = 0; bx < BN / 64; ++bx)
          tma_load_2d_hint(side_base + (j & 1u) * C::kSideBytes + bx * 16384, &tmS, &sidef[j & 1u], n0 + bx * 64, m0,
                           pol);
      }
      return true;
    };
    uint32_t side_issued = 0;  // loads issued (meaningful in the issuing thread)
    if (Epi::kSide && slot < tiles && side_issuer) {
      if (side_load(0u, slot)) side_issued = 1; else *abort_s = 1;
    }
    for (int t = slot; t < items; t += gridDim.x, ++acc_it) {
      const uint32_t a = acc_it & 1u, aph = (acc_it >> 1) & 1u;
      if (Epi::kSide && t + (int)gridDim.x < tiles && side_issuer) {  // prefetch the next tile's side operand
        if (side_load(acc_it + 1u, t + gridDim.x)) ++side_issued; else *abort_s = 1;
      }
      if (!mbar_wait_warp(&accf[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      if (acc_it == 0 && warp == 2 && lane == 0) stamp(trace, 6, clk());
      if (Epi::kSide && !mbar_wait_warp(&sidef[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      tmem_fence_after_sync();
      const int tile = t / ksplit;
      const int m0 = tile_m0(tile), n0 = tile_n0(tile);
      const int row = q * 32 + lane;
      const int m = m0 + row;
      const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + a * BN;
      const uint8_t* side = Epi::kSide ? side_base + a * C::kSideBytes : nullptr;
      if constexpr (SPLIT) {  // push this piece's partial of every unit to the unit's owner
        constexpr int U = C::kUnits;
        const int piece = (int)blockIdx.x % ksplit;
        const int nmax = (U + ksplit - 1) / ksplit;
        const uint32_t recv = smem_u32(recv_buf);
        if (!waited_first) {
          cluster_wait();  // every CTA of the cluster is running
          waited_first = true;
        }
        // up to 64 columns of TMEM loads in flight per wait: one load latency per batch rather than
        // one per 16-column unit
        constexpr int kCh = BN >= 64 ? 64 : BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += kCh) {
          uint32_t r[kCh];
#pragma unroll
          for (int h = 0; h < kCh / 16; ++h) tmem_ld16(taddr + c0 + 16 * h, &r[16 * h]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kCh / 16; ++h) {
            const int u = ((c0 + 16 * h) >> 4) * kBM + row;
            const int o = unit_owner(u, ksplit, U);
            const int li = u - unit_first(o, ksplit, U);
            const uint32_t base = cluster_map(recv, o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t* q4 = &r[16 * h + 4 * j];
              reg_fence(q4[0]); reg_fence(q4[1]); reg_fence(q4[2]); reg_fence(q4[3]);
              st_cluster_f4(base + slot_offset(piece * nmax + li, li, j), __uint_as_float(q4[0]),
                            __uint_as_float(q4[1]), __uint_as_float(q4[2]), __uint_as_float(q4[3]));
            }
          }
        }
        tmem_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[a]);
        continue;
      }
      m_last = m;
      // Software pipeline over 32-column steps of this warp's CW columns: the next step's TMEM
      // loads are in flight while this step is processed; one wait per step (it covers the loads
      // issued just before).
      constexpr int kStep = CW >= 32 ? 32 : 16, kSteps = CW / kStep;
      uint32_t r[2][kStep];
      tmem_ld16(taddr + cb, &r[0][0]);
      if (kStep == 32) tmem_ld16(taddr + cb + 16, &r[0][16]);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < kSteps; ++k) {
        uint32_t(&cur)[kStep] = r[k & 1];
#pragma unroll
        for (int j = 0; j < kStep; ++j) reg_fence(cur[j]);
        if (k + 1 < kSteps) {
          tmem_ld16(taddr + cb + (k + 1) * kStep, &r[(k + 1) & 1][0]);
          if (kStep == 32) tmem_ld16(taddr + cb + (k + 1) * kStep + 16, &r[(k + 1) & 1][16]);
        }
#pragma unroll
        for (int h = 0; h < kStep / 16; ++h) {
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(cur[16 * h + j]);
          const int c = cb + k * kStep + 16 * h;
          epi.apply(est, m, n0 + c, v, N, side, row, c);
        }
        if (k + 1 < kSteps) tmem_wait_ld();
      }
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acce[a]);
        if (Epi::kSide) mbar_arrive(&sidee[a]);
      }
      if (acc_it == 0 && warp == 2 && lane == 0) stamp(trace, 13, clk());
    }
    if (m_last >= 0) epi.finish(est, m_last);
    if (warp == 2 && lane == 0) {
      stamp(trace, 7, clk());
      stamp(trace, 12, acc_it);
    }
    // no side copy may be in flight at exit: wait for the last ones issued
    if (Epi::kSide && side_issuer) {
      int never = 0;
      for (uint32_t k = (side_issued > 2u ? side_issued - 2u : 0u); k < side_issued; ++k)
        mbar_wait_bounded(&sidef[k & 1u], (k >> 1) & 1u, kDrainPolls, &never);
    }
  }

  if constexpr (SPLIT) {
    __syncwarp();
    // threads that pushed nothing pass the first cluster barrier here; then the second one: every
    // piece of every unit has landed in its owner's receive buffer
    if (!waited_first) cluster_wait();
    cluster_arrive_release();
    cluster_wait();
    if (threadIdx.x == 64) stamp(trace, 8, clk());
    if (warp >= 2) {
      constexpr int U = C::kUnits;
      const int tile = blockIdx.x / ksplit, piece = blockIdx.x - tile * ksplit;
      const int m0 = tile_m0(tile), n0 = tile_n0(tile);
      const int nmax = (U + ksplit - 1) / ksplit;
      const int u0 = unit_first(piece, ksplit, U), u1 = unit_first(piece + 1, ksplit, U);
      const uint8_t* recv = recv_buf;
      typename Epi::State est;
      epi.init(est);
      for (int li = (int)threadIdx.x - 64; li < u1 - u0; li += 128 * EpiWarps<Epi>::kGroups) {
        const int u = u0 + li, g = u / kBM, row = u - g * kBM;
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
#pragma unroll 1
        for (int pc = 0; pc < ksplit; ++pc) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 x = *reinterpret_cast<const float4*>(recv + slot_offset(pc * nmax + li, li, j));
            v[4 * j] += x.x; v[4 * j + 1] += x.y; v[4 * j + 2] += x.z; v[4 * j + 3] += x.w;
          }
        }
        epi.apply(est, m0 + row, n0 + g * 16, v, N, nullptr, row, g * 16);
      }
      if (threadIdx.x == 64) stamp(trace, 9, clk());
    }
  }

  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (warp == 1) tmem_dealloc(tbase, C::kTmemCols);
  if (threadIdx.x == 0 && *abort_s && status) set_status(status, DOMINO_STATUS_DEVICE_TIMEOUT);
  if (threadIdx.x == 0) {
    stamp(trace, 10, clk());
    stamp(trace, 1, globaltimer_ns());
  }
}

// ---- tensor maps ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 matrix [rows x cols] (row-major, row stride ld elements) seen as tiles of box_rows x 64.
bool tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, uint64_t ld = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {(ld ? ld : cols) * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// The kernel's dynamic shared memory opt-in, set once per device.
template <int BN, class Epi, bool SPLIT>
cudaError_t set_smem_once(size_t smem) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN, Epi, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int BN, class Epi>
cudaError_t launch_gemm(const void* A, const void* Bm, int M, int N, int K, const Epi& epi, int32_t* status,
                        uint64_t limit, cudaStream_t st, uint64_t lda = 0, uint64_t ldb = 0, int a_kwrap = 0,
                        const void* side = nullptr, uint64_t lds = 0, const void* A2 = nullptr, int a_split = 0,
                        uint64_t lda2 = 0, int ksplit = 1, int a_stream = 0, int indep = 0,
                        uint32_t* claim = nullptr, uint32_t epoch = 0, int mfirst = 0) {
  CUtensorMap ta, ta2, tb, ts;
  const uint64_t ka = a_kwrap ? (uint64_t)a_kwrap : (uint64_t)K;
  const uint64_t rows_a = a_split ? (uint64_t)a_split : (uint64_t)M;
  if (!tmap_bf16(&ta, A, rows_a, ka, kBM, lda) || !tmap_bf16(&tb, Bm, (uint64_t)N, (uint64_t)K, BN, ldb))
    return cudaErrorInvalidValue;
  if (a_split) {  // rows [a_split, M) of A come from A2
    if (!A2 || !tmap_bf16(&ta2, A2, (uint64_t)(M - a_split), ka, kBM, lda2)) return cudaErrorInvalidValue;
  } else {
    ta2 = ta;
  }
  if (Epi::kSide) {  // side operand: M rows x N columns, row stride lds
    if (!side || !tmap_bf16(&ts, side, (uint64_t)M, (uint64_t)N, kBM, lds)) return cudaErrorInvalidValue;
  } else {
    ts = ta;
  }
  if (Epi::kARes && (M > kBM || K > 4 * kBK || K % (2 * kBK) != 0)) return cudaErrorInvalidValue;
  const long long tiles = (long long)((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
  const long long grid_ctas = ksplit > 1 ? tiles * ksplit : std::min<long long>(tiles, (long long)sm_count());
  unsigned long long* trace = nullptr;
  int ntrace = 0;
  debug_trace(&trace, &ntrace);
  if (trace && (long long)ntrace < grid_ctas * kTraceSlots) trace = nullptr;
  if constexpr (!Epi::kSide && !Epi::kARes && !WarpCoop<Epi>::value) {
    if (ksplit > 1) {  // one cluster of ksplit CTAs per output tile
      if (ksplit > 8 || K / kBK < ksplit || tiles * ksplit > (1LL << 30)) return cudaErrorInvalidValue;
      auto kern = k_gemm_tc<BN, Epi, true>;
      const size_t smem = Cfg<BN, false, false, true>::kSmem;
      cudaError_t e = set_smem_once<BN, Epi, true>(smem);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * ksplit));
    cfg.blockDim = dim3(EpiWarps<Epi>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)ksplit;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return note_launch(cudaLaunchKernelEx(&cfg, kern, ta, ta2, tb, ts, M, N, K, epi, status,
                                          (unsigned long long)limit, a_kwrap, a_split, ksplit, a_stream, indep,
                                          (uint32_t*)nullptr, 0u, trace, 0));
    }
  }
  if (ksplit > 1) return cudaErrorInvalidValue;
  auto kern = k_gemm_tc<BN, Epi, false>;
  const size_t smem = Cfg<BN, Epi::kSide, Epi::kARes, false, StaticSmemOf<Epi>::value>::kSmem;
  cudaError_t e = set_smem_once<BN, Epi, false>(smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)grid_ctas;
  return note_launch(launch_pdl(kern, dim3(grid), dim3(EpiWarps<Epi>::kThreads), smem, st, ta, ta2, tb, ts, M, N, K, epi, status,
                                (unsigned long long)limit, a_kwrap, a_split, 1, a_stream, indep,
                                grid == sm_count() ? claim : nullptr, epoch, trace, mfirst));
}

// A is a weight operand (no earlier kernel writes it): its first tiles are prefetched to L2.
template <class Epi>
cudaError_t launch_gemm_bn(const void* A, const void* Bm, int M, int N, int K, const Epi& epi, int32_t* status,
                           uint64_t limit, cudaStream_t st) {
#define DOMINO_GEMM_BN(W) launch_gemm<W>(A, Bm, M, N, K, epi, status, limit, st, 0, 0, 0, nullptr, 0, nullptr, 0, 0, 1, 0, 1)
  if (N <= 16) return DOMINO_GEMM_BN(16);
  if (N <= 32) return DOMINO_GEMM_BN(32);
  if (N <= 64) return DOMINO_GEMM_BN(64);
  if (N <= 128) return DOMINO_GEMM_BN(128);
  return DOMINO_GEMM_BN(256);
#undef DOMINO_GEMM_BN
}

// Clusters of `ks` CTAs of k_gemm_tc<BN, Epi> that fit on the GPU at once (cached per device).
template <int BN, class Epi>
int max_clusters(int ks) {
  static std::mutex mu;
  static int cache[64][9];
  static bool init = false;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || ks < 2 || ks > 8) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    for (auto& row : cache)
      for (int& v : row) v = -1;
    init = true;
  }
  if (cache[dev][ks] < 0) {
    auto kern = k_gemm_tc<BN, Epi, true>;
    const size_t smem = Cfg<BN, false, false, true>::kSmem;
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ks * 16));
    cfg.blockDim = dim3(EpiWarps<Epi>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)ks;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (set_smem_once<BN, Epi, true>(smem) != cudaSuccess || cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess)
      n = 0;
    cudaGetLastError();  // a refused query leaves no sticky error behind
    cache[dev][ks] = n;
  }
  return cache[dev][ks];
}

struct SkinnyPlan {
  int bn, ks;
};

// Tile width and K split for a skinny product (N = a batch of rows).  The critical path of a CTA
// is the bytes it streams: (128 + BN) x 2 x K / ks operand bytes per item, times the items it
// runs, plus parking and reducing a 128 x BN fp32 tile when the tile is split.  A split is only
// taken when all its clusters fit on the GPU at once.
template <class Epi>
SkinnyPlan plan_skinny(int M, int N, int K) {
  const int sms = sm_count();
  const int kblocks = K / kBK;
  const long long m_tiles = (M + kBM - 1) / kBM;
  SkinnyPlan best{16, 1};
  if (sms <= 0) return best;
  double best_cost = 1e300;
  const int bns[4] = {16, 32, 64, 128};
  for (int bn : bns) {
    if (bn > 16 && (bn / 2) >= N) break;  // wider tiles only add padding
    const long long tiles = m_tiles * ((N + bn - 1) / bn);
    for (int ks = 1; ks <= 8; ++ks) {
      double cost;
      if (ks == 1) {
        const long long waves = (tiles + sms - 1) / sms;
        cost = (double)waves * (kBM + bn) * 2.0 * K;
      } else {
        if (kblocks < 2 * ks || tiles * ks > sms) break;
        const int fit = bn == 16 ? max_clusters<16, Epi>(ks)
                                 : bn == 32 ? max_clusters<32, Epi>(ks)
                                            : bn == 64 ? max_clusters<64, Epi>(ks) : max_clusters<128, Epi>(ks);
        if (tiles > fit) continue;
        cost = (double)(kBM + bn) * 2.0 * ((kblocks + ks - 1) / ks) * kBK + 2.0 * kBM * bn * 4.0;
      }
      if (cost < best_cost * 0.98) {
        best_cost = cost;
        best = SkinnyPlan{bn, ks};
      }
    }
  }
  return best;
}

// Skinny products (N = a batch of rows): tiles as wide as N up to 128 so that A is read once per
// 128 columns, K split over a cluster when the tiles alone do not occupy the SMs.
template <class Epi>
cudaError_t launch_gemm_skinny(const void* A, const void* Bm, int M, int N, int K, const Epi& epi, int32_t* status,
                               uint64_t limit, cudaStream_t st, uint64_t lda, int a_kwrap, const void* A2 = nullptr,
                               int a_split = 0, uint64_t lda2 = 0, int a_stream = 0, int indep = 1) {
  const SkinnyPlan p = plan_skinny<Epi>(M, N, K);
  switch (p.bn) {
    case 16:
      return launch_gemm<16>(A, Bm, M, N, K, epi, status, limit, st, lda, 0, a_kwrap, nullptr, 0, A2, a_split, lda2,
                             p.ks, a_stream, indep);
    case 32:
      return launch_gemm<32>(A, Bm, M, N, K, epi, status, limit, st, lda, 0, a_kwrap, nullptr, 0, A2, a_split, lda2,
                             p.ks, a_stream, indep);
    case 64:
      return launch_gemm<64>(A, Bm, M, N, K, epi, status, limit, st, lda, 0, a_kwrap, nullptr, 0, A2, a_split, lda2,
                             p.ks, a_stream, indep);
    default:
      return launch_gemm<128>(A, Bm, M, N, K, epi, status, limit, st, lda, 0, a_kwrap, nullptr, 0, A2, a_split,
                              lda2, p.ks, a_stream, indep);
  }
}

}  // namespace

bool tmap_bf16_tiles(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, uint64_t ld) {
  return tmap_bf16(tm, base, rows, cols, box_rows, ld);
}

bool tmap_f32_3d(CUtensorMap* tm, void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || n0 % 4 != 0) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {n0 * 4, n0 * n1 * 4};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool tmap_bf16_3d(CUtensorMap* tm, const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || n0 % 8 != 0) return false;
  cuuint64_t dims[3] = {n0, n1, n2};
  cuuint64_t strides[2] = {n0 * 2, n0 * n1 * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBK, 1, box2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tmap_bf16_chunks(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      uint32_t box_chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || cols % kBK != 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kBK, rows, cols / kBK};
  cuuint64_t strides[2] = {cols * 2, (cuuint64_t)kBK * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBK, box_rows, box_chunks};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

cudaError_t gemm_tc_debug(const bf16* A, const bf16* Bm, int M, int N, int K, int a_kwrap, float* out, long long ldo,
                          int trans, int bn, int ks, int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiStore e{out, M, ldo, trans};
  if (bn == 0 && ks == 0) return launch_gemm_skinny(A, Bm, M, N, K, e, status, limit, st, 0, a_kwrap);
  if (ks < 1 || ks > 8) return cudaErrorInvalidValue;
  switch (bn) {
    case 16: return launch_gemm<16>(A, Bm, M, N, K, e, status, limit, st, 0, 0, a_kwrap, nullptr, 0, nullptr, 0, 0, ks);
    case 32: return launch_gemm<32>(A, Bm, M, N, K, e, status, limit, st, 0, 0, a_kwrap, nullptr, 0, nullptr, 0, 0, ks);
    case 64: return launch_gemm<64>(A, Bm, M, N, K, e, status, limit, st, 0, 0, a_kwrap, nullptr, 0, nullptr, 0, 0, ks);
    case 128:
      return launch_gemm<128>(A, Bm, M, N, K, e, status, limit, st, 0, 0, a_kwrap, nullptr, 0, nullptr, 0, 0, ks);
    default: return cudaErrorInvalidValue;
  }
}

void gemm_tc_skinny_plan(int M, int N, int K, int* bn, int* ks) {
  const SkinnyPlan p = plan_skinny<EpiStore>(M, N, K);
  *bn = p.bn;
  *ks = p.ks;
}

bool gemm_tc_supported(int M, int N, int K, const void* A, const void* Bm) {
  return M >= 1 && N >= 1 && K >= kBK && K % kBK == 0 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(Bm) & 15u) == 0 && encode_fn() != nullptr;
}

cudaError_t gemm_tc_store_f32(const bf16* A, const bf16* Bm, int M, int N, int K, float* out, long long ldo,
                              int32_t* status, uint64_t limit, cudaStream_t st, int trans) {
  EpiStore e{out, M, ldo, trans};
  return launch_gemm_bn(A, Bm, M, N, K, e, status, limit, st);
}

cudaError_t gemm_tc_argmax(const bf16* U, const bf16* W2, int M, int V, int r, const bf16* Lb, long long ldl,
                           uint64_t* keys, float* out, long long ldo, int32_t* status, uint64_t limit,
                           cudaStream_t st, uint32_t* claim, uint32_t epoch) {
  if (claim) {
    cudaError_t e = ensure_sm_rank(st);
    if (e != cudaSuccess) return e;
  }
  if (r % 128 == 0 && r <= 256) {  // the activation band stays in shared memory for every vocabulary tile
    EpiArgmaxT<true> e{keys, M, out, ldo};
    return launch_gemm<128>(U, W2, M, V, r, e, status, limit, st, 0, 0, 0, Lb, (uint64_t)ldl, nullptr, 0, 0, 1, 0, 2,
                            claim, epoch);
  }
  EpiArgmaxT<false> e{keys, M, out, ldo};
  return launch_gemm<128>(U, W2, M, V, r, e, status, limit, st, 0, 0, 0, Lb, (uint64_t)ldl, nullptr, 0, 0, 1, 0, 2,
                          claim, epoch);
}

cudaError_t gemm_tc_gru_u(const bf16* W_hh, const bf16* W1s, long long ldw, const bf16* S_hl, int Hs, int r, int N,
                          float* Gh, const float* P, long long ldp, bf16* u16, int32_t* status, uint64_t limit,
                          cudaStream_t st) {
  EpiGruU e{Gh, 3 * Hs, 3 * Hs, P, ldp, u16, r};
  return launch_gemm_skinny(W_hh, S_hl, 3 * Hs + r, N, 2 * Hs, e, status, limit, st, 0, Hs, W1s, 3 * Hs,
                            (uint64_t)ldw);
}

cudaError_t gemm_tc_silu_u(const bf16* W1s, long long ldw, const bf16* S_hl, int r, int N, int Hs, const float* P,
                           long long ldp, bf16* u16, float* uf, int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiSiluU e{P, ldp, u16, uf, r};
  return launch_gemm_skinny(W1s, S_hl, r, N, 2 * Hs, e, status, limit, st, (uint64_t)ldw, Hs);
}

cudaError_t gemm_tc_store_f32_t(const bf16* A, const bf16* Bm, int M, int N, int K, int a_kwrap, float* out,
                                long long ldo, int32_t* status, uint64_t limit, cudaStream_t st, int a_stream,
                                long long lda) {
  EpiStore e{out, M, ldo, 1};
  return launch_gemm_skinny(A, Bm, M, N, K, e, status, limit, st, (uint64_t)lda, a_kwrap, nullptr, 0, 0, a_stream);
}

template <typename OutT>
cudaError_t logits_t(const bf16* W2, const bf16* U, int V, int N, int r, const bf16* Lb, OutT* logits, int32_t* status,
                     uint64_t limit, cudaStream_t st, uint32_t* claim, uint32_t epoch) {
  if (N >= 64) {  // enough rows for the row-major orientation: vector loads and stores in the epilogue
    // The row bands of one vocabulary tile run side by side on CTAs of consecutive work slots --
    // neighbouring SMs when the slots are taken by SM (claim) -- so each W2 tile is read from HBM once.
    if (claim) {
      cudaError_t e = ensure_sm_rank(st);
      if (e != cudaSuccess) return e;
    }
    EpiLogitsRowT<OutT> e{Lb, logits, N, (long long)V};
    return launch_gemm<128>(U, W2, N, V, r, e, status, limit, st, 0, 0, 0, Lb, (uint64_t)V, nullptr, 0, 0, 1, 0, 2,
                            claim, epoch, 1);
  }
  EpiLogitsT<OutT> e{Lb, logits, V};
  return launch_gemm_bn(W2, U, V, N, r, e, status, limit, st);
}

cudaError_t gemm_tc_logits(const bf16* W2, const bf16* U, int V, int N, int r, const bf16* Lb, void* logits,
                           int out_bf16, int32_t* status, uint64_t limit, cudaStream_t st, uint32_t* claim,
                           uint32_t epoch) {
  return out_bf16 ? logits_t(W2, U, V, N, r, Lb, static_cast<bf16*>(logits), status, limit, st, claim, epoch)
                  : logits_t(W2, U, V, N, r, Lb, static_cast<float*>(logits), status, limit, st, claim, epoch);
}

}  // namespace domino
