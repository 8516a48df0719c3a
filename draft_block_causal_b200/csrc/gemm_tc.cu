// gemm_tc.cu -- persistent tcgen05 GEMM with fused epilogues (bf16 x bf16 -> fp32 in TMEM).
//
//   D[m][n] = sum_k A[m][k] * B[n][k]      A: [M x K], B: [N x K], both bf16, K-major
//
// One CTA per SM walks output tiles of 128 x BN.  Warp roles:
//   warp 0, one thread : TMA producer -- 128x64 A tile + BNx64 B tile per k-block into a ring of
//                        S shared-memory stages (128-byte swizzle), signalled on full[s]
//   warp 1, one thread : MMA issuer   -- four tcgen05.mma (K = 16) per k-block into one of two TMEM
//                        accumulators; tcgen05.commit frees the stage (empty[s]) and, after the
//                        last k-block, publishes the accumulator (acc_full[a])
//   warps 2..5         : epilogue     -- tcgen05.ld of the accumulator (warp w reads TMEM lanes
//                        32*(w%4).., i.e. output rows), then the epilogue functor; acc_empty[a]
// Every mbarrier wait is bounded.  A role that gives up raises a CTA-wide abort flag; the others
// stop at their next wait, the producer waits for its copies still in flight, TMEM is freed and
// DOMINO_STATUS_DEVICE_TIMEOUT is reported.
//
// Uses in this library:
//   - the W2 product of teacher forcing: A = W2 [V x r], B = u [B*L x r] (bf16), epilogue adds
//     L_base and writes fp32 logits -- the logit-space residual of the Domino head equation;
//   - the input projection of the embedding table: A = embed [V x d], B = W_ih [3Hs x d],
//     epilogue stores fp32 [V x 3Hs] (the GRU's input half for every token at once).
#include "common.cuh"
#include "gemm_tc.h"
#include "umma.cuh"

#include <mutex>

namespace domino {

namespace {

constexpr int kBM = 128, kBK = 64;
constexpr int kGemmThreads = 192;
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
struct EpiStore {  // out[m * ldo + n] = D
  static constexpr bool kSide = false;
  using State = NoState;
  float* out;
  int M;
  long long ldo;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m >= M) return;
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
struct EpiLogits {  // logits[n][m] = D + Lb[n][m]   (m = vocabulary row, n = (row, position))
  static constexpr bool kSide = false;
  using State = NoState;
  const bf16* Lb;
  float* logits;
  int M;
  __device__ __forceinline__ void init(State&) const {}
  __device__ __forceinline__ void finish(State&, int) const {}
  __device__ __forceinline__ void apply(State&, int m, int n0, const float (&v)[16], int N, const uint8_t*, int,
                                        int) const {
    if (m >= M) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int n = n0 + j;
      if (n < N) {
        const size_t at = (size_t)n * M + m;
        logits[at] = v[j] + __bfloat162float(Lb[at]);
      }
    }
  }
};

// Greedy step, batch-major: m = batch row b (< M), n = vocabulary row v.
//   z = D + Lb[b][v] (Lb row stride ldl), running argmax over the thread's columns (ascending,
//   strict > keeps the lowest index), finish: keys[b] = max(keys[b], key(best)).  When out is
//   set, z is also stored to out[b * ldo + v].
struct EpiArgmax {
  static constexpr bool kSide = true;  // the L_base tile [128 rows b x BN columns v]
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
    for (int j = 0; j < 16; ++j) {
      z[j] = v[j] + l[j];
      if (n0 + j < N && z[j] > s.best) { s.best = z[j]; s.idx = n0 + j; }
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

// u[n][m] = SiLU(P[n * ldp + m] + D) as bf16 (and fp32 when uf is set): m = rank index (M = r), n = row.
struct EpiSiluU {
  static constexpr bool kSide = false;
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
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int n = n0 + j;
      if (n < N) {
        const float u = siluf_(P[(size_t)n * ldp + m] + v[j]);
        u16[(size_t)n * M + m] = __float2bfloat16_rn(u);
        if (uf) uf[(size_t)n * M + m] = u;
      }
    }
  }
};

// Shared memory (from a 1024-aligned base): the stage ring, 1024 bytes for the mbarriers and the
// TMEM slot, then (side epilogues) two side tiles; plus 1024 bytes of slack for the alignment.
template <int BN, bool SIDE> struct Cfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStage = kABytes + kBBytes;
  static constexpr size_t kSideBytes = SIDE ? (size_t)kBM * BN * 2 : 0;  // one side tile
  static constexpr size_t kBudget = 232448 - 2048 - 2 * kSideBytes;     // 227 KB per CTA
  static constexpr int kStagesFit = (int)(kBudget / kStage);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kTmemCols = (2 * BN) <= 32 ? 32 : ((2 * BN) <= 64 ? 64 : ((2 * BN) <= 128 ? 128 : ((2 * BN) <= 256 ? 256 : 512)));
  static constexpr size_t kSmem = (size_t)kStages * kStage + 2048 + 2 * kSideBytes;
  static_assert(kStages >= 2, "shared memory too small for the pipeline");
};

template <int BN, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmS, int M, int N, int K, Epi epi, int32_t* status,
              unsigned long long limit, int a_kwrap) {
  using C = Cfg<BN, Epi::kSide>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStage);
  uint64_t* empty = full + S;
  uint64_t* accf = empty + S;
  uint64_t* acce = accf + 2;
  uint64_t* mma_done = acce + 2;
  uint64_t* sidef = mma_done + 1;  // [2] side tile landed
  uint64_t* sidee = sidef + 2;     // [2] side buffer read by all four epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sidee + 2);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 4); }
    mbar_init(mma_done, 1);
    mbar_init(&sidef[0], 1);
    mbar_init(&sidef[1], 1);
    mbar_init(&sidee[0], 4);
    mbar_init(&sidee[1], 4);
    *abort_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
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

  const int m_tiles = (M + kBM - 1) / kBM, n_tiles = (N + BN - 1) / BN, kblocks = K / kBK;
  const int tiles = m_tiles * n_tiles;

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer ----
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_s)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], C::kStage);
          uint8_t* st = smem + s * C::kStage;
          // with a_kwrap, A's k coordinate wraps (A repeated along K, e.g. W [W | W])
          tma_load_2d(st, &tmA, &full[s], a_kwrap ? (kb * kBK) % a_kwrap : kb * kBK, m0);
          tma_load_2d(st + kABytes, &tmB, &full[s], kb * kBK, n0);
        }
      }
      if (!ok) *abort_s = 1;
      // no copy may be in flight when the CTA exits: wait for the last S issued stages
      int never = 0;
      for (uint32_t j = (it > (uint32_t)S ? it - S : 0u); j < it; ++j)
        mbar_wait_bounded(&full[j % S], (j / S) & 1u, limit, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      const uint32_t idesc = idesc_bf16_f32(kBM, BN);
      uint32_t it = 0, acc_it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++acc_it) {
        const uint32_t a = acc_it & 1u, aph = (acc_it >> 1) & 1u;
        if (!mbar_wait_bounded(&acce[a], aph ^ 1u, limit, abort_s)) { ok = false; break; }
        tmem_fence_after_sync();
        const uint32_t d_tmem = tbase + a * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait_bounded(&full[s], ph, limit, abort_s)) { ok = false; break; }
          tmem_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + s * C::kStage), b_addr = a_addr + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, sw128_desc(a_addr + 32 * k), sw128_desc(b_addr + 32 * k), idesc, (kb | k) != 0);
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&accf[a]);
      }
      if (!ok) *abort_s = 1;
      // TMEM may only be freed once every issued MMA has finished
      int never = 0;
      umma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0u, limit, &never);
    }
  } else {  // ---- epilogue: warps 2..5 ----
    const int q = warp & 3;
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
        const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * BN;
        mbar_arrive_expect_tx(&sidef[j & 1u], (uint32_t)C::kSideBytes);
        for (int bx = 0; bx < BN / 64; ++bx)
          tma_load_2d(side_base + (j & 1u) * C::kSideBytes + bx * 16384, &tmS, &sidef[j & 1u], n0 + bx * 64, m0);
      }
      return true;
    };
    uint32_t side_issued = 0;  // loads issued (meaningful in the issuing thread)
    if (Epi::kSide && (int)blockIdx.x < tiles && side_issuer) {
      if (side_load(0u, blockIdx.x)) side_issued = 1; else *abort_s = 1;
    }
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++acc_it) {
      const uint32_t a = acc_it & 1u, aph = (acc_it >> 1) & 1u;
      if (Epi::kSide && t + (int)gridDim.x < tiles && side_issuer) {  // prefetch the next tile's side operand
        if (side_load(acc_it + 1u, t + gridDim.x)) ++side_issued; else *abort_s = 1;
      }
      if (!mbar_wait_warp(&accf[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      if (Epi::kSide && !mbar_wait_warp(&sidef[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      tmem_fence_after_sync();
      const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * BN;
      const int row = q * 32 + lane;
      const int m = m0 + row;
      m_last = m;
      const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + a * BN;
      const uint8_t* side = Epi::kSide ? side_base + a * C::kSideBytes : nullptr;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c0, r);
        tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) { reg_fence(r[j]); v[j] = __uint_as_float(r[j]); }
        epi.apply(est, m, n0 + c0, v, N, side, row, c0);
      }
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&acce[a]);
        if (Epi::kSide) mbar_arrive(&sidee[a]);
      }
    }
    if (m_last >= 0) epi.finish(est, m_last);
    // no side copy may be in flight at exit: wait for the last ones issued
    if (Epi::kSide && side_issuer) {
      int never = 0;
      for (uint32_t k = (side_issued > 2u ? side_issued - 2u : 0u); k < side_issued; ++k)
        mbar_wait_bounded(&sidef[k & 1u], (k >> 1) & 1u, limit, &never);
    }
  }

  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (warp == 1) tmem_dealloc(tbase, C::kTmemCols);
  if (threadIdx.x == 0 && *abort_s && status) set_status(status, DOMINO_STATUS_DEVICE_TIMEOUT);
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

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <int BN, class Epi>
cudaError_t launch_gemm(const void* A, const void* Bm, int M, int N, int K, const Epi& epi, int32_t* status,
                        uint64_t limit, cudaStream_t st, uint64_t lda = 0, uint64_t ldb = 0, int a_kwrap = 0,
                        const void* side = nullptr, uint64_t lds = 0) {
  CUtensorMap ta, tb, ts;
  const uint64_t ka = a_kwrap ? (uint64_t)a_kwrap : (uint64_t)K;
  if (!tmap_bf16(&ta, A, (uint64_t)M, ka, kBM, lda) || !tmap_bf16(&tb, Bm, (uint64_t)N, (uint64_t)K, BN, ldb))
    return cudaErrorInvalidValue;
  if (Epi::kSide) {  // side operand: M rows x N columns, row stride lds
    if (!side || !tmap_bf16(&ts, side, (uint64_t)M, (uint64_t)N, kBM, lds)) return cudaErrorInvalidValue;
  } else {
    ts = ta;
  }
  auto kern = k_gemm_tc<BN, Epi>;
  const size_t smem = Cfg<BN, Epi::kSide>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<long long>(tiles, (long long)sm_count());
  kern<<<grid, kGemmThreads, smem, st>>>(ta, tb, ts, M, N, K, epi, status, (unsigned long long)limit, a_kwrap);
  return note_launch(cudaGetLastError());
}

template <class Epi>
cudaError_t launch_gemm_bn(const void* A, const void* Bm, int M, int N, int K, const Epi& epi, int32_t* status,
                           uint64_t limit, cudaStream_t st) {
  if (N <= 16) return launch_gemm<16>(A, Bm, M, N, K, epi, status, limit, st);
  if (N <= 32) return launch_gemm<32>(A, Bm, M, N, K, epi, status, limit, st);
  if (N <= 64) return launch_gemm<64>(A, Bm, M, N, K, epi, status, limit, st);
  if (N <= 128) return launch_gemm<128>(A, Bm, M, N, K, epi, status, limit, st);
  return launch_gemm<256>(A, Bm, M, N, K, epi, status, limit, st);
}

}  // namespace

bool gemm_tc_supported(int M, int N, int K, const void* A, const void* Bm) {
  return M >= 1 && N >= 1 && K >= kBK && K % kBK == 0 && (reinterpret_cast<uintptr_t>(A) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(Bm) & 15u) == 0 && encode_fn() != nullptr;
}

cudaError_t gemm_tc_store_f32(const bf16* A, const bf16* Bm, int M, int N, int K, float* out, long long ldo,
                              int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiStore e{out, M, ldo};
  return launch_gemm_bn(A, Bm, M, N, K, e, status, limit, st);
}

cudaError_t gemm_tc_argmax(const bf16* U, const bf16* W2, int M, int V, int r, const bf16* Lb, long long ldl,
                           uint64_t* keys, float* out, long long ldo, int32_t* status, uint64_t limit,
                           cudaStream_t st) {
  EpiArgmax e{keys, M, out, ldo};
  return launch_gemm<128>(U, W2, M, V, r, e, status, limit, st, 0, 0, 0, Lb, (uint64_t)ldl);
}

cudaError_t gemm_tc_silu_u(const bf16* W1s, long long ldw, const bf16* S_hl, int r, int N, int Hs, const float* P,
                           long long ldp, bf16* u16, float* uf, int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiSiluU e{P, ldp, u16, uf, r};
  if (N <= 16) return launch_gemm<16>(W1s, S_hl, r, N, 2 * Hs, e, status, limit, st, (uint64_t)ldw, 0, Hs);
  return launch_gemm<32>(W1s, S_hl, r, N, 2 * Hs, e, status, limit, st, (uint64_t)ldw, 0, Hs);
}

cudaError_t gemm_tc_store_f32_bn64(const bf16* A, const bf16* Bm, int M, int N, int K, long long ldb, float* out,
                                  long long ldo, int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiStore e{out, M, ldo};
  return launch_gemm<64>(A, Bm, M, N, K, e, status, limit, st, 0, (uint64_t)ldb);
}

cudaError_t gemm_tc_store_f32_bn32(const bf16* A, const bf16* Bm, int M, int N, int K, int a_kwrap, float* out,
                                  long long ldo, int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiStore e{out, M, ldo};
  return launch_gemm<32>(A, Bm, M, N, K, e, status, limit, st, 0, 0, a_kwrap);
}

cudaError_t gemm_tc_logits(const bf16* W2, const bf16* U, int V, int N, int r, const bf16* Lb, float* logits,
                           int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiLogits e{Lb, logits, V};
  return launch_gemm_bn(W2, U, V, N, r, e, status, limit, st);
}

}  // namespace domino
