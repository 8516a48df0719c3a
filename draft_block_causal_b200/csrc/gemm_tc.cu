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

// ---- epilogues: apply(m, n0, v[16], N) for 16 consecutive output columns of row m ----
struct EpiStore {  // out[m * ldo + n] = D
  float* out;
  int M;
  long long ldo;
  __device__ __forceinline__ void apply(int m, int n0, const float (&v)[16], int N) const {
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
  const bf16* Lb;
  float* logits;
  int M;
  __device__ __forceinline__ void apply(int m, int n0, const float (&v)[16], int N) const {
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

template <int BN> struct Cfg {
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStage = kABytes + kBBytes;
  static constexpr int kStages = (196608 / kStage) > 8 ? 8 : (196608 / kStage);
  static constexpr int kTmemCols = (2 * BN) <= 32 ? 32 : ((2 * BN) <= 64 ? 64 : ((2 * BN) <= 128 ? 128 : ((2 * BN) <= 256 ? 256 : 512)));
  static constexpr size_t kSmem = (size_t)kStages * kStage + 1024 + 256;
};

template <int BN, class Epi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
              Epi epi, int32_t* status, unsigned long long limit) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStage);
  uint64_t* empty = full + S;
  uint64_t* accf = empty + S;
  uint64_t* acce = accf + 2;
  uint64_t* mma_done = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], 4); }
    mbar_init(mma_done, 1);
    *abort_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
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
          tma_load_2d(st, &tmA, &full[s], kb * kBK, m0);
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
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++acc_it) {
      const uint32_t a = acc_it & 1u, aph = (acc_it >> 1) & 1u;
      if (!mbar_wait_bounded(&accf[a], aph, limit, abort_s)) { *abort_s = 1; break; }
      tmem_fence_after_sync();
      const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * BN;
      const int m = m0 + q * 32 + lane;
      const uint32_t taddr = tbase + ((uint32_t)(q * 32) << 16) + a * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c0, r);
        tmem_wait_ld();
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) { reg_fence(r[j]); v[j] = __uint_as_float(r[j]); }
        epi.apply(m, n0 + c0, v, N);
      }
      tmem_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);
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

// bf16 matrix [rows x cols] (row-major, cols contiguous) seen as tiles of box_rows x 64.
bool tmap_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
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
                        uint64_t limit, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (!tmap_bf16(&ta, A, (uint64_t)M, (uint64_t)K, kBM) || !tmap_bf16(&tb, Bm, (uint64_t)N, (uint64_t)K, BN))
    return cudaErrorInvalidValue;
  auto kern = k_gemm_tc<BN, Epi>;
  const size_t smem = Cfg<BN>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<long long>(tiles, (long long)sm_count());
  kern<<<grid, kGemmThreads, smem, st>>>(ta, tb, M, N, K, epi, status, (unsigned long long)limit);
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

cudaError_t gemm_tc_logits(const bf16* W2, const bf16* U, int V, int N, int r, const bf16* Lb, float* logits,
                           int32_t* status, uint64_t limit, cudaStream_t st) {
  EpiLogits e{Lb, logits, V};
  return launch_gemm_bn(W2, U, V, N, r, e, status, limit, st);
}

}  // namespace domino
