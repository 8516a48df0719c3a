// gemm_tc.h -- host entry points of the tcgen05 GEMM (gemm_tc.cu).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "domino.h"
#include "internal.h"

namespace domino {

// A bf16 matrix [rows x cols] (row stride ld elements; 0 = cols) as a TMA tensor map of
// box_rows x 64 tiles with 128-byte swizzling -- the shared-memory layout the tcgen05 descriptors
// of this library expect.  False when the driver's encoder is missing or refuses the map.
bool tmap_bf16_tiles(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                     uint64_t ld = 0);
// bf16 tensor [n2][n1][n0] (contiguous, n0 innermost) seen as boxes of 64 x 1 x box2 with 128-byte
// swizzling: one box is box2 rows of 64 elements at one index of the middle dimension, laid out in
// shared memory as a box_rows x 64 tile of tmap_bf16_tiles.  n0 must be a multiple of 8.
bool tmap_bf16_3d(CUtensorMap* tm, const void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t box2);
// bf16 matrix [rows][cols] (row-major, cols a multiple of 64) seen as 64-column chunks: one box is
// box_chunks consecutive chunks of box_rows rows, laid out in shared memory chunk by chunk, each a
// box_rows x 64 tile of tmap_bf16_tiles (128-byte swizzle).
bool tmap_bf16_chunks(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      uint32_t box_chunks);
// fp32 tensor [n2][n1][n0] (contiguous, n0 innermost, a multiple of 4) seen as boxes of
// box0 x box1 x 1, no swizzle: a box is box1 rows of box0 elements in shared memory.
bool tmap_f32_3d(CUtensorMap* tm, void* base, uint64_t n0, uint64_t n1, uint64_t n2, uint32_t box0, uint32_t box1);
// SM count of the current device.
int sm_count();

// True when the tensor-core GEMM handles these sizes and pointers (K a multiple of 64, 16-byte
// aligned operands, the driver's tensor-map encoder available).
bool gemm_tc_supported(int M, int N, int K, const void* A, const void* Bm);

// out[m * ldo + n] (or out[n * ldo + m] when trans) = sum_k A[m][k] Bm[n][k]
// (A [M x K], Bm [N x K] bf16; out fp32)
cudaError_t gemm_tc_store_f32(const __nv_bfloat16* A, const __nv_bfloat16* Bm, int M, int N, int K, float* out,
                              long long ldo, int32_t* status, uint64_t limit, cudaStream_t st, int trans = 0);

// Greedy step over a band of M <= 128 batch rows: for each row b < M,
//   keys[b] = max(keys[b], key of argmax_v (Lb[b*ldl + v] + sum_k U[b][k] W2[v][k]))
// (U [M x r], W2 [V x r] bf16; the argmax key orders by value, then lowest index).  When out is
// non-null the logits are also stored: out[b * ldo + v].
// claim (optional): work-slot claim words (at least one per SM, zero before the first launch that
// uses them) and epoch (nonzero, distinct for every launch sharing them): the CTAs then pick
// their vocabulary tiles by the SM they run on, so that each W2 tile stays with one SM across
// launches (see k_gemm_tc).
cudaError_t gemm_tc_argmax(const __nv_bfloat16* U, const __nv_bfloat16* W2, int M, int V, int r,
                           const __nv_bfloat16* Lb, long long ldl, uint64_t* keys, float* out, long long ldo,
                           int32_t* status, uint64_t limit, cudaStream_t st, uint32_t* claim = nullptr,
                           uint32_t epoch = 0);

// The same greedy step as gemm_tc_argmax on the dedicated kernel of w2_argmax.cu (activations
// resident in TMEM, W2 kept in L2 across positions, balanced vocabulary ranges): M <= 128 rows,
// r a multiple of 64 up to 256, U, W2 and Lb 16-byte aligned, Lb's row stride ldl (elements) a
// multiple of 8.  w2_argmax_supported tells whether a call qualifies.  last: this is the call's last
// read of W2 (its lines are then marked evict-first rather than evict-last).  claim / epoch: as for
// gemm_tc_argmax (vocabulary ranges taken by the SM a CTA runs on).
bool w2_argmax_supported(int M, int V, int r, const void* U, const void* W2, const void* Lb, long long ldl);
cudaError_t w2_argmax(const __nv_bfloat16* U, const __nv_bfloat16* W2, int M, int V, int r, const __nv_bfloat16* Lb,
                      long long ldl, uint64_t* keys, float* out, long long ldo, bool last, uint32_t* claim,
                      uint32_t epoch, int32_t* status, uint64_t limit, cudaStream_t st);

// u16[n][k] = bf16(SiLU(P[n * ldp + k] + sum_j W1s[k][j] S[n][j])) for k < r, n < N, where the
// fp32 state arrives as its two-term bf16 split S_hl [N x 2Hs] and W1s [r x Hs] has row stride ldw
// (the state block of W1).  uf (optional) receives the fp32 activations.
cudaError_t gemm_tc_silu_u(const __nv_bfloat16* W1s, long long ldw, const __nv_bfloat16* S_hl, int r, int N, int Hs,
                           const float* P, long long ldp, __nv_bfloat16* u16, float* uf, int32_t* status,
                           uint64_t limit, cudaStream_t st);

// One GEMM for both state products of a GRU step, on the two-term split S_hl [N x 2Hs]:
//   Gh[n * 3Hs + m] = sum_j W_hh[m][j] S[n][j]                            (m < 3Hs)
//   u16[n * r + k] = bf16(SiLU(P[n * ldp + k] + sum_j W1s[k][j] S[n][j])) (k < r)
// W1s [r x Hs] has row stride ldw (the state block of W1).  3Hs must be a multiple of 128.
cudaError_t gemm_tc_gru_u(const __nv_bfloat16* W_hh, const __nv_bfloat16* W1s, long long ldw,
                          const __nv_bfloat16* S_hl, int Hs, int r, int N, float* Gh, const float* P, long long ldp,
                          __nv_bfloat16* u16, int32_t* status, uint64_t limit, cudaStream_t st);

// out[n * ldo + m] = sum_k A[m][k mod a_kwrap] Bm[n][k] (a_kwrap = 0: no wrap) for a skinny Bm
// (N = a batch of rows), stored transposed (n-major) so that per-row consumers read contiguously.
// With a_kwrap = K/2 and Bm = [hi | lo] this applies A to a two-term bf16 split of an fp32 operand.
// a_stream: A is read once per call (no reuse by later calls): its lines are evicted from L2 first.
// lda: row stride of A in elements (0: K, or a_kwrap when set).
cudaError_t gemm_tc_store_f32_t(const __nv_bfloat16* A, const __nv_bfloat16* Bm, int M, int N, int K, int a_kwrap,
                                float* out, long long ldo, int32_t* status, uint64_t limit, cudaStream_t st,
                                int a_stream = 0, long long lda = 0);

// One store-epilogue product with a forced plan (bn in {16, 32, 64, 128}, ks in 1..8) or the
// automatic skinny plan (bn = ks = 0); out[m * ldo + n], or out[n * ldo + m] when trans.
cudaError_t gemm_tc_debug(const __nv_bfloat16* A, const __nv_bfloat16* Bm, int M, int N, int K, int a_kwrap,
                          float* out, long long ldo, int trans, int bn, int ks, int32_t* status, uint64_t limit,
                          cudaStream_t st);
// The automatic skinny plan for an M x N x K product (tile width bn, K split ks).
void gemm_tc_skinny_plan(int M, int N, int K, int* bn, int* ks);

// logits[n][v] = Lb[n][v] + sum_k W2[v][k] U[n][k]   (W2 [V x r], U [N x r], Lb [N x V] bf16); logits
// fp32, or bf16 (round to nearest even) when out_bf16.  claim / epoch (optional, as for
// gemm_tc_argmax): work slots taken by the SM a CTA runs on.
cudaError_t gemm_tc_logits(const __nv_bfloat16* W2, const __nv_bfloat16* U, int V, int N, int r,
                           const __nv_bfloat16* Lb, void* logits, int out_bf16, int32_t* status, uint64_t limit,
                           cudaStream_t st, uint32_t* claim = nullptr, uint32_t epoch = 0);

}  // namespace domino
