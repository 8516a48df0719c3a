// gemm_tc.h -- host entry points of the tcgen05 GEMM (gemm_tc.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "domino.h"
#include "internal.h"

namespace domino {

// True when the tensor-core GEMM handles these sizes and pointers (K a multiple of 64, 16-byte
// aligned operands, the driver's tensor-map encoder available).
bool gemm_tc_supported(int M, int N, int K, const void* A, const void* Bm);

// out[m * ldo + n] = sum_k A[m][k] Bm[n][k]   (A [M x K], Bm [N x K] bf16; out fp32)
cudaError_t gemm_tc_store_f32(const __nv_bfloat16* A, const __nv_bfloat16* Bm, int M, int N, int K, float* out,
                              long long ldo, int32_t* status, uint64_t limit, cudaStream_t st);

// logits[n][v] = Lb[n][v] + sum_k W2[v][k] U[n][k]   (W2 [V x r], U [N x r], Lb [N x V] bf16)
cudaError_t gemm_tc_logits(const __nv_bfloat16* W2, const __nv_bfloat16* U, int V, int N, int r,
                           const __nv_bfloat16* Lb, float* logits, int32_t* status, uint64_t limit, cudaStream_t st);

}  // namespace domino
