// internal.h -- host-side declarations shared by the libdomino translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "domino.h"

namespace domino {

// Host-side argument checks shared by the entry points (DOMINO_OK or a negative DOMINO_ERR_*).
int check_shape(const domino_shape_t* s);
int check_weights(const domino_weights_t* w);

struct Shape {
  int B, L, d, Hs, r, V, dtype;
};

// Scratch layout inside the caller's workspace.  Every region starts on a 256-byte boundary.
struct Workspace {
  int32_t* status;     // fallback status word when the caller passes no status pointer
  uint32_t* sync;      // barrier counters of the persistent kernels (kSyncWords words)
  uint32_t* claim;     // [kClaimWords] work-slot claims of SM-affine GEMM launches (zeroed per call)
  uint64_t* keys;      // [L][B]   greedy argmax keys per position
  uint64_t* acc_keys;  // [B*L]    target-logit argmax keys (accept length)
  uint32_t* acc_count; // [B*L]    chunks finished per (row, position); then [B] first mismatch (as L - j);
                       //          then one grid-completion word -- contiguous with acc_keys (one memset)
  float* P;            // [B*L][r] W1 . H for every position
  float* u;            // [B*L][r] SiLU activations
  float* S;            // [2][B][Hs] greedy state ping-pong
  float* states;       // [B][L][Hs] teacher-forced states when the caller keeps none
  __nv_bfloat16* u16;  // [B*L][r] activations rounded to bf16 (tensor-core W2 product)
  __nv_bfloat16* X;    // [B*L][d] gathered embedding rows (tensor-core GRU input product)
  float* Gx;           // [B*L][3Hs] W_ih . x for every gathered row
  float* Gh;           // [B][3Hs] W_hh . S
  __nv_bfloat16* S_hl; // [B*L][2Hs] two-term bf16 split of states
  unsigned long long* a_acc;  // [2][kAccReplicas][B][r] W1 state-block sums of the fused kernels
                              // (fixed point, see fix_add; ping-pong over positions)
  float* part;         // partial sums of the persistent batched kernel (batched_partial_floats)
  size_t bytes;
};
constexpr int kSyncWords = 64;
constexpr int kClaimWords = 1024;
// The fused greedy kernels spread the W1 state-block partial sums over this many copies of the
// accumulator (fewer atomics per address); the reader adds the copies.
constexpr int kAccReplicas = 4;
// Bytes of the fused kernels' accumulator ping-pong for B rows of rank r.
constexpr size_t acc_bytes(int B, int r) { return (size_t)2 * kAccReplicas * B * r * sizeof(unsigned long long); }

Workspace layout_workspace(const Shape& s, void* base);

// Phase-trace buffer set by domino_debug_set_trace (null when off).
void debug_trace(unsigned long long** buf, int* n);

// Counts one enqueued kernel when `e` reports success; returns `e`.
cudaError_t note_launch(cudaError_t e);
size_t accept_workspace_bytes(int B, int L);

// ---- step kernels (one launch per phase; any storage type, any batch) ----
cudaError_t launch_hproj(const Shape& s, const void* W1, const void* hidden, int N, float* P, cudaStream_t st);
// u16 (optional): the same activations rounded to bf16, for the tensor-core W2 product.
cudaError_t launch_u(const Shape& s, const void* W1, const float* P, int p_mul, int p_add, const float* S,
                     size_t s_stride, int M, float* u, cudaStream_t st, __nv_bfloat16* u16 = nullptr);
cudaError_t launch_w2(const Shape& s, const void* W2, const float* u, int M, const void* Lb, int l_mul,
                      int l_add, uint64_t* keys, float* logits, cudaStream_t st);
cudaError_t launch_gru(const Shape& s, const void* embed, const void* W_ih, const void* W_hh, const void* b_ih,
                       const void* b_hh, const uint64_t* tok_keys, const int32_t* tokens, int tok_mul, int tok_add,
                       const float* Sin, size_t sin_stride, float* Sout, size_t sout_stride, float* Sout2,
                       size_t sout2_stride, int M, int32_t* status, cudaStream_t st, const float* Xp = nullptr);
// Xp[v][n] = sum_c W_ih[n][c] embed[v][c] on CUDA cores (the tensor-core path lives in gemm_tc).
cudaError_t launch_project_simple(const Shape& s, const void* embed, const void* W_ih, float* Xp, cudaStream_t st);
// Large-batch GRU pieces for the tensor-core path (step_kernels.cu).
cudaError_t launch_split_state(const float* S, size_t s_stride, int B, int Hs, __nv_bfloat16* S_hl, cudaStream_t st);
cudaError_t launch_gather_rows(const __nv_bfloat16* embed, const uint64_t* keys, const int32_t* tokens, int per, int ld,
                               int N, int d, int V, __nv_bfloat16* X, cudaStream_t st);
cudaError_t launch_cell(const Shape& s, const float* Gx, int ldx, int xper, int xoff, const float* Xp, const float* Gh,
                        const void* b_ih, const void* b_hh, const uint64_t* keys, const int32_t* tokens, int tok_mul,
                        int tok_add, const float* Sin, size_t sin_stride, float* Sout, size_t sout_stride,
                        float* Sout2, size_t sout2_stride, int32_t* status, cudaStream_t st,
                        __nv_bfloat16* S_hl = nullptr);
// One launch: accept lengths with early exit (k_accept_early).  keys [B*L] and count
// [B*L + B + 1] must be zero.
cudaError_t launch_accept_early(const float* T, const int32_t* draft, int B, int L, int V, uint64_t* keys,
                                uint32_t* count, int32_t* out, cudaStream_t st);
cudaError_t launch_tokens_from_keys(const uint64_t* keys, int B, int L, int32_t* tokens, cudaStream_t st);
cudaError_t launch_copy_rows(const float* src, size_t src_stride, float* dst, size_t dst_stride, int rows, int n,
                             cudaStream_t st);

}  // namespace domino
