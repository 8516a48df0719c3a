// sm_affinity.cuh -- work slots chosen by the SM a CTA runs on.
//
// A persistent launch with one CTA per SM walks work slot = its rank, rank + grid, ...  Choosing the
// slot from the SM the CTA runs on (rather than from blockIdx) gives every slot the same SM at every
// launch, so that the operand lines of the slot stay in the L2 next to that SM across launches (B200
// has one L2 per die).  g_sm_rank maps %smid to a dense rank, filled once per device by k_sm_probe /
// k_sm_rank; each launch claims slots with atomicExch against a per-launch epoch, so that every slot
// is taken exactly once even when the scheduler places two CTAs on one SM.  Every translation unit
// that includes this header has its own table (internal linkage) and fills it itself.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "gemm_tc.h"

namespace domino {
namespace {

constexpr int kMaxSmid = 1024;
__device__ int g_sm_of_cta[kMaxSmid];
__device__ int g_sm_rank[kMaxSmid];

__device__ __forceinline__ unsigned sm_id() {
  unsigned s;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
  return s;
}
// Launched with more than half an SM's shared memory (unused): one CTA per SM.
__global__ void k_sm_probe(int n) {
  if (threadIdx.x == 0 && blockIdx.x < (unsigned)n) g_sm_of_cta[blockIdx.x] = (int)sm_id();
}
__global__ void k_sm_rank(int n) {  // one thread: dense rank of each recorded smid
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  for (int s = 0; s < kMaxSmid; ++s) g_sm_rank[s] = -1;
  for (int i = 0; i < n; ++i) {
    const int s = g_sm_of_cta[i];
    if (s >= 0 && s < kMaxSmid) g_sm_rank[s] = 0;  // present
  }
  int r = 0;
  for (int s = 0; s < kMaxSmid; ++s)
    if (g_sm_rank[s] == 0) g_sm_rank[s] = ++r;
  for (int s = 0; s < kMaxSmid; ++s)
    if (g_sm_rank[s] > 0) --g_sm_rank[s];  // ranks 0 .. r-1
}
// Work slot of this CTA (thread 0 only).  claim == null: blockIdx.x.
__device__ int claim_slot(uint32_t* claim, uint32_t epoch) {
  if (!claim) return (int)blockIdx.x;
  const int G = (int)gridDim.x;
  const unsigned s = sm_id();
  const int pref = s < (unsigned)kMaxSmid ? g_sm_rank[s] : -1;
  if (pref >= 0 && pref < G && atomicExch(claim + pref, epoch) != epoch) return pref;
  for (int k = 0; k < G; ++k) {  // taken (or no rank): the next free slot
    const int c = ((int)blockIdx.x + k) % G;
    if (atomicExch(claim + c, epoch) != epoch) return c;
  }
  return (int)blockIdx.x;  // unreachable: G CTAs, G slots
}

// Fills g_sm_rank once per device (two small launches on `st`, no host synchronisation).
cudaError_t ensure_sm_rank(cudaStream_t st) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const int n = std::min(sm_count(), kMaxSmid);
  const int hold = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM
  cudaError_t e = cudaFuncSetAttribute(k_sm_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, hold);
  if (e != cudaSuccess) return e;
  k_sm_probe<<<n, 32, hold, st>>>(n);
  k_sm_rank<<<1, 32, 0, st>>>(n);
  e = cudaGetLastError();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace
}  // namespace domino
