// debug.cu -- measurement aids for roofline reporting.
#include "common.cuh"
#include "domino.h"
#include "internal.h"

namespace domino {
namespace {

__device__ unsigned g_read_sink;

// One CTA per SM (forced by the launch's shared memory request) re-reads its contiguous slice of
// `buf` `passes` times with 16-byte read-only loads -- the access pattern of the fused kernel's W2
// pass -- so that passes after the first are served by L2 when the buffer fits.
// Eight independent loads in flight per thread (the fused kernel's W2 loop double-buffers its
// rows in registers the same way), so the measurement is not bound by one load's latency.
__global__ void __launch_bounds__(512, 1) k_read_passes(const uint4* __restrict__ buf, size_t n16, int passes) {
  const size_t G = gridDim.x, c = blockIdx.x;
  const size_t v0 = n16 * c / G, v1 = n16 * (c + 1) / G;
  const size_t step = (size_t)blockDim.x * 8;
  unsigned acc = 0;
  for (int p = 0; p < passes; ++p)
    for (size_t i0 = v0 + threadIdx.x; i0 < v1; i0 += step) {
      uint4 q[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const size_t i = i0 + (size_t)k * blockDim.x;
        q[k] = i < v1 ? __ldg(buf + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) acc ^= q[k].x ^ q[k].y ^ q[k].z ^ q[k].w;
    }
  if (acc == 0x9E3779B9u) g_read_sink = acc;  // keeps the loads; practically never taken
}

}  // namespace
}  // namespace domino

using namespace domino;

extern "C" int domino_debug_read_passes(const void* buf, size_t bytes, int32_t passes, domino_stream_t stream) {
  if (!buf || (reinterpret_cast<uintptr_t>(buf) & 15u) || bytes < 16 || passes < 1 || passes > 1000)
    return DOMINO_ERR_INVALID_ARGUMENT;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return DOMINO_ERR_CUDA;
  const int smem = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM
  if (cudaFuncSetAttribute(k_read_passes, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DOMINO_ERR_CUDA;
  k_read_passes<<<sms, 512, smem, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(buf), bytes / 16,
                                                                       passes);
  return note_launch(cudaGetLastError()) == cudaSuccess ? DOMINO_OK : DOMINO_ERR_CUDA;
}
