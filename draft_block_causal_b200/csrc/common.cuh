// common.cuh -- device helpers shared by the libdomino kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace domino {

using bf16 = __nv_bfloat16;

// Elements of storage type T per 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<bf16> { static constexpr int N = 8; };

// Widen one 16-byte vector of stored elements to fp32 (exact for both storage types).
__device__ __forceinline__ void widen(const uint4& q, float (&f)[8]) {
  f[0] = __uint_as_float(q.x << 16); f[1] = __uint_as_float(q.x & 0xffff0000u);
  f[2] = __uint_as_float(q.y << 16); f[3] = __uint_as_float(q.y & 0xffff0000u);
  f[4] = __uint_as_float(q.z << 16); f[5] = __uint_as_float(q.z & 0xffff0000u);
  f[6] = __uint_as_float(q.w << 16); f[7] = __uint_as_float(q.w & 0xffff0000u);
}
__device__ __forceinline__ void widen(const uint4& q, float (&f)[4]) {
  f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
  f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<bf16>(bf16 x) { return __bfloat162float(x); }

// Read-only 16-byte load through the non-coherent path.
__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Logistic function and SiLU on the CUDA math library's expf.
__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return x / (1.0f + expf(-x)); }

// Argmax keys: one u64 per (value, index) that orders like "larger value, then lower index",
// so atomicMax over keys is a deterministic argmax with the lowest-index tie rule.
//   high 32 bits: fp32 bits mapped monotonically onto u32 (-0 folded onto +0)
//   low 32 bits : 0xFFFFFFFF - index
// Key 0 never arises from a finite value and serves as "empty".
__device__ __forceinline__ uint64_t argmax_key(float z, int v) {
  uint32_t u = __float_as_uint(z);
  if (u == 0x80000000u) u = 0u;
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(0xFFFFFFFFu - static_cast<uint32_t>(v));
}
__device__ __forceinline__ int key_index(uint64_t k) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
}
__device__ __forceinline__ float key_value(uint64_t k) {
  uint32_t u = static_cast<uint32_t>(k >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}
__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }

// Fixed-point partial sums.  A sum whose partials arrive from many threads or CTAs in an order
// that varies from run to run is kept as a signed 64-bit integer count of 2^-32 units: each fp32
// partial is rounded once to that grid (|error| <= 2^-33) and integer addition is associative, so
// the total -- and every result computed from it -- is the same bits on every run.  Sums must stay
// below 2^31 in magnitude.  fix_add works on global and shared memory (generic address).
constexpr float kFixOne = 4294967296.0f;  // 2^32 units per 1.0
__device__ __forceinline__ unsigned long long fix_of(float x) {
  return static_cast<unsigned long long>(__float2ll_rn(x * kFixOne));
}
__device__ __forceinline__ void fix_add(unsigned long long* p, float x) { atomicAdd(p, fix_of(x)); }
__device__ __forceinline__ float fix_value(unsigned long long s) {
  return __ll2float_rn(static_cast<long long>(s)) * (1.0f / kFixOne);
}

// First problem wins; the library never clears the word.
__device__ __forceinline__ void set_status(int32_t* st, int code) { atomicCAS(st, 0, code); }

}  // namespace domino
