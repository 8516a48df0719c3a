// sample.cu -- sampled (temperature > 0) verification of a draft block.
//
// The pages call Domino's verification lossless (review page, section 一: the target checks the
// whole block in one parallel pass; researchpapers.dev summary) and spell out only its greedy
// setting.  For sampling, the rule that keeps verification lossless is speculative sampling's
// acceptance test (Leviathan, Kalman and Matias, ICML 2023; Chen et al. 2023):
//
//   p_j = softmax(target[b, j] / T),  q_j = softmax(draft[b, j] / T)  (one-hot on the draft token
//         for a greedy draft: draft logits absent)
//   accept x_j while u[b, j] < p_j(x_j) / q_j(x_j); at the first rejected position k draw the
//   replacement from res(v) = max(0, p_k(v) - q_k(v)) by inverse transform with u[b, L]: the
//   smallest v whose running sum of res exceeds u[b, L] * sum(res).
//
// The random draws are inputs (uniforms [B, L + 1]), so a run is reproducible and checkable.
// Two launches:
//   k_sample_stats  one block per (row, position, 8192-column chunk), issued position-major: the
//                   chunk's max and sum of exp((t - max) / T) for the target (and draft) logits; the
//                   last chunk block of a (row, position) merges the chunks in chunk order, takes
//                   the decision and records a rejection as first[b] = max(first[b], L - j).  A block
//                   whose position lies past a recorded rejection of its row skips its reads: such a
//                   position cannot change the result (a rejection recorded for it can only follow
//                   an earlier one, which wins the max).
//   k_sample_finish one block per row: k = L - first[b]; the replacement at (b, k) from the residual,
//                   recomputed from the merged statistics, with coalesced tiles and a fixed-order
//                   double-precision block scan carried across tiles.
// Both are memory-bound on the logits they read: at most B*L*V*4 bytes of target (and as many of
// draft) logits, plus one target (and draft) row per rejected row.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace domino {

namespace {

constexpr int kChunk = 8192;        // columns per statistics block
constexpr int kStatThreads = 256;   // 8 float4 per thread per logits row
constexpr int kFinThreads = 1024;

struct SampleArgs {
  const float* T;        // target logits [B][L][V]
  const float* D;        // draft logits [B][L][V], or null (greedy draft: one-hot)
  const int32_t* draft;  // [B][L]
  const float* uni;      // [B][L + 1]
  float inv_t;           // 1 / temperature
  int B, L, V, nchunks;
  float4* part;          // [B*L][nchunks] (max_t, sum_t, max_d, sum_d) per chunk
  float4* stats;         // [B*L] merged
  float2* xv;            // [B*L] (t[x], d[x]) at the draft token
  uint32_t* count;       // [B*L] finished chunks, then [B] first-rejection words (as L - j)
  int32_t* status;
};

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
  return m;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) s += red[w];  // fixed order
  return s;
}

// Chunk max and sum of exp((v - max) * inv_t) of one logits row segment [v0, v1).
__device__ __forceinline__ float2 chunk_stats(const float* row, int v0, int v1, float inv_t, float* red) {
  float x[kChunk / kStatThreads];
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kChunk / kStatThreads / 4; ++k) {
    const int v = v0 + 4 * (threadIdx.x + k * kStatThreads);
    float4 q = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    if (v + 4 <= v1) q = __ldcs(reinterpret_cast<const float4*>(row + v));
    else if (v < v1) {  // V is a multiple of 8, so a chunk end is 4-aligned: not reached
      q.x = row[v];
      if (v + 1 < v1) q.y = row[v + 1];
      if (v + 2 < v1) q.z = row[v + 2];
    }
    x[4 * k] = q.x; x[4 * k + 1] = q.y; x[4 * k + 2] = q.z; x[4 * k + 3] = q.w;
    m = fmaxf(fmaxf(m, fmaxf(q.x, q.y)), fmaxf(q.z, q.w));
  }
  m = block_max(m, red);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kChunk / kStatThreads; ++k) s += expf((x[k] - m) * inv_t);
  s = block_sum(s, red);
  return make_float2(m, s);
}

__global__ void __launch_bounds__(kStatThreads) k_sample_stats(SampleArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[kStatThreads / 32];
  __shared__ bool last_chunk, skip_s;
  const int y = blockIdx.y, j = y / a.B, b = y % a.B;
  const size_t n = (size_t)b * a.L + j;
  uint32_t* const first = a.count + (size_t)a.B * a.L;
  // one read of the row's rejection word for the whole block (another block may raise it meanwhile)
  if (threadIdx.x == 0) skip_s = *reinterpret_cast<volatile uint32_t*>(first + b) > (uint32_t)(a.L - j);
  __syncthreads();
  if (skip_s) return;
  const int c = blockIdx.x, v0 = c * kChunk, v1 = min(a.V, v0 + kChunk);
  const float2 st = chunk_stats(a.T + n * a.V, v0, v1, a.inv_t, red);
  float2 sd = make_float2(0.f, 0.f);
  if (a.D) sd = chunk_stats(a.D + n * a.V, v0, v1, a.inv_t, red);
  if (threadIdx.x == 0) {
    a.part[n * a.nchunks + c] = make_float4(st.x, st.y, sd.x, sd.y);
    const int x = a.draft[n];
    if (x >= v0 && x < v1) a.xv[n] = make_float2(a.T[n * a.V + x], a.D ? a.D[n * a.V + x] : 0.f);
    __threadfence();  // this chunk's record before its count
    last_chunk = atomicAdd(a.count + n, 1u) == (uint32_t)a.nchunks - 1;
  }
  __syncthreads();
  if (!last_chunk || threadIdx.x != 0) return;
  __threadfence();
  // merge the chunks in chunk order
  float mt = -INFINITY, md = -INFINITY;
  for (int k = 0; k < a.nchunks; ++k) {
    const float4 pk = __ldcg(a.part + n * a.nchunks + k);
    mt = fmaxf(mt, pk.x);
    md = fmaxf(md, pk.z);
  }
  float sumt = 0.f, sumd = 0.f;
  for (int k = 0; k < a.nchunks; ++k) {
    const float4 pk = __ldcg(a.part + n * a.nchunks + k);
    sumt += pk.y * expf((pk.x - mt) * a.inv_t);
    if (a.D) sumd += pk.w * expf((pk.z - md) * a.inv_t);
  }
  a.stats[n] = make_float4(mt, sumt, md, sumd);
  const int x = a.draft[n];
  float ratio = 0.f;
  if (x < 0 || x >= a.V) {
    set_status(a.status, DOMINO_STATUS_BAD_TOKEN);  // p(x) = 0: the position is rejected
  } else {
    const float2 v = __ldcg(a.xv + n);
    const float px = expf((v.x - mt) * a.inv_t) / sumt;
    const float qx = a.D ? expf((v.y - md) * a.inv_t) / sumd : 1.f;
    ratio = px / qx;
  }
  if (!(a.uni[(size_t)b * (a.L + 1) + j] < ratio)) atomicMax(first + b, (uint32_t)(a.L - j));
}

// Residual mass max(0, p(v) - q(v)) at one position from its merged statistics.
__device__ __forceinline__ float residual_of(const SampleArgs& a, float t, float d, bool one_hot, const float4& st) {
  const float p = expf((t - st.x) * a.inv_t) / st.y;
  const float q = one_hot ? 0.f : expf((d - st.z) * a.inv_t) / st.w;
  return fmaxf(p - q, 0.f);
}

// The four residuals of columns v .. v + 3 (v a multiple of 4; V is a multiple of 8).
__device__ __forceinline__ void residual4(const SampleArgs& a, const float* trow, const float* drow, int x,
                                          const float4& st, int v, float (&r)[4]) {
  const float4 t = __ldcs(reinterpret_cast<const float4*>(trow + v));
  const float4 d = drow ? __ldcs(reinterpret_cast<const float4*>(drow + v)) : make_float4(0.f, 0.f, 0.f, 0.f);
  r[0] = residual_of(a, t.x, d.x, !drow, st);
  r[1] = residual_of(a, t.y, d.y, !drow, st);
  r[2] = residual_of(a, t.z, d.z, !drow, st);
  r[3] = residual_of(a, t.w, d.w, !drow, st);
  if (!drow) {  // the one-hot draft removes the draft token's whole mass: res(x) = max(0, p(x) - 1)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (v + e == x) r[e] = fmaxf(expf((((const float*)&t)[e] - st.x) * a.inv_t) / st.y - 1.f, 0.f);
  }
}

// Block-wide inclusive scan of one double per thread in thread order (fixed): within each warp, then
// over the warp totals.  Returns the inclusive prefix; *excl receives the exclusive one -- equal, bit
// for bit, to the inclusive prefix of the previous thread -- and *total the block total.
__device__ __forceinline__ double block_scan(double v, double* wsum, double* excl, double* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  double exc = __shfl_up_sync(0xffffffffu, inc, 1);
  if (lane == 0) exc = 0.0;
  __syncthreads();  // wsum is free (its previous use has been read)
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  double before = 0.0, tot = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    if (w == wid) before = tot;
    tot += wsum[w];
  }
  *excl = before + exc;
  *total = tot;
  return before + inc;
}

// One block per row.  Pass 1: the residual's total Z (fixed-order sum).  Pass 2: walk the row in
// tiles of 4 columns per thread, coalesced; a block scan of the per-thread sums gives every thread an
// interval [lo, hi) of the running sum that tiles the row exactly (the tile base carries over
// bit-exactly); the thread whose interval holds u * Z finds the column among its four.
__global__ void __launch_bounds__(kFinThreads) k_sample_finish(SampleArgs a, int32_t* __restrict__ accept_out,
                                                                int32_t* __restrict__ next_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ double wsum[kFinThreads / 32];
  __shared__ int y_s, last_s, done_s;
  const int b = blockIdx.x, tid = threadIdx.x;
  const uint32_t f = __ldcg(a.count + (size_t)a.B * a.L + b);
  const int k = a.L - (int)f;
  if (k >= a.L) {
    if (tid == 0) { accept_out[b] = a.L; next_out[b] = -1; }
    return;
  }
  const size_t n = (size_t)b * a.L + k;
  const int x = a.draft[n];
  const float4 st = __ldcg(a.stats + n);
  const float* trow = a.T + n * a.V;
  const float* drow = a.D ? a.D + n * a.V : nullptr;
  constexpr int kTile = 4 * kFinThreads;
  if (tid == 0) { y_s = -1; last_s = -1; done_s = 0; }
  // pass 1: the total, and the last column with mass
  double own = 0.0;
  int lastpos = -1;
  for (int v = 4 * tid; v < a.V; v += kTile) {
    float r[4];
    residual4(a, trow, drow, x, st, v, r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      own += (double)r[e];
      if (r[e] > 0.f) lastpos = v + e;
    }
  }
  double excl, total;
  block_scan(own, wsum, &excl, &total);
  if (lastpos >= 0) atomicMax(&last_s, lastpos);
  const double target = (double)a.uni[(size_t)b * (a.L + 1) + a.L] * total;
  // pass 2: the tile and column where the running sum first exceeds the target
  double base = 0.0;
  for (int v0 = 0; v0 < a.V; v0 += kTile) {
    const int v = v0 + 4 * tid;
    float r[4] = {0.f, 0.f, 0.f, 0.f};
    if (v < a.V) residual4(a, trow, drow, x, st, v, r);
    const double s4 = (((double)r[0] + (double)r[1]) + (double)r[2]) + (double)r[3];
    double ex, tile_total;
    const double inc = block_scan(s4, wsum, &ex, &tile_total);
    const double lo = base + ex, hi = base + inc;
    if (lo <= target && target < hi) {  // exactly one thread of one tile
      double run = lo;
      int y = -1, lp = -1;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        run += (double)r[e];
        if (r[e] > 0.f) lp = v + e;
        if (y < 0 && run > target && r[e] > 0.f) y = v + e;
      }
      y_s = y >= 0 ? y : lp;  // rounding within the four: the last of them with mass
      done_s = 1;
    }
    base = base + tile_total;
    __syncthreads();
    if (done_s) break;  // block-uniform
  }
  __syncthreads();
  if (tid == 0) {
    accept_out[b] = k;
    next_out[b] = y_s >= 0 ? y_s : last_s;  // the draw lies past the running total: the last v with mass
  }
}

inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct SampleLayout {
  size_t status, part, stats, xv, count, bytes;
};
SampleLayout sample_layout(int B, int L, int V) {
  const size_t BL = (size_t)B * L, nch = (size_t)(V + kChunk - 1) / kChunk;
  SampleLayout s{};
  s.status = 0;  // the status word used when the caller passes none
  s.part = 256;
  s.stats = s.part + al256(BL * nch * sizeof(float4));
  s.xv = s.stats + al256(BL * sizeof(float4));
  s.count = s.xv + al256(BL * sizeof(float2));
  s.bytes = s.count + al256((BL + B) * sizeof(uint32_t));
  return s;
}

}  // namespace

}  // namespace domino

using namespace domino;

extern "C" size_t domino_accept_sample_workspace_bytes(int32_t B, int32_t L, int32_t V) {
  if (B < 1 || L < 1 || L > DOMINO_MAX_L || V < 8 || V % 8) return 0;
  return sample_layout(B, L, V).bytes;
}

extern "C" int domino_accept_sample(int32_t B, int32_t L, int32_t V, const int32_t* draft_tokens,
                                    const float* draft_logits, const float* target_logits, float temperature,
                                    const float* uniforms, int32_t* accept_out, int32_t* next_out,
                                    void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                    domino_stream_t stream) {
  auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (B < 1 || L < 1 || L > DOMINO_MAX_L || V < 8 || V % 8) return DOMINO_ERR_INVALID_ARGUMENT;
  if ((int64_t)B * L > 65535) return DOMINO_ERR_UNSUPPORTED;
  if (!(temperature > 0.f) || !(temperature < INFINITY)) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!draft_tokens || !target_logits || !uniforms || !accept_out || !next_out) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!a16(target_logits) || (draft_logits && !a16(draft_logits))) return DOMINO_ERR_INVALID_ARGUMENT;
  const SampleLayout lay = sample_layout(B, L, V);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < lay.bytes)
    return DOMINO_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  SampleArgs a{};
  a.T = target_logits;
  a.D = draft_logits;
  a.draft = draft_tokens;
  a.uni = uniforms;
  a.inv_t = 1.0f / temperature;
  a.B = B; a.L = L; a.V = V;
  a.nchunks = (V + kChunk - 1) / kChunk;
  a.part = reinterpret_cast<float4*>(ws + lay.part);
  a.stats = reinterpret_cast<float4*>(ws + lay.stats);
  a.xv = reinterpret_cast<float2*>(ws + lay.xv);
  a.count = reinterpret_cast<uint32_t*>(ws + lay.count);
  a.status = status_dev ? status_dev : reinterpret_cast<int32_t*>(ws + lay.status);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(a.count, 0, ((size_t)B * L + B) * sizeof(uint32_t), cs);
  if (e == cudaSuccess)
    e = note_launch(launch_pdl(k_sample_stats, dim3((unsigned)a.nchunks, (unsigned)(B * L)), dim3(kStatThreads), 0, cs,
                               a));
  if (e == cudaSuccess)
    e = note_launch(launch_pdl(k_sample_finish, dim3((unsigned)B), dim3(kFinThreads), 0, cs, a, accept_out, next_out));
  return e == cudaSuccess ? DOMINO_OK : DOMINO_ERR_CUDA;
}
