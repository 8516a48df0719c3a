// step_kernels.cu -- one-launch-per-phase kernels of the Domino head (any storage type, any
// batch).  They compute, phase by phase, the equations of the Domino review page, section 二:
//   P = W1[:, :d] . H                 (H-projection, all positions)
//   u = SiLU(P + W1[:, d:] . S)        (low-rank activation)
//   z = L_base + W2 . u, argmax        (logit-space residual, fused vocabulary argmax)
//   S' = GRUCell(embed[t], S)          (causal encoder update)
// and the accept-length check.  A warp owns one output row of the weight matrix and applies it
// to a tile of up to kTileM right-hand vectors, so each weight row is read once per tile.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace domino {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTileM = 8;

// fp32 vector of N elements at p (16-byte aligned), N in {4, 8}.
template <int N> __device__ __forceinline__ void load_f32(const float* p, float (&f)[N]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    float4 v = __ldg(q + i);
    f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
  }
}

// P[n][k] = sum_c W1[k][c] H[n][c]
template <typename T>
__global__ void __launch_bounds__(kThreads) k_hproj(const T* __restrict__ W1, int ldw, const T* __restrict__ H,
                                                    int N, int d, int r, float* __restrict__ P) {
  constexpr int E = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * kWarps + warp;
  if (k >= r) return;
  const int n0 = blockIdx.y * kTileM;
  float acc[kTileM];
#pragma unroll
  for (int m = 0; m < kTileM; ++m) acc[m] = 0.f;
  const T* wrow = W1 + (size_t)k * ldw;
  for (int q = lane; q < d / E; q += 32) {
    float w[E];
    widen(ldg16(wrow + q * E), w);
#pragma unroll
    for (int m = 0; m < kTileM; ++m) {
      if (n0 + m < N) {
        float h[E];
        widen(ldg16(H + (size_t)(n0 + m) * d + q * E), h);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[m] = fmaf(w[e], h[e], acc[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kTileM; ++m) {
    float s = warp_sum(acc[m]);
    if (lane == 0 && n0 + m < N) P[(size_t)(n0 + m) * r + k] = s;
  }
}

// u[m][k] = SiLU(P[m*p_mul + p_add][k] + sum_j W1[k][d+j] S[m][j])
template <typename T>
__global__ void __launch_bounds__(kThreads) k_u(const T* __restrict__ W1, int ldw, int d, int Hs, int r,
                                                const float* __restrict__ P, int p_mul, int p_add,
                                                const float* __restrict__ S, size_t s_stride, int M,
                                                float* __restrict__ u, bf16* __restrict__ u16) {
  constexpr int E = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * kWarps + warp;
  if (k >= r) return;
  const int m0 = blockIdx.y * kTileM;
  float acc[kTileM];
#pragma unroll
  for (int m = 0; m < kTileM; ++m) acc[m] = 0.f;
  const T* wrow = W1 + (size_t)k * ldw + d;
  for (int q = lane; q < Hs / E; q += 32) {
    float w[E];
    widen(ldg16(wrow + q * E), w);
#pragma unroll
    for (int m = 0; m < kTileM; ++m) {
      if (m0 + m < M) {
        float h[E];
        load_f32<E>(S + (size_t)(m0 + m) * s_stride + q * E, h);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[m] = fmaf(w[e], h[e], acc[m]);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < kTileM; ++m) {
    float s = warp_sum(acc[m]);
    if (lane == 0 && m0 + m < M) {
      float a = P[(size_t)((m0 + m) * p_mul + p_add) * r + k] + s;
      const float v = siluf_(a);
      u[(size_t)(m0 + m) * r + k] = v;
      if (u16) u16[(size_t)(m0 + m) * r + k] = __float2bfloat16_rn(v);
    }
  }
}

// z[m][v] = Lb[row(m)][v] + sum_k W2[v][k] u[m][k],  row(m) = m*l_mul + l_add, for a tile of MT
// rows m.  keys != null: keys[m] = max(keys[m], argmax_key(z, v)).  logits != null:
// logits[row(m)][v] = z.  u sits in shared memory as [m][vector][E + pad] so that the 16-byte
// reads of 32 lanes (one vector each) hit distinct bank groups.
template <typename T> struct UPad { static constexpr int v = 0; };
template <> struct UPad<bf16> { static constexpr int v = 4; };

template <typename T, int MT>
__global__ void __launch_bounds__(kThreads) k_w2(const T* __restrict__ W2, int r, int V, const float* __restrict__ u,
                                                 int M, const T* __restrict__ Lb, int l_mul, int l_add,
                                                 uint64_t* __restrict__ keys, float* __restrict__ logits) {
  constexpr int E = Vec<T>::N;
  constexpr int VS = E + UPad<T>::v;
  extern __shared__ __align__(16) float u_s[];  // [MT][r/E][VS]
  __shared__ uint64_t best_s[kWarps][MT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqv = r / E;
  const int m0 = blockIdx.y * MT;
  const int mt = min(MT, M - m0);
  for (int i = threadIdx.x; i < MT * r; i += kThreads) {
    const int m = i / r, k = i % r;
    u_s[(m * nqv + k / E) * VS + k % E] = (m < mt) ? u[(size_t)(m0 + m) * r + k] : 0.f;
  }
  __syncthreads();
  uint64_t best[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) best[m] = 0ull;
  for (int v = blockIdx.x * kWarps + warp; v < V; v += gridDim.x * kWarps) {
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    const T* wrow = W2 + (size_t)v * r;
    for (int q = lane; q < nqv; q += 32) {
      float w[E];
      widen(ldg16(wrow + q * E), w);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4* up = reinterpret_cast<const float4*>(u_s + (m * nqv + q) * VS);
#pragma unroll
        for (int h = 0; h < E / 4; ++h) {
          const float4 x = up[h];
          acc[m] = fmaf(w[4 * h], x.x, acc[m]);
          acc[m] = fmaf(w[4 * h + 1], x.y, acc[m]);
          acc[m] = fmaf(w[4 * h + 2], x.z, acc[m]);
          acc[m] = fmaf(w[4 * h + 3], x.w, acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float s = warp_sum(acc[m]);
      if (lane == 0 && m < mt) {
        size_t row = (size_t)(m0 + m) * l_mul + l_add;
        float z = to_f32(Lb[row * V + v]) + s;
        if (logits) logits[row * V + v] = z;
        best[m] = umax64(best[m], argmax_key(z, v));
      }
    }
  }
  if (keys) {
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < MT; ++m) best_s[warp][m] = best[m];
    }
    __syncthreads();
    if (threadIdx.x < mt) {
      uint64_t b = 0ull;
      for (int w = 0; w < kWarps; ++w) b = umax64(b, best_s[w][threadIdx.x]);
      atomicMax(reinterpret_cast<unsigned long long*>(keys + m0 + threadIdx.x), (unsigned long long)b);
    }
  }
}

// GRU update, PyTorch GRUCell form, for every row m < M and unit j < Hs:
//   t = tok_keys ? index(tok_keys[m]) : tokens[m*tok_mul + tok_add];  x = embed[t];  h = Sin[m]
//   r = sig(gi_r + gh_r), z = sig(gi_z + gh_z), n = tanh(gi_n + r * gh_n), h' = (1-z) n + z h[j]
// gi = W_ih x is read from the projection table Xp[t] when one is given, else computed here.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_gru(const T* __restrict__ embed, const T* __restrict__ W_ih,
                                                  const T* __restrict__ W_hh, const T* __restrict__ b_ih,
                                                  const T* __restrict__ b_hh, int d, int Hs, int V,
                                                  const uint64_t* __restrict__ tok_keys,
                                                  const int32_t* __restrict__ tokens, int tok_mul, int tok_add,
                                                  const float* __restrict__ Sin, size_t sin_stride,
                                                  float* __restrict__ Sout, size_t sout_stride,
                                                  float* __restrict__ Sout2, size_t sout2_stride, int M,
                                                  int32_t* __restrict__ status, const float* __restrict__ Xp) {
  constexpr int E = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * kWarps + warp;
  if (j >= Hs) return;
  const int m0 = blockIdx.y * kTileM;
  const T* xrow[kTileM];
  int tk[kTileM];
  bool ok[kTileM];
#pragma unroll
  for (int m = 0; m < kTileM; ++m) {
    int t = 0;
    ok[m] = false;
    if (m0 + m < M) {
      t = tok_keys ? key_index(tok_keys[m0 + m]) : tokens[(size_t)(m0 + m) * tok_mul + tok_add];
      ok[m] = (t >= 0 && t < V);
      if (!ok[m] && lane == 0 && j == 0) set_status(status, 2 /* DOMINO_STATUS_BAD_TOKEN */);
    }
    tk[m] = ok[m] ? t : 0;
    xrow[m] = embed + (size_t)tk[m] * d;
  }
  float gi[3][kTileM], gh[3][kTileM];
#pragma unroll
  for (int g = 0; g < 3; ++g)
#pragma unroll
    for (int m = 0; m < kTileM; ++m) gi[g][m] = gh[g][m] = 0.f;
  for (int q = lane; q < (Xp ? 0 : d / E); q += 32) {
    float w[3][E];
#pragma unroll
    for (int g = 0; g < 3; ++g) widen(ldg16(W_ih + ((size_t)g * Hs + j) * d + q * E), w[g]);
#pragma unroll
    for (int m = 0; m < kTileM; ++m) {
      if (ok[m]) {
        float x[E];
        widen(ldg16(xrow[m] + q * E), x);
#pragma unroll
        for (int g = 0; g < 3; ++g)
#pragma unroll
          for (int e = 0; e < E; ++e) gi[g][m] = fmaf(w[g][e], x[e], gi[g][m]);
      }
    }
  }
  for (int q = lane; q < Hs / E; q += 32) {
    float w[3][E];
#pragma unroll
    for (int g = 0; g < 3; ++g) widen(ldg16(W_hh + ((size_t)g * Hs + j) * Hs + q * E), w[g]);
#pragma unroll
    for (int m = 0; m < kTileM; ++m) {
      if (m0 + m < M) {
        float h[E];
        load_f32<E>(Sin + (size_t)(m0 + m) * sin_stride + q * E, h);
#pragma unroll
        for (int g = 0; g < 3; ++g)
#pragma unroll
          for (int e = 0; e < E; ++e) gh[g][m] = fmaf(w[g][e], h[e], gh[g][m]);
      }
    }
  }
  float bi[3], bh[3];
#pragma unroll
  for (int g = 0; g < 3; ++g) {
    bi[g] = to_f32(b_ih[(size_t)g * Hs + j]);
    bh[g] = to_f32(b_hh[(size_t)g * Hs + j]);
  }
#pragma unroll
  for (int m = 0; m < kTileM; ++m) {
    float si[3], sh[3];
#pragma unroll
    for (int g = 0; g < 3; ++g) {
      si[g] = (Xp ? (ok[m] ? Xp[(size_t)tk[m] * 3 * Hs + (size_t)g * Hs + j] : 0.f) : warp_sum(gi[g][m])) + bi[g];
      sh[g] = warp_sum(gh[g][m]) + bh[g];
    }
    if (lane == 0 && m0 + m < M) {
      float h = Sin[(size_t)(m0 + m) * sin_stride + j];
      float rg = sigmoidf_(si[0] + sh[0]);
      float zg = sigmoidf_(si[1] + sh[1]);
      float ng = tanhf(si[2] + rg * sh[2]);
      float hn = (1.f - zg) * ng + zg * h;
      Sout[(size_t)(m0 + m) * sout_stride + j] = hn;
      if (Sout2) Sout2[(size_t)(m0 + m) * sout2_stride + j] = hn;
    }
  }
}

// Xp[v][n] = sum_c W_ih[n][c] embed[v][c] on CUDA cores (any storage type): a warp per (v, 8 n).
template <typename T>
__global__ void __launch_bounds__(kThreads) k_project(const T* __restrict__ embed, const T* __restrict__ W_ih, int V,
                                                      int d, int N, float* __restrict__ Xp) {
  constexpr int E = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v = blockIdx.y;
  const int n0 = (blockIdx.x * kWarps + warp) * 8;
  if (n0 >= N) return;
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  for (int q = lane; q < d / E; q += 32) {
    float x[E];
    widen(ldg16(embed + (size_t)v * d + q * E), x);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (n0 + k < N) {
        float w[E];
        widen(ldg16(W_ih + (size_t)(n0 + k) * d + q * E), w);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[k] = fmaf(w[e], x[e], acc[k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float s = warp_sum(acc[k]);
    if (lane == 0 && n0 + k < N) Xp[(size_t)v * N + n0 + k] = s;
  }
}

// Two-term bf16 split of the fp32 state for the tensor cores: S_hl[b] = [hi | lo] with
// hi = bf16(S), lo = bf16(S - hi), so hi + lo = S within 2^-16 |S|.
__global__ void k_split_state(const float* __restrict__ S, size_t s_stride, int B, int Hs, bf16* __restrict__ S_hl) {
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < B * Hs; t += gridDim.x * blockDim.x) {
    const int b = t / Hs, k = t % Hs;
    const float v = S[(size_t)b * s_stride + k];
    const bf16 hi = __float2bfloat16_rn(v);
    S_hl[(size_t)b * 2 * Hs + k] = hi;
    S_hl[(size_t)b * 2 * Hs + Hs + k] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// X[n] = embed[t_n] for n < N, t_n = key_index(keys[n]) (keys != null) or tokens[(n / per) * ld + n % per].
__global__ void k_gather_rows(const bf16* __restrict__ embed, const uint64_t* __restrict__ keys,
                              const int32_t* __restrict__ tokens, int per, int ld, int N, int d, int V,
                              bf16* __restrict__ X) {
  pdl_wait();
  pdl_trigger();
  const int nv = d / 8;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < N * nv; t += gridDim.x * blockDim.x) {
    const int n = t / nv, q = t % nv;
    int tok = keys ? key_index(keys[n]) : tokens[(size_t)(n / per) * ld + n % per];
    tok = min(max(tok, 0), V - 1);  // out-of-range tokens are reported by the cell kernel
    reinterpret_cast<uint4*>(X + (size_t)n * d)[q] = ldg16(embed + (size_t)tok * d + q * 8);
  }
}

// GRU cell from precomputed gate pre-activations, PyTorch GRUCell form, for b < B, j < Hs:
//   gi[g] = (Xp ? Xp[t][g*Hs + j] : Gx[cx(b) * ldx + g*Hs + j]) + b_ih,  gh[g] = Gh[b * 3Hs + g*Hs + j] + b_hh
//   h' = (1 - z) n + z h,  r = sig(gi_r + gh_r), z = sig(gi_z + gh_z), n = tanh(gi_n + r gh_n)
// cx(b) = b * xper + xoff.  Writes Sout (and Sout2) rows; t from keys[b] or tokens[b * tok_mul + tok_add].
template <typename T>
__global__ void k_cell(const float* __restrict__ Gx, int ldx, int xper, int xoff, const float* __restrict__ Xp,
                       const float* __restrict__ Gh, const T* __restrict__ b_ih, const T* __restrict__ b_hh,
                       const uint64_t* __restrict__ keys, const int32_t* __restrict__ tokens, int tok_mul, int tok_add,
                       const float* __restrict__ Sin, size_t sin_stride, float* __restrict__ Sout, size_t sout_stride,
                       float* __restrict__ Sout2, size_t sout2_stride, int B, int Hs, int V,
                       int32_t* __restrict__ status, bf16* __restrict__ S_hl) {
  pdl_wait();
  pdl_trigger();
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < B * Hs; t += gridDim.x * blockDim.x) {
    const int b = t / Hs, j = t % Hs;
    int tok = keys ? key_index(keys[b]) : tokens[(size_t)b * tok_mul + tok_add];
    const bool ok = tok >= 0 && tok < V;
    if (!ok && j == 0) set_status(status, 2 /* DOMINO_STATUS_BAD_TOKEN */);
    tok = ok ? tok : 0;
    float gi[3], gh[3];
#pragma unroll
    for (int g = 0; g < 3; ++g) {
      const size_t row = (size_t)g * Hs + j;
      gi[g] = (Xp ? Xp[(size_t)tok * 3 * Hs + row] : Gx[((size_t)b * xper + xoff) * ldx + row]) + to_f32(b_ih[row]);
      gh[g] = Gh[(size_t)b * 3 * Hs + row] + to_f32(b_hh[row]);
    }
    const float rg = sigmoidf_(gi[0] + gh[0]);
    const float zg = sigmoidf_(gi[1] + gh[1]);
    const float ng = tanhf(gi[2] + rg * gh[2]);
    const float hn = (1.f - zg) * ng + zg * Sin[(size_t)b * sin_stride + j];
    Sout[(size_t)b * sout_stride + j] = hn;
    if (Sout2) Sout2[(size_t)b * sout2_stride + j] = hn;
    if (S_hl) {  // two-term bf16 split of the new state for the next tensor-core products
      const bf16 hi = __float2bfloat16_rn(hn);
      S_hl[(size_t)b * 2 * Hs + j] = hi;
      S_hl[(size_t)b * 2 * Hs + Hs + j] = __float2bfloat16_rn(hn - __bfloat162float(hi));
    }
  }
}

__global__ void k_tokens_from_keys(const uint64_t* __restrict__ keys, int B, int L, int32_t* __restrict__ tokens) {
  pdl_wait();
  pdl_trigger();
  int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= B * L) return;
  int b = n / L, i = n % L;
  tokens[n] = key_index(keys[(size_t)i * B + b]);
}

__global__ void k_copy_rows(const float* __restrict__ src, size_t src_stride, float* __restrict__ dst,
                            size_t dst_stride, int rows, int n) {
  pdl_wait();
  pdl_trigger();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * n; i += gridDim.x * blockDim.x) {
    int m = i / n, c = i % n;
    dst[(size_t)m * dst_stride + c] = src[(size_t)m * src_stride + c];
  }
}

// Columns of one target row that one block of the accept-length kernel reads.
constexpr int kArgChunk = 8192;

// Greedy accept length with early exit, in one launch.  Block (c, y) reads chunk c (kArgChunk
// columns) of the target row of position j = y / B, batch row b = y % B: position-major, so that a
// row's earlier positions are issued first.  It folds the chunk's argmax key into keys[b * L + j].
// The last chunk block of a (row, position) compares the finished argmax with the draft token and,
// on a mismatch, records it: first[b] = max(first[b], L - j), so 0 means "none" and the largest
// value is the earliest mismatch.  A block whose position lies past a recorded mismatch of its row
// skips its reads; such a position cannot change the row's result, because a mismatch can only
// be recorded for it after an earlier one has been, and the earlier one wins the max.  The last
// block of the grid writes out[b] = L - first[b].
// count = [B*L chunk counters][B first-mismatch words][1 grid counter], all zero at launch.
__global__ void __launch_bounds__(256) k_accept_early(const float* __restrict__ T, const int32_t* __restrict__ draft,
                                                      int B, int L, int V, uint64_t* __restrict__ keys,
                                                      uint32_t* __restrict__ count, int32_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t red[8];
  __shared__ bool last_chunk, last_block, skip_s;
  const int y = blockIdx.y, j = y / B, b = y % B;
  const size_t n = (size_t)b * L + j;
  uint32_t* const first = count + (size_t)B * L;
  uint32_t* const done = first + B;
  // one read of the row's mismatch word for the whole block: another block may raise it at any
  // moment, and every thread must take the same branch around the block barriers below
  if (threadIdx.x == 0) skip_s = *reinterpret_cast<volatile uint32_t*>(first + b) > (uint32_t)(L - j);
  __syncthreads();
  const bool skip = skip_s;
  if (!skip) {  // block-uniform
    const int v0 = blockIdx.x * kArgChunk, v1 = min(V, v0 + kArgChunk);
    const float* row = T + n * V;
    uint64_t best = 0ull;
    for (int v = v0 + 4 * threadIdx.x; v < v1; v += 4 * blockDim.x) {
      const float4 q = __ldcs(reinterpret_cast<const float4*>(row + v));
      best = umax64(best, argmax_key(q.x, v));
      best = umax64(best, argmax_key(q.y, v + 1));
      best = umax64(best, argmax_key(q.z, v + 2));
      best = umax64(best, argmax_key(q.w, v + 3));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = umax64(best, __shfl_xor_sync(0xffffffffu, best, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w) best = umax64(best, red[w]);
      atomicMax(reinterpret_cast<unsigned long long*>(keys + n), (unsigned long long)best);
    }
  }
  if (threadIdx.x == 0) {
    __threadfence();  // this block's key before its count
    last_chunk = atomicAdd(count + n, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (last_chunk) {
      __threadfence();
      const uint64_t k = atomicAdd(reinterpret_cast<unsigned long long*>(keys + n), 0ull);
      if (draft[n] != key_index(k)) atomicMax(first + b, (uint32_t)(L - j));
    }
    __threadfence();  // this block's record before its completion
    last_block = atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1;
  }
  __syncthreads();
  if (last_block) {
    __threadfence();
    for (int r = threadIdx.x; r < B; r += blockDim.x)
      out[r] = L - (int)*reinterpret_cast<volatile uint32_t*>(first + r);
  }
}

inline unsigned cdiv(size_t a, size_t b) { return (unsigned)((a + b - 1) / b); }

}  // namespace

cudaError_t launch_hproj(const Shape& s, const void* W1, const void* hidden, int N, float* P, cudaStream_t st) {
  dim3 grid(cdiv(s.r, kWarps), cdiv(N, kTileM));
  if (s.dtype == 0)
    k_hproj<float><<<grid, kThreads, 0, st>>>((const float*)W1, s.d + s.Hs, (const float*)hidden, N, s.d, s.r, P);
  else
    k_hproj<bf16><<<grid, kThreads, 0, st>>>((const bf16*)W1, s.d + s.Hs, (const bf16*)hidden, N, s.d, s.r, P);
  return note_launch(cudaGetLastError());
}

cudaError_t launch_u(const Shape& s, const void* W1, const float* P, int p_mul, int p_add, const float* S,
                     size_t s_stride, int M, float* u, cudaStream_t st, bf16* u16) {
  dim3 grid(cdiv(s.r, kWarps), cdiv(M, kTileM));
  if (s.dtype == 0)
    k_u<float><<<grid, kThreads, 0, st>>>((const float*)W1, s.d + s.Hs, s.d, s.Hs, s.r, P, p_mul, p_add, S,
                                          s_stride, M, u, u16);
  else
    k_u<bf16><<<grid, kThreads, 0, st>>>((const bf16*)W1, s.d + s.Hs, s.d, s.Hs, s.r, P, p_mul, p_add, S,
                                         s_stride, M, u, u16);
  return note_launch(cudaGetLastError());
}

template <typename T, int MT>
cudaError_t launch_w2_t(const Shape& s, const void* W2, const float* u, int M, const void* Lb, int l_mul, int l_add,
                        uint64_t* keys, float* logits, unsigned gx, cudaStream_t st) {
  constexpr int E = Vec<T>::N;
  dim3 grid(gx, cdiv(M, MT));
  size_t smem = (size_t)MT * (s.r / E) * (E + UPad<T>::v) * sizeof(float);
  auto kern = k_w2<T, MT>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, kThreads, smem, st>>>((const T*)W2, s.r, s.V, u, M, (const T*)Lb, l_mul, l_add, keys, logits);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_w2_dt(const Shape& s, const void* W2, const float* u, int M, const void* Lb, int l_mul, int l_add,
                         uint64_t* keys, float* logits, unsigned gx, cudaStream_t st) {
  if (M >= 8) return launch_w2_t<T, 8>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st);
  if (M >= 4) return launch_w2_t<T, 4>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st);
  if (M >= 2) return launch_w2_t<T, 2>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st);
  return launch_w2_t<T, 1>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st);
}

cudaError_t launch_w2(const Shape& s, const void* W2, const float* u, int M, const void* Lb, int l_mul, int l_add,
                      uint64_t* keys, float* logits, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  unsigned gx = (unsigned)min((size_t)sms * 4, (size_t)cdiv(s.V, kWarps));
  cudaError_t e = (s.dtype == 0) ? launch_w2_dt<float>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st)
                                 : launch_w2_dt<bf16>(s, W2, u, M, Lb, l_mul, l_add, keys, logits, gx, st);
  return note_launch(e);
}

cudaError_t launch_gru(const Shape& s, const void* embed, const void* W_ih, const void* W_hh, const void* b_ih,
                       const void* b_hh, const uint64_t* tok_keys, const int32_t* tokens, int tok_mul, int tok_add,
                       const float* Sin, size_t sin_stride, float* Sout, size_t sout_stride, float* Sout2,
                       size_t sout2_stride, int M, int32_t* status, cudaStream_t st, const float* Xp) {
  dim3 grid(cdiv(s.Hs, kWarps), cdiv(M, kTileM));
  if (s.dtype == 0)
    k_gru<float><<<grid, kThreads, 0, st>>>((const float*)embed, (const float*)W_ih, (const float*)W_hh,
                                            (const float*)b_ih, (const float*)b_hh, s.d, s.Hs, s.V, tok_keys, tokens,
                                            tok_mul, tok_add, Sin, sin_stride, Sout, sout_stride, Sout2,
                                            sout2_stride, M, status, Xp);
  else
    k_gru<bf16><<<grid, kThreads, 0, st>>>((const bf16*)embed, (const bf16*)W_ih, (const bf16*)W_hh,
                                           (const bf16*)b_ih, (const bf16*)b_hh, s.d, s.Hs, s.V, tok_keys, tokens,
                                           tok_mul, tok_add, Sin, sin_stride, Sout, sout_stride, Sout2, sout2_stride,
                                           M, status, Xp);
  return note_launch(cudaGetLastError());
}

cudaError_t launch_project_simple(const Shape& s, const void* embed, const void* W_ih, float* Xp, cudaStream_t st) {
  const int N = 3 * s.Hs;
  dim3 grid(cdiv(N, kWarps * 8), s.V);
  if (s.dtype == 0)
    k_project<float><<<grid, kThreads, 0, st>>>((const float*)embed, (const float*)W_ih, s.V, s.d, N, Xp);
  else
    k_project<bf16><<<grid, kThreads, 0, st>>>((const bf16*)embed, (const bf16*)W_ih, s.V, s.d, N, Xp);
  return note_launch(cudaGetLastError());
}

cudaError_t launch_split_state(const float* S, size_t s_stride, int B, int Hs, bf16* S_hl, cudaStream_t st) {
  cudaError_t e = launch_pdl(k_split_state, dim3(min(cdiv((size_t)B * Hs, 256), 4096u)), dim3(256), 0, st, S, s_stride,
                             B, Hs, S_hl);
  return note_launch(e);
}

cudaError_t launch_gather_rows(const bf16* embed, const uint64_t* keys, const int32_t* tokens, int per, int ld, int N,
                               int d, int V, bf16* X, cudaStream_t st) {
  cudaError_t e = launch_pdl(k_gather_rows, dim3(min(cdiv((size_t)N * (d / 8), 256), 8192u)), dim3(256), 0, st, embed,
                             keys, tokens, per, ld, N, d, V, X);
  return note_launch(e);
}

cudaError_t launch_cell(const Shape& s, const float* Gx, int ldx, int xper, int xoff, const float* Xp, const float* Gh,
                        const void* b_ih, const void* b_hh, const uint64_t* keys, const int32_t* tokens, int tok_mul,
                        int tok_add, const float* Sin, size_t sin_stride, float* Sout, size_t sout_stride,
                        float* Sout2, size_t sout2_stride, int32_t* status, cudaStream_t st, bf16* S_hl) {
  const unsigned g = min(cdiv((size_t)s.B * s.Hs, 256), 4096u);
  cudaError_t e;
  if (s.dtype == 0)
    e = launch_pdl(k_cell<float>, dim3(g), dim3(256), 0, st, Gx, ldx, xper, xoff, Xp, Gh, (const float*)b_ih,
                   (const float*)b_hh, keys, tokens, tok_mul, tok_add, Sin, sin_stride, Sout, sout_stride, Sout2,
                   sout2_stride, s.B, s.Hs, s.V, status, S_hl);
  else
    e = launch_pdl(k_cell<bf16>, dim3(g), dim3(256), 0, st, Gx, ldx, xper, xoff, Xp, Gh, (const bf16*)b_ih,
                   (const bf16*)b_hh, keys, tokens, tok_mul, tok_add, Sin, sin_stride, Sout, sout_stride, Sout2,
                   sout2_stride, s.B, s.Hs, s.V, status, S_hl);
  return note_launch(e);
}

cudaError_t launch_tokens_from_keys(const uint64_t* keys, int B, int L, int32_t* tokens, cudaStream_t st) {
  cudaError_t e = launch_pdl(k_tokens_from_keys, dim3(cdiv((size_t)B * L, 256)), dim3(256), 0, st, keys, B, L, tokens);
  return note_launch(e);
}

cudaError_t launch_copy_rows(const float* src, size_t src_stride, float* dst, size_t dst_stride, int rows, int n,
                             cudaStream_t st) {
  unsigned g = min(cdiv((size_t)rows * n, 256), 4096u);
  cudaError_t e = launch_pdl(k_copy_rows, dim3(g), dim3(256), 0, st, src, src_stride, dst, dst_stride, rows, n);
  return note_launch(e);
}

cudaError_t launch_accept_early(const float* T, const int32_t* draft, int B, int L, int V, uint64_t* keys,
                                uint32_t* count, int32_t* out, cudaStream_t st) {
  dim3 grid(cdiv(V, kArgChunk), (unsigned)(B * L));  // B * L <= 65535 (shape checks)
  cudaError_t e = launch_pdl(k_accept_early, grid, dim3(256), 0, st, T, draft, B, L, V, keys, count, out);
  return note_launch(e);
}

}  // namespace domino
