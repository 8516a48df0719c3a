// persistent_tmem.cu -- fused greedy drafting of a whole block, small batch, with the GRU weights
// resident in Tensor Memory.
//
// Same equations and phase structure as k_greedy_persistent (Domino review page, section 二:
// z_i = L_base + W2 . SiLU(W1 . [H_i ; S_{i-1}]), greedy t_i = argmax z_i, S_i = GRU(embed[t_i],
// S_{i-1})), with three changes aimed at the B200 memory system:
//
//  1. Each CTA copies its GRU rows (3 gates x its units, of W_ih and of W_hh: ~213 KB at d=4096)
//     into TMEM once per call and reads them from there at every position with tcgen05.ld.
//     Only W2 (77.8 MB at V=151936) then cycles through L2 between positions, which fits; with
//     the GRU rows also streaming, the ~110 MB per-position working set thrashed L2.
//     TMEM layout: lane l holds elements [l*d/128, (l+1)*d/128) of every row, row R of W_ih in
//     columns [R*d/256, (R+1)*d/256) and the W_hh rows after them (packed bf16 pairs).
//  2. The W2 stream is register double-buffered (the next chunk's loads are issued before the
//     current chunk is reduced) and its first chunk is issued between barrier arrival and wait.
//     (Staging it through shared memory -- a ring of 1-D bulk copies, or of cp.async chunks three
//     ahead per warp -- measured slower: 198 and 191 us for the W2 pass against 129 us.)
//  3. The W1 state-block partials are spread over kRep replicas of the accumulator, cutting the
//     number of same-address atomics per replica from G to G/kRep.  Every partial sum that
//     several CTAs or warps add into (these accumulators, and the GRU gate sums in shared
//     memory) is kept in 64-bit fixed point (fix_add), so the order in which the atomics land
//     does not change a single bit: two calls on the same inputs give identical outputs.
// Teacher-forced mode (tf_tokens set): the given tokens drive the GRU, so the kernel runs only the
// L - 1 state updates (TMEM-resident rows, one grid barrier each) and writes every state; the
// activations and logits of all positions then come from two batched tensor-core products.
// Every wait is bounded; on a timeout the CTA frees its TMEM and returns.
#include "common.cuh"
#include "persistent.h"
#include "tmem.cuh"

#include <algorithm>
#include <type_traits>

namespace domino {

namespace {

constexpr int kThreads2 = 512;
constexpr int kWarps2 = kThreads2 / 32;
constexpr int kR2 = 256;
constexpr int kRep = kAccReplicas;
constexpr int kTmemCols = 512;
constexpr size_t kMinSmem = 120 * 1024;  // more than half an SM's shared memory: one CTA per SM

struct TArgs {
  const bf16 *embed, *W_ih, *W_hh, *b_ih, *b_hh, *W1, *W2;
  const bf16 *Lb, *H;
  const float* S0;
  int32_t* tokens;
  float* logits;
  float* states;
  uint64_t* keys;   // [L][B]
  unsigned long long* a_acc;  // [2][kRep][B][r] W1 state-block sums, fixed point, position i in slot i & 1
  float* P;         // [L][B][r] W1[:, :d] . H[b, i]
  float* Sbuf;      // [2][B][Hs]
  unsigned* bar;
  int32_t* status;
  int B, L, d, Hs, V, maxu;
  unsigned long long spin_limit;
  unsigned long long* trace;  // [ntrace] SM clock stamps, or null
  int ntrace;
  const float* Xp;  // [V][3Hs] input projection of the embedding table, or null
  const int32_t* tf_tokens;  // [B][L] given tokens (teacher-forced mode), or null (greedy)
  const float* Gx;           // teacher-forced mode: [B][L-1][3Hs] W_ih . embed[y_i] precomputed, or null
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_s32(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
// W2 rows are re-read at every position: a plain non-coherent load keeps them in L2.  (With an
// L1::no_allocate qualifier the lines were not retained in L2 either and every position
// streamed W2 from HBM.)
__device__ __forceinline__ uint4 ldg16_w2(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Optional phase trace (set through domino_debug_set_trace): SM clock of CTA 0, thread 0.
__device__ __forceinline__ void stamp(unsigned long long* trace, int ntrace, int k) {
  if (trace && k < ntrace && blockIdx.x == 0 && threadIdx.x == 0) trace[k] = clock64();
}

// Split-phase grid barrier on a monotonic counter: arrive, do independent work, then wait.  (A
// separate release flag written by the last arrival was measured slower: its extra round trip is
// serial, while polling the counter itself costs nothing the waits can feel.)
__device__ __forceinline__ void grid_arrive(const TArgs& p, unsigned& epoch) {
  __syncthreads();
  ++epoch;
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(p.bar, 1u);
  }
}
__device__ bool grid_wait(const TArgs& p, unsigned epoch, int* flag_s) {
  if (threadIdx.x == 0) {
    const unsigned target = epoch * gridDim.x;
    bool ok = false;
    for (unsigned long long it = 0; it < p.spin_limit; ++it) {
      if (ld_acquire_u32(p.bar) >= target) { ok = true; break; }
      if ((it & 31) == 31 && ld_relaxed_s32(p.status) == DOMINO_STATUS_DEVICE_TIMEOUT) break;
    }
    if (!ok) set_status(p.status, DOMINO_STATUS_DEVICE_TIMEOUT);
    __threadfence();
    *flag_s = ok ? 1 : 0;
  }
  __syncthreads();
  const bool ok = *flag_s != 0;
  __syncthreads();
  return ok;
}

template <int ROWS>
__device__ __forceinline__ float transpose_reduce2(float (&v)[ROWS], int lane) {
#pragma unroll
  for (int n = ROWS, m = 16; n > 1; n >>= 1, m >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int k = 0; k < n / 2; ++k) {
      const float send = up ? v[k] : v[k + n / 2];
      const float keep = up ? v[k + n / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  float s = v[0];
#pragma unroll
  for (int m = (32 / ROWS) >> 1; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  return s;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Dot products of TMEM-resident rows with per-lane input slices, for the rows R of this warp's
// group (R = group, group + 4, ...), four rows per pass.  Row R sits at columns
// [col0 + R*cpr, col0 + (R+1)*cpr) of every lane.  Input for batch row b, word c of lane l is
//   bf16 pair x_t[(b*cpr + c)*128 + l]           (In = uint32_t, the embedding row), or
//   floats    s_t[(b*2cpr + 2c + {0,1})*128 + l] (In = float, the previous state).
// Sums go to acc_s[b*acc_stride + R] with fixed-point shared-memory atomics (4 warps share each
// row; the total does not depend on their order).
template <int BMAX, typename In, int CH>
__device__ void tmem_rows_dot_ch(uint32_t tbase, int col0, int cpr, int nrows, const In* in_t, int B,
                                 unsigned long long* acc_s, int acc_stride, int warp, int lane) {
  const int q = warp & 3, group = warp >> 2;
  const int l = q * 32 + lane;
  const uint32_t taddr_lane = tbase + ((uint32_t)(q * 32) << 16);
  for (int r0 = group; r0 < nrows; r0 += 16) {  // rows r0, r0+4, r0+8, r0+12
    float acc[BMAX][4];
#pragma unroll
    for (int b = 0; b < BMAX; ++b)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[b][k] = 0.f;
    for (int c = 0; c < cpr; c += CH) {
      // CH columns of four rows in flight, one wait
      uint32_t w[4][CH];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int R = r0 + 4 * k;
        const int Rc = R < nrows ? R : r0;  // keep the warp's loads uniform; masked below
        tmem_ld<CH>(taddr_lane + (uint32_t)(col0 + Rc * cpr + c), w[k]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int e = 0; e < CH; ++e) reg_fence(w[k][e]);
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        if (b < B) {
#pragma unroll
          for (int e = 0; e < CH; ++e) {
            float x0, x1;
            if constexpr (!std::is_same<In, float>::value) {
              const uint32_t xa = in_t[((size_t)b * cpr + c + e) * 128 + l];
              x0 = bf_lo(xa); x1 = bf_hi(xa);
            } else {
              x0 = in_t[((size_t)b * 2 * cpr + 2 * (c + e)) * 128 + l];
              x1 = in_t[((size_t)b * 2 * cpr + 2 * (c + e) + 1) * 128 + l];
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc[b][k] = fmaf(bf_lo(w[k][e]), x0, acc[b][k]);
              acc[b][k] = fmaf(bf_hi(w[k][e]), x1, acc[b][k]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BMAX; ++b) {
      if (b < B) {
        const float s = transpose_reduce2<4>(acc[b], lane);
        const int R = r0 + 4 * (lane >> 3);
        if ((lane & 7) == 0 && R < nrows) fix_add(acc_s + b * acc_stride + R, s);
      }
    }
  }
}

// Dot products of TMEM-resident rows with per-lane input slices, for the rows R of this warp's
// group (R = group, group + 4, ...), four rows per pass.  Row R sits at columns
// [col0 + R*cpr, col0 + (R+1)*cpr) of every lane.  Input for batch row b, word c of lane l is
//   bf16 pair x_t[(b*cpr + c)*128 + l]           (In = uint32_t, the embedding row), or
//   floats    s_t[(b*2cpr + 2c + {0,1})*128 + l] (In = float, the previous state).
// Sums go to acc_s[b*acc_stride + R] in fixed point (see tmem_rows_dot_ch).
// cpr is even; the widest load that divides it is used.
template <int BMAX, typename In>
__device__ void tmem_rows_dot(uint32_t tbase, int col0, int cpr, int nrows, const In* in_t, int B,
                              unsigned long long* acc_s, int acc_stride, int warp, int lane) {
  if (cpr % 8 == 0)
    tmem_rows_dot_ch<BMAX, In, 8>(tbase, col0, cpr, nrows, in_t, B, acc_s, acc_stride, warp, lane);
  else if (cpr % 4 == 0)
    tmem_rows_dot_ch<BMAX, In, 4>(tbase, col0, cpr, nrows, in_t, B, acc_s, acc_stride, warp, lane);
  else
    tmem_rows_dot_ch<BMAX, In, 2>(tbase, col0, cpr, nrows, in_t, B, acc_s, acc_stride, warp, lane);
}

template <int BMAX, int ROWS>
__device__ __forceinline__ void w2_load(const TArgs& p, int v0, int v1, int ch, int lane, size_t lrow, int L,
                                        uint4 (&q)[ROWS], float (&lb)[BMAX]) {
  const int vb = v0 + ch * ROWS;
#pragma unroll
  for (int k = 0; k < ROWS; ++k)
    q[k] = (vb + k < v1) ? ldg16_w2(p.W2 + (size_t)(vb + k) * kR2 + lane * 8) : make_uint4(0u, 0u, 0u, 0u);
  const int v = vb + (lane / (32 / ROWS));
#pragma unroll
  for (int b = 0; b < BMAX; ++b)
    lb[b] = (b < p.B && (lane & (32 / ROWS - 1)) == 0 && v < v1)
                ? __bfloat162float(p.Lb[lrow + (size_t)b * L * p.V + v]) : 0.f;
}

template <int BMAX, int ROWS>
__device__ __forceinline__ void w2_chunk(const TArgs& p, int v0, int v1, int ch, int lane, size_t lrow, int L,
                                         const uint4 (&q)[ROWS], const float (&lb)[BMAX],
                                         const float (&uv)[BMAX][8], uint64_t (&best)[BMAX]) {
  float acc[BMAX][ROWS];
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    float w[8];
    widen(q[k], w);
#pragma unroll
    for (int b = 0; b < BMAX; ++b) {
      float a = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) a = fmaf(w[e], uv[b][e], a);
      acc[b][k] = a;
    }
  }
  const int v = v0 + ch * ROWS + lane / (32 / ROWS);
#pragma unroll
  for (int b = 0; b < BMAX; ++b) {
    if (b < p.B) {
      const float s = transpose_reduce2<ROWS>(acc[b], lane);
      if ((lane & (32 / ROWS - 1)) == 0 && v < v1) {
        const float z = lb[b] + s;
        if (p.logits) p.logits[lrow + (size_t)b * L * p.V + v] = z;
        best[b] = umax64(best[b], argmax_key(z, v));
      }
    }
  }
}

template <int BMAX, int ROWS>
__global__ void __launch_bounds__(kThreads2, 1) k_greedy_tmem(TArgs p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int G = gridDim.x, c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = p.B, L = p.L, d = p.d, Hs = p.Hs, V = p.V, maxu = p.maxu;
  const int v0 = (int)((long long)V * c / G), v1 = (int)((long long)V * (c + 1) / G);
  const int j0 = (int)((long long)Hs * c / G), j1 = (int)((long long)Hs * (c + 1) / G);
  const int nu = j1 - j0;
  const int ldw1 = d + Hs;
  const int cpri = d / 256, cprh = Hs / 256;       // TMEM columns per W_ih / W_hh row
  // GRU input half gathered from the projection table (per token) or from precomputed teacher-forced
  // gates (per row and position): the W_ih rows are then not kept in TMEM
  const bool proj = p.Xp != nullptr || p.Gx != nullptr;
  const int colh = proj ? 0 : 3 * nu * cpri;       // first W_hh column
  const int rep = c % kRep;

  // shared memory
  float* u_s = reinterpret_cast<float*>(smem);                          // [BMAX][256]
  float* s_t = u_s + BMAX * kR2;                                        // [BMAX][2*cprh][128] S_{i-1}
  uint32_t* x_t = reinterpret_cast<uint32_t*>(s_t + (size_t)BMAX * Hs); // [BMAX][cpri][128]  embed[t_i]
  float* w1s_s = reinterpret_cast<float*>(x_t + (size_t)BMAX * (d / 2));  // [maxu][256]
  // gate sums W_hh . S and W_ih . x for the own units, fixed point (8-byte aligned: every piece
  // before them is a multiple of 8 bytes)
  unsigned long long* gh_s = reinterpret_cast<unsigned long long*>(w1s_s + (size_t)maxu * kR2);  // [BMAX][3*maxu]
  unsigned long long* gi_s = gh_s + BMAX * 3 * maxu;                    // [BMAX][3*maxu]
  float* sn_s = reinterpret_cast<float*>(gi_s + BMAX * 3 * maxu);       // [BMAX][maxu]
  float* bias_s = sn_s + ((BMAX * maxu + 3) & ~3);                      // [2][3][maxu] b_ih, b_hh (own units)
  uint64_t* best_s = reinterpret_cast<uint64_t*>(bias_s + ((6 * maxu + 3) & ~3));  // [warps][BMAX]
  int* tok_s = reinterpret_cast<int*>(best_s + kWarps2 * BMAX);        // [BMAX]
  int* flag_s = tok_s + BMAX;
  uint32_t* tbase_s = reinterpret_cast<uint32_t*>(flag_s + 1);
  unsigned epoch = 0;

  // ---- TMEM: one allocation for the whole call ----
  if (warp == 0) {
    tmem_alloc(tbase_s, kTmemCols);
    tmem_relinquish();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *tbase_s;
  auto leave = [&]() {
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, kTmemCols);
  };

  stamp(p.trace, p.ntrace, 0);
  // ---- prologue ----
  // GRU rows into TMEM.  Warp (quadrant q, group g) stores rows R = g, g+4, ... of its lanes:
  // the same warps read them back later, so no cross-warp ordering is involved.
  {
    const int q = warp & 3, group = warp >> 2, l = q * 32 + lane;
    const uint32_t ta = tbase + ((uint32_t)(q * 32) << 16);
    // cpri and cprh are even; rows are copied in 16-byte (x4) or 8-byte (x2) pieces
    for (int R = group; R < 3 * nu; R += 4) {
      const int g = R / nu, jj = R % nu;
      const uint32_t* ri = reinterpret_cast<const uint32_t*>(p.W_ih + ((size_t)g * Hs + j0 + jj) * d) + l * cpri;
      const uint32_t* rh = reinterpret_cast<const uint32_t*>(p.W_hh + ((size_t)g * Hs + j0 + jj) * Hs) + l * cprh;
      if (proj) {
      } else if (cpri % 4 == 0) {
        for (int cc = 0; cc < cpri; cc += 4)
          tmem_st4(ta + (uint32_t)(R * cpri + cc), __ldg(reinterpret_cast<const uint4*>(ri + cc)));
      } else {
        for (int cc = 0; cc < cpri; cc += 2) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(ri + cc));
          tmem_st2(ta + (uint32_t)(R * cpri + cc), v.x, v.y);
        }
      }
      if (cprh % 4 == 0) {
        for (int cc = 0; cc < cprh; cc += 4)
          tmem_st4(ta + (uint32_t)(colh + R * cprh + cc), __ldg(reinterpret_cast<const uint4*>(rh + cc)));
      } else {
        for (int cc = 0; cc < cprh; cc += 2) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(rh + cc));
          tmem_st2(ta + (uint32_t)(colh + R * cprh + cc), v.x, v.y);
        }
      }
    }
    tmem_wait_st();
  }
  const bool tf = p.tf_tokens != nullptr;
  for (int k = tid; k < maxu * kR2 && !tf; k += kThreads2) {
    const int jj = k / kR2, kk = k % kR2;
    w1s_s[k] = (jj < nu) ? __bfloat162float(p.W1[(size_t)kk * ldw1 + d + j0 + jj]) : 0.f;
  }
  for (int k = tid; k < BMAX * 6 * maxu; k += kThreads2) gh_s[k] = 0ull;  // gh_s and gi_s
  for (int k = tid; k < 6 * maxu; k += kThreads2) {  // the own units' biases, read at every update
    const int h = k / (3 * maxu), g = (k / maxu) % 3, jj = k % maxu;
    bias_s[k] = jj < nu ? __bfloat162float((h ? p.b_hh : p.b_ih)[(size_t)g * Hs + j0 + jj]) : 0.f;
  }
  // P[i][b][k] = W1[k, :d] . H[b, i]  for the rank rows k = c, c + G, ... (one warp per value)
  if (!tf) {
    const int nk = (kR2 - c + G - 1) / G;
    const int npos = B * L;
    const int nseg = d / 256;
    for (int item = warp; item < nk * npos; item += kWarps2) {
      const int k = c + (item / npos) * G, n = item % npos;
      const bf16* wr = p.W1 + (size_t)k * ldw1;
      const bf16* hr = p.H + (size_t)n * d;
      float acc0 = 0.f, acc1 = 0.f;
      int s = 0;
      for (; s + 1 < nseg; s += 2) {
        const uint4 h0 = ldg16(hr + s * 256 + lane * 8), w0 = ldg16(wr + s * 256 + lane * 8);
        const uint4 h1 = ldg16(hr + (s + 1) * 256 + lane * 8), w1 = ldg16(wr + (s + 1) * 256 + lane * 8);
        float x[8], y[8];
        widen(h0, x); widen(w0, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc0 = fmaf(y[e], x[e], acc0);
        widen(h1, x); widen(w1, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc1 = fmaf(y[e], x[e], acc1);
      }
      for (; s < nseg; ++s) {
        float x[8], y[8];
        widen(ldg16(hr + s * 256 + lane * 8), x);
        widen(ldg16(wr + s * 256 + lane * 8), y);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc0 = fmaf(y[e], x[e], acc0);
      }
      const float acc = warp_sum(acc0 + acc1);
      const int b = n / L, i = n % L;
      if (lane == 0) p.P[((size_t)i * B + b) * kR2 + k] = acc;
    }
  }
  __syncthreads();
  // a_acc[0][rep][b] += W1[:, d + own units] . S0[b, own units];  states_out[b, 0] = S0[b]
  // (slot 1 is zero at launch; slot i & 1 is cleared again once every CTA has read it)
  for (int t = tid; t < BMAX * (kR2 / 4) && !tf; t += kThreads2) {
    const int b = t / (kR2 / 4), k4 = (t % (kR2 / 4)) * 4;
    if (b < B && nu > 0) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int jj = 0; jj < nu; ++jj) {
        const float h = p.S0[(size_t)b * Hs + j0 + jj];
        const float* w = w1s_s + jj * kR2 + k4;
        s.x = fmaf(w[0], h, s.x); s.y = fmaf(w[1], h, s.y); s.z = fmaf(w[2], h, s.z); s.w = fmaf(w[3], h, s.w);
      }
      unsigned long long* acc = p.a_acc + ((size_t)rep * B + b) * kR2 + k4;
      fix_add(acc, s.x); fix_add(acc + 1, s.y); fix_add(acc + 2, s.z); fix_add(acc + 3, s.w);
    }
  }
  if (p.states)
    for (int t = tid; t < B * nu; t += kThreads2) {
      const int b = t / nu, jj = t % nu;
      p.states[(size_t)b * L * Hs + j0 + jj] = p.S0[(size_t)b * Hs + j0 + jj];
    }
  // L_base rows of position 0 towards L2
  for (int t = tid; t < B * ((v1 - v0 + 63) / 64) && !tf; t += kThreads2) {
    const int b = t / ((v1 - v0 + 63) / 64), ln = t % ((v1 - v0 + 63) / 64);
    if (v0 + ln * 64 < v1) prefetch_l2(p.Lb + (size_t)b * L * V + v0 + ln * 64);
  }

  const int nrows = v1 - v0;
  const int nch = (nrows + ROWS - 1) / ROWS;
  uint4 qa[ROWS], qb[ROWS];
  float lba[BMAX], lbb[BMAX];

  stamp(p.trace, p.ntrace, 1);
  grid_arrive(p, epoch);
  if (!tf && warp < nch) w2_load<BMAX, ROWS>(p, v0, v1, warp, lane, 0, L, qa, lba);
  if (!grid_wait(p, epoch, flag_s)) { leave(); return; }
  stamp(p.trace, p.ntrace, 2);

  for (int i = 0; i < L; ++i) {
    const size_t lrow = (size_t)i * V;
    if (tf) {  // ---- teacher-forced step: t_i given; W_hh . S_{i-1} for the own units ----
      if (i == L - 1) break;
      if (tid < B) {
        int tok = p.tf_tokens[(size_t)tid * L + i];
        if (tok < 0 || tok >= V) {
          set_status(p.status, DOMINO_STATUS_BAD_TOKEN);
          tok = 0;
        }
        tok_s[tid] = tok;
      }
      const float* Sprev = (i == 0) ? p.S0 : p.Sbuf + (size_t)((i - 1) & 1) * B * Hs;
      for (int t = tid; t < B * Hs; t += kThreads2) {
        const int b = t / Hs, j = t % Hs;
        s_t[((size_t)b * 2 * cprh + j % (2 * cprh)) * 128 + j / (2 * cprh)] = __ldcg(Sprev + t);
      }
      __syncthreads();
      if (nu > 0) tmem_rows_dot<BMAX, float>(tbase, colh, cprh, 3 * nu, s_t, B, gh_s, 3 * maxu, warp, lane);
      stamp(p.trace, p.ntrace, 4 + 10 * i + 3);
    } else {
    // u = SiLU(P + the state block: the accumulator replicas, added as integers)
    for (int t = tid; t < BMAX * kR2; t += kThreads2) {
      const int b = t / kR2, k = t % kR2;
      float a = 0.f;
      if (b < B) {
        unsigned long long q = 0ull;
#pragma unroll
        for (int r = 0; r < kRep; ++r) q += __ldcg(p.a_acc + (((size_t)(i & 1) * kRep + r) * B + b) * kR2 + k);
        a = __ldcg(p.P + ((size_t)i * B + b) * kR2 + k) + fix_value(q);
      }
      u_s[t] = (b < B) ? siluf_(a) : 0.f;
    }
    // L_base rows of the next position towards L2
    if (i + 1 < L)
      for (int t = tid; t < B * ((nrows + 63) / 64); t += kThreads2) {
        const int b = t / ((nrows + 63) / 64), ln = t % ((nrows + 63) / 64);
        if (v0 + ln * 64 < v1) prefetch_l2(p.Lb + lrow + V + (size_t)b * L * V + v0 + ln * 64);
      }
    __syncthreads();
    const int tb = 4 + 10 * i;
    stamp(p.trace, p.ntrace, tb + 0);

    stamp(p.trace, p.ntrace, tb + 1);

    // z = L_base + W2 . u over [v0, v1) with the argmax folded in; register double-buffered
    {
      float uv[BMAX][8];
#pragma unroll
      for (int b = 0; b < BMAX; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) uv[b][e] = u_s[b * kR2 + lane * 8 + e];
      uint64_t best[BMAX];
#pragma unroll
      for (int b = 0; b < BMAX; ++b) best[b] = 0ull;
      for (int ch = warp; ch < nch; ch += 2 * kWarps2) {
        if (ch + kWarps2 < nch) w2_load<BMAX, ROWS>(p, v0, v1, ch + kWarps2, lane, lrow, L, qb, lbb);
        w2_chunk<BMAX, ROWS>(p, v0, v1, ch, lane, lrow, L, qa, lba, uv, best);
        if (ch + kWarps2 >= nch) break;
        if (ch + 2 * kWarps2 < nch) w2_load<BMAX, ROWS>(p, v0, v1, ch + 2 * kWarps2, lane, lrow, L, qa, lba);
        w2_chunk<BMAX, ROWS>(p, v0, v1, ch + kWarps2, lane, lrow, L, qb, lbb, uv, best);
      }
#pragma unroll
      for (int b = 0; b < BMAX; ++b) {
        uint64_t m = best[b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = umax64(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) best_s[warp * BMAX + b] = m;
      }
      __syncthreads();
      if (tid < B) {
        uint64_t m = 0ull;
        for (int w = 0; w < kWarps2; ++w) m = umax64(m, best_s[w * BMAX + tid]);
        atomicMax(reinterpret_cast<unsigned long long*>(p.keys + (size_t)i * B + tid), (unsigned long long)m);
        tok_s[tid] = min(max(key_index(m), 0), V - 1);
      }
    }
    stamp(p.trace, p.ntrace, tb + 2);
    grid_arrive(p, epoch);
    // While the other CTAs finish their vocabulary slices: pull this CTA's own best row of the
    // embedding table into L2 (the global winner's row is then an L2 hit for every CTA), and do
    // the W_hh half of the GRU, which does not depend on the argmax.
    if (i < L - 1) {
      if (proj) {
        for (int t = tid; t < B * (3 * Hs / 32); t += kThreads2) {
          const int b = t / (3 * Hs / 32), ln = t % (3 * Hs / 32);
          prefetch_l2(p.Xp + (size_t)tok_s[b] * 3 * Hs + ln * 32);
        }
      } else {
        for (int t = tid; t < B * (d / 64); t += kThreads2) {
          const int b = t / (d / 64), ln = t % (d / 64);
          prefetch_l2(p.embed + (size_t)tok_s[b] * d + ln * 64);
        }
      }
      const float* Sprev = (i == 0) ? p.S0 : p.Sbuf + (size_t)((i - 1) & 1) * B * Hs;
      for (int t = tid; t < B * Hs; t += kThreads2) {
        const int b = t / Hs, j = t % Hs;
        s_t[((size_t)b * 2 * cprh + j % (2 * cprh)) * 128 + j / (2 * cprh)] = __ldcg(Sprev + t);
      }
      __syncthreads();
      if (nu > 0) tmem_rows_dot<BMAX, float>(tbase, colh, cprh, 3 * nu, s_t, B, gh_s, 3 * maxu, warp, lane);
    }
    if (!grid_wait(p, epoch, flag_s)) { leave(); return; }
    stamp(p.trace, p.ntrace, tb + 3);
    if (i == L - 1) break;
    // every CTA has read slot i & 1 (before the barrier just passed): clear this CTA's share of it
    // for position i + 2, whose sums are added only after the next barrier
    {
      const int n = kRep * B * kR2, z0 = (int)((long long)n * c / G), z1 = (int)((long long)n * (c + 1) / G);
      for (int t = z0 + tid; t < z1; t += kThreads2) p.a_acc[(size_t)(i & 1) * n + t] = 0ull;
    }
    }  // greedy step
    const int tb = 4 + 10 * i;

    // t_i; gi = W_ih . embed[t_i] for the own units: gathered from the projection table, or
    // computed from TMEM with the embedding row staged in the lane-sliced layout; GRU cell -> S_i
    if (!tf) {  // the global argmax of each row, read once (tok_s held this CTA's own candidate)
      if (tid < B) tok_s[tid] = min(max(key_index(__ldcg(p.keys + (size_t)i * B + tid)), 0), V - 1);
      __syncthreads();
    }
    if (proj) {
      for (int t = tid; t < B * 3 * nu; t += kThreads2) {
        const int b = t / (3 * nu), R = t % (3 * nu), g = R / nu, jj = R % nu;
        if (p.Gx) {  // teacher forcing: the gates of (row b, position i) were computed up front
          gi_s[b * 3 * maxu + R] = fix_of(__ldg(p.Gx + ((size_t)b * (L - 1) + i) * 3 * Hs + (size_t)g * Hs + j0 + jj));
          continue;
        }
        gi_s[b * 3 * maxu + R] = fix_of(__ldg(p.Xp + (size_t)tok_s[b] * 3 * Hs + (size_t)g * Hs + j0 + jj));
      }
      __syncthreads();
      stamp(p.trace, p.ntrace, tb + 4);
    } else {
      for (int t = tid; t < B * (d / 2); t += kThreads2) {
        const int b = t / (d / 2), w = t % (d / 2);
        x_t[((size_t)b * cpri + w % cpri) * 128 + w / cpri] =
            __ldg(reinterpret_cast<const uint32_t*>(p.embed + (size_t)tok_s[b] * d) + w);
      }
      __syncthreads();
      stamp(p.trace, p.ntrace, tb + 4);
      if (nu > 0) tmem_rows_dot<BMAX, uint32_t>(tbase, 0, cpri, 3 * nu, x_t, B, gi_s, 3 * maxu, warp, lane);
    }
    __syncthreads();
    stamp(p.trace, p.ntrace, tb + 5);
    float* Snext = p.Sbuf + (size_t)(i & 1) * B * Hs;
    for (int t = tid; t < B * nu; t += kThreads2) {
      const int b = t / nu, jj = t % nu, j = j0 + jj;
      float gi[3], gh[3];
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        gi[g] = fix_value(gi_s[b * 3 * maxu + g * nu + jj]) + bias_s[g * maxu + jj];
        gh[g] = fix_value(gh_s[b * 3 * maxu + g * nu + jj]) + bias_s[(3 + g) * maxu + jj];
        gi_s[b * 3 * maxu + g * nu + jj] = 0ull;
        gh_s[b * 3 * maxu + g * nu + jj] = 0ull;
      }
      const float rg = sigmoidf_(gi[0] + gh[0]);
      const float zg = sigmoidf_(gi[1] + gh[1]);
      const float ng = tanhf(gi[2] + rg * gh[2]);
      const float hprev = s_t[((size_t)b * 2 * cprh + j % (2 * cprh)) * 128 + j / (2 * cprh)];
      const float hn = (1.f - zg) * ng + zg * hprev;
      sn_s[b * maxu + jj] = hn;
      Snext[(size_t)b * Hs + j] = hn;
      if (p.states) p.states[((size_t)b * L + i + 1) * Hs + j] = hn;
    }
    __syncthreads();
    for (int t = tid; t < BMAX * (kR2 / 4) && !tf; t += kThreads2) {
      const int b = t / (kR2 / 4), k4 = (t % (kR2 / 4)) * 4;
      if (b < B && nu > 0) {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int jj = 0; jj < nu; ++jj) {
          const float h = sn_s[b * maxu + jj];
          const float* w = w1s_s + jj * kR2 + k4;
          s.x = fmaf(w[0], h, s.x); s.y = fmaf(w[1], h, s.y); s.z = fmaf(w[2], h, s.z); s.w = fmaf(w[3], h, s.w);
        }
        unsigned long long* acc = p.a_acc + (((size_t)((i + 1) & 1) * kRep + rep) * B + b) * kR2 + k4;
        fix_add(acc, s.x); fix_add(acc + 1, s.y); fix_add(acc + 2, s.z); fix_add(acc + 3, s.w);
      }
    }
    stamp(p.trace, p.ntrace, tb + 6);
    grid_arrive(p, epoch);
    if (!tf && warp < nch) w2_load<BMAX, ROWS>(p, v0, v1, warp, lane, lrow + V, L, qa, lba);
    if (!grid_wait(p, epoch, flag_s)) { leave(); return; }
    stamp(p.trace, p.ntrace, tb + 7);
  }
  if (c == 0 && !tf)
    for (int t = tid; t < B * L; t += kThreads2) {
      const int b = t / L, i = t % L;
      p.tokens[t] = key_index(__ldcg(p.keys + (size_t)i * B + b));
    }
  stamp(p.trace, p.ntrace, 3);
  leave();
}

// Shared memory of the kernel's working arrays.
size_t smem_work_bytes(int bmax, int d, int Hs, int maxu) {
  size_t bytes = ((size_t)bmax * kR2 + (size_t)bmax * Hs) * 4 + (size_t)bmax * (d / 2) * 4;
  bytes += ((size_t)maxu * kR2 + (((size_t)bmax * maxu + 3) & ~(size_t)3) + ((6 * (size_t)maxu + 3) & ~(size_t)3)) * 4 +
           6 * (size_t)bmax * maxu * 8;
  bytes += (size_t)kWarps2 * bmax * 8 + (size_t)bmax * 4 + 16;
  return (bytes + 15) & ~(size_t)15;
}
size_t smem_bytes_tmem(int bmax, int d, int Hs, int maxu) {
  const size_t bytes = smem_work_bytes(bmax, d, Hs, maxu);
  return bytes < kMinSmem ? kMinSmem : bytes;
}

template <int BMAX, int ROWS>
cudaError_t launch_tmem_t(const TArgs& a, int G, size_t smem, cudaStream_t st) {
  auto kern = k_greedy_tmem<BMAX, ROWS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads2, smem);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorCooperativeLaunchTooLarge;  // TMEM plan needs exactly one CTA per SM
  TArgs args = a;
  void* params[] = {&args};
  return cudaLaunchCooperativeKernel((const void*)kern, dim3(G), dim3(kThreads2), params, smem, st);
}

}  // namespace

bool tmem_plan_fits(const Shape& s, int G, bool proj) {
  if (G < 1 || s.d % 512 != 0 || s.Hs % 512 != 0) return false;
  const int maxu = (s.Hs + G - 1) / G;
  return 3 * maxu * ((proj ? 0 : s.d / 256) + s.Hs / 256) <= kTmemCols &&
         smem_bytes_tmem(4, s.d, s.Hs, maxu) <= 200 * 1024;
}

namespace {
cudaError_t launch_tmem_common(const Shape& s, const domino_weights_t& w, const void* base_logits, const void* hidden,
                               const float* S0, int32_t* tokens_out, float* logits_out, float* states_out,
                               const Workspace& ws, int32_t* status, uint64_t spin, int G, cudaStream_t st,
                               const int32_t* tf_tokens, const float* Gx) {
  TArgs a{};
  a.tf_tokens = tf_tokens;
  a.Gx = Gx;
  a.embed = (const bf16*)w.embed; a.W_ih = (const bf16*)w.W_ih; a.W_hh = (const bf16*)w.W_hh;
  a.b_ih = (const bf16*)w.b_ih; a.b_hh = (const bf16*)w.b_hh; a.W1 = (const bf16*)w.W1; a.W2 = (const bf16*)w.W2;
  a.Lb = (const bf16*)base_logits; a.H = (const bf16*)hidden; a.S0 = S0;
  a.tokens = tokens_out; a.logits = logits_out; a.states = states_out;
  a.keys = ws.keys; a.a_acc = ws.a_acc; a.P = ws.P; a.Sbuf = ws.S; a.bar = ws.sync; a.status = status;
  a.B = s.B; a.L = s.L; a.d = s.d; a.Hs = s.Hs; a.V = s.V;
  a.maxu = (s.Hs + G - 1) / G;
  a.spin_limit = spin;
  a.Xp = w.embed_proj;
  debug_trace(&a.trace, &a.ntrace);
  // barrier counter, argmax keys and accumulators are contiguous in the workspace: one memset
  const size_t zero_bytes = (size_t)((char*)ws.a_acc + acc_bytes(s.B, s.r) - (char*)ws.sync);
  cudaError_t e = cudaMemsetAsync(ws.sync, 0, zero_bytes, st);
  if (e != cudaSuccess) return e;
  const int bmax = s.B <= 1 ? 1 : (s.B <= 2 ? 2 : 4);
  const size_t smem = smem_bytes_tmem(bmax, s.d, s.Hs, a.maxu);
  if (bmax == 1) e = launch_tmem_t<1, 8>(a, G, smem, st);
  else if (bmax == 2) e = launch_tmem_t<2, 8>(a, G, smem, st);
  else e = launch_tmem_t<4, 4>(a, G, smem, st);
  return note_launch(e);
}
}  // namespace

cudaError_t launch_greedy_tmem(const Shape& s, const domino_weights_t& w, const void* base_logits, const void* hidden,
                               const float* S0, int32_t* tokens_out, float* logits_out, float* states_out,
                               const Workspace& ws, int32_t* status, uint64_t spin, int G, cudaStream_t st) {
  return launch_tmem_common(s, w, base_logits, hidden, S0, tokens_out, logits_out, states_out, ws, status, spin, G, st,
                            nullptr, nullptr);
}

cudaError_t launch_tf_recurrence_tmem(const Shape& s, const domino_weights_t& w, const float* S0, const int32_t* tokens,
                                      const float* Gx, float* states, const Workspace& ws, int32_t* status,
                                      uint64_t spin, int G, cudaStream_t st) {
  return launch_tmem_common(s, w, nullptr, nullptr, S0, nullptr, nullptr, states, ws, status, spin, G, st, tokens, Gx);
}

}  // namespace domino
