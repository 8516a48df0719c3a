// api.cu -- the C ABI of libdomino: argument checks, workspace layout and launch sequencing.
// Every entry point validates on the host, then enqueues kernels on the caller's stream; it
// never synchronises and never allocates.
#include "domino.h"
#include "internal.h"
#include "gemm_tc.h"
#include "persistent.h"

#include <algorithm>
#include <atomic>
#include <string>

namespace domino {

namespace {

std::atomic<uint64_t> g_spin_limit{0};
std::atomic<uint64_t> g_launches{0};
std::atomic<unsigned long long*> g_trace{nullptr};
std::atomic<int> g_ntrace{0};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Largest B * L any entry point accepts (grid y of the row-per-block launches).
constexpr int64_t kMaxRows = 65535;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// K dimension in 16-byte vectors: a multiple of 32 vectors, or a power of two up to 32.
inline bool vec_layout_ok(int K, int dtype) {
  int nv = K / (dtype == DOMINO_DTYPE_F32 ? 4 : 8);
  if (nv < 1) return false;
  if (nv % 32 == 0) return true;
  return nv <= 32 && (nv & (nv - 1)) == 0;
}

}  // namespace

int check_shape(const domino_shape_t* s) {
  if (!s) return DOMINO_ERR_INVALID_ARGUMENT;
  if (s->dtype != DOMINO_DTYPE_F32 && s->dtype != DOMINO_DTYPE_BF16) return DOMINO_ERR_INVALID_ARGUMENT;
  if (s->B < 1 || s->L < 1 || s->L > DOMINO_MAX_L || s->d < 8 || s->Hs < 8 || s->r < 8 || s->V < 8)
    return DOMINO_ERR_INVALID_ARGUMENT;
  if (s->d % 8 || s->Hs % 8 || s->r % 8 || s->V % 8) return DOMINO_ERR_INVALID_ARGUMENT;
  // launches with one row (or row tile) per block along grid y need B*L <= 65535; element loops over
  // B*Hs and B*L*d/8 count in 32-bit integers
  const int64_t BL = (int64_t)s->B * s->L;
  if (BL > kMaxRows || BL * std::max<int64_t>(s->Hs, s->d / 8) > INT32_MAX) return DOMINO_ERR_UNSUPPORTED;
  if (s->r > 1024) return DOMINO_ERR_UNSUPPORTED;
  if (!vec_layout_ok(s->d, s->dtype) || !vec_layout_ok(s->Hs, s->dtype) || !vec_layout_ok(s->r, s->dtype))
    return DOMINO_ERR_UNSUPPORTED;
  return DOMINO_OK;
}

int check_weights(const domino_weights_t* w) {
  if (!w) return DOMINO_ERR_INVALID_ARGUMENT;
  const void* p[] = {w->embed, w->W_ih, w->W_hh, w->b_ih, w->b_hh, w->W1, w->W2};
  for (const void* q : p)
    if (!q || !aligned16(q)) return DOMINO_ERR_INVALID_ARGUMENT;
  if (w->embed_proj && !aligned16(w->embed_proj)) return DOMINO_ERR_INVALID_ARGUMENT;
  return DOMINO_OK;
}

namespace {

Shape to_shape(const domino_shape_t* s) { return Shape{s->B, s->L, s->d, s->Hs, s->r, s->V, s->dtype}; }

inline int cuda_rc(cudaError_t e) { return e == cudaSuccess ? DOMINO_OK : DOMINO_ERR_CUDA; }

}  // namespace

// One GRU update on the tensor cores for B rows: gh = W_hh . S from the two-term bf16 split of S
// held in ws.S_hl (one GEMM with W_hh repeated along K), gi = W_ih . embed[t] from precomputed
// columns of Gx, or a gather + GEMM here (need_gx), or the projection table; then the cell kernel,
// which also refreshes ws.S_hl with the split of the new state.  Tokens come from keys[b] or
// tokens[b * tok_mul + tok_add]; the Gx column of row b is b*xper + xoff.
cudaError_t gru_step_tc(const Shape& s, const domino_weights_t& w, const Workspace& ws, const float* S_in,
                        size_t s_stride, const uint64_t* keys, const int32_t* tokens, int tok_mul, int tok_add,
                        float* Gx, int ldx, int xper, int xoff, bool need_gx, float* S_out, size_t so_stride,
                        float* S_keep, size_t sk_stride, int32_t* status, cudaStream_t cs) {
  using bf = __nv_bfloat16;
  cudaError_t e = gemm_tc_store_f32_t((const bf*)w.W_hh, ws.S_hl, 3 * s.Hs, s.B, 2 * s.Hs, s.Hs, ws.Gh, 3 * s.Hs,
                                      status, spin_limit(), cs);
  if (e == cudaSuccess && !w.embed_proj && need_gx) {
    e = launch_gather_rows((const bf*)w.embed, keys, tokens, 1, tok_mul, s.B, s.d, s.V, ws.X, cs);
    if (e == cudaSuccess)
      e = gemm_tc_store_f32_t((const bf*)w.W_ih, ws.X, 3 * s.Hs, s.B, s.d, 0, Gx, 3 * s.Hs, status,
                              spin_limit(), cs, 1);
  }
  if (e == cudaSuccess)
    e = launch_cell(s, Gx, ldx, xper, xoff, w.embed_proj, ws.Gh, w.b_ih, w.b_hh, keys, tokens, tok_mul, tok_add,
                    S_in, s_stride, S_out, so_stride, S_keep, sk_stride, status, cs, ws.S_hl);
  return e;
}

Workspace layout_workspace(const Shape& s, void* base) {
  Workspace w{};
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return p ? p + o : nullptr;
  };
  const size_t BL = (size_t)s.B * s.L;
  w.status = reinterpret_cast<int32_t*>(take(sizeof(int32_t)));
  w.sync = reinterpret_cast<uint32_t*>(take(kSyncWords * sizeof(uint32_t)));
  // sync, claim, keys and a_acc are adjacent so that one memset clears them together
  w.claim = reinterpret_cast<uint32_t*>(take(kClaimWords * sizeof(uint32_t)));
  w.keys = reinterpret_cast<uint64_t*>(take(BL * sizeof(uint64_t)));
  w.a_acc = reinterpret_cast<unsigned long long*>(take(acc_bytes(s.B, s.r)));
  w.acc_keys = reinterpret_cast<uint64_t*>(take(BL * sizeof(uint64_t)));
  w.acc_count = reinterpret_cast<uint32_t*>(take((BL + s.B + 1) * sizeof(uint32_t)));
  w.P = reinterpret_cast<float*>(take(BL * s.r * sizeof(float)));
  w.u = reinterpret_cast<float*>(take(BL * s.r * sizeof(float)));
  w.S = reinterpret_cast<float*>(take(2 * (size_t)s.B * s.Hs * sizeof(float)));
  w.states = reinterpret_cast<float*>(take(BL * s.Hs * sizeof(float)));
  w.u16 = reinterpret_cast<__nv_bfloat16*>(take(BL * s.r * sizeof(__nv_bfloat16)));
  w.X = reinterpret_cast<__nv_bfloat16*>(take(BL * s.d * sizeof(__nv_bfloat16)));
  w.Gx = reinterpret_cast<float*>(take(3 * (size_t)s.Hs * BL * sizeof(float)));
  w.Gh = reinterpret_cast<float*>(take(3 * (size_t)s.Hs * s.B * sizeof(float)));
  w.S_hl = reinterpret_cast<__nv_bfloat16*>(take(2 * BL * s.Hs * sizeof(__nv_bfloat16)));
  w.part = reinterpret_cast<float*>(take(batched_partial_floats(s) * sizeof(float)));
  w.bytes = off;
  return w;
}

size_t accept_workspace_bytes(int B, int L) {
  // the accept path uses the status word and acc_keys of the general layout
  Shape s{B, L, 8, 8, 8, 8, DOMINO_DTYPE_F32};
  Workspace w = layout_workspace(s, nullptr);
  return w.bytes;
}

void debug_trace(unsigned long long** buf, int* n) {
  *buf = g_trace.load(std::memory_order_relaxed);
  *n = *buf ? g_ntrace.load(std::memory_order_relaxed) : 0;
}

cudaError_t note_launch(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

uint64_t spin_limit() {
  uint64_t v = g_spin_limit.load(std::memory_order_relaxed);
  return v ? v : kDefaultSpinLimit;
}

}  // namespace domino

using namespace domino;

extern "C" {

int32_t domino_abi_version(void) { return DOMINO_ABI_VERSION; }

uint64_t domino_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* domino_greedy_plan(const domino_shape_t* shape) {
  if (check_shape(shape) != DOMINO_OK) return "invalid shape";
  const Shape s = to_shape(shape);
  if (use_persistent_greedy(s)) return persistent_plan(s);
  if (batched_shape_ok(s)) return batched_plan();
  if (s.dtype == DOMINO_DTYPE_BF16 && s.d % 64 == 0 && s.r % 64 == 0) {
    if (s.Hs % 64 != 0)
      return "per-phase kernels: tcgen05 H-projection GEMM, then per position k_u + tcgen05 W2 GEMM with the argmax "
             "in its epilogue + k_gru, then k_tokens";
    static thread_local std::string text;
    int bn_h = 0, ks_h = 0, bn_i = 0, ks_i = 0;
    gemm_tc_skinny_plan(3 * s.Hs + s.r, s.B, 2 * s.Hs, &bn_h, &ks_h);
    gemm_tc_skinny_plan(3 * s.Hs, s.B, s.d, &bn_i, &ks_i);
    text = std::string("per-phase kernels: tcgen05 H-projection GEMM; per position ") +
           (s.r <= 256 ? "k_w2_argmax (tcgen05 W2 product, activations in TMEM, L_base and the argmax fused)"
                       : "a tcgen05 W2 GEMM with the argmax in its epilogue") +
           ", the GRU input half (" +
           std::string("embedding gather + W_ih GEMM, tiles 128x") + std::to_string(bn_i) + " K-split " +
           std::to_string(ks_i) + ", or a projection-table gather), k_cell, and one stacked W_hh|W1 GEMM (tiles 128x" +
           std::to_string(bn_h) + " K-split " + std::to_string(ks_h) + ") for the next gh and activations; k_tokens";
    return text.c_str();
  }
  return "per-phase kernels: k_hproj, then per position k_u + k_w2 (fused argmax) + k_gru, then k_tokens";
}

const char* domino_teacher_forced_plan(const domino_shape_t* shape) {
  if (check_shape(shape) != DOMINO_OK) return "invalid shape";
  const Shape s = to_shape(shape);
  const bool tc = s.dtype == DOMINO_DTYPE_BF16 && s.d % 64 == 0 && s.r % 64 == 0 && s.Hs % 64 == 0;
  if (tc && use_persistent_greedy(s) && tmem_plan_fits(s, persistent_grid(), true) &&
      (s.L > 1 || tmem_plan_fits(s, persistent_grid(), false)))
    return "embedding gather + tcgen05 W_ih GEMM over all given tokens, k_greedy_tmem in teacher-forced mode (the "
           "recurrence), then tcgen05 GEMMs for the activations and the logits of all positions";
  if (tc && batched_shape_ok(s))
    return tf_units_ok(s) ? "embedding gather + tcgen05 W_ih GEMM over all given tokens, k_tf_units (the recurrence: "
                            "each CTA owns eight state units, loads gated by a write counter), then tcgen05 GEMMs for the "
                            "activations and the logits of all positions"
                          : "embedding gather + tcgen05 W_ih GEMM over all given tokens, k_greedy_batched in "
                            "teacher-forced mode (the recurrence), then tcgen05 GEMMs for the activations and the "
                            "logits of all positions";
  if (tc)
    return "embedding gather + tcgen05 W_ih GEMM over all given tokens, per update a tcgen05 gh GEMM + k_cell, then "
           "tcgen05 GEMMs for the activations and the logits of all positions";
  return "CUDA-core kernels: k_hproj, k_gru per update, then k_u + k_w2 for the logits";
}

int domino_debug_gemm(const void* A, const void* Bm, int32_t M, int32_t N, int32_t K, int32_t a_kwrap, float* out,
                      int64_t ldo, int32_t trans, int32_t bn, int32_t ks, int32_t* status_dev,
                      domino_stream_t stream) {
  if (!A || !Bm || !out || M < 1 || N < 1 || K < 64 || K % 64 || a_kwrap < 0 || (a_kwrap && (a_kwrap % 64 || K % a_kwrap)))
    return DOMINO_ERR_INVALID_ARGUMENT;
  if (ldo < (trans ? M : N) || !aligned16(A) || !aligned16(Bm) || !aligned16(out)) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!((bn == 0 && ks == 0) || ((bn == 16 || bn == 32 || bn == 64 || bn == 128) && ks >= 1 && ks <= 8)))
    return DOMINO_ERR_INVALID_ARGUMENT;
  if (!gemm_tc_supported(M, N, K, A, Bm)) return DOMINO_ERR_UNSUPPORTED;
  return cuda_rc(gemm_tc_debug((const __nv_bfloat16*)A, (const __nv_bfloat16*)Bm, M, N, K, a_kwrap, out, ldo, trans,
                               bn, ks, status_dev, spin_limit(), static_cast<cudaStream_t>(stream)));
}

int domino_debug_set_trace(void* device_buf, int32_t n_entries) {
  if (device_buf && (n_entries < 1 || (reinterpret_cast<uintptr_t>(device_buf) & 7u))) return DOMINO_ERR_INVALID_ARGUMENT;
  g_ntrace.store(device_buf ? n_entries : 0, std::memory_order_relaxed);
  g_trace.store(static_cast<unsigned long long*>(device_buf), std::memory_order_relaxed);
  return DOMINO_OK;
}

int domino_debug_set_spin_limit(uint64_t limit) {
  g_spin_limit.store(limit, std::memory_order_relaxed);
  return DOMINO_OK;
}

const char* domino_status_string(int code) {
  switch (code) {
    case DOMINO_OK: return "ok";
    case DOMINO_ERR_INVALID_ARGUMENT: return "invalid argument (null pointer, bad shape or misalignment)";
    case DOMINO_ERR_UNSUPPORTED: return "unsupported shape, layout or device";
    case DOMINO_ERR_CUDA: return "CUDA launch or query failed";
    case DOMINO_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DOMINO_ERR_SCRATCH_LIMIT: return "shape needs more scratch than the library-owned array holds";
    case DOMINO_STATUS_DEVICE_TIMEOUT: return "device: a bounded wait gave up (outputs invalid)";
    case DOMINO_STATUS_BAD_TOKEN: return "device: teacher-forcing token outside [0, V)";
    default: return "unknown code";
  }
}

size_t domino_embed_proj_bytes(const domino_shape_t* shape) {
  if (check_shape(shape) != DOMINO_OK) return 0;
  return (size_t)shape->V * 3 * shape->Hs * sizeof(float);
}

int domino_project_embeddings(const domino_shape_t* shape, const domino_weights_t* w, float* embed_proj,
                              int32_t* status_dev, domino_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  if (!w || !w->embed || !w->W_ih || !embed_proj || !aligned16(w->embed) || !aligned16(w->W_ih) ||
      !aligned16(embed_proj))
    return DOMINO_ERR_INVALID_ARGUMENT;
  const Shape s = to_shape(shape);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t* st = status_dev;
  cudaError_t e;
  if (s.dtype == DOMINO_DTYPE_BF16 && gemm_tc_supported(s.V, 3 * s.Hs, s.d, w->embed, w->W_ih))
    e = gemm_tc_store_f32((const __nv_bfloat16*)w->embed, (const __nv_bfloat16*)w->W_ih, s.V, 3 * s.Hs, s.d,
                          embed_proj, 3 * s.Hs, st, spin_limit(), cs);
  else
    e = launch_project_simple(s, w->embed, w->W_ih, embed_proj, cs);
  return cuda_rc(e);
}

size_t domino_workspace_bytes(const domino_shape_t* shape) {
  if (check_shape(shape) != DOMINO_OK) return 0;
  return layout_workspace(to_shape(shape), nullptr).bytes;
}

size_t domino_accept_workspace_bytes(int32_t B, int32_t L) {
  if (B < 1 || L < 1 || L > DOMINO_MAX_L) return 0;
  return accept_workspace_bytes(B, L);
}

int domino_draft_greedy(const domino_shape_t* shape, const domino_weights_t* w, const void* base_logits,
                        const void* hidden, const float* S0, int32_t* tokens_out, float* logits_out,
                        float* states_out, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                        domino_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  if ((rc = check_weights(w)) != DOMINO_OK) return rc;
  if (!base_logits || !hidden || !S0 || !tokens_out) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!aligned16(base_logits) || !aligned16(hidden) || !aligned16(S0) || !aligned16(tokens_out) ||
      (logits_out && !aligned16(logits_out)) || (states_out && !aligned16(states_out)))
    return DOMINO_ERR_INVALID_ARGUMENT;
  const Shape s = to_shape(shape);
  const Workspace need = layout_workspace(s, nullptr);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need.bytes)
    return DOMINO_ERR_WORKSPACE;
  const Workspace ws = layout_workspace(s, workspace);
  int32_t* st = status_dev ? status_dev : ws.status;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  if (use_persistent_greedy(s)) return cuda_rc(launch_persistent_greedy(s, *w, base_logits, hidden, S0, tokens_out,
                                                                         logits_out, states_out, ws, st,
                                                                         spin_limit(), cs));
  if (use_greedy_batched(s, *w, base_logits)) {
    // the barrier counter, the work-slot claims and the argmax keys are adjacent: one memset
    cudaError_t e =
        cudaMemsetAsync(ws.sync, 0, (char*)(ws.keys + (size_t)s.B * s.L) - (char*)ws.sync, cs);
    if (e == cudaSuccess)  // P[n][k] = sum_c W1[k][c] H[n][c] for every (row, position) n
      e = gemm_tc_store_f32_t((const __nv_bfloat16*)w->W1, (const __nv_bfloat16*)hidden, s.r, s.B * s.L, s.d, 0,
                              ws.P, s.r, st, spin_limit(), cs, 0, s.d + s.Hs);
    if (e == cudaSuccess)
      e = launch_greedy_batched(s, *w, base_logits, S0, logits_out, states_out, ws, st, spin_limit(), cs);
    if (e == cudaSuccess) e = launch_tokens_from_keys(ws.keys, s.B, s.L, tokens_out, cs);
    return cuda_rc(e);
  }

  const size_t BL = (size_t)s.B * s.L;
  // Batches the fused kernel does not take: one launch per phase and position.  With bf16 storage
  // the H-projection and the W2 product run on the tensor cores (tcgen05 GEMMs; the W2 product
  // batch-major with the argmax folded into its epilogue), else on CUDA cores.
  const bool tc = s.dtype == DOMINO_DTYPE_BF16 && s.d % 64 == 0 && s.r % 64 == 0 &&
                  gemm_tc_supported((int)BL, s.r, s.d, hidden, w->W1) &&
                  gemm_tc_supported(s.B, s.V, s.r, ws.u16, w->W2);
  const bool tc_gru = tc && s.Hs % 64 == 0;
  // work-slot claims and argmax keys are adjacent: one memset clears both
  cudaError_t e = cudaMemsetAsync(ws.claim, 0, (char*)(ws.keys + BL) - (char*)ws.claim, cs);
  if (e == cudaSuccess) {
    if (tc)  // P[n][k] = sum_c W1[k][c] H[n][c]: the first d columns of W1 (row stride d + Hs) against
             // the B*L hidden rows, a skinny product (split over K when its tiles do not cover the SMs)
      e = gemm_tc_store_f32_t((const __nv_bfloat16*)w->W1, (const __nv_bfloat16*)hidden, s.r, (int)BL, s.d, 0, ws.P,
                              s.r, st, spin_limit(), cs, 0, s.d + s.Hs);
    else
      e = launch_hproj(s, w->W1, hidden, (int)BL, ws.P, cs);
  }
  if (e == cudaSuccess && states_out) e = launch_copy_rows(S0, s.Hs, states_out, (size_t)s.L * s.Hs, s.B, s.Hs, cs);
  const float* S_cur = S0;
  using bf = __nv_bfloat16;
  const bf* W1s = (const bf*)w->W1 + s.d;  // state block of W1, row stride d + Hs
  // tensor-core GRU: the split state feeds one GEMM that yields W_hh . S (for the next cell) and the
  // next position's activations u = SiLU(P + W1_s . S)
  const bool stacked = tc_gru && (3 * s.Hs) % 128 == 0;
  if (e == cudaSuccess && tc_gru) {
    e = launch_split_state(S0, s.Hs, s.B, s.Hs, ws.S_hl, cs);
    if (e == cudaSuccess)
      e = stacked ? gemm_tc_gru_u((const bf*)w->W_hh, W1s, s.d + s.Hs, ws.S_hl, s.Hs, s.r, s.B, ws.Gh, ws.P,
                                  (long long)s.L * s.r, ws.u16, st, spin_limit(), cs)
                  : gemm_tc_silu_u(W1s, s.d + s.Hs, ws.S_hl, s.r, s.B, s.Hs, ws.P, (long long)s.L * s.r, ws.u16,
                                   nullptr, st, spin_limit(), cs);
  }
  for (int i = 0; i < s.L && e == cudaSuccess; ++i) {
    if (!tc_gru) e = launch_u(s, w->W1, ws.P, s.L, i, S_cur, s.Hs, s.B, ws.u, cs, tc ? ws.u16 : nullptr);
    if (e == cudaSuccess && tc) {
      for (int b0 = 0; b0 < s.B && e == cudaSuccess; b0 += 128) {  // bands of <= 128 batch rows
        const size_t row0 = (size_t)b0 * s.L + i;                   // (row b0, position i)
        // epochs distinct per launch of this call (the claims were zeroed above)
        const uint32_t epoch = (uint32_t)(i * ((s.B + 127) / 128) + b0 / 128 + 1);
        const bf* Ub = ws.u16 + (size_t)b0 * s.r;
        const bf* Lbp = (const bf*)base_logits + row0 * s.V;
        const int Mb = std::min(128, s.B - b0);
        float* lo = logits_out ? logits_out + row0 * s.V : nullptr;
        if (w2_argmax_supported(Mb, s.V, s.r, Ub, w->W2, Lbp, (long long)s.L * s.V))
          e = w2_argmax(Ub, (const bf*)w->W2, Mb, s.V, s.r, Lbp, (long long)s.L * s.V, ws.keys + (size_t)i * s.B + b0,
                        lo, (long long)s.L * s.V, i == s.L - 1 && b0 + 128 >= s.B, ws.claim, epoch, st,
                        spin_limit(), cs);
        else
          e = gemm_tc_argmax(Ub, (const bf*)w->W2, Mb, s.V, s.r, Lbp, (long long)s.L * s.V,
                             ws.keys + (size_t)i * s.B + b0, lo, (long long)s.L * s.V, st, spin_limit(), cs, ws.claim,
                             epoch);
      }
    } else if (e == cudaSuccess) {
      e = launch_w2(s, w->W2, ws.u, s.B, base_logits, s.L, i, ws.keys + (size_t)i * s.B, logits_out, cs);
    }
    if (e == cudaSuccess && i < s.L - 1) {
      float* S_next = ws.S + (size_t)(i & 1) * s.B * s.Hs;
      float* S_keep = states_out ? states_out + (size_t)(i + 1) * s.Hs : nullptr;
      const uint64_t* keys_i = ws.keys + (size_t)i * s.B;
      if (tc_gru) {
        if (!stacked)
          e = gemm_tc_store_f32_t((const bf*)w->W_hh, ws.S_hl, 3 * s.Hs, s.B, 2 * s.Hs, s.Hs, ws.Gh, 3 * s.Hs,
                                  st, spin_limit(), cs);
        if (e == cudaSuccess && !w->embed_proj) {  // gi = W_ih . embed[t_i] for every row
          e = launch_gather_rows((const bf*)w->embed, keys_i, nullptr, 1, 0, s.B, s.d, s.V, ws.X, cs);
          if (e == cudaSuccess)
            e = gemm_tc_store_f32_t((const bf*)w->W_ih, ws.X, 3 * s.Hs, s.B, s.d, 0, ws.Gx, 3 * s.Hs, st,
                                    spin_limit(), cs, 1);
        }
        if (e == cudaSuccess)
          e = launch_cell(s, ws.Gx, 3 * s.Hs, 1, 0, w->embed_proj, ws.Gh, w->b_ih, w->b_hh, keys_i, nullptr, 0, 0, S_cur,
                          s.Hs, S_next, s.Hs, S_keep, (size_t)s.L * s.Hs, st, cs, ws.S_hl);
        if (e == cudaSuccess) {  // gh for the next cell and the next position's activations
          const float* P_next = ws.P + (size_t)(i + 1) * s.r;
          if (stacked && i + 1 < s.L - 1)
            e = gemm_tc_gru_u((const bf*)w->W_hh, W1s, s.d + s.Hs, ws.S_hl, s.Hs, s.r, s.B, ws.Gh, P_next,
                              (long long)s.L * s.r, ws.u16, st, spin_limit(), cs);
          else
            e = gemm_tc_silu_u(W1s, s.d + s.Hs, ws.S_hl, s.r, s.B, s.Hs, P_next, (long long)s.L * s.r, ws.u16,
                               nullptr, st, spin_limit(), cs);
        }
      } else {
        e = launch_gru(s, w->embed, w->W_ih, w->W_hh, w->b_ih, w->b_hh, keys_i, nullptr, 0, 0, S_cur, s.Hs, S_next,
                       s.Hs, S_keep, (size_t)s.L * s.Hs, s.B, st, cs, w->embed_proj);
      }
      S_cur = S_next;
    }
  }
  if (e == cudaSuccess) e = launch_tokens_from_keys(ws.keys, s.B, s.L, tokens_out, cs);
  return cuda_rc(e);
}

}  // extern "C"

namespace {

// Teacher forcing with fp32 or bf16 logits (logits_dtype: DOMINO_DTYPE_F32 or DOMINO_DTYPE_BF16).
int teacher_forced_impl(const domino_shape_t* shape, const domino_weights_t* w, const void* base_logits,
                        const void* hidden, const float* S0, const int32_t* tokens, void* logits_out,
                        int logits_dtype, float* states_out, void* workspace, size_t workspace_bytes,
                        int32_t* status_dev, domino_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  if ((rc = check_weights(w)) != DOMINO_OK) return rc;
  if (!base_logits || !hidden || !S0 || !tokens || !logits_out) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!aligned16(base_logits) || !aligned16(hidden) || !aligned16(S0) || !aligned16(tokens) ||
      !aligned16(logits_out) || (states_out && !aligned16(states_out)))
    return DOMINO_ERR_INVALID_ARGUMENT;
  const Shape s = to_shape(shape);
  const Workspace need = layout_workspace(s, nullptr);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need.bytes)
    return DOMINO_ERR_WORKSPACE;
  const Workspace ws = layout_workspace(s, workspace);
  int32_t* st = status_dev ? status_dev : ws.status;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);

  const size_t BL = (size_t)s.B * s.L;
  // bf16 logits come from the tensor-core W2 product only
  const bool tc_w2 = s.dtype == DOMINO_DTYPE_BF16 && gemm_tc_supported(s.V, (int)BL, s.r, w->W2, ws.u16);
  if (logits_dtype == DOMINO_DTYPE_BF16 && !tc_w2) return DOMINO_ERR_UNSUPPORTED;
  float* SB = states_out ? states_out : ws.states;  // [B][L][Hs]
  const size_t row = (size_t)s.L * s.Hs;
  using bf = __nv_bfloat16;
  const bool tc = s.dtype == DOMINO_DTYPE_BF16 && s.d % 64 == 0 && s.r % 64 == 0 && s.Hs % 64 == 0 &&
                  gemm_tc_supported((int)BL, s.r, s.d, hidden, w->W1);
  // every check has passed: from here on work is enqueued.  The logits GEMM claims its work slots by
  // SM (epoch 1 against words zeroed here).
  cudaError_t e = cudaMemsetAsync(ws.claim, 0, kClaimWords * sizeof(uint32_t), cs);
  if (e == cudaSuccess)
    e = tc ? gemm_tc_store_f32_t((const bf*)w->W1, (const bf*)hidden, s.r, (int)BL, s.d, 0, ws.P, s.r, st,
                                 spin_limit(), cs, 0, s.d + s.Hs)
           : launch_hproj(s, w->W1, hidden, (int)BL, ws.P, cs);
  // Small batches whose GRU rows fit in TMEM: the whole recurrence in one fused kernel (one grid
  // barrier per update), then the activations and logits of all positions as below.
  // The input half of every update is known up front: one gather + W_ih product over all B*(L-1)
  // given tokens (unless the projection table holds it), so TMEM keeps only the W_hh rows.
  // (With a single position no gates are precomputed and the kernel keeps W_ih rows as in greedy
  // drafting, so that plan must fit then.)
  const bool fused = tc && use_persistent_greedy(s) && tmem_plan_fits(s, persistent_grid(), true) &&
                     (s.L > 1 || w->embed_proj || tmem_plan_fits(s, persistent_grid(), false));
  if (fused) {
    const int NXf = s.B * (s.L - 1);
    const float* gx = nullptr;
    if (e == cudaSuccess && !w->embed_proj && NXf > 0) {
      e = launch_gather_rows((const bf*)w->embed, nullptr, tokens, s.L - 1, s.L, NXf, s.d, s.V, ws.X, cs);
      if (e == cudaSuccess)
        e = gemm_tc_store_f32_t((const bf*)w->W_ih, ws.X, 3 * s.Hs, NXf, s.d, 0, ws.Gx, 3 * s.Hs, st, spin_limit(),
                                cs, 1);
      gx = ws.Gx;
    }
    if (e == cudaSuccess)
      e = launch_tf_recurrence_tmem(s, *w, S0, tokens, gx, SB, ws, st, spin_limit(), persistent_grid(), cs);
  } else {
  // 5..128 rows: the recurrence in one launch of the persistent batched kernel (it writes the
  // states' first position and the split of S0 itself); otherwise one gh GEMM + cell per update
  const bool batched = tc && use_greedy_batched(s, *w, base_logits);
  if (e == cudaSuccess && !batched) e = launch_copy_rows(S0, s.Hs, SB, row, s.B, s.Hs, cs);
  if (e == cudaSuccess && tc && !batched) e = launch_split_state(S0, s.Hs, s.B, s.Hs, ws.S_hl, cs);
  // The GRU input half for every given token at once (one GEMM over B*(L-1) gathered rows), unless
  // the projection table already holds it.
  const int NX = s.B * (s.L - 1);
  if (e == cudaSuccess && tc && !w->embed_proj && NX > 0) {
    e = launch_gather_rows((const bf*)w->embed, nullptr, tokens, s.L - 1, s.L, NX, s.d, s.V, ws.X, cs);
    if (e == cudaSuccess)
      e = gemm_tc_store_f32_t((const bf*)w->W_ih, ws.X, 3 * s.Hs, NX, s.d, 0, ws.Gx, 3 * s.Hs, st, spin_limit(), cs,
                              1);
  }
  if (batched) {
    if (e == cudaSuccess) e = cudaMemsetAsync(ws.sync, 0, kSyncWords * sizeof(uint32_t), cs);
    if (e == cudaSuccess)
      e = tf_units_ok(s) ? launch_tf_units(s, *w, S0, tokens, ws.Gx, SB, ws, st, spin_limit(), cs)
                         : launch_tf_batched(s, *w, base_logits, S0, tokens, ws.Gx, SB, ws, st, spin_limit(), cs);
  }
  for (int i = 0; i + 1 < s.L && e == cudaSuccess && !batched; ++i) {
    if (tc)
      e = gru_step_tc(s, *w, ws, SB + (size_t)i * s.Hs, row, nullptr, tokens, s.L, i, ws.Gx, 3 * s.Hs, s.L - 1, i, false,
                      SB + (size_t)(i + 1) * s.Hs, row, nullptr, 0, st, cs);
    else
      e = launch_gru(s, w->embed, w->W_ih, w->W_hh, w->b_ih, w->b_hh, nullptr, tokens, s.L, i,
                     SB + (size_t)i * s.Hs, row, SB + (size_t)(i + 1) * s.Hs, row, nullptr, 0, s.B, st, cs,
                     w->embed_proj);
  }
  }  // per-update recurrence
  // W2 product over all B*L positions at once: a tcgen05 GEMM with the L_base add fused into its
  // epilogue (activations rounded to bf16 for the tensor cores), or the CUDA-core kernel.
  if (e == cudaSuccess && tc && tc_w2) {  // u for every position: one GEMM on the split of all states
    e = launch_split_state(SB, s.Hs, (int)BL, s.Hs, ws.S_hl, cs);
    if (e == cudaSuccess)
      e = gemm_tc_silu_u((const __nv_bfloat16*)w->W1 + s.d, s.d + s.Hs, ws.S_hl, s.r, (int)BL, s.Hs, ws.P, s.r,
                         ws.u16, nullptr, st, spin_limit(), cs);
  } else if (e == cudaSuccess) {
    e = launch_u(s, w->W1, ws.P, 1, 0, SB, s.Hs, (int)BL, ws.u, cs, tc_w2 ? ws.u16 : nullptr);
  }
  if (e == cudaSuccess) {
    if (tc_w2)
      e = gemm_tc_logits((const __nv_bfloat16*)w->W2, ws.u16, s.V, (int)BL, s.r, (const __nv_bfloat16*)base_logits,
                         logits_out, logits_dtype == DOMINO_DTYPE_BF16, st, spin_limit(), cs, ws.claim, 1u);
    else
      e = launch_w2(s, w->W2, ws.u, (int)BL, base_logits, 1, 0, nullptr, static_cast<float*>(logits_out), cs);
  }
  return cuda_rc(e);
}

}  // namespace

extern "C" {

int domino_teacher_forced(const domino_shape_t* shape, const domino_weights_t* w, const void* base_logits,
                          const void* hidden, const float* S0, const int32_t* tokens, float* logits_out,
                          float* states_out, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                          domino_stream_t stream) {
  return teacher_forced_impl(shape, w, base_logits, hidden, S0, tokens, logits_out, DOMINO_DTYPE_F32, states_out,
                             workspace, workspace_bytes, status_dev, stream);
}

int domino_teacher_forced_ex(const domino_shape_t* shape, const domino_weights_t* w, const void* base_logits,
                             const void* hidden, const float* S0, const int32_t* tokens, void* logits_out,
                             int32_t logits_dtype, float* states_out, void* workspace, size_t workspace_bytes,
                             int32_t* status_dev, domino_stream_t stream) {
  if (logits_dtype != DOMINO_DTYPE_F32 && logits_dtype != DOMINO_DTYPE_BF16) return DOMINO_ERR_INVALID_ARGUMENT;
  return teacher_forced_impl(shape, w, base_logits, hidden, S0, tokens, logits_out, logits_dtype, states_out,
                             workspace, workspace_bytes, status_dev, stream);
}

int domino_accept_len(int32_t B, int32_t L, int32_t V, const int32_t* draft_tokens, const float* target_logits,
                      int32_t* accept_out, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                      domino_stream_t stream) {
  (void)status_dev;
  if (B < 1 || L < 1 || L > DOMINO_MAX_L || V < 8 || V % 8) return DOMINO_ERR_INVALID_ARGUMENT;
  if ((int64_t)B * L > kMaxRows) return DOMINO_ERR_UNSUPPORTED;
  if (!draft_tokens || !target_logits || !accept_out) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!aligned16(target_logits)) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < accept_workspace_bytes(B, L))
    return DOMINO_ERR_WORKSPACE;
  Shape s{B, L, 8, 8, 8, 8, DOMINO_DTYPE_F32};
  const Workspace ws = layout_workspace(s, workspace);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t BL = (size_t)B * L;
  // keys, counters, first-mismatch words and the completion word: adjacent, cleared together
  const size_t clear = reinterpret_cast<char*>(ws.acc_count + BL + B + 1) - reinterpret_cast<char*>(ws.acc_keys);
  cudaError_t e = cudaMemsetAsync(ws.acc_keys, 0, clear, cs);
  if (e == cudaSuccess)
    e = launch_accept_early(target_logits, draft_tokens, B, L, V, ws.acc_keys, ws.acc_count, accept_out, cs);
  return cuda_rc(e);
}

}  // extern "C"
