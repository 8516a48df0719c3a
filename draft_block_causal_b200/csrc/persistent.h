// persistent.h -- the fused, persistent greedy-drafting kernel (small batch).
#pragma once

#include "domino.h"
#include "internal.h"

namespace domino {

// Default iteration limit of bounded device-wide waits (about a second of polling).
constexpr uint64_t kDefaultSpinLimit = 1ull << 22;
uint64_t spin_limit();

// True when the fused persistent kernel handles this shape (else the step kernels do).
bool use_persistent_greedy(const Shape& s);
const char* persistent_plan(const Shape& s);

// The TMEM-resident variant (persistent_tmem.cu): fits when d and Hs are multiples of 512 and a
// CTA's GRU rows fit in its 512 TMEM columns.
bool tmem_plan_fits(const Shape& s, int G, bool proj);
cudaError_t launch_greedy_tmem(const Shape& s, const domino_weights_t& w, const void* base_logits, const void* hidden,
                               const float* S0, int32_t* tokens_out, float* logits_out, float* states_out,
                               const Workspace& ws, int32_t* status, uint64_t spin, int G, cudaStream_t st);

// Teacher-forced GRU recurrence of the TMEM-resident kernel: states [B][L][Hs] (states[b][0] = S0)
// for the given tokens [B][L]; out-of-range tokens set DOMINO_STATUS_BAD_TOKEN and read token 0.
// Gx (optional): [B][L-1][3Hs] fp32 W_ih . embed[y_i], computed up front; else the projection
// table of the weights, else the TMEM-resident W_ih rows give the input half.
cudaError_t launch_tf_recurrence_tmem(const Shape& s, const domino_weights_t& w, const float* S0, const int32_t* tokens,
                                      const float* Gx, float* states, const Workspace& ws, int32_t* status,
                                      uint64_t spin, int G, cudaStream_t st);
// Grid of the fused kernels (one CTA per SM of the current device).
int persistent_grid();

cudaError_t launch_persistent_greedy(const Shape& s, const domino_weights_t& w, const void* base_logits,
                                     const void* hidden, const float* S0, int32_t* tokens_out, float* logits_out,
                                     float* states_out, const Workspace& ws, int32_t* status, uint64_t spin_limit,
                                     cudaStream_t st);

// The persistent batched kernel (persistent_batched.cu): greedy drafting of 5..128 rows in one
// cooperative launch, bf16 storage.  The caller computes ws.P (W1[:, :d] . H for every position)
// and zeroes ws.sync, ws.claim and ws.keys before the launch, and turns the keys into tokens after.
bool batched_shape_ok(const Shape& s);
bool use_greedy_batched(const Shape& s, const domino_weights_t& w, const void* base_logits);
const char* batched_plan();
// Floats of ws.part the kernel needs for shape s (0 when the kernel does not take the shape).
size_t batched_partial_floats(const Shape& s);
cudaError_t launch_greedy_batched(const Shape& s, const domino_weights_t& w, const void* base_logits,
                                  const float* S0, float* logits_out, float* states_out, const Workspace& ws,
                                  int32_t* status, uint64_t spin, cudaStream_t st);
// Its teacher-forced recurrence: states [B][L][Hs] (states[b][0] = S0) for the given tokens [B][L];
// Gx: [B * (L - 1)][3Hs] fp32 W_ih . embed[y_i] (row b * (L - 1) + i), unless the weights carry the
// projection table.  Out-of-range tokens set DOMINO_STATUS_BAD_TOKEN and read token 0.  The caller
// zeroes ws.sync and ws.claim first.
cudaError_t launch_tf_batched(const Shape& s, const domino_weights_t& w, const void* base_logits, const float* S0,
                              const int32_t* tokens, const float* Gx, float* states, const Workspace& ws,
                              int32_t* status, uint64_t spin, cudaStream_t st);

// The unit-owned teacher-forced recurrence (tf_units.cu): every CTA owns eight state units and
// keeps their W_hh rows in shared memory; no grid barrier (a write counter).  Same contract as
// launch_tf_batched (ws.S_hl's first 2B rows serve as its two split-state buffers); the caller
// zeroes ws.sync first.
bool tf_units_ok(const Shape& s);
const char* tf_units_plan();
cudaError_t launch_tf_units(const Shape& s, const domino_weights_t& w, const float* S0, const int32_t* tokens,
                            const float* Gx, float* states, const Workspace& ws, int32_t* status, uint64_t spin,
                            cudaStream_t st);

}  // namespace domino
