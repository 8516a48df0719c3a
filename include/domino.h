/*
 * domino.h -- C ABI of libdomino, the B200 (sm_100a) implementation of the Domino head.
 *
 * The Domino head (Domino review page, paper.oopus.info, section 二 "Domino Head") turns the
 * parallel backbone's outputs for one draft block -- hidden states H[i] and base logits
 * L_base[i] at every position i -- into corrected logits
 *
 *     L_final[i] = L_base[i] + W2 . SiLU(W1 . [H[i] ; S_{i-1}])
 *
 * where S_{i-1} is the state of a GRU causal encoder (hidden size Hs, 1024 on the pages) that has
 * read the embeddings of the tokens drafted before position i.  W1 is rank r (256 on the pages)
 * and W2 maps r -> V over the whole vocabulary; the LM head is not recomputed.
 *
 * Conventions shared by every entry point
 *   - Every pointer is caller-owned device memory (cudaMalloc / PyTorch), row-major, contiguous
 *     and 16-byte aligned, unless stated otherwise.  The library allocates nothing: scratch
 *     memory is the caller's workspace.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     never synchronises the host.  Calls that share a workspace must be ordered on the GPU.
 *   - Calls run on the calling thread's current device, which must hold every pointer passed.
 *     Several host threads may call at once; calls whose GPU work overlaps need separate
 *     workspaces (and see domino_draft_greedy_noalloc).  The debug hooks' settings are
 *     process-wide.
 *   - Host-side checks happen before any launch: on a negative return code nothing was enqueued.
 *   - Device-side problems (a bounded wait that gave up, a token outside [0, V)) are reported by
 *     writing a positive DOMINO_STATUS_* code to *status_dev with an atomic compare-and-swap from
 *     0, so the first problem wins.  The library never clears *status_dev: zero it before the
 *     call and read it after your own synchronisation.  status_dev may be NULL, in which case
 *     the code lands in a word inside the workspace.
 *   - Storage type (`dtype`): DOMINO_DTYPE_BF16 means embed, W_ih, W_hh, b_ih, b_hh, W1, W2,
 *     base_logits and hidden are bf16; DOMINO_DTYPE_F32 means they are fp32.  S0, states,
 *     logits and target logits are always fp32; tokens are int32.  Arithmetic accumulates in
 *     fp32 in every mode.
 *   - Shapes: 1 <= B, 1 <= L <= DOMINO_MAX_L; d, Hs and r must each be a multiple of 8 and, in
 *     16-byte vectors, either a multiple of 32 vectors or a power of two up to 32 vectors; V must
 *     be a multiple of 8 (else DOMINO_ERR_INVALID_ARGUMENT).  B * L <= 65535, r <= 1024 and
 *     B * L * max(Hs, d / 8) < 2^31 (else DOMINO_ERR_UNSUPPORTED).
 */
#ifndef DOMINO_H_
#define DOMINO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DOMINO_API __attribute__((visibility("default")))
#else
#define DOMINO_API
#endif

#define DOMINO_ABI_VERSION 2
#define DOMINO_MAX_L 64

/* Storage type of the weights, embedding table, base logits and hidden states. */
#define DOMINO_DTYPE_F32 0
#define DOMINO_DTYPE_BF16 1

/* Host return codes. */
#define DOMINO_OK 0
#define DOMINO_ERR_INVALID_ARGUMENT (-1) /* null required pointer, bad shape, misalignment      */
#define DOMINO_ERR_UNSUPPORTED (-2)      /* valid but not handled (dims layout, device, grid)   */
#define DOMINO_ERR_CUDA (-3)             /* a CUDA launch or query failed                       */
#define DOMINO_ERR_WORKSPACE (-4)        /* workspace missing, misaligned (256 B) or too small  */
#define DOMINO_ERR_SCRATCH_LIMIT (-5)    /* shape needs more than DOMINO_NOALLOC_SCRATCH_BYTES  */

/* Device status codes written to *status_dev. */
#define DOMINO_STATUS_OK 0
#define DOMINO_STATUS_DEVICE_TIMEOUT 1 /* a bounded device-wide wait gave up; outputs invalid */
#define DOMINO_STATUS_BAD_TOKEN 2      /* a teacher-forcing token was outside [0, V)          */

/* cudaStream_t, kept opaque so this header needs no CUDA include. */
typedef void* domino_stream_t;

/* Problem shape.  B rows, L positions per draft block, embedding / hidden width d, GRU hidden
 * size Hs, correction rank r, vocabulary V, storage type dtype (DOMINO_DTYPE_*). */
typedef struct {
  int32_t B, L, d, Hs, r, V, dtype;
} domino_shape_t;

/* Head weights (device pointers, storage type = shape.dtype):
 *   embed [V, d]      token embedding table, shared with the backbone
 *   W_ih  [3Hs, d]    GRU input weights, gate blocks in the order (r | z | n)
 *   W_hh  [3Hs, Hs]   GRU recurrent weights, same gate order
 *   b_ih  [3Hs], b_hh [3Hs]
 *   W1    [r, d+Hs]   columns 0..d-1 multiply H[i], columns d..d+Hs-1 multiply S_{i-1}
 *   W2    [V, r]
 * The GRU cell is the PyTorch nn.GRUCell form:
 *   r = sig(W_ir x + b_ir + W_hr h + b_hr), z = sig(W_iz x + b_iz + W_hz h + b_hz),
 *   n = tanh(W_in x + b_in + r * (W_hn h + b_hn)), h' = (1 - z) * n + z * h.
 *   embed_proj [V, 3Hs] fp32, optional (NULL = not prepared): the GRU input half of every token,
 *                     embed_proj[v][g*Hs + j] = sum_c W_ih[g*Hs + j][c] * embed[v][c], filled once
 *                     per weight set by domino_project_embeddings.  When present, every entry point
 *                     gathers the drafted (or given) token's row instead of multiplying W_ih by the
 *                     embedding at each position.                                          */
typedef struct {
  const void *embed, *W_ih, *W_hh, *b_ih, *b_hh, *W1, *W2;
  const float* embed_proj;
} domino_weights_t;

/* Bytes of the optional input-projection table (V * 3Hs * 4), or 0 for an invalid shape. */
DOMINO_API size_t domino_embed_proj_bytes(const domino_shape_t* shape);

/* Fills embed_proj [V, 3Hs] fp32 with embed . W_ih^T (the GRU's input projection applied to every
 * row of the embedding table at once) -- an algebraic precomputation of the encoder's input half
 * (the drafted tokens' embeddings feed the GRU: review page section 二, GRU causal encoder), done
 * once per weight set.  bf16 storage uses the tensor cores (fp32 accumulation); fp32 storage a
 * CUDA-core kernel.  Only shape->d, Hs, V and dtype are used.  weights->embed_proj is ignored.
 * Returns DOMINO_OK or a negative DOMINO_ERR_* code (nothing launched). */
DOMINO_API int domino_project_embeddings(const domino_shape_t* shape, const domino_weights_t* weights,
                                         float* embed_proj, int32_t* status_dev, domino_stream_t stream);

/* ---- Weight arena and L2 residency (opt-in) ----
 *
 * Every position of a block re-reads W2, W1's state block, W_hh and (without the projection
 * table) W_ih: about 110 MB at the pages' Qwen3-8B shapes, which B200's L2 (126 MB) can hold
 * between positions and, with a persisting window, between blocks.
 *
 * domino_arena_bytes: bytes of one contiguous arena holding W2, W1, W_hh, W_ih, b_ih and b_hh in
 * that order (each region 256-byte aligned; the embedding table and the projection table stay
 * where the caller keeps them), or 0 for an invalid shape.  Only d, Hs, r, V and dtype are used.
 *
 * domino_pack_weights: copies the six tensors of `src` into `arena` (device memory, 256-byte
 * aligned, at least domino_arena_bytes long; caller-owned) with device-to-device copies on
 * `stream`, and fills `packed` with pointers into the arena (embed and embed_proj are copied
 * from `src` unchanged).  `packed` is usable by every entry point once the copies have run.
 * Returns DOMINO_OK, DOMINO_ERR_INVALID_ARGUMENT, DOMINO_ERR_WORKSPACE (arena missing, misaligned
 * or too small) or DOMINO_ERR_CUDA.
 *
 * domino_set_l2_persistence: with 0 < hit_ratio <= 1, sets the access-policy window of `stream`
 * (a created stream, not the legacy default stream) over the packed hot range -- W2 through W_ih,
 * or through W_hh when weights->embed_proj is set -- with persisting hits and streaming misses,
 * and raises this context's persisting-L2 set-aside to min(range, device maximum); when the
 * range exceeds the set-aside, only that fraction of its lines (times hit_ratio) is marked
 * persisting.  Kernels launched on `stream` afterwards keep those weights in L2 across calls.
 * hit_ratio = 0 clears the window, returns persisting lines to normal and restores the
 * set-aside the context had before the first window.  The set-aside belongs to the calling
 * process's context on the current device and ends with it.  Returns DOMINO_OK,
 * DOMINO_ERR_INVALID_ARGUMENT (weights not packed, stream NULL, hit_ratio outside [0, 1]),
 * DOMINO_ERR_UNSUPPORTED (no persisting L2 on this device) or DOMINO_ERR_CUDA. */
DOMINO_API size_t domino_arena_bytes(const domino_shape_t* shape);
DOMINO_API int domino_pack_weights(const domino_shape_t* shape, const domino_weights_t* src, void* arena,
                                   size_t arena_bytes, domino_weights_t* packed, domino_stream_t stream);
DOMINO_API int domino_set_l2_persistence(const domino_shape_t* shape, const domino_weights_t* weights,
                                         domino_stream_t stream, float hit_ratio);

/* Workspace bytes needed by domino_draft_greedy, domino_teacher_forced and domino_accept_len
 * for `shape` (the largest of the three), or 0 if the shape is invalid.  The workspace must be
 * device memory aligned to 256 bytes; its contents need no initialisation. */
DOMINO_API size_t domino_workspace_bytes(const domino_shape_t* shape);

/* Greedy drafting of one block per row (review page section 二: GRU causal encoder + low-rank
 * logit-space correction; news.sig.ai article: the greedy decoding setting).
 *
 * For every row b and position i = 0..L-1, with S_{-1} = S0[b]:
 *   z_i = L_base[b,i] + W2 . SiLU(W1 . [H[b,i] ; S_{i-1}])
 *   t_i = argmax_v z_i[v]            (lowest index on ties; decided on fp32 z)
 *   S_i = GRU(embed[t_i], S_{i-1})   for i < L-1 (the state after the last position is unused)
 * Inputs:  base_logits [B, L, V], hidden [B, L, d] (storage type), S0 [B, Hs] fp32.
 * Outputs: tokens_out [B, L] int32 (required);
 *          logits_out [B, L, V] fp32 = z_i, or NULL to skip (the greedy path then never writes
 *          logits: the argmax is fused into the W2 product);
 *          states_out [B, L, Hs] fp32 = the state each position consumed (states_out[b,0] = S0),
 *          or NULL.
 * Returns DOMINO_OK or a negative DOMINO_ERR_* code (nothing launched). */
DOMINO_API int domino_draft_greedy(const domino_shape_t* shape, const domino_weights_t* weights,
                        const void* base_logits, const void* hidden, const float* S0,
                        int32_t* tokens_out, float* logits_out, float* states_out,
                        void* workspace, size_t workspace_bytes, int32_t* status_dev,
                        domino_stream_t stream);

/* Teacher-forced causal encoding (review page section 二, "Teacher Forcing": the GRU reads the
 * given tokens instead of its own predictions).  Same equations as greedy drafting with
 * t_i := tokens[b, i]; no argmax is taken.
 * Inputs:  as domino_draft_greedy plus tokens [B, L] int32 (each in [0, V); an out-of-range
 *          token sets DOMINO_STATUS_BAD_TOKEN and its row's later outputs are unspecified;
 *          tokens[b, L-1] feeds no GRU update and is not read).
 * Outputs: logits_out [B, L, V] fp32 (required); states_out [B, L, Hs] fp32 or NULL.
 * Returns DOMINO_OK or a negative DOMINO_ERR_* code. */
DOMINO_API int domino_teacher_forced(const domino_shape_t* shape, const domino_weights_t* weights,
                          const void* base_logits, const void* hidden, const float* S0,
                          const int32_t* tokens, float* logits_out, float* states_out,
                          void* workspace, size_t workspace_bytes, int32_t* status_dev,
                          domino_stream_t stream);

/* domino_teacher_forced with a choice of logits storage: logits_dtype DOMINO_DTYPE_F32 (logits_out
 * is float [B, L, V], as domino_teacher_forced) or DOMINO_DTYPE_BF16 (logits_out is bf16 [B, L, V],
 * each value the fp32 logit rounded to nearest even: half the bytes of the largest output).
 * bf16 logits need bf16 storage (shape->dtype) and the tensor-core W2 product, else
 * DOMINO_ERR_UNSUPPORTED; another logits_dtype gives DOMINO_ERR_INVALID_ARGUMENT.  Nothing is
 * launched when a negative code is returned. */
DOMINO_API int domino_teacher_forced_ex(const domino_shape_t* shape, const domino_weights_t* weights,
                                        const void* base_logits, const void* hidden, const float* S0,
                                        const int32_t* tokens, void* logits_out, int32_t logits_dtype,
                                        float* states_out, void* workspace, size_t workspace_bytes,
                                        int32_t* status_dev, domino_stream_t stream);

/* Greedy accept length (the accept-length metric of the review page, section 四; the target
 * verifies the whole block in one pass and keeps the longest agreeing prefix, sections 一 and
 * the researchpapers.dev summary):
 *   accept_out[b] = number of leading positions j (0 <= j < L) with
 *                   draft_tokens[b, j] == argmax_v target_logits[b, j, v]  (lowest index on ties)
 * No bonus token is counted.  draft_tokens [B, L] int32, target_logits [B, L, V] fp32,
 * accept_out [B] int32.  One kernel launch; the target logits of a row's positions after its first
 * mismatch may be left unread (the result is the same).  Needs domino_accept_workspace_bytes(B, L)
 * bytes of workspace (a workspace sized by domino_workspace_bytes for the same B and L also
 * suffices).  Returns DOMINO_OK or a negative DOMINO_ERR_* code. */
DOMINO_API size_t domino_accept_workspace_bytes(int32_t B, int32_t L);
DOMINO_API int domino_accept_len(int32_t B, int32_t L, int32_t V, const int32_t* draft_tokens,
                      const float* target_logits, int32_t* accept_out, void* workspace,
                      size_t workspace_bytes, int32_t* status_dev, domino_stream_t stream);

/* Sampled (temperature > 0) verification of a draft block.  The pages call Domino's verification
 * lossless (review page, section 一: the target model checks the whole block in one parallel pass;
 * researchpapers.dev summary) and spell out only the greedy setting (domino_accept_len).  For a
 * target that samples at temperature T, this is the published speculative-sampling rule that keeps
 * verification lossless (Leviathan, Kalman and Matias, ICML 2023; Chen et al. 2023):
 *   p_j = softmax(target_logits[b, j] / T)
 *   q_j = softmax(draft_logits[b, j] / T), or, when draft_logits is NULL, the one-hot distribution
 *         on draft_tokens[b, j] (greedy drafting, as domino_draft_greedy does, is that case)
 *   position j is accepted when uniforms[b, j] < p_j(x) / q_j(x), x = draft_tokens[b, j]; the row
 *   stops at its first rejected position k, whose replacement token is drawn from the residual
 *   max(0, p_k - q_k) by inverse transform with uniforms[b, L]: the smallest v whose running sum
 *   (ascending v) exceeds uniforms[b, L] times the residual's total.
 * Inputs: draft_tokens [B, L] int32 (each in [0, V); an out-of-range token sets
 *         DOMINO_STATUS_BAD_TOKEN and is rejected), draft_logits [B, L, V] fp32 or NULL,
 *         target_logits [B, L, V] fp32, uniforms [B, L + 1] fp32 in [0, 1) -- the random draws are
 *         the caller's, so a call is reproducible -- and 0 < temperature < infinity.
 * Outputs: accept_out [B] int32 = k (L when every position is accepted); next_out [B] int32 = the
 *          replacement token at position k, or -1 when all L positions were accepted (no bonus
 *          token: there are no target logits past the block).
 * Two launches; logits of a row's positions after its first rejection may be left unread (the
 * result is the same).  Needs domino_accept_sample_workspace_bytes(B, L, V) bytes of workspace
 * (device memory, 256-byte aligned).  Returns DOMINO_OK, DOMINO_ERR_INVALID_ARGUMENT (null pointer,
 * misaligned logits, bad shape or temperature), DOMINO_ERR_UNSUPPORTED (B * L > 65535),
 * DOMINO_ERR_WORKSPACE or DOMINO_ERR_CUDA; nothing is launched on a negative code. */
DOMINO_API size_t domino_accept_sample_workspace_bytes(int32_t B, int32_t L, int32_t V);
DOMINO_API int domino_accept_sample(int32_t B, int32_t L, int32_t V, const int32_t* draft_tokens,
                                    const float* draft_logits, const float* target_logits, float temperature,
                                    const float* uniforms, int32_t* accept_out, int32_t* next_out,
                                    void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                    domino_stream_t stream);

/* Human-readable text for a DOMINO_ERR_* or DOMINO_STATUS_* code (static storage). */
DOMINO_API const char* domino_status_string(int code);

/* DOMINO_ABI_VERSION of the loaded library. */
DOMINO_API int32_t domino_abi_version(void);

/* Number of kernels this library has enqueued in this process so far (all entry points, all
 * devices).  Reading it before and after a region counts the library's launches in it. */
DOMINO_API uint64_t domino_launch_count(void);

/* Short static description of the kernel sequence domino_draft_greedy runs for `shape`
 * (e.g. which fused kernel, or the per-phase kernels), or "invalid shape". */
DOMINO_API const char* domino_greedy_plan(const domino_shape_t* shape);

/* The same for domino_teacher_forced and domino_teacher_forced_ex (weights without the embedding
 * projection table). */
DOMINO_API const char* domino_teacher_forced_plan(const domino_shape_t* shape);

/* Greedy drafting without a workspace, for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is a deployment convenience of this library.  Callers
 * that cannot hand over a workspace include serving processes that reserved all free device
 * memory for weights and KV cache at start-up (a later cudaMalloc would fail or fragment those
 * pools), plugins whose host runtime owns the device allocator, and latency-critical loops that
 * must not pay an allocation's implicit synchronisation.
 *
 * Same arguments, equations and outputs as domino_draft_greedy, minus the workspace.  The
 * scratch memory is a library-owned, file-scope device array of DOMINO_NOALLOC_SCRATCH_BYTES
 * bytes that every GPU which loads the library holds until the process exits; nothing is ever
 * allocated or freed by this call.  Limits:
 *   - only shapes the fused small-batch kernel handles (bf16, r = 256, B <= 4, d and Hs
 *     multiples of 256) are accepted, else DOMINO_ERR_UNSUPPORTED;
 *   - the kernel's scratch (4*B*L*r + 64*B*r + 8*B*L + 8*B*Hs + 512 bytes, each piece rounded
 *     up to 256) must fit the array, else DOMINO_ERR_SCRATCH_LIMIT -- e.g. B=4, L=16, Hs=1024
 *     needs 164,864 bytes and fits; B=4, L=64 needs 363,008 and does not;
 *   - every call on a device shares that device's array, and the array keeps the previous
 *     call's contents (the call clears what must start at zero).  Calls whose kernels overlap
 *     on the GPU -- on different streams, or from different host threads -- race on the array
 *     and give wrong results: order them on one stream.
 *   - the first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture begins.
 * status_dev may be NULL (the code then lands in the array).  Returns DOMINO_OK or a negative
 * DOMINO_ERR_* code (nothing launched). */
#define DOMINO_NOALLOC_SCRATCH_BYTES (256u * 1024u)
DOMINO_API int domino_draft_greedy_noalloc(const domino_shape_t* shape, const domino_weights_t* weights,
                                           const void* base_logits, const void* hidden, const float* S0,
                                           int32_t* tokens_out, float* logits_out, float* states_out,
                                           int32_t* status_dev, domino_stream_t stream);

/* Profiling hook: when `device_buf` is non-NULL (8-byte aligned device memory of n_entries u64),
 * the TMEM-resident fused greedy kernel records the SM clock of CTA 0 at its phase boundaries:
 * [0] start, [1] prologue done, [2] first barrier passed, [3] end, and for position i at
 * 4 + 10*i + {0: inputs staged, 1: W_hh products done, 2: W2 pass + CTA argmax done,
 * 3: argmax barrier passed, 4: embedding row staged, 5: W_ih products done, 6: state and W1
 * partials done, 7: state barrier passed}.  The persistent batched kernel (5..128 rows) records the
 * globaltimer (ns) of CTA 0: [0] start, [e] when it passed grid barrier e (phases C0, D, E, then per
 * position A, B, C, D, E -- B absent with a projection table -- and A alone at the last position),
 * then its end.  The teacher-forced recurrence of 5..128 rows (k_tf_units) records the globaltimer
 * of CTA 0: [0] start, [1] set-up issued, [i + 2] update i done, [L + 1] end; and, from entry 128,
 * per CTA c the milestones k of update 1 at [128 + k * G + c] (G = Hs / 8 CTAs; k: 0 start, 1 copies
 * issued, 2 copies landed, 3 MMAs issued, 4 accumulator in the epilogue, 5 cell done and counted).
 * NULL turns it off.  Process-wide. */
DOMINO_API int domino_debug_set_trace(void* device_buf, int32_t n_entries);

/* Test and tuning hook for the tensor-core GEMM engine behind the batched paths:
 *   out[m * ldo + n] = sum_k A[m][k mod K'] * B[n][k]      (trans = 0)
 *   out[n * ldo + m] = the same                             (trans = 1)
 * A [M, K'] bf16 with K' = a_kwrap (0: K' = K; else K is a multiple of K'), B [N, K] bf16, out fp32,
 * all device memory, 16-byte aligned; K a multiple of 64.  bn (16, 32, 64 or 128: output tile width)
 * and ks (1..8: K split over a cluster of ks CTAs, partials added in a fixed order) force a plan;
 * bn = ks = 0 takes the plan the library would choose for a batch-sized N.  The profiling hook
 * (domino_debug_set_trace) also receives this kernel's per-CTA stamps when its buffer holds
 * 16 entries per CTA.  Returns DOMINO_OK, DOMINO_ERR_INVALID_ARGUMENT, DOMINO_ERR_UNSUPPORTED or
 * DOMINO_ERR_CUDA (e.g. a forced cluster that cannot launch). */
DOMINO_API int domino_debug_gemm(const void* A, const void* B, int32_t M, int32_t N, int32_t K, int32_t a_kwrap,
                                 float* out, int64_t ldo, int32_t trans, int32_t bn, int32_t ks,
                                 int32_t* status_dev, domino_stream_t stream);

/* Measurement aid: one launch in which each of one CTA per SM re-reads its contiguous slice of
 * `buf` (device memory, 16-byte aligned, `bytes` long) `passes` times (1..1000) with 16-byte
 * read-only loads, the access pattern of the fused kernel's W2 pass.  Timing 1 and n passes of a
 * buffer that fits L2 gives the L2 re-read bandwidth used for the reuse-aware roofline.  Returns
 * DOMINO_OK, DOMINO_ERR_INVALID_ARGUMENT or DOMINO_ERR_CUDA. */
DOMINO_API int domino_debug_read_passes(const void* buf, size_t bytes, int32_t passes, domino_stream_t stream);

/* Test hook: iteration limit of the library's bounded device-wide waits (0 restores the
 * default, about one second).  A tiny limit makes waits give up early, which exercises the
 * DOMINO_STATUS_DEVICE_TIMEOUT path without faulting or hanging the GPU.  Process-wide; takes
 * effect at the next launch.  Returns DOMINO_OK. */
DOMINO_API int domino_debug_set_spin_limit(uint64_t limit);

#ifdef __cplusplus
}
#endif

#endif /* DOMINO_H_ */
