/*
 * gdn.h — C ABI of the B200 (sm_100a) gated delta rule library, libgdn.so.
 *
 * The method. Per head, an fp32 recurrent state S (dk x dv) evolves token by
 * token as the gated delta rule (Yang, Kautz, Hatamizadeh, "Gated Delta
 * Networks: Improving Mamba2 with Delta Rule", ICLR 2025):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t,                alpha_t = exp(g_t)
 *
 * The gated delta product (kernel family cake_gated_delta_product_mtp on the
 * FlashInfer PR #7156 page, "Cake GDP kernel: shared-memory reduction and
 * direct register loads", introduction and section 1) applies, per token, the
 * gate once and then n_h Householder updates (I - beta_j k_j k_j^T) S +
 * beta_j k_j v_j^T in order j = 1..n_h, then emits one output.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent) unless
 *    stated otherwise, densely packed, innermost dimension contiguous, 16-byte
 *    aligned. No stride arguments: the layouts are the ones documented here.
 *  - States are stored K-last: S^T row-major, [.., dv, dk] (fp32), the layout the
 *    FlashInfer PR #7156 page (section 1) loads as float4 rows over k, and the
 *    FlashInfer PR #3866 page ("CP delta-rule precompute at ultra-low
 *    parallelism", section 2) contracts over the second index.
 *  - The caller owns every buffer. The library never allocates, frees or
 *    synchronises; it only enqueues kernels on `stream` (a cudaStream_t passed as
 *    void*, NULL = legacy default stream). Calls are therefore capturable into CUDA
 *    graphs once the workspace size is known (the "prepare before capture" pattern
 *    of the FlashInfer PR #6291 page, section 3).
 *  - Every host-checkable error (null or misaligned pointer, bad size, unsupported
 *    combination, small workspace) returns a non-OK status BEFORE anything is
 *    launched; gdn_last_error() then gives a message (thread-local). This follows the
 *    host launcher of the FlashInfer PR #4593 page (section 1), which checks its
 *    arguments and reports each failure with a message before any launch. Errors that
 *    only the data can show (slot id out of range, non-monotone cu_seqlens) are
 *    detected on the device: the offending unit is skipped (never an out-of-bounds
 *    access) and a sticky device error word is set, read by gdn_get_device_error().
 *  - Input dtype: q, k, v are GDN_BF16 or GDN_F32 (same dtype for all three); g
 *    and beta are always fp32; o is GDN_BF16 (round-to-nearest-even) or GDN_F32.
 *  - Heads. H counts the value heads: v, g, beta, o and the states have H heads.
 *    q and k may have fewer, H_qk, with H a multiple of H_qk: value head h reads
 *    query/key head h / (H / H_qk), so consecutive value heads share one q/k head
 *    (grouped value heads, the layout of models whose q/k projections are repeated
 *    over value heads). H_qk = H is the one-to-one case. This and the q/k
 *    normalisation below are plain extensions of the recurrence; the pages do not
 *    discuss them.
 *  - flags: GDN_QK_L2NORM scales q and every k to unit Euclidean length per token
 *    (and per q/k head) inside the kernels before use, in fp32 (a zero vector
 *    stays zero); without it q and k are used as given.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative or inconsistent sizes */
  GDN_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dims, dtype, chunk, algorithm) */
  GDN_ERR_WORKSPACE = 3,     /* workspace pointer null or smaller than required */
  GDN_ERR_CUDA = 4,          /* a CUDA runtime call failed (message has the CUDA error) */
  GDN_ERR_DEVICE_DATA = 5    /* returned by gdn_get_device_error when the device flagged data */
} gdn_status_t;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype_t;

/* flags of gdn_decode / gdn_chunk_prefill */
#define GDN_QK_L2NORM 0x1u  /* normalise q and k to unit length per token, in the kernel */

/* Bits of the sticky device error word (gdn_get_device_error). */
#define GDN_DEVERR_SLOT_OUT_OF_RANGE 0x1u  /* a slot id >= num_slots was skipped */
#define GDN_DEVERR_BAD_CU_SEQLENS 0x2u     /* cu_seqlens not 0-based / non-decreasing / > total_T */
#define GDN_DEVERR_TIMEOUT 0x4u            /* a bounded wait inside a kernel gave up (2 s); the kernel unwound */

/*
 * gdn_decode — one decode step over a slot-indexed state pool, updated in place.
 *
 * Computes, for every batch row b with slot s = slot_ids[b] and every head h,
 * T tokens in order, each: S <- alpha_t S, then n_h Householder updates, then
 * o[b,t,h,:] = scale * S^T q[b,t,h,:]; the final S is written back to the pool
 * slot. n_h = 1, T = 1 is the gated delta rule decode step (the T=1 split-V
 * variant of the FlashInfer PR #7156 page); n_h > 1 and/or T > 1 is the gated
 * delta product multi-token step of the same page.
 *
 *   q          [B, T, H_qk, dk]       in_dtype
 *   k          [B, T, H_qk, n_h, dk]  in_dtype
 *   v          [B, T, H, n_h, dv]     in_dtype
 *   g          [B, T, H]            fp32, log-space gate (alpha = exp(g); -inf allowed)
 *   beta       [B, T, H, n_h]       fp32
 *   state_pool [num_slots, H, dv, dk] fp32, K-last; read and written in place
 *   slot_ids   [B] int32. Negative id: row skipped (pool untouched, o rows set to 0).
 *              Id >= num_slots: same, and GDN_DEVERR_SLOT_OUT_OF_RANGE is set.
 *              Ids must be distinct (duplicates race: undefined result).
 *   o          [B, T, H, dv]        out_dtype
 *
 * Supported: dk == dv in {32, 64, 128}; T in {1, 2, 4, 8}, n_h in {1, 2, 4}, T * n_h <= 8.
 * scale: usually 1/sqrt(dk). Returns GDN_OK after enqueueing one kernel.
 */
gdn_status_t gdn_decode(const void* q, const void* k, const void* v, const float* g,
                        const float* beta, float* state_pool, int num_slots,
                        const int32_t* slot_ids, void* o, int B, int T, int H, int H_qk,
                        int dk, int dv, int n_h, float scale, uint32_t flags,
                        gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream);

/*
 * gdn_decode_mtp — gdn_decode that also records the state after every token, for
 * speculative (multi-token prediction) verification: the T tokens of a step are
 * draft tokens, and once the caller knows how many were accepted it restores the
 * state after the last accepted one (a rollback). The kernel family on the
 * FlashInfer PR #7156 page (introduction) carries "mtp" in its name; recording the
 * per-token states is the reading adopted here.
 *
 *   token_states [B, T, H, dv, dk] fp32, K-last, or NULL: the state of (b, h) after
 *                token t (after its gate and all n_h Householder updates). Rows of a
 *                skipped batch row (slot id < 0 or >= num_slots) are written as zeros.
 *   update_pool  1: the final state is written back to the pool slot (as gdn_decode);
 *                0: the pool is only read (verification without committing).
 *
 * Everything else, including validation, is as gdn_decode, which is this call with
 * token_states = NULL and update_pool = 1. The per-token states add T * dk * dv * 4
 * bytes of writes per (batch row, head).
 */
gdn_status_t gdn_decode_mtp(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float* state_pool, int num_slots,
                            const int32_t* slot_ids, void* o, float* token_states, int B, int T, int H,
                            int H_qk, int dk, int dv, int n_h, float scale, uint32_t flags, int update_pool,
                            gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream);

/* Prefill algorithm selection (gdn_chunk_prefill / gdn_chunk_prefill_workspace_size). */
typedef enum {
  GDN_PREFILL_AUTO = 0,       /* library picks from (N, H, total_T, dims) */
  GDN_PREFILL_FUSED = 1,      /* tcgen05 chunk pipeline, state kept on chip across chunks;
                                 dk == dv == 128, chunk == 64 */
  GDN_PREFILL_TRANSFER = 2,   /* chunk-parallel local states + transfer matrices, then the
                                 inter-chunk fixup scan, then outputs (the CP precompute
                                 structure of the FlashInfer PR #3866 page, section 2);
                                 for few (sequence, head) pairs with long sequences;
                                 dk == dv == 128, chunk == 64 */
  GDN_PREFILL_SEQUENTIAL = 3  /* token-sequential SIMT kernel, any dk == dv in {32, 64,
                                 128}; the chunk size does not change its arithmetic */
} gdn_prefill_algo_t;

/*
 * gdn_chunk_prefill_workspace_size — bytes of device workspace gdn_chunk_prefill
 * needs for these sizes and this algorithm (0 is a valid answer). Host-only, no
 * CUDA call: call it before stream capture. Returns (size_t)-1 for arguments
 * gdn_chunk_prefill would reject (see gdn_last_error).
 */
size_t gdn_chunk_prefill_workspace_size(int N, int64_t total_T, int H, int dk, int dv, int chunk,
                                        gdn_prefill_algo_t algo);

/*
 * gdn_chunk_prefill — chunked prefill over varlen sequences packed by cu_seqlens.
 *
 * For each sequence n (tokens cu_seqlens[n] .. cu_seqlens[n+1]-1) and head h,
 * runs the recurrence from initial_state[n,h] (or zero) over the sequence,
 * writes o for every token and the state after the last token to
 * final_state[n,h]. Internally the sequence is cut into chunks of `chunk` tokens
 * starting at the sequence start (the last chunk may be partial); within a chunk
 * the WY/UT form with T = (I + tril(diag(beta) decay * K K^T))^{-1} is used, and
 * the chunk states are passed along as S_{c+1} = M_c S_c + H_c (transfer M_c,
 * local state H_c; FlashInfer PR #3866 page, section 2). An empty sequence
 * copies its initial state (or zeros) to final_state.
 *
 *   q, k          [total_T, H_qk, dk] in_dtype
 *   v             [total_T, H, dv]   in_dtype
 *   g, beta       [total_T, H]       fp32 (g finite)
 *   cu_seqlens    [N + 1] int32, DEVICE; cu[0] = 0, non-decreasing, cu[N] = total_T
 *   initial_state [N, H, dv, dk] fp32 or NULL (zero state)
 *   final_state   [N, H, dv, dk] fp32 or NULL (not written); may alias initial_state
 *   o             [total_T, H, dv]   out_dtype
 *   workspace     device buffer of >= gdn_chunk_prefill_workspace_size(...) bytes
 *                 (may be NULL when that size is 0), 256-byte aligned, owned by the
 *                 caller; must not be shared by calls that overlap on the GPU.
 *
 * Numerics: tensor-core products use fp16 operands with fp32 accumulation; the
 * state is carried in fp32. Inputs must therefore lie within the fp16 range
 * (|x| < 65504) on the FUSED and TRANSFER algorithms.
 */
gdn_status_t gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const int32_t* cu_seqlens, int N,
                               int64_t total_T, const float* initial_state, float* final_state,
                               void* o, int H, int H_qk, int dk, int dv, int chunk, float scale,
                               uint32_t flags, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                               gdn_prefill_algo_t algo, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * gdn_chunk_prefill_static_scratch — gdn_chunk_prefill with GDN_PREFILL_TRANSFER,
 * for callers that cannot allocate device memory when they call (a plugin whose
 * host framework owns every device allocation, a serving engine that has
 * reserved the whole device for its own pool, a loop that may not block on the
 * allocator). It allocates nothing: the transfer algorithm's scratch lives in a
 * 32 MiB array the library places in device memory, held on every GPU that loads
 * the library until the process exits. The pages have no counterpart of this
 * entry point; it is an addition of this library.
 *
 * Arguments, layouts and numerics are those of gdn_chunk_prefill (no workspace
 * arguments). A shape whose transfer workspace
 * (gdn_chunk_prefill_workspace_size(..., GDN_PREFILL_TRANSFER)) exceeds 32 MiB is
 * rejected with GDN_ERR_WORKSPACE before anything is launched. All calls on a
 * device share the one scratch array, which keeps the previous call's contents
 * (nothing in it needs clearing); calls that overlap on the GPU race on it and
 * must be serialised by the caller. The first call on each device looks up the
 * array's device address; make it before any stream capture.
 */
gdn_status_t gdn_chunk_prefill_static_scratch(const void* q, const void* k, const void* v, const float* g,
                                              const float* beta, const int32_t* cu_seqlens, int N,
                                              int64_t total_T, const float* initial_state,
                                              float* final_state, void* o, int H, int H_qk, int dk,
                                              int dv, int chunk, float scale, uint32_t flags,
                                              gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream);

/*
 * Context parallelism for long prefills (the chunk/context-parallel state passing
 * of the FlashInfer PR #3866 page, section 2, generalised from chunks to ranks).
 * The tokens of each of the N sequences are split into consecutive slices held by
 * consecutive ranks 0..ranks-1 (one GPU each). The recurrence is affine in the
 * state over any run of tokens, S_end = M S_start + H, so each rank:
 *   1. gdn_cp_local_state on its slice: H (from a zero state) and M (from the
 *      identity with the values taken as zero), both [N, H, dv, dk] fp32 K-last
 *      (the transfer as M^T row-major, i.e. K-last like a state);
 *   2. all-gathers both across ranks in rank order (by the caller, e.g. NCCL):
 *      rank-major [ranks, N, H, dv, dk];
 *   3. gdn_cp_combine: its start state from the pairs of ranks 0..rank-1 and the
 *      sequences' initial state (NULL = zero): S^T <- S^T M_r^T + H_r^T in fp32;
 *   4. gdn_chunk_prefill on its slice with initial_state = that start state, or
 *      gdn_cp_finish (below), which reuses step 1's segments; the last rank's final
 *      state is the sequences' final state.
 * gdn_cp_local_state: dk == dv == 128, chunk == 64; the slice's sequences are cut
 * into segments processed in parallel by the fused tensor-core kernel (local states
 * and transfers of every segment), then two fixup scans fold the segments' pairs;
 * workspace: gdn_cp_local_state_workspace_size bytes, 16-byte aligned (the transfer
 * prefill's), GDN_ERR_WORKSPACE otherwise; other arguments as gdn_chunk_prefill.
 * gdn_cp_combine: dk == dv == 128; rank 0 copies the initial state (or zeros);
 * start_state may alias initial_state. Both only enqueue on `stream`.
 */
gdn_status_t gdn_cp_local_state_workspace_size(int N, int64_t total_T, int H, int dk, int dv, int chunk,
                                               size_t* bytes);
gdn_status_t gdn_cp_local_state(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const int32_t* cu_seqlens, int N, int64_t total_T,
                                float* local_state, float* transfer, int H, int H_qk, int dk, int dv,
                                int chunk, uint32_t flags, gdn_dtype_t in_dtype, void* workspace,
                                size_t workspace_bytes, void* stream);
/*
 * gdn_cp_finish — step 4 without recomputing step 1: the slice's outputs o and final
 * state (NULL: not written) from the rank's start state (NULL = zero), reusing the
 * segments' local states and transfers that gdn_cp_local_state left in `workspace`.
 * The call must use the same slice (q, k, v, g, beta, cu_seqlens, N, total_T, H,
 * H_qk, dk, dv, chunk, flags) and the same workspace as that gdn_cp_local_state call,
 * with nothing else writing the workspace in between; the result then equals
 * gdn_chunk_prefill with GDN_PREFILL_TRANSFER on the slice. Other arguments and
 * errors as gdn_chunk_prefill.
 */
gdn_status_t gdn_cp_finish(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const int32_t* cu_seqlens, int N, int64_t total_T, const float* start_state,
                           float* final_state, void* o, int H, int H_qk, int dk, int dv, int chunk, float scale,
                           uint32_t flags, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* workspace,
                           size_t workspace_bytes, void* stream);
gdn_status_t gdn_cp_combine(const float* local_states, const float* transfers, int ranks, int rank, int N,
                            int H, int dk, int dv, const float* initial_state, float* start_state,
                            void* stream);

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* gdn_last_error(void);

/*
 * gdn_chunk_prefill_backward — derivatives of a loss L with respect to the inputs
 * of gdn_chunk_prefill, given dL/do (d_o) and dL/dS_final (d_final_state, NULL =
 * zero), for training. The pages give no backward pass: this is the chain rule on
 * the gated delta rule's token relations S_t = alpha_t (I - beta_t k_t k_t^T)
 * S_{t-1} + beta_t k_t v_t^T, o_t = scale S_t^T q_t, alpha_t = exp(g_t), walked from
 * the last token to the first (one Householder per token). With GDN_QK_L2NORM the
 * relations read k / |k| and q / |q| (as in gdn_chunk_prefill) and the derivatives
 * are taken through that normalisation (zero for a zero vector).
 *
 * Inputs as gdn_chunk_prefill (q, k [total_T, H_qk, dk]; v [total_T, H, dv]; g, beta
 * [total_T, H] fp32; cu_seqlens [N+1] int32 on the device; initial_state [N, H, dv,
 * dk] fp32 K-last or NULL), plus d_o [total_T, H, dv] in in_dtype. Outputs, fp32,
 * caller-owned: d_q, d_k [total_T, H_qk, dk] (value heads that share a q/k head add
 * up), d_v [total_T, H, dv], d_g, d_beta [total_T, H] (d_q, d_k, d_g and d_beta are
 * cleared on `stream` first), d_initial_state [N, H, dv, dk] K-last or NULL (not
 * written).
 * dk == dv in {32, 64, 128}; flags: GDN_QK_L2NORM or 0 (GDN_ERR_INVALID_ARG otherwise);
 * q, k, v, d_o, d_q, d_k and the state pointers 16-byte aligned.
 *
 * Token-sequential, one CTA (one warp) per 1024 / dk value columns of a (sequence,
 * head) (the columns of the state evolve independently): a forward pass writes the state at the start of
 * every `chunk` tokens to the workspace, then each chunk, last to first, is
 * recomputed from its checkpoint into the workspace and walked backwards. d_q, d_k,
 * d_g and d_beta are sums over column blocks (and grouped heads) taken with fp32
 * atomics: their last bits may differ between calls; d_v and d_initial_state are
 * written directly and are reproducible. The
 * workspace (gdn_chunk_prefill_backward_workspace_size; 16-byte aligned, contents
 * need no clearing) holds H x (total_T / chunk + N + 1) checkpoints and N x H x
 * (chunk + 1) recomputed states of dk x dv fp32. Errors: GDN_ERR_INVALID_ARG /
 * GDN_ERR_UNSUPPORTED / GDN_ERR_WORKSPACE before anything is launched; a malformed
 * cu_seqlens pair sets GDN_DEVERR_BAD_CU_SEQLENS and skips that sequence. Only
 * enqueues on `stream` (four memsets and one kernel).
 */
gdn_status_t gdn_chunk_prefill_backward_workspace_size(int N, int64_t total_T, int H, int dk, int dv, int chunk,
                                                       size_t* bytes);
gdn_status_t gdn_chunk_prefill_backward(const void* q, const void* k, const void* v, const float* g,
                                        const float* beta, const int32_t* cu_seqlens, int N, int64_t total_T,
                                        const float* initial_state, const void* d_o, const float* d_final_state,
                                        float* d_q, float* d_k, float* d_v, float* d_g, float* d_beta,
                                        float* d_initial_state, int H, int H_qk, int dk, int dv, int chunk,
                                        float scale, uint32_t flags, gdn_dtype_t in_dtype, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * gdn_get_device_error — read and clear the sticky device error word of the
 * current CUDA device (GDN_DEVERR_* bits). Synchronous: waits for all prior work
 * on the device. Returns GDN_OK when the word was 0, GDN_ERR_DEVICE_DATA when a
 * bit was set (*flags gets the word), GDN_ERR_CUDA on a CUDA failure.
 */
gdn_status_t gdn_get_device_error(uint32_t* flags);

/*
 * gdn_selftest_wait_timeout — a check of the failure reporting, for tests and
 * health checks. Every wait inside the library's kernels (on an mbarrier phase) is
 * bounded; when one gives up the kernel sets GDN_DEVERR_TIMEOUT in the device
 * error word and unwinds instead of hanging. This call enqueues one small kernel
 * that performs such a bounded wait, for wait_us microseconds, on a barrier that
 * nothing completes, so the wait always gives up: afterwards gdn_get_device_error
 * reports GDN_DEVERR_TIMEOUT and the CUDA context remains usable. wait_us must be in
 * [1, 10^7]; GDN_ERR_INVALID_ARG otherwise (nothing launched). The pages have no
 * counterpart (the error conventions follow the checked errors of the FlashInfer
 * PR #4593 page, section 1, host launcher).
 */
gdn_status_t gdn_selftest_wait_timeout(uint32_t wait_us, void* stream);

/* Library version, e.g. "gdn 0.1.0 sm_100a". */
const char* gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
