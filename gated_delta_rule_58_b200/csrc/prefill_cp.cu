// Context parallelism for long prefills: the tokens of every sequence are split
// into consecutive slices held by consecutive ranks (GPUs). The chunk recurrence
// is affine in the state, S_end = M S_start + H over any run of tokens (the
// local-state / transfer / fixed-state structure of the FlashInfer PR #3866 page,
// "CP delta-rule precompute at ultra-low parallelism", section 2, generalised
// from chunks to ranks), so a rank
//   1. computes its slice's local state H (zero start) and transfer M (identity
//      start, values taken as zero) with the transfer path's segment passes (the
//      fused chunk kernel over segments of every sequence, in parallel) and two
//      fixup scans that fold the segments' pairs (gdn_cp_local_state),
//   2. receives the pairs of all ranks (an all-gather by the caller, e.g. NCCL over
//      NVLink; 2 x 64 KiB per (sequence, head) and rank),
//   3. folds the pairs of the ranks before it into its start state, S^T <- S^T M^T
//      + H^T in fp32 from the sequence's initial state (gdn_cp_combine, the fixup
//      scan kernel over ranks), and
//   4. runs gdn_chunk_prefill on its slice from that start state, or gdn_cp_finish,
//      which reuses the segments' local states and transfers of step 1 from the
//      workspace (a fixup scan from the start state, then the output pass).
// The exchange is one collective of (M, H) pairs; nothing waits on another rank
// inside a kernel.
#include <string>

#include "prefill.cuh"

using gdn::fail;

namespace {

bool ptr_ok(const void* p) { return p != nullptr && gdn::aligned16(p); }

}  // namespace

extern "C" gdn_status_t gdn_cp_local_state_workspace_size(int N, int64_t total_T, int H, int dk, int dv, int chunk,
                                                          size_t* bytes) {
  if (!bytes) return fail(GDN_ERR_INVALID_ARG, "gdn_cp_local_state_workspace_size: bytes is NULL");
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H};
  gdn_prefill_algo_t resolved;
  const gdn_status_t st = gdn::prefill_resolve(s, GDN_BF16, 0, GDN_PREFILL_FUSED, &resolved);
  if (st != GDN_OK) return st;
  *bytes = gdn::prefill_transfer_workspace_bytes(s);
  return gdn::ok();
}

extern "C" gdn_status_t gdn_cp_local_state(const void* q, const void* k, const void* v, const float* g,
                                           const float* beta, const int32_t* cu_seqlens, int N, int64_t total_T,
                                           float* local_state, float* transfer, int H, int H_qk, int dk, int dv,
                                           int chunk, uint32_t flags, gdn_dtype_t in_dtype, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (!(in_dtype == GDN_BF16 || in_dtype == GDN_F32)) return fail(GDN_ERR_INVALID_ARG, "gdn_cp_local_state: unknown dtype");
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H_qk};
  gdn_prefill_algo_t resolved;
  gdn_status_t st = gdn::prefill_resolve(s, in_dtype, flags, GDN_PREFILL_FUSED, &resolved);
  if (st != GDN_OK) return st;
  if (N == 0) return gdn::ok();
  if (cu_seqlens == nullptr) return fail(GDN_ERR_INVALID_ARG, "gdn_cp_local_state: cu_seqlens is NULL");
  if (total_T > 0 && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || g == nullptr || beta == nullptr))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_local_state: q, k, v must be non-NULL and 16-byte aligned; g, beta non-NULL");
  if (!ptr_ok(local_state) || !ptr_ok(transfer))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_local_state: local_state and transfer must be non-NULL and 16-byte aligned");
  const size_t need = gdn::prefill_transfer_workspace_bytes(s);
  if (workspace == nullptr || workspace_bytes < need || !gdn::aligned16(workspace))
    return fail(GDN_ERR_WORKSPACE, "gdn_cp_local_state: workspace missing, misaligned or smaller than "
                                   "gdn_cp_local_state_workspace_size");
  unsigned int* err = nullptr;
  st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  gdn::PrefillArgs a{q, k, v, g, beta, cu_seqlens, nullptr, nullptr, nullptr, 1.f,
                     in_dtype, GDN_BF16, workspace, err, gdn::kPrefillOutputs, flags};
  return gdn::cp_local_state_launch(s, a, local_state, transfer, gdn::as_stream(stream));
}

extern "C" gdn_status_t gdn_cp_finish(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                      const int32_t* cu_seqlens, int N, int64_t total_T, const float* start_state,
                                      float* final_state, void* o, int H, int H_qk, int dk, int dv, int chunk,
                                      float scale, uint32_t flags, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!(in_dtype == GDN_BF16 || in_dtype == GDN_F32) || !(out_dtype == GDN_BF16 || out_dtype == GDN_F32))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_finish: unknown dtype");
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H_qk};
  gdn_prefill_algo_t resolved;
  gdn_status_t st = gdn::prefill_resolve(s, in_dtype, flags, GDN_PREFILL_FUSED, &resolved);
  if (st != GDN_OK) return st;
  if (N == 0) return gdn::ok();
  if (cu_seqlens == nullptr) return fail(GDN_ERR_INVALID_ARG, "gdn_cp_finish: cu_seqlens is NULL");
  if (total_T > 0 && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(o) || g == nullptr || beta == nullptr))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_finish: q, k, v, o must be non-NULL and 16-byte aligned; g, beta non-NULL");
  if ((start_state && !ptr_ok(start_state)) || (final_state && !ptr_ok(final_state)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_finish: state pointers must be 16-byte aligned");
  const size_t need = gdn::prefill_transfer_workspace_bytes(s);
  if (workspace == nullptr || workspace_bytes < need || !gdn::aligned16(workspace))
    return fail(GDN_ERR_WORKSPACE, "gdn_cp_finish: workspace missing, misaligned or smaller than "
                                   "gdn_cp_local_state_workspace_size");
  unsigned int* err = nullptr;
  st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  gdn::PrefillArgs a{q, k, v, g, beta, cu_seqlens, start_state, final_state, o, scale,
                     in_dtype, out_dtype, workspace, err, gdn::kPrefillOutputs, flags};
  return gdn::cp_finish_launch(s, a, gdn::as_stream(stream));
}

extern "C" gdn_status_t gdn_cp_combine(const float* local_states, const float* transfers, int ranks, int rank, int N,
                                       int H, int dk, int dv, const float* initial_state, float* start_state,
                                       void* stream) {
  if (ranks < 1 || rank < 0 || rank >= ranks || N < 0 || H < 1)
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_combine: need 0 <= rank < ranks, N >= 0, H >= 1");
  if (dk != 128 || dv != 128) return fail(GDN_ERR_UNSUPPORTED, "gdn_cp_combine: dk == dv == 128");
  if (N == 0) return gdn::ok();
  if (rank > 0 && (!ptr_ok(local_states) || !ptr_ok(transfers)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_combine: local_states and transfers must be non-NULL and 16-byte aligned");
  if (!ptr_ok(start_state)) return fail(GDN_ERR_INVALID_ARG, "gdn_cp_combine: start_state must be non-NULL and 16-byte aligned");
  if (initial_state && !ptr_ok(initial_state))
    return fail(GDN_ERR_INVALID_ARG, "gdn_cp_combine: initial_state is not 16-byte aligned");
  unsigned int* err = nullptr;
  gdn_status_t st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  return gdn::cp_combine_launch(local_states, transfers, ranks, rank, N, H, initial_state, start_state, err,
                                gdn::as_stream(stream));
}
