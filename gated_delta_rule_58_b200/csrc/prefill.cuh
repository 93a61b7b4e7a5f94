// Internal prefill interfaces shared by the prefill translation units.
#pragma once

#include "common.cuh"

namespace gdn {

struct PrefillShape {
  int N;            // sequences
  int64_t total_T;  // packed tokens
  int H, dk, dv, chunk;
  int Hqk;          // query/key heads (H is a multiple); value head h reads q/k head h / (H / Hqk)
};

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  const int32_t* cu_seqlens;
  const float* initial_state;
  float* final_state;
  void* o;
  float scale;
  gdn_dtype_t in_dtype, out_dtype;
  void* workspace;
  unsigned int* err;
  // Fused-kernel mode. kPrefillOutputs: the normal prefill. kPrefillLocalState:
  // zero initial state, no outputs (final state = the local state H of each
  // sequence). kPrefillTransfer: identity initial state, values taken as zero, no
  // outputs (final state = the transfer matrix M^T of each sequence, K-last).
  int mode;
  uint32_t flags;  // GDN_QK_L2NORM
};

constexpr int kPrefillOutputs = 0;
constexpr int kPrefillLocalState = 1;
constexpr int kPrefillTransfer = 2;

// Validates the shape for `requested` and resolves GDN_PREFILL_AUTO.
gdn_status_t prefill_resolve(const PrefillShape& s, gdn_dtype_t in, uint32_t flags, gdn_prefill_algo_t requested,
                             gdn_prefill_algo_t* resolved);
// AUTO choice between the two tensor-core algorithms (dk == dv == 128, chunk == 64).
gdn_prefill_algo_t prefill_auto_tensor_core(const PrefillShape& s);
size_t prefill_workspace_bytes(const PrefillShape& s, gdn_prefill_algo_t resolved);
gdn_status_t prefill_launch(const PrefillShape& s, const PrefillArgs& a, gdn_prefill_algo_t resolved,
                            cudaStream_t stream);

gdn_status_t prefill_sequential_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream);
gdn_status_t prefill_fused_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream);
size_t prefill_transfer_workspace_bytes(const PrefillShape& s);
// Chunks per segment (G) the transfer algorithm uses for this shape.
int prefill_transfer_segment_chunks(const PrefillShape& s);
gdn_status_t prefill_transfer_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream);
// Context parallelism: a slice's local state and transfer over segments (transfer
// path workspace).
gdn_status_t cp_local_state_launch(const PrefillShape& s, const PrefillArgs& a, float* local_out, float* transfer_out,
                                   cudaStream_t stream);
// Context parallelism: the slice's outputs and final state from the rank's start
// state, reusing the segments left in the workspace by cp_local_state_launch.
gdn_status_t cp_finish_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream);
// Context parallelism: the start state of rank `rank` from the (local state,
// transfer) pairs of ranks 0..rank-1, rank-major [ranks][N][H][128][128] (K-last).
gdn_status_t cp_combine_launch(const float* local_states, const float* transfers, int ranks, int rank, int N, int H,
                               const float* initial_state, float* start_state, unsigned int* err,
                               cudaStream_t stream);

// Reads cu_seqlens[n], cu_seqlens[n+1] and validates them against total_T; on a bad
// pair sets GDN_DEVERR_BAD_CU_SEQLENS and returns false (the caller skips the unit).
__device__ __forceinline__ bool seq_bounds(const int32_t* cu, int n, int64_t total_T,
                                           unsigned int* err, int64_t* bos, int64_t* eos) {
  const int32_t a = __ldg(cu + n), b = __ldg(cu + n + 1);
  if (a < 0 || b < a || (int64_t)b > total_T || (n == 0 && a != 0)) {
    raise_device_error(err, GDN_DEVERR_BAD_CU_SEQLENS);
    return false;
  }
  *bos = a;
  *eos = b;
  return true;
}

}  // namespace gdn
