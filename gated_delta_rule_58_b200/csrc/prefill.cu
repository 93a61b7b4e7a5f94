// Prefill algorithm selection and dispatch (host side).
#include <string>

#include "prefill.cuh"

namespace gdn {

// AUTO may pick the transfer (chunk-parallel fixup) algorithm.
constexpr bool kTransferPrefillBuilt = true;

gdn_prefill_algo_t prefill_auto_tensor_core(const PrefillShape& s) {
  if (!kTransferPrefillBuilt) return GDN_PREFILL_FUSED;
  // Few (sequence, head) pairs with long sequences leave most SMs idle on the fused
  // path (one chain of chunks per pair); the transfer path spreads the chunks of a
  // chain over all SMs and leaves only the short fixup scan serial.
  const long long pairs = (long long)s.N * s.H;
  const long long avg_len = s.N > 0 ? s.total_T / s.N : 0;
  if (pairs <= 16 && avg_len >= 8192) return GDN_PREFILL_TRANSFER;
  return GDN_PREFILL_FUSED;
}

gdn_status_t prefill_resolve(const PrefillShape& s, gdn_dtype_t in, gdn_prefill_algo_t requested,
                             gdn_prefill_algo_t* resolved) {
  (void)in;
  if (s.N < 0 || s.total_T < 0 || s.H < 1 || s.dk < 1 || s.dv < 1 || s.chunk < 1)
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: need N >= 0, total_T >= 0, H, dk, dv, chunk >= 1");
  if (s.total_T > (int64_t)INT32_MAX)
    return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill: total_T must fit int32 (cu_seqlens is int32)");
  const bool seq_ok = s.dk == s.dv && (s.dk == 32 || s.dk == 64 || s.dk == 128);
  const bool tc_ok = s.dk == 128 && s.dv == 128 && s.chunk == 64;
  switch (requested) {
    case GDN_PREFILL_SEQUENTIAL:
      if (!seq_ok) return fail(GDN_ERR_UNSUPPORTED, "sequential prefill: dk == dv in {32, 64, 128}");
      *resolved = requested;
      return ok();
    case GDN_PREFILL_FUSED:
    case GDN_PREFILL_TRANSFER:
      if (!tc_ok) return fail(GDN_ERR_UNSUPPORTED, "tensor-core prefill: dk == dv == 128, chunk == 64");
      *resolved = requested;
      return ok();
    case GDN_PREFILL_AUTO:
      if (tc_ok) {
        *resolved = prefill_auto_tensor_core(s);
        return ok();
      }
      if (seq_ok) {
        *resolved = GDN_PREFILL_SEQUENTIAL;
        return ok();
      }
      return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill: dk == dv in {32, 64, 128} required");
    default:
      return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: unknown algorithm");
  }
}

size_t prefill_workspace_bytes(const PrefillShape& s, gdn_prefill_algo_t resolved) {
  if (resolved == GDN_PREFILL_TRANSFER) return prefill_transfer_workspace_bytes(s);
  return 0;
}

gdn_status_t prefill_launch(const PrefillShape& s, const PrefillArgs& a, gdn_prefill_algo_t resolved,
                            cudaStream_t stream) {
  switch (resolved) {
    case GDN_PREFILL_SEQUENTIAL: return prefill_sequential_launch(s, a, stream);
    case GDN_PREFILL_FUSED: return prefill_fused_launch(s, a, stream);
    case GDN_PREFILL_TRANSFER: return prefill_transfer_launch(s, a, stream);
    default: return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: unresolved algorithm");
  }
}

}  // namespace gdn
