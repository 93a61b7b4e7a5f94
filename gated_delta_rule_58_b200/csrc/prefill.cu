// Prefill algorithm selection and dispatch (host side).
#include <string>

#include "prefill.cuh"

namespace gdn {

// AUTO may pick the transfer (chunk-parallel fixup) algorithm.
constexpr bool kTransferPrefillBuilt = true;

gdn_prefill_algo_t prefill_auto_tensor_core(const PrefillShape& s) {
  if (!kTransferPrefillBuilt) return GDN_PREFILL_FUSED;
  // Cost model in units of one chunk step of one CTA (the fused kernel's period).
  // Fused: one CTA per (sequence, head) walks its chunks, so the time is the
  // chunks per sequence (times the waves when the pairs exceed the SMs). Transfer:
  // three passes of the same kernel over segments of G chunks (one wave of
  // segment CTAs, or more when G is capped), plus a serial fixup scan whose step
  // costs about 0.7 of a chunk step, plus the launches. The constants were
  // measured on B200 (148 SMs). The average sequence length stands in for
  // the lengths (they are on the device); transfer is taken only when it is
  // clearly cheaper.
  constexpr long long kSms = 148;
  const long long pairs = (long long)s.N * s.H;
  if (pairs <= 0 || pairs > kSms || s.total_T <= 0) return GDN_PREFILL_FUSED;
  const long long chunks = (s.total_T / s.N + 63) / 64;  // per sequence, average
  const long long g = prefill_transfer_segment_chunks(s);
  const long long seg_per_seq = (chunks + g - 1) / g;
  const long long waves = (pairs * seg_per_seq + kSms - 1) / kSms;
  // + about 7 chunk steps of fixed cost: the segment map and three kernel launches
  const double transfer = 3.0 * (double)g * (double)waves + 0.7 * (double)seg_per_seq + 7.0;
  const double fused = (double)chunks;
  return transfer < 0.8 * fused ? GDN_PREFILL_TRANSFER : GDN_PREFILL_FUSED;
}

gdn_status_t prefill_resolve(const PrefillShape& s, gdn_dtype_t in, uint32_t flags, gdn_prefill_algo_t requested,
                             gdn_prefill_algo_t* resolved) {
  (void)in;
  if (s.N < 0 || s.total_T < 0 || s.H < 1 || s.dk < 1 || s.dv < 1 || s.chunk < 1)
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: need N >= 0, total_T >= 0, H, dk, dv, chunk >= 1");
  if (s.Hqk < 1 || s.H % s.Hqk != 0)
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: H_qk must be >= 1 and divide H");
  if ((flags & ~GDN_QK_L2NORM) != 0) return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: unknown flags");
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
