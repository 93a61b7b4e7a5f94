// Fused tensor-core chunk prefill (placeholder until the tcgen05 pipeline lands).
#include "prefill.cuh"

namespace gdn {
gdn_status_t prefill_fused_launch(const PrefillShape&, const PrefillArgs&, cudaStream_t) {
  return fail(GDN_ERR_UNSUPPORTED, "fused tensor-core prefill is not built yet");
}
}  // namespace gdn
