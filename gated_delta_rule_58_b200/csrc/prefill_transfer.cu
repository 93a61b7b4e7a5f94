// Chunk-parallel transfer/fixup prefill (placeholder until implemented).
#include "prefill.cuh"

namespace gdn {
size_t prefill_transfer_workspace_bytes(const PrefillShape&) { return 0; }
gdn_status_t prefill_transfer_launch(const PrefillShape&, const PrefillArgs&, cudaStream_t) {
  return fail(GDN_ERR_UNSUPPORTED, "transfer prefill is not built yet");
}
}  // namespace gdn
