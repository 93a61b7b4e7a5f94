// Decode step dispatch: builds the kernel parameters and picks the head-size
// translation unit. The kernels and their design are in decode_impl.cuh.
#include "decode.cuh"

namespace gdn {

gdn_status_t decode_launch(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, float* pool, int num_slots, const int32_t* slot_ids,
                           void* o, int B, int T, int H, int Hqk, int dk, int dv, int nh, float scale,
                           uint32_t flags, float* token_states, int update_pool, gdn_dtype_t in,
                           gdn_dtype_t out, unsigned int* err, cudaStream_t stream) {
  (void)dv;
  DecodeParams p{q, k, v, g, beta, pool, slot_ids, o, err, B, H, num_slots, 0, scale, Hqk, flags,
                 token_states, update_pool};
  switch (dk) {
    case 32: return decode_launch_d32(p, T, nh, in, out, stream);
    case 64: return decode_launch_d64(p, T, nh, in, out, stream);
    case 128: return decode_launch_d128(p, T, nh, in, out, stream);
    default: return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: dk must be 32, 64 or 128");
  }
}

}  // namespace gdn
