// Decode kernels instantiated for dk = dv = 64 (one translation unit per head size
// so that the many (T, n_h, dtype) instantiations compile in parallel).
#include "decode_impl.cuh"

namespace gdn {

gdn_status_t decode_launch_d64(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s) {
  return launch_steps<64>(p, T, nh, in, out, s);
}

}  // namespace gdn
