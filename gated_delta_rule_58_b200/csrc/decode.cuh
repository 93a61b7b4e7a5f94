// Internal interface between the decode dispatcher (decode.cu) and the per-head-size
// translation units that instantiate the decode kernels (decode_d32.cu,
// decode_d64.cu, decode_d128.cu; the kernels themselves are in decode_impl.cuh).
#pragma once

#include "common.cuh"

namespace gdn {

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  float* pool;
  const int32_t* slot_ids;
  void* o;
  unsigned int* err;
  int B, H, num_slots;
  int n_items;
  float scale;
  int Hqk;         // query/key heads; value head h reads q/k head h / (H / Hqk)
  uint32_t flags;  // GDN_QK_L2NORM
  float* token_states;  // [B, T, H, dv, dk] state after each token, or null
  int update_pool;      // 0: the pool is only read (speculative verification)
};

// Launches the decode step for one head size (dk = dv = 32, 64 or 128).
gdn_status_t decode_launch_d32(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s);
gdn_status_t decode_launch_d64(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s);
gdn_status_t decode_launch_d128(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s);

}  // namespace gdn
