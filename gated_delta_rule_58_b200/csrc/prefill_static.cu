// gdn_chunk_prefill_static_scratch: the transfer prefill with library-owned
// scratch, for callers that cannot allocate device memory when they call.
//
// Some callers cannot call cudaMalloc (or any allocator) on their hot path: a
// plugin whose host framework owns every device allocation and forbids others,
// a serving engine that has reserved the whole device for its own memory pool,
// or a real-time loop that may not block on the driver's allocator. They can
// use this entry point: it is gdn_chunk_prefill with GDN_PREFILL_TRANSFER, except
// that the scratch the transfer algorithm needs (segment map, local states,
// transfer matrices, fixed states) lives in a fixed-size array that the library
// itself places in device memory.
//
// Limits and sharing:
//  - The array holds kStaticScratchBytes (32 MiB) on EVERY GPU that loads the
//    library, for as long as the process lives.
//  - Shapes whose transfer workspace exceeds that size are rejected with
//    GDN_ERR_WORKSPACE before anything is launched.
//  - All calls on a device share the one array. It keeps whatever the previous
//    call left in it; the transfer algorithm writes every scratch entry it later
//    reads, so nothing has to be cleared between calls. Calls that overlap on the
//    GPU (different streams, or work still running from another host thread)
//    race on the array and give undefined results: serialise them.
//  - The first call on each device looks the array's device address up (once,
//    with that device current). Make that first call before any stream capture.
#include <mutex>
#include <string>

#include "prefill.cuh"

namespace gdn {
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

// The scratch itself. In host code this name is only a handle to the symbol: the
// device address comes from cudaGetSymbolAddress below and is what the kernels get.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
void* g_static_scratch_addr[kMaxScratchDevices] = {nullptr};
std::mutex g_static_scratch_mutex;

// Device address of the scratch array on the current device (looked up once).
gdn_status_t static_scratch_address(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxScratchDevices) return fail(GDN_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_addr[dev]) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_static_scratch);
    if (e != cudaSuccess)
      return fail(GDN_ERR_CUDA, std::string("static scratch: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_static_scratch_addr[dev] = addr;
  }
  *ptr = g_static_scratch_addr[dev];
  return GDN_OK;
}

bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

}  // namespace
}  // namespace gdn

extern "C" gdn_status_t gdn_chunk_prefill_static_scratch(
    const void* q, const void* k, const void* v, const float* g, const float* beta, const int32_t* cu_seqlens,
    int N, int64_t total_T, const float* initial_state, float* final_state, void* o, int H, int H_qk, int dk,
    int dv, int chunk, float scale, uint32_t flags, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream) {
  using gdn::fail;
  if (!((in_dtype == GDN_BF16 || in_dtype == GDN_F32) && (out_dtype == GDN_BF16 || out_dtype == GDN_F32)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_static_scratch: unknown dtype");
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H_qk};
  gdn_prefill_algo_t resolved;
  gdn_status_t st = gdn::prefill_resolve(s, in_dtype, flags, GDN_PREFILL_TRANSFER, &resolved);
  if (st != GDN_OK) return st;
  if (N == 0) return gdn::ok();
  if (cu_seqlens == nullptr) return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_static_scratch: cu_seqlens is NULL");
  if (total_T > 0 && (!gdn::ptr_ok(q) || !gdn::ptr_ok(k) || !gdn::ptr_ok(v) || g == nullptr || beta == nullptr ||
                      o == nullptr))
    return fail(GDN_ERR_INVALID_ARG,
                "gdn_chunk_prefill_static_scratch: q, k, v must be non-NULL and 16-byte aligned; g, beta, o non-NULL");
  if ((initial_state && !gdn::ptr_ok(initial_state)) || (final_state && !gdn::ptr_ok(final_state)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_static_scratch: states must be 16-byte aligned");
  const size_t need = gdn::prefill_workspace_bytes(s, GDN_PREFILL_TRANSFER);
  if (need > gdn::kStaticScratchBytes)
    return fail(GDN_ERR_WORKSPACE, "gdn_chunk_prefill_static_scratch: this shape needs " + std::to_string(need) +
                                       " bytes of scratch; the library's static scratch holds " +
                                       std::to_string(gdn::kStaticScratchBytes) +
                                       " bytes (use gdn_chunk_prefill with a caller-provided workspace)");
  void* scratch = nullptr;
  st = gdn::static_scratch_address(&scratch);
  if (st != GDN_OK) return st;
  unsigned int* err = nullptr;
  st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  gdn::PrefillArgs a{q, k, v, g, beta, cu_seqlens, initial_state, final_state, o, scale,
                     in_dtype, out_dtype, scratch, err, gdn::kPrefillOutputs, flags};
  return gdn::prefill_transfer_launch(s, a, gdn::as_stream(stream));
}
