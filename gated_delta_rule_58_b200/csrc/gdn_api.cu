// C ABI entry points of libgdn.so: argument validation, dispatch, error reporting.
// Declared in include/gdn.h; every check here runs before anything is launched.
#include <cstdio>
#include <mutex>
#include <string>

#include "common.cuh"
#include "prefill.cuh"
#include "tcgen05.cuh"

namespace gdn {

// Sticky device error word (GDN_DEVERR_* bits), one per device context.
__device__ unsigned int g_device_error_word = 0;

namespace {
thread_local std::string t_last_error;

constexpr int kMaxDevices = 64;
unsigned int* g_error_word_addr[kMaxDevices] = {nullptr};
std::mutex g_error_word_mutex;
}  // namespace

gdn_status_t fail(gdn_status_t st, const std::string& msg) {
  t_last_error = msg;
  return st;
}

gdn_status_t ok() {
  t_last_error.clear();
  return GDN_OK;
}

gdn_status_t check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(GDN_ERR_CUDA, std::string(what) + ": launch failed: " + cudaGetErrorString(e));
  return ok();
}

gdn_status_t device_error_word(unsigned int** word) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(GDN_ERR_UNSUPPORTED, "device index too large");
  std::lock_guard<std::mutex> lock(g_error_word_mutex);
  if (!g_error_word_addr[dev]) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_device_error_word);
    if (e != cudaSuccess)
      return fail(GDN_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_error_word_addr[dev] = static_cast<unsigned int*>(addr);
  }
  *word = g_error_word_addr[dev];
  return GDN_OK;
}

gdn_status_t decode_launch(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, float* pool, int num_slots, const int32_t* slot_ids,
                           void* o, int B, int T, int H, int Hqk, int dk, int dv, int nh, float scale,
                           uint32_t flags, float* token_states, int update_pool, gdn_dtype_t in,
                           gdn_dtype_t out, unsigned int* err, cudaStream_t stream);

namespace {

// One thread waits, with the kernels' bounded wait, for a phase of a shared-memory
// mbarrier that nothing completes, then reports the timeout the way every kernel
// of the library does. No copies or tensor-memory allocations are in flight, so
// the kernel simply returns.
__global__ void gdn_selftest_timeout_kernel(unsigned int* err, uint64_t wait_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, wait_ns)) raise_device_error(err, GDN_DEVERR_TIMEOUT);
}

}  // namespace
}  // namespace gdn

using gdn::fail;

namespace {

bool valid_dtype(gdn_dtype_t d) { return d == GDN_BF16 || d == GDN_F32; }

#define GDN_REQUIRE(cond, st, msg) \
  do {                             \
    if (!(cond)) return fail(st, std::string(msg)); \
  } while (0)

#define GDN_REQUIRE_PTR(p, name)                                                          \
  do {                                                                                    \
    GDN_REQUIRE((p) != nullptr, GDN_ERR_INVALID_ARG, std::string(name) + " is NULL");      \
    GDN_REQUIRE(gdn::aligned16(p), GDN_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned"); \
  } while (0)

}  // namespace

extern "C" {

const char* gdn_last_error(void) { return gdn::t_last_error.c_str(); }

const char* gdn_version(void) { return "gdn 0.1.0 sm_100a"; }

gdn_status_t gdn_get_device_error(uint32_t* flags) {
  GDN_REQUIRE(flags != nullptr, GDN_ERR_INVALID_ARG, "gdn_get_device_error: flags is NULL");
  unsigned int* word = nullptr;
  gdn_status_t st = gdn::device_error_word(&word);
  if (st != GDN_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("gdn_get_device_error: ") + cudaGetErrorString(e));
  unsigned int value = 0;
  e = cudaMemcpy(&value, word, sizeof(value), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(word, 0, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("gdn_get_device_error: ") + cudaGetErrorString(e));
  *flags = value;
  if (value) return fail(GDN_ERR_DEVICE_DATA, "device flagged invalid data (see flags)");
  return gdn::ok();
}

gdn_status_t gdn_decode_mtp(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float* state_pool, int num_slots,
                            const int32_t* slot_ids, void* o, float* token_states, int B, int T, int H,
                            int H_qk, int dk, int dv, int n_h, float scale, uint32_t flags, int update_pool,
                            gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream) {
  GDN_REQUIRE(B >= 0 && T >= 1 && H >= 1 && n_h >= 1 && num_slots >= 0, GDN_ERR_INVALID_ARG,
              "gdn_decode: need B >= 0, T >= 1, H >= 1, n_h >= 1, num_slots >= 0");
  GDN_REQUIRE(H_qk >= 1 && H % H_qk == 0, GDN_ERR_INVALID_ARG,
              "gdn_decode: H_qk must be >= 1 and divide H");
  GDN_REQUIRE((flags & ~GDN_QK_L2NORM) == 0, GDN_ERR_INVALID_ARG, "gdn_decode: unknown flags");
  GDN_REQUIRE(update_pool == 0 || update_pool == 1, GDN_ERR_INVALID_ARG, "gdn_decode_mtp: update_pool must be 0 or 1");
  GDN_REQUIRE(valid_dtype(in_dtype) && valid_dtype(out_dtype), GDN_ERR_INVALID_ARG,
              "gdn_decode: unknown dtype");
  GDN_REQUIRE(dk == dv, GDN_ERR_UNSUPPORTED, "gdn_decode: dk must equal dv");
  GDN_REQUIRE(dk == 32 || dk == 64 || dk == 128, GDN_ERR_UNSUPPORTED,
              "gdn_decode: dk must be 32, 64 or 128");
  if (B == 0) return gdn::ok();
  GDN_REQUIRE_PTR(q, "gdn_decode: q");
  GDN_REQUIRE_PTR(k, "gdn_decode: k");
  GDN_REQUIRE_PTR(v, "gdn_decode: v");
  GDN_REQUIRE(g != nullptr && beta != nullptr, GDN_ERR_INVALID_ARG, "gdn_decode: g or beta is NULL");
  GDN_REQUIRE(slot_ids != nullptr, GDN_ERR_INVALID_ARG, "gdn_decode: slot_ids is NULL");
  GDN_REQUIRE_PTR(state_pool, "gdn_decode: state_pool");
  GDN_REQUIRE(o != nullptr, GDN_ERR_INVALID_ARG, "gdn_decode: o is NULL");
  if (token_states) GDN_REQUIRE_PTR(token_states, "gdn_decode_mtp: token_states");
  GDN_REQUIRE((long long)B * H * ((dv + 63) / 64) < (1LL << 31), GDN_ERR_UNSUPPORTED,
              "gdn_decode: B * H too large for one launch");
  unsigned int* err = nullptr;
  gdn_status_t st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  return gdn::decode_launch(q, k, v, g, beta, state_pool, num_slots, slot_ids, o, B, T, H, H_qk, dk, dv,
                            n_h, scale, flags, token_states, update_pool, in_dtype, out_dtype, err,
                            gdn::as_stream(stream));
}

gdn_status_t gdn_decode(const void* q, const void* k, const void* v, const float* g,
                        const float* beta, float* state_pool, int num_slots,
                        const int32_t* slot_ids, void* o, int B, int T, int H, int H_qk,
                        int dk, int dv, int n_h, float scale, uint32_t flags,
                        gdn_dtype_t in_dtype, gdn_dtype_t out_dtype, void* stream) {
  return gdn_decode_mtp(q, k, v, g, beta, state_pool, num_slots, slot_ids, o, nullptr, B, T, H, H_qk, dk, dv,
                        n_h, scale, flags, 1, in_dtype, out_dtype, stream);
}

gdn_status_t gdn_selftest_wait_timeout(uint32_t wait_us, void* stream) {
  GDN_REQUIRE(wait_us >= 1 && wait_us <= 10000000u, GDN_ERR_INVALID_ARG,
              "gdn_selftest_wait_timeout: wait_us must be in [1, 10^7]");
  unsigned int* err = nullptr;
  gdn_status_t st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  gdn::gdn_selftest_timeout_kernel<<<1, 32, 0, gdn::as_stream(stream)>>>(err, (uint64_t)wait_us * 1000u);
  return gdn::check_launch("gdn_selftest_wait_timeout");
}

size_t gdn_chunk_prefill_workspace_size(int N, int64_t total_T, int H, int dk, int dv, int chunk,
                                        gdn_prefill_algo_t algo) {
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H};
  gdn_prefill_algo_t resolved;
  if (gdn::prefill_resolve(s, GDN_BF16, 0, algo, &resolved) != GDN_OK) return (size_t)-1;
  return gdn::prefill_workspace_bytes(s, resolved);
}

gdn_status_t gdn_chunk_prefill(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const int32_t* cu_seqlens, int N,
                               int64_t total_T, const float* initial_state, float* final_state,
                               void* o, int H, int H_qk, int dk, int dv, int chunk, float scale,
                               uint32_t flags, gdn_dtype_t in_dtype, gdn_dtype_t out_dtype,
                               gdn_prefill_algo_t algo, void* workspace, size_t workspace_bytes,
                               void* stream) {
  GDN_REQUIRE(valid_dtype(in_dtype) && valid_dtype(out_dtype), GDN_ERR_INVALID_ARG,
              "gdn_chunk_prefill: unknown dtype");
  gdn::PrefillShape s{N, total_T, H, dk, dv, chunk, H_qk};
  gdn_prefill_algo_t resolved;
  gdn_status_t st = gdn::prefill_resolve(s, in_dtype, flags, algo, &resolved);
  if (st != GDN_OK) return st;
  if (N == 0) return gdn::ok();
  GDN_REQUIRE(cu_seqlens != nullptr, GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: cu_seqlens is NULL");
  if (total_T > 0) {
    GDN_REQUIRE_PTR(q, "gdn_chunk_prefill: q");
    GDN_REQUIRE_PTR(k, "gdn_chunk_prefill: k");
    GDN_REQUIRE_PTR(v, "gdn_chunk_prefill: v");
    GDN_REQUIRE(g != nullptr && beta != nullptr, GDN_ERR_INVALID_ARG,
                "gdn_chunk_prefill: g or beta is NULL");
    GDN_REQUIRE(o != nullptr, GDN_ERR_INVALID_ARG, "gdn_chunk_prefill: o is NULL");
  }
  if (initial_state) GDN_REQUIRE_PTR(initial_state, "gdn_chunk_prefill: initial_state");
  if (final_state) GDN_REQUIRE_PTR(final_state, "gdn_chunk_prefill: final_state");
  const size_t need = gdn::prefill_workspace_bytes(s, resolved);
  if (need > 0) {
    GDN_REQUIRE(workspace != nullptr && workspace_bytes >= need, GDN_ERR_WORKSPACE,
                "gdn_chunk_prefill: workspace needs " + std::to_string(need) + " bytes, got " +
                    std::to_string(workspace ? workspace_bytes : 0));
    GDN_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, GDN_ERR_INVALID_ARG,
                "gdn_chunk_prefill: workspace is not 256-byte aligned");
  }
  unsigned int* err = nullptr;
  st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  gdn::PrefillArgs a{q, k, v, g, beta, cu_seqlens, initial_state, final_state, o, scale,
                     in_dtype, out_dtype, workspace, err, gdn::kPrefillOutputs, flags};
  return gdn::prefill_launch(s, a, resolved, gdn::as_stream(stream));
}

}  // extern "C"
