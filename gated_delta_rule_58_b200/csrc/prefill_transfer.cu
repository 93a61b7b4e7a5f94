// Chunk-parallel prefill with an inter-segment fixup scan, for few (sequence,
// head) pairs with long sequences.
//
// The chunk recurrence is affine in the state: S_{c+1} = M_c S_c + H_c with the
// transfer matrix M_c and the local state H_c (the local-state / transfer /
// fixed-state structure of the FlashInfer PR #3866 page, "CP delta-rule
// precompute at ultra-low parallelism", section 2). Affine maps compose, so a
// segment of G consecutive chunks is again S_end = M_seg S_start + H_seg. The
// path runs:
//
//   1. segment map: cuts every sequence into segments of G chunks (G * 64
//      tokens, the last one partial) and lists their token boundaries;
//   2. local states: the fused chunk kernel over all segments at once, each from
//      a zero state, final state = H_seg (K-last, i.e. H_seg^T);
//   3. transfers: the same kernel from the identity state with the values taken
//      as zero, final state = M_seg (stored K-last, i.e. M_seg^T row-major);
//   4. fixup scan (SIMT, fp32): per (sequence, head), the state rows split across
//      CTAs, fixed[s] = S; S^T <- S^T M_seg^T + H_seg^T over the sequence's
//      segments, then the final state (the serial part; the PR #3866 page's SIMT
//      fixup loop, with the next segment's transfer matrix staged ahead);
//   5. outputs: the fused kernel over all segments, each from its fixed state.
//
// Steps 2, 3 and 5 use every SM even for a single sequence; only step 4 is
// serial, with G times fewer steps than there are chunks. G is the smallest
// power of two that fits steps 2/3/5 into about one wave of CTAs (one per SM):
// more segments would add fixup steps without shortening those passes.
#include <string>

#include "device_once.h"
#include "prefill.cuh"
#include "tcgen05.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int kFixRows = 4;       // state rows (value indices) per fixup CTA
constexpr int kFixRPT = kFixRows / 4;  // rows per thread (four row groups per warp)
constexpr int kFixThreads = 128;  // 4 warps; each thread a kFixRPT x 4 tile of the block

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct TransferLayout {
  int seg_chunks;     // G
  int max_segments;   // upper bound on segments over all sequences
  size_t off_seg_cu, off_seg_of_seq, off_local, off_transfer, off_fixed, total;
};

// Segment CTAs wanted per state run: one per SM of a B200 (148 SMs). A constant,
// so that the workspace size is a pure function of the shape.
constexpr long long kTargetSegmentCtas = 148;

TransferLayout layout_for(const PrefillShape& s) {
  TransferLayout L{};
  const long long chunks = (s.total_T + C - 1) / C + s.N;  // upper bound on chunks
  int g = 1;
  while (g < 64 && (long long)s.H * chunks / g > kTargetSegmentCtas) g *= 2;
  L.seg_chunks = g;
  L.max_segments = (int)(s.total_T / ((long long)g * C) + s.N);
  const size_t state_bytes = (size_t)s.H * D * D * sizeof(float);
  size_t off = 0;
  L.off_seg_cu = off;
  off = align256(off + sizeof(int32_t) * ((size_t)L.max_segments + 1));
  L.off_seg_of_seq = off;
  off = align256(off + sizeof(int32_t) * ((size_t)s.N + 1));
  L.off_local = off;
  off = align256(off + state_bytes * L.max_segments);
  L.off_transfer = off;
  off = align256(off + state_bytes * L.max_segments);
  L.off_fixed = off;
  off = align256(off + state_bytes * L.max_segments);
  L.total = off;
  return L;
}

// 1. Segment map (one CTA): seg_of_seq[n] = index of sequence n's first segment
//    (exclusive prefix sum of ceil(L_n / (G C))), seg_cu = token boundaries of all
//    segments; unused tail entries are empty segments at the end of the last sequence.
__global__ void __launch_bounds__(1024)
gdn_segment_map_kernel(const int32_t* cu, int N, int64_t total_T, int seg_len, int max_segments,
                       int32_t* seg_cu, int32_t* seg_of_seq, unsigned int* err) {
  __shared__ int32_t carry;
  __shared__ int32_t warp_sums[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += 1024) {
    const int n = base + tid;
    int cnt = 0;
    if (n < N) {
      const int32_t a = cu[n], b = cu[n + 1];
      if (a < 0 || b < a || (int64_t)b > total_T || (n == 0 && a != 0)) {
        raise_device_error(err, GDN_DEVERR_BAD_CU_SEQLENS);
      } else {
        cnt = (b - a + seg_len - 1) / seg_len;
      }
    }
    // block-wide exclusive scan of cnt
    int x = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int excl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x - cnt;
    if (n < N) {
      seg_of_seq[n] = excl;
      const int32_t a = cu[n];
      for (int k = 0; k < cnt && excl + k < max_segments; ++k) seg_cu[excl + k] = a + k * seg_len;
    }
    __syncthreads();
    if (tid == 1023) carry = excl + cnt;
    __syncthreads();
  }
  const int total = carry;
  if (tid == 0) seg_of_seq[N] = total;
  // the last real segment ends where the last sequence ends
  const int32_t end = (N > 0) ? cu[N] : 0;
  for (int i = total + tid; i <= max_segments; i += 1024) seg_cu[i] = end;
}

// 4. Fixup scan over the segments of one (sequence, head), kFixRows rows of S^T
//    per CTA: fixed[s] = S, then S^T <- S^T M^T + H^T, in fp32 (the products
//    compose along the whole sequence, so no reduced-precision operands here).
//    Each segment's transfer matrix (64 KiB) and local-state rows are staged in
//    shared memory by one bulk copy, one segment ahead (two buffers). Thread
//    (warp w, lane = 8 rg + cg) owns kFixRPT rows from kFixRPT * rg and columns
//    32w + 4cg .. +3
//    of the block; the state block is kept transposed in shared memory (sT[i][j])
//    for the products and in registers (the thread's own tile) for the stores.
constexpr uint32_t kFixMtBytes = D * D * 4;
constexpr uint32_t kFixLocBytes = kFixRows * D * 4;
constexpr uint32_t kFixSmem = 2 * kFixMtBytes + 2 * kFixLocBytes + D * kFixRows * 4 + 64;
constexpr uint64_t kFixWaitNs = 2000000000ull;

// `local` may be null: the local states are then zero and only the transfer is copied.
__device__ __forceinline__ void fixup_issue(float* mt, float* loc, uint64_t* bar, const float* transfer,
                                            const float* local, size_t off, int r0) {
  tc::fence_proxy_async_smem();  // earlier generic reads of this buffer precede the copy
  tc::mbar_arrive_expect_tx(bar, kFixMtBytes + (local ? kFixLocBytes : 0u));
  tc::bulk_load(tc::smem_u32(mt), transfer + off, kFixMtBytes, bar);
  if (local) tc::bulk_load(tc::smem_u32(loc), local + off + (size_t)r0 * D, kFixLocBytes, bar);
}

// The segments of sequence n: seg_of_seq[n] .. seg_of_seq[n+1]-1 (the transfer
// path), or, with seg_of_seq null, the context-parallel ranks 0 .. cp_count-1 of a
// rank-major [ranks][N] list: entries n, n + cp_stride, ... (cp_stride = N). A launch
// may carry two folds over the same transfers (blockIdx.y picks the job). In a job,
// `fixed` may be null (only the final state is wanted); `local` null means zero local
// states; init_identity starts from the identity instead of initial_state (which is
// then ignored), so the fold yields the composed transfer.
struct FixupJob {
  const float* local;
  const float* initial_state;
  int init_identity;
  float* fixed;
  float* final_state;
};

__global__ void __launch_bounds__(kFixThreads)
gdn_fixup_scan_kernel(const int32_t* seg_of_seq, int cp_stride, int cp_count, int H, const float* transfer,
                      const FixupJob job0, const FixupJob job1, unsigned int* err) {
  const FixupJob job = blockIdx.y ? job1 : job0;
  const float* local = job.local;
  const float* initial_state = job.initial_state;
  const int init_identity = job.init_identity;
  float* fixed = job.fixed;
  float* final_state = job.final_state;
  extern __shared__ __align__(16) uint8_t fsm[];
  float* mt = reinterpret_cast<float*>(fsm);                 // [2][D][D]
  float* loc = mt + 2 * D * D;                                // [2][kFixRows][D]
  float* sT = loc + 2 * kFixRows * D;                         // [D][kFixRows]
  uint64_t* full = reinterpret_cast<uint64_t*>(sT + D * kFixRows);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int rg = lane >> 3, cg = lane & 7;
  const int jr = kFixRPT * rg;           // first of my rows (within the block)
  const int l0 = 32 * w + 4 * cg;        // first of my four columns
  const int rblocks = D / kFixRows;
  const int rb = blockIdx.x % rblocks;
  const int nh = blockIdx.x / rblocks;
  const int n = nh / H, h = nh - (nh / H) * H;
  const int r0 = rb * kFixRows;
  const size_t ssz = (size_t)D * D;
  const size_t soff = ((size_t)n * H + h) * ssz;
  const int first = seg_of_seq ? seg_of_seq[n] : n;
  const int stride = seg_of_seq ? 1 : cp_stride;
  const int count = seg_of_seq ? seg_of_seq[n + 1] - first : cp_count;

  if (tid == 0) {
    tc::mbar_init(&full[0], 1);
    tc::mbar_init(&full[1], 1);
    tc::fence_mbar_init();
  }
  // my tile of the initial state (registers) and the transposed block (shared)
  float cur[kFixRPT][4];
#pragma unroll
  for (int a = 0; a < kFixRPT; ++a) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    const int row = r0 + jr + a;
    if (init_identity)
      x = make_float4(row == l0 ? 1.f : 0.f, row == l0 + 1 ? 1.f : 0.f, row == l0 + 2 ? 1.f : 0.f,
                      row == l0 + 3 ? 1.f : 0.f);
    else if (initial_state)
      x = *reinterpret_cast<const float4*>(initial_state + soff + (size_t)row * D + l0);
    cur[a][0] = x.x; cur[a][1] = x.y; cur[a][2] = x.z; cur[a][3] = x.w;
#pragma unroll
    for (int x4 = 0; x4 < 4; ++x4) sT[(l0 + x4) * kFixRows + jr + a] = cur[a][x4];
  }
  __syncthreads();
  if (tid == 0 && count > 0)
    fixup_issue(mt, loc, &full[0], transfer, local, ((size_t)first * H + h) * ssz, r0);

  int it = 0;
  bool pending_other = false;  // a prefetch into the other buffer is in flight
  for (int i = 0; i < count; ++i, ++it) {
    const int sg = first + i * stride;
    const int b = it & 1;
    pending_other = false;
    if (tid == 0 && i + 1 < count) {
      fixup_issue(mt + (b ^ 1) * D * D, loc + (b ^ 1) * kFixRows * D, &full[b ^ 1], transfer, local,
                  ((size_t)(sg + stride) * H + h) * ssz, r0);
      pending_other = true;
    }
    const bool got = tc::mbar_wait(&full[b], (it >> 1) & 1, kFixWaitNs);
    if (!__syncthreads_and(got)) {
      if (tid == 0) {
        raise_device_error(err, GDN_DEVERR_TIMEOUT);
        if (pending_other) tc::mbar_wait(&full[b ^ 1], ((it + 1) >> 1) & 1, kFixWaitNs);
      }
      return;
    }
    const size_t off = ((size_t)sg * H + h) * ssz;
    const float* m = mt + b * D * D;
    const float* lr = loc + b * kFixRows * D;
    float acc[kFixRPT][4];
#pragma unroll
    for (int a = 0; a < kFixRPT; ++a) {
      // the state at the segment start, then the local state as the accumulator
      if (fixed)
        *reinterpret_cast<float4*>(fixed + off + (size_t)(r0 + jr + a) * D + l0) =
            make_float4(cur[a][0], cur[a][1], cur[a][2], cur[a][3]);
      const float4 x = local ? *reinterpret_cast<const float4*>(lr + (jr + a) * D + l0)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      acc[a][0] = x.x; acc[a][1] = x.y; acc[a][2] = x.z; acc[a][3] = x.w;
    }
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float4 mv = *reinterpret_cast<const float4*>(m + i * D + l0);
#pragma unroll
      for (int a = 0; a < kFixRPT; ++a) {
        const float sv = sT[i * kFixRows + jr + a];
        acc[a][0] = fmaf(sv, mv.x, acc[a][0]);
        acc[a][1] = fmaf(sv, mv.y, acc[a][1]);
        acc[a][2] = fmaf(sv, mv.z, acc[a][2]);
        acc[a][3] = fmaf(sv, mv.w, acc[a][3]);
      }
    }
    __syncthreads();  // every read of sT and of this buffer is done
#pragma unroll
    for (int a = 0; a < kFixRPT; ++a)
#pragma unroll
      for (int x4 = 0; x4 < 4; ++x4) {
        cur[a][x4] = acc[a][x4];
        sT[(l0 + x4) * kFixRows + jr + a] = acc[a][x4];
      }
    __syncthreads();
  }
  if (final_state) {
#pragma unroll
    for (int a = 0; a < kFixRPT; ++a)
      *reinterpret_cast<float4*>(final_state + soff + (size_t)(r0 + jr + a) * D + l0) =
          make_float4(cur[a][0], cur[a][1], cur[a][2], cur[a][3]);
  }
}

}  // namespace

size_t prefill_transfer_workspace_bytes(const PrefillShape& s) { return layout_for(s).total; }

int prefill_transfer_segment_chunks(const PrefillShape& s) { return layout_for(s).seg_chunks; }

gdn_status_t prefill_transfer_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  const TransferLayout L = layout_for(s);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int32_t* seg_cu = reinterpret_cast<int32_t*>(ws + L.off_seg_cu);
  int32_t* seg_of_seq = reinterpret_cast<int32_t*>(ws + L.off_seg_of_seq);
  float* local = reinterpret_cast<float*>(ws + L.off_local);
  float* transfer = reinterpret_cast<float*>(ws + L.off_transfer);
  float* fixed = reinterpret_cast<float*>(ws + L.off_fixed);
  if ((long long)L.max_segments * s.H >= (1LL << 31) || (long long)s.N * s.H * (D / kFixRows) >= (1LL << 31))
    return fail(GDN_ERR_UNSUPPORTED, "transfer prefill: too many segments");

  gdn_segment_map_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, s.N, s.total_T, L.seg_chunks * C, L.max_segments,
                                                  seg_cu, seg_of_seq, a.err);
  gdn_status_t st = check_launch("transfer prefill: segment map");
  if (st != GDN_OK) return st;

  PrefillShape seg = s;
  seg.N = L.max_segments;
  PrefillArgs loc = a;
  loc.cu_seqlens = seg_cu;
  loc.initial_state = nullptr;
  loc.o = nullptr;
  loc.final_state = local;
  loc.mode = kPrefillLocalState;
  st = prefill_fused_launch(seg, loc, stream);
  if (st != GDN_OK) return st;
  PrefillArgs tr = loc;
  tr.final_state = transfer;
  tr.mode = kPrefillTransfer;
  st = prefill_fused_launch(seg, tr, stream);
  if (st != GDN_OK) return st;

  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("transfer prefill: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(gdn_fixup_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFixSmem);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("transfer prefill: setup: ") +
                    (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  const FixupJob job{local, a.initial_state, 0, fixed, a.final_state};
  gdn_fixup_scan_kernel<<<(unsigned)((long long)s.N * s.H * (D / kFixRows)), kFixThreads, kFixSmem, stream>>>(
      seg_of_seq, 0, 0, s.H, transfer, job, job, a.err);
  st = check_launch("transfer prefill: fixup scan");
  if (st != GDN_OK) return st;

  PrefillArgs out = a;
  out.cu_seqlens = seg_cu;
  out.initial_state = fixed;
  out.final_state = nullptr;
  out.mode = kPrefillOutputs;
  return prefill_fused_launch(seg, out, stream);
}

// Context parallelism, step 1, for any number of sequences: the slice's local state
// H (zero start) and transfer M (identity start, values zero), both K-last, from the
// transfer path's segment passes and two fixup scans over the segments (one from
// zero with the local states, one from the identity with zero local states). Uses
// the transfer prefill's workspace.
gdn_status_t cp_local_state_launch(const PrefillShape& s, const PrefillArgs& a, float* local_out, float* transfer_out,
                                   cudaStream_t stream) {
  const TransferLayout L = layout_for(s);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int32_t* seg_cu = reinterpret_cast<int32_t*>(ws + L.off_seg_cu);
  int32_t* seg_of_seq = reinterpret_cast<int32_t*>(ws + L.off_seg_of_seq);
  float* local = reinterpret_cast<float*>(ws + L.off_local);
  float* transfer = reinterpret_cast<float*>(ws + L.off_transfer);
  if ((long long)L.max_segments * s.H >= (1LL << 31) || (long long)s.N * s.H * (D / kFixRows) >= (1LL << 31))
    return fail(GDN_ERR_UNSUPPORTED, "cp local state: too many segments");
  gdn_segment_map_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, s.N, s.total_T, L.seg_chunks * C, L.max_segments,
                                                  seg_cu, seg_of_seq, a.err);
  gdn_status_t st = check_launch("cp local state: segment map");
  if (st != GDN_OK) return st;
  PrefillShape seg = s;
  seg.N = L.max_segments;
  PrefillArgs loc = a;
  loc.cu_seqlens = seg_cu;
  loc.initial_state = nullptr;
  loc.o = nullptr;
  loc.final_state = local;
  loc.mode = kPrefillLocalState;
  st = prefill_fused_launch(seg, loc, stream);
  if (st != GDN_OK) return st;
  PrefillArgs tr = loc;
  tr.final_state = transfer;
  tr.mode = kPrefillTransfer;
  st = prefill_fused_launch(seg, tr, stream);
  if (st != GDN_OK) return st;
  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("cp local state: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(gdn_fixup_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFixSmem);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("cp local state: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  // both folds in one launch: y = 0 the local states from zero, y = 1 the transfers
  // from the identity with zero local states
  const dim3 grid((unsigned)((long long)s.N * s.H * (D / kFixRows)), 2);
  const FixupJob fold_local{local, nullptr, 0, nullptr, local_out};
  const FixupJob fold_transfer{nullptr, nullptr, 1, nullptr, transfer_out};
  gdn_fixup_scan_kernel<<<grid, kFixThreads, kFixSmem, stream>>>(seg_of_seq, 0, 0, s.H, transfer, fold_local,
                                                                  fold_transfer, a.err);
  return check_launch("cp local state: fixup scans");
}

// Context parallelism, step 4, after cp_local_state_launch on the same slice and
// workspace: the segments' start states from the rank's start state (a.initial_state),
// the final state, and the outputs of every segment, reusing the segment map, local
// states and transfers left in the workspace.
gdn_status_t cp_finish_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  const TransferLayout L = layout_for(s);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int32_t* seg_cu = reinterpret_cast<int32_t*>(ws + L.off_seg_cu);
  int32_t* seg_of_seq = reinterpret_cast<int32_t*>(ws + L.off_seg_of_seq);
  float* local = reinterpret_cast<float*>(ws + L.off_local);
  float* transfer = reinterpret_cast<float*>(ws + L.off_transfer);
  float* fixed = reinterpret_cast<float*>(ws + L.off_fixed);
  if ((long long)L.max_segments * s.H >= (1LL << 31) || (long long)s.N * s.H * (D / kFixRows) >= (1LL << 31))
    return fail(GDN_ERR_UNSUPPORTED, "cp finish: too many segments");
  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("cp finish: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(gdn_fixup_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFixSmem);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("cp finish: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  const FixupJob job{local, a.initial_state, 0, fixed, a.final_state};
  gdn_fixup_scan_kernel<<<(unsigned)((long long)s.N * s.H * (D / kFixRows)), kFixThreads, kFixSmem, stream>>>(
      seg_of_seq, 0, 0, s.H, transfer, job, job, a.err);
  gdn_status_t st = check_launch("cp finish: fixup scan");
  if (st != GDN_OK) return st;
  PrefillShape seg = s;
  seg.N = L.max_segments;
  PrefillArgs out = a;
  out.cu_seqlens = seg_cu;
  out.initial_state = fixed;
  out.final_state = nullptr;
  out.mode = kPrefillOutputs;
  return prefill_fused_launch(seg, out, stream);
}

gdn_status_t cp_combine_launch(const float* local_states, const float* transfers, int ranks, int rank, int N, int H,
                               const float* initial_state, float* start_state, unsigned int* err,
                               cudaStream_t stream) {
  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("cp combine: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(gdn_fixup_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFixSmem);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("cp combine: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  (void)ranks;
  if ((long long)N * H * (D / kFixRows) >= (1LL << 31)) return fail(GDN_ERR_UNSUPPORTED, "cp combine: N * H too large");
  const FixupJob job{local_states, initial_state, 0, nullptr, start_state};
  gdn_fixup_scan_kernel<<<(unsigned)((long long)N * H * (D / kFixRows)), kFixThreads, kFixSmem, stream>>>(
      nullptr, N, rank, H, transfers, job, job, err);
  return check_launch("gdn_cp_combine");
}

}  // namespace gdn
