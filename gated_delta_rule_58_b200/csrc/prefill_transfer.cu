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
//   4. fixup scan (SIMT): per (sequence, head), the state rows split across CTAs,
//      fixed[s] = S; S^T <- S^T M_seg^T + H_seg^T over the sequence's segments,
//      then the final state (the serial part; the PR #3866 page's SIMT fixup
//      loop, with the next segment's transfer rows preloaded);
//   5. outputs: the fused kernel over all segments, each from its fixed state.
//
// Steps 2, 3 and 5 use every SM even for a single sequence; only step 4 is
// serial, with G times fewer steps than there are chunks. G is picked so that
// steps 2/3/5 have about four segment CTAs per SM.
#include <string>

#include "prefill.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int D = 128;
constexpr int kFixRows = 8;       // state rows (value indices) per fixup CTA
constexpr int kFixThreads = 128;  // one thread per key column

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct TransferLayout {
  int seg_chunks;     // G
  int max_segments;   // upper bound on segments over all sequences
  size_t off_seg_cu, off_seg_of_seq, off_local, off_transfer, off_fixed, total;
};

// Segment CTAs wanted per state run: about four per SM of a B200 (148 SMs). A
// constant, so that the workspace size is a pure function of the shape.
constexpr long long kTargetSegmentCtas = 4LL * 148;

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
      const int32_t a = cu[n], b = cu[n + 1];
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
//    per CTA: fixed[s] = S, then S^T <- S^T M^T + H^T. Thread l owns column l.
__global__ void __launch_bounds__(kFixThreads)
gdn_fixup_scan_kernel(const int32_t* seg_of_seq, int H, const float* local, const float* transfer,
                      float* fixed, const float* initial_state, float* final_state) {
  __shared__ __align__(16) float srow[kFixRows][D];
  const int l = threadIdx.x;
  const int rblocks = D / kFixRows;
  const int rb = blockIdx.x % rblocks;
  const int nh = blockIdx.x / rblocks;
  const int n = nh / H, h = nh - (nh / H) * H;
  const int r0 = rb * kFixRows;
  const size_t ssz = (size_t)D * D;
#pragma unroll
  for (int j = 0; j < kFixRows; ++j)
    srow[j][l] = initial_state ? initial_state[((size_t)n * H + h) * ssz + (size_t)(r0 + j) * D + l] : 0.f;
  __syncthreads();
  const int s0 = seg_of_seq[n], s1 = seg_of_seq[n + 1];
  for (int sg = s0; sg < s1; ++sg) {
    const size_t off = ((size_t)sg * H + h) * ssz;
    float acc[kFixRows];
#pragma unroll
    for (int j = 0; j < kFixRows; ++j) {
      acc[j] = local[off + (size_t)(r0 + j) * D + l];
      fixed[off + (size_t)(r0 + j) * D + l] = srow[j][l];  // state at the segment start
    }
    // acc[j] += sum_i S^T[j][i] * M^T[i][l], transfer rows streamed 16 at a time
    const float* mt = transfer + off + l;
    for (int i0 = 0; i0 < D; i0 += 16) {
      float m[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) m[i] = mt[(size_t)(i0 + i) * D];
#pragma unroll
      for (int j = 0; j < kFixRows; ++j) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 sv = *reinterpret_cast<const float4*>(&srow[j][i0 + 4 * q]);
          acc[j] = fmaf(sv.x, m[4 * q], acc[j]);
          acc[j] = fmaf(sv.y, m[4 * q + 1], acc[j]);
          acc[j] = fmaf(sv.z, m[4 * q + 2], acc[j]);
          acc[j] = fmaf(sv.w, m[4 * q + 3], acc[j]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kFixRows; ++j) srow[j][l] = acc[j];
    __syncthreads();
  }
  if (final_state) {
#pragma unroll
    for (int j = 0; j < kFixRows; ++j)
      final_state[((size_t)n * H + h) * ssz + (size_t)(r0 + j) * D + l] = srow[j][l];
  }
}

}  // namespace

size_t prefill_transfer_workspace_bytes(const PrefillShape& s) { return layout_for(s).total; }

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

  gdn_fixup_scan_kernel<<<(unsigned)((long long)s.N * s.H * (D / kFixRows)), kFixThreads, 0, stream>>>(
      seg_of_seq, s.H, local, transfer, fixed, a.initial_state, a.final_state);
  st = check_launch("transfer prefill: fixup scan");
  if (st != GDN_OK) return st;

  PrefillArgs out = a;
  out.cu_seqlens = seg_cu;
  out.initial_state = fixed;
  out.final_state = nullptr;
  out.mode = kPrefillOutputs;
  return prefill_fused_launch(seg, out, stream);
}

}  // namespace gdn
