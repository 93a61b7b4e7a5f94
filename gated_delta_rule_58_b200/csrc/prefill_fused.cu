// Fused chunked prefill on the sm_100a tensor cores (tcgen05 + TMEM).
//
// One CTA per (sequence, head) walks the sequence chunk by chunk (C = 64
// tokens, dk = dv = 128) and keeps the fp32 state in tensor memory the whole
// time, so the only HBM traffic is q, k, v, g, beta in, o out, and the initial /
// final state once. Per chunk, with G the cumulative log gate inside the chunk,
// gamma = exp(G), S the state at the chunk start (dk x dv):
//
//   A  = strict_lower(beta_i exp(G_i - G_j) k_i.k_j)      (from K K^T)
//   T  = (I + A)^{-1}                                     (SIMT, 16x16 blocks)
//   W^T = K^T (T diag(beta gamma))^T,  U~^T = V^T (T diag(beta))^T
//   U^T = U~^T - S^T W^T                                  (the corrected values)
//   O^T = scale [ S^T Q^T diag(gamma) + U^T P^T ],  P = tril(exp(G_r - G_i) Q K^T)
//   S^T <- gamma_C S^T + U^T diag(exp(G_C - G_i)) K
//
// Every product is written with the value or key dimension on the MMA's M side,
// so all MMAs are M = 128 (cta_group::1) with fp16 operands in 128-byte-swizzled
// shared memory (the fp16 copy of the state is read straight from TMEM as the A
// operand) and fp32 accumulators in TMEM. fp16 (10-bit mantissa) keeps the
// result within the 2e-3 tolerance where bf16 operands do not; bf16 inputs are
// converted in shared memory. The decay factors exp(G_i - G_j) are taken on
// differences of cumulative gates (the cumulative decay idiom of the FlashInfer
// PR #6291 page, section 2), never as a ratio. The chunk step is the local-state /
// transfer update S_{c+1} = M_c S_c + H_c of the FlashInfer PR #3866 page
// (section 2) evaluated without materialising M_c or H_c.
//
// Warp specialisation (13 warps) and the chunk pipeline:
//   loader  (warps 8-11): TMA tensor loads of chunk c's q/k/v rows (bf16) straight
//            into the 128-byte-swizzled MMA tiles, g/beta, the cumulative gates
//            and decays; once [K;Q]K^T has read the raw tiles, their in-place
//            conversion to fp16. fp32 inputs are loaded and converted by the
//            threads instead. Runs up to two chunks ahead.
//   prep    (warps 4-7):  A and P from [K;Q]K^T, the triangular solve, the fp16
//            T diag(beta gamma) / T diag(beta) tiles. Works on chunk c+1 while
//            the state warps finish chunk c.
//   state   (warps 0-3):  W^T -> fp16 tile, U^T -> fp16 tiles, the new state ->
//            fp16 TMEM operand (and the gamma_C rescale of the fp32 TMEM state),
//            outputs -> HBM.
//   mma     (warp 12):    one thread issues the chunk's tcgen05.mma products in
//            dependency order. [K;Q]K^T is issued by the loader's first thread
//            instead, as soon as its tiles are in and the prep warps have read the
//            previous chunk's, so the chain's MMAs never wait on future tiles.
// Hand-offs are mbarriers: tcgen05.commit for MMA completion, one elected arrive
// per warpgroup (after a named barrier) for thread-produced tiles. Every wait is
// bounded; a timeout sets GDN_DEVERR_TIMEOUT and unwinds all roles.
#include <cstring>
#include <type_traits>

#include "device_once.h"
#include "prefill.cuh"
#include "tcgen05.cuh"
#include "tensor_map.cuh"

namespace gdn {
namespace {

constexpr int C = 64;      // chunk
constexpr int D = 128;     // dk = dv
constexpr int kThreads = 13 * 32;
constexpr int kPrepWarp0 = 4, kLoadWarp0 = 8, kMmaWarp = 12;  // state warps are 0-3
constexpr uint32_t kBarState = 1, kBarPrep = 2, kBarLoad = 3;  // named barrier ids
constexpr uint64_t kWaitNs = 2000000000ull;                     // 2 s
constexpr int kLptMaxSeqs = 64;  // longest-first launch order up to this many sequences

// Shared memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_KQ = 0;          // 2 buffers: [2 dk halves][128 rows: K 0-63, Q 64-127][64] fp16
constexpr uint32_t KQ_BUF = 32768;
constexpr uint32_t KQ_HALF = 16384;
constexpr uint32_t OFF_V = 65536;       // 2 buffers: [2 dv halves][64 tokens][64] fp16
constexpr uint32_t V_BUF = 16384;
constexpr uint32_t V_HALF = 8192;
constexpr uint32_t OFF_W16 = 98304;     // W^T [128 dk rows][64 tokens] fp16 (MN-major B)
constexpr uint32_t OFF_U16 = 114688;    // U^T [128 dv rows][64 tokens] fp16 (K-major A)
constexpr uint32_t OFF_UDD = 131072;    // U^T diag(exp(G_C - G_i))
constexpr uint32_t OFF_TP = 147456;     // T diag(beta gamma) [64][64] fp16 (K-major B)
constexpr uint32_t OFF_TPP = 155648;    // T diag(beta)
constexpr uint32_t OFF_P16 = 163840;    // 2 buffers: P [64][64] fp16 (K-major B)
constexpr uint32_t P_BUF = 8192;
constexpr uint32_t OFF_A = 180224;      // A fp32 [64][64], 16-byte chunks XOR-swizzled by row
constexpr uint32_t OFF_T = 196608;      // T fp32 [64][64], same swizzle
constexpr uint32_t OFF_VEC = 212992;    // 3 buffers (chunk % 3) x {G, gamma, dd, beta, beta*gamma} x 64 fp32
                                        // + 128 inverse q/k norms
constexpr uint32_t VEC_BUF = 7 * C * 4;
constexpr uint32_t OFF_BAR = OFF_VEC + 3 * VEC_BUF;
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for the 1024-byte alignment

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t COL_S = 0;     // S^T: lane = dv row, columns = dk
constexpr uint32_t COL_D1 = 128;  // [K;Q] K^T (lanes 0-63 K K^T, 64-127 Q K^T)
constexpr uint32_t COL_SH = 192;  // fp16 S^T as the MMA A operand: two halves per column
constexpr uint32_t COL_W = 256;   // W^T: lane = dk, column = token
constexpr uint32_t COL_U = 320;   // U~^T then U^T: lane = dv, column = token
constexpr uint32_t COL_O1 = 384;  // S^T Q^T
constexpr uint32_t COL_O2 = 448;  // U^T P^T
constexpr uint32_t TMEM_COLS = 512;

// mbarrier slots
enum Bar : int {
  B_L0 = 0, B_L1,      // loader -> chunk tiles ready (per buffer)
  B_T0, B_T1,          // TMA -> raw bf16 tiles landed (per buffer)
  B_LC0, B_LC1,        // loader -> fp16 tiles converted (per buffer)
  B_M1,                // MMA: D1 ready
  B_M2,                // MMA: W^T, U~^T ready
  B_M3A,               // MMA: U^T ready (S16, W16 consumed)
  B_M4B,               // MMA: new state ready
  B_M4A,               // MMA: O2 ready (all chunk MMAs done)
  B_E1,                // prep: D1 consumed (one arrival per prep warp)
  B_E2,                // prep: T', T'', P ready
  B_E3,                // state: W16 ready, W region consumed
  B_E5,                // state: U16/UDD ready, U region consumed
  B_E6A,               // state: S16 ready, TMEM state rescaled
  B_E6B,               // state: O1/O2 consumed
  B_FREE0, B_FREE1,    // state: a tile buffer's last reader (the state update) is done (fp32 inputs)
  B_DRAIN_M, B_DRAIN_L,  // abort path: the MMA thread's / the loader's MMAs have completed
  B_COUNT
};

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_sw128_chunk(uint8_t* tile, uint32_t row, uint32_t chunk, const float* v) {
  uint4 u;
  u.x = pack_half2(v[0], v[1]);
  u.y = pack_half2(v[2], v[3]);
  u.z = pack_half2(v[4], v[5]);
  u.w = pack_half2(v[6], v[7]);
  *reinterpret_cast<uint4*>(tile + tc::sw128_offset(row, chunk, 1024)) = u;
}

// [64][64] fp32 matrices: element (i, j) lives at i*64 + (j ^ ((i & 7) << 2)), i.e.
// the 16-byte chunks of a row are XOR-swizzled so that row-wise float4 accesses by
// consecutive rows and column-wise scalar accesses are both bank-conflict free.
__device__ __forceinline__ int sidx(int i, int j) { return i * 64 + (j ^ ((i & 7) << 2)); }

struct Smem {
  uint8_t* base;
  __device__ float* A() const { return reinterpret_cast<float*>(base + OFF_A); }
  __device__ float* T() const { return reinterpret_cast<float*>(base + OFF_T); }
  __device__ float* vec(int b) const { return reinterpret_cast<float*>(base + OFF_VEC + b * VEC_BUF); }
  __device__ uint64_t* bar(int i) const { return reinterpret_cast<uint64_t*>(base + OFF_BAR) + i; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_BAR + 8 * B_COUNT); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(base + OFF_BAR + 8 * B_COUNT + 4);
  }
  // per tile buffer: copies issued into it, and copies whose landing the loader saw
  // (an aborting CTA waits for the difference before it exits)
  __device__ volatile uint32_t* loads_issued() const {
    return reinterpret_cast<volatile uint32_t*>(base + OFF_BAR + 8 * B_COUNT + 8);
  }
  __device__ volatile uint32_t* loads_landed() const {
    return reinterpret_cast<volatile uint32_t*>(base + OFF_BAR + 8 * B_COUNT + 16);
  }
  __device__ uint32_t u32(uint32_t off) const { return tc::smem_u32(base + off); }
};
// vec(b) layout: [0,64) G log2(e) (cumulative log gate in base 2), [64,128) gamma,
// [128,192) dd, [192,256) beta, [256,320) beta*gamma, [320,448) 1/|k_i| then 1/|q_i|
// (with the q/k normalisation only)
constexpr int V_G = 0, V_GAM = 64, V_DD = 128, V_BETA = 192, V_BG = 256, V_RN = 320;
constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (exp(y) = 2^(y log2 e)); results below the
// normal range flush to zero, which only drops decays under 1e-38. Not volatile,
// so independent calls can be scheduled back to back.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_bar(const Smem& sm, int b, uint32_t parity, unsigned int* err) {
  if (tc::mbar_wait(sm.bar(b), parity, kWaitNs, sm.abort_flag())) return true;
  if (*sm.abort_flag() == 0) raise_device_error(err, GDN_DEVERR_TIMEOUT);
  *sm.abort_flag() = 1;
  return false;
}

// Warpgroup hand-off: writers' smem visible to the async proxy and TMEM accesses
// ordered, the group synchronised, then one elected arrive.
__device__ __forceinline__ void group_signal(const Smem& sm, uint32_t bar_id, int b) {
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  tc::named_sync(bar_id, 128);
  if ((threadIdx.x & 127) == 0) tc::mbar_arrive(sm.bar(b));
}

// ---------------------------------------------------------------- loader role

struct QkvMaps {
  CUtensorMap q, k, v;  // bf16 [total_T][H][128] as {128, H, total_T}; box {64, 1, 64}
  CUtensorMap o;        // o [total_T][H][128] as {128, H, total_T}; box {128, 1, 64}, not swizzled
};

// TMA loads of the raw bf16 K, Q (and V) tiles of the chunk starting at token t0
// into tile buffer b, completing on B_T0 + b. Issued by one thread, once the
// buffer's previous chunk (two chunks back) has had its last MMA complete.
__device__ __forceinline__ void issue_tile_loads(const Smem& sm, const QkvMaps& maps, int b, int h, int hq,
                                                 int64_t t0, bool zero_values) {
  uint8_t* kq = sm.base + OFF_KQ + b * KQ_BUF;
  uint8_t* v16 = sm.base + OFF_V + b * V_BUF;
  tc::fence_proxy_async_smem();  // the previous generic writes of these tiles precede the copies
  sm.loads_issued()[b] = sm.loads_issued()[b] + 1;
  tc::mbar_arrive_expect_tx(sm.bar(B_T0 + b), (zero_values ? 2u : 3u) * 16384u);
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    tc::tma_load_3d(tc::smem_u32(kq + hf * KQ_HALF), &maps.k, 64 * hf, hq, (int)t0, sm.bar(B_T0 + b));
    tc::tma_load_3d(tc::smem_u32(kq + hf * KQ_HALF + C * 128), &maps.q, 64 * hf, hq, (int)t0, sm.bar(B_T0 + b));
    if (!zero_values)
      tc::tma_load_3d(tc::smem_u32(v16 + hf * V_HALF), &maps.v, 64 * hf, h, (int)t0, sm.bar(B_T0 + b));
  }
}

// bf16 -> fp16 of one 16-byte chunk (8 elements) in place, times `sc` if kScale.
template <bool kScale>
__device__ __forceinline__ void convert_chunk_bf16(uint8_t* p, float sc = 1.f) {
  uint4* q = reinterpret_cast<uint4*>(p);
  const uint4 raw = *q;
  const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&raw);
  uint4 u;
  float2 f0 = __bfloat1622float2(hb[0]), f1 = __bfloat1622float2(hb[1]);
  float2 f2 = __bfloat1622float2(hb[2]), f3 = __bfloat1622float2(hb[3]);
  if (kScale) {
    f0.x *= sc; f0.y *= sc; f1.x *= sc; f1.y *= sc;
    f2.x *= sc; f2.y *= sc; f3.x *= sc; f3.y *= sc;
  }
  u.x = pack_half2(f0.x, f0.y);
  u.y = pack_half2(f1.x, f1.y);
  u.z = pack_half2(f2.x, f2.y);
  u.w = pack_half2(f3.x, f3.y);
  *q = u;
}

// D1 = [K;Q] K^T for chunk buffer b (raw bf16 tiles, or fp16 ones for fp32 inputs).
__device__ __forceinline__ void issue_m1(const Smem& sm, uint32_t tmem, int b, int raw_bf16) {
  const uint32_t kq = sm.u32(OFF_KQ + b * KQ_BUF);
  const uint32_t id = tc::idesc_f16(128, 64, 0, 0, 0, raw_bf16);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t off = (ks >> 2) * KQ_HALF + (ks & 3) * 32;
    tc::mma_f16(tmem + COL_D1, tc::sw128_desc(kq + off, 16, 1024), tc::sw128_desc(kq + off, 16, 1024), id, ks > 0);
  }
  tc::mma_commit(sm.bar(B_M1));
}

// Chunk c's [K;Q]K^T, issued by the loader's first thread as soon as the tiles
// are in (L0 signalled) and the prep group has read chunk c-1's D1 from TMEM, so
// the MMA role never waits on future tiles before this chunk's products.
__device__ __forceinline__ bool issue_d1(const Smem& sm, uint32_t tmem, int c, int b, int raw_bf16, unsigned int* err) {
  if (c >= 1 && !wait_bar(sm, B_E1, (c - 1) & 1, err)) return false;
  tc::fence_after_sync();
  issue_m1(sm, tmem, b, raw_bf16);
  return true;
}

template <typename TIn>
__device__ void loader_role(const Smem& sm, const PrefillShape& s, const PrefillArgs& a, const QkvMaps& maps,
                            uint32_t tmem, int h, int64_t bos, int64_t eos, int nchunks) {
  constexpr bool kTma = std::is_same<TIn, __nv_bfloat16>::value;
  const int t = threadIdx.x - kLoadWarp0 * 32;  // 0..127
  const bool zero_values = (a.mode == kPrefillTransfer);  // transfer run: V taken as 0
  const int hq = h / (s.H / s.Hqk);                       // the value head's query/key head
  // With the q/k normalisation K and Q are scaled by their inverse norms while
  // they are converted to fp16, and the conversion happens before [K;Q]K^T, which
  // then reads the fp16 tiles (as for fp32 inputs).
  const bool l2 = (a.flags & GDN_QK_L2NORM) != 0;
  if (zero_values) {  // both V buffers stay zero for the whole run
    for (int i = t; i < 2 * V_BUF / 16; i += 128)
      *reinterpret_cast<uint4*>(sm.base + OFF_V + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const int64_t t0 = bos + (int64_t)c * C;
    const int Lc = (int)((eos - t0) < C ? (eos - t0) : C);
    float* vec = sm.vec(c % 3);  // three gate buffers: chunk c-2's output epilogue may still read its own
    uint8_t* kq = sm.base + OFF_KQ + b * KQ_BUF;
    uint8_t* v16 = sm.base + OFF_V + b * V_BUF;
    // g and beta (zero past the sequence end), into registers first
    float gv = 0.f, bv = 0.f;
    if (t < Lc) {
      const size_t th = (size_t)(t0 + t) * s.H + h;
      gv = __ldg(a.g + th);
      bv = __ldg(a.beta + th);
    }
    // Chunk c-2 (same tile and gate buffers) must be done with K, Q, V: its state
    // update, the last MMA to read them, has completed (so have the earlier ones).
    // With TMA loads the state warps issue chunk c's copies as soon as that update
    // completes (chunks 0 and 1 are issued here), so the landing of the copies
    // implies it; the fp32 path waits for it directly.
    if constexpr (kTma) {
      // rows past the sequence end load the next tokens (or zeros past the tensor);
      // they are zeroed once the copies have landed, and their beta and g are 0
      if (c < 2 && t == 0) issue_tile_loads(sm, maps, b, h, hq, t0, zero_values);
      if (!wait_bar(sm, B_T0 + b, (c >> 1) & 1, a.err)) return;
      if (t == 0) sm.loads_landed()[b] = sm.loads_landed()[b] + 1;
    } else {
      // the buffer's release barrier completes once per use of the buffer, so its
      // parity names the use (chunk c-2) without depending on timing
      if (c >= 2 && !wait_bar(sm, B_FREE0 + b, ((c - 2) >> 1) & 1, a.err)) return;
    }
    if (t < C) {
      vec[V_G + t] = gv;
      vec[V_BETA + t] = bv;
    }
    tc::named_sync(kBarLoad, 128);
    if (t < 32) {
      // inclusive cumulative sum of the chunk's log gates (two per lane), decays
      const float x0 = vec[V_G + 2 * t], x1 = vec[V_G + 2 * t + 1];
      float pre = x0 + x1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, pre, off);
        if (t >= off) pre += y;
      }
      const float Gc = __shfl_sync(0xffffffffu, pre, 31) * kLog2e;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * t + e;
        const float Gi = (e ? pre : pre - x1) * kLog2e;
        const float gm = exp2_approx(Gi);
        vec[V_G + i] = Gi;
        vec[V_GAM + i] = gm;
        vec[V_DD + i] = exp2_approx(Gc - Gi);
        vec[V_BG + i] = vec[V_BETA + i] * gm;
      }
    }
    tc::named_sync(kBarLoad, 128);
    if constexpr (kTma) {
      // the raw bf16 tiles feed [K;Q] K^T directly (bf16 MMA, exact inputs); they
      // are converted to fp16 in place once that MMA has read them
      if (Lc < C) {
        // Rows past the sequence end hold the next sequence's tokens (or zeros past
        // the tensor). They are zeroed before any product reads them: beta = g = 0
        // alone would leave 0 * x in the products, which is NaN for a non-finite x
        // of the neighbour (or one outside the fp16 range after the conversion).
        // In the 128-byte-swizzled tiles row r is the 128 bytes at r * 128.
        const int nrows = C - Lc;
        const int per_tile = nrows * 8;  // 16-byte chunks of the padded rows of one half tile
        const int n_tiles = zero_values ? 4 : 6;  // K and Q halves, then V halves
        for (int i = t; i < n_tiles * per_tile; i += 128) {
          const int tile = i / per_tile, rem = i - tile * per_tile;
          const int row = Lc + (rem >> 3), ch = rem & 7;
          uint8_t* base = (tile < 4) ? kq + (tile >> 1) * KQ_HALF + (tile & 1) * (C * 128)
                                     : v16 + (tile - 4) * V_HALF;
          *reinterpret_cast<uint4*>(base + row * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (l2) {
        // thread t: 1 / |row t| of the [K;Q] tile stack from the raw bf16 row (both
        // 64-column halves; the chunk order within a row does not matter)
        tc::named_sync(kBarLoad, 128);  // the zeroed rows are written
        float ss = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 raw = *reinterpret_cast<const uint4*>(kq + hf * KQ_HALF + t * 128 + ch * 16);
            const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float2 f = __bfloat1622float2(hb[x]);
              ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
            }
          }
        vec[V_RN + t] = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        tc::named_sync(kBarLoad, 128);
#pragma unroll 4
        for (int i = t; i < 3 * C * 16; i += 128) {
          const int mat = i >> 10, rem = i & 1023;  // 0 K, 1 Q, 2 V; 64 rows x 16 chunks each
          const int row = rem >> 4, ch = rem & 15;
          if (mat == 2 && zero_values) continue;
          uint8_t* tile = (mat == 2) ? v16 + (ch >> 3) * V_HALF : kq + (ch >> 3) * KQ_HALF;
          const int trow = row + (mat == 1 ? C : 0);
          if (mat < 2)  // warp-uniform: the matrices are 1024 chunks apart
            convert_chunk_bf16<true>(tile + tc::sw128_offset(trow, ch & 7, 1024), vec[V_RN + trow]);
          else
            convert_chunk_bf16<false>(tile + tc::sw128_offset(trow, ch & 7, 1024));
        }
        group_signal(sm, kBarLoad, B_L0 + b);
        if (t == 0 && !issue_d1(sm, tmem, c, b, 0, a.err)) return;
      } else {
        group_signal(sm, kBarLoad, B_L0 + b);
        if (t == 0 && !issue_d1(sm, tmem, c, b, 1, a.err)) return;
        if (!wait_bar(sm, B_M1, c & 1, a.err)) return;
        tc::fence_after_sync();
#pragma unroll 4
        for (int i = t; i < 3 * C * 16; i += 128) {
          const int mat = i >> 10, rem = i & 1023;  // 0 K, 1 Q, 2 V; 64 rows x 16 chunks each
          const int row = rem >> 4, ch = rem & 15;
          if (mat == 2 && zero_values) continue;
          uint8_t* tile = (mat == 2) ? v16 + (ch >> 3) * V_HALF : kq + (ch >> 3) * KQ_HALF;
          const int trow = row + (mat == 1 ? C : 0);
          convert_chunk_bf16<false>(tile + tc::sw128_offset(trow, ch & 7, 1024));
        }
      }
    } else {
      if (l2) {  // thread t: 1 / |row t| of [K;Q] (zero past the sequence end)
        const int row = t & 63;
        float ss = 0.f;
        if (row < Lc) {
          const TIn* src = static_cast<const TIn*>(t < C ? a.k : a.q) + ((size_t)(t0 + row) * s.Hqk + hq) * D;
#pragma unroll 4
          for (int e = 0; e < D; e += 8) {
            float v8[8];
            load8_f32(src + e, v8);
#pragma unroll
            for (int x = 0; x < 8; ++x) ss = fmaf(v8[x], v8[x], ss);
          }
        }
        vec[V_RN + t] = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
        tc::named_sync(kBarLoad, 128);
      }
#pragma unroll
      for (int mat = 0; mat < 3; ++mat) {
        if (mat == 2 && zero_values) continue;
        const TIn* src0 = static_cast<const TIn*>(mat == 0 ? a.k : (mat == 1 ? a.q : a.v));
        uint8_t* base = (mat == 2) ? v16 : kq;
        const uint32_t half = (mat == 2) ? V_HALF : KQ_HALF;
        const int roff = (mat == 1) ? C : 0;
#pragma unroll 4
        for (int i = t; i < C * 16; i += 128) {
          const int row = i >> 4, ch = i & 15;
          float v8[8];
          if (row < Lc) {
            const size_t tok = (mat == 2) ? (size_t)(t0 + row) * s.H + h : (size_t)(t0 + row) * s.Hqk + hq;
            load8_f32(src0 + tok * D + ch * 8, v8);
            if (l2 && mat < 2) {
              const float r = vec[V_RN + row + roff];
#pragma unroll
              for (int x = 0; x < 8; ++x) v8[x] *= r;
            }
          } else {
#pragma unroll
            for (int x = 0; x < 8; ++x) v8[x] = 0.f;
          }
          st_sw128_chunk(base + (ch >> 3) * half, row + roff, ch & 7, v8);
        }
      }
      group_signal(sm, kBarLoad, B_L0 + b);
      if (t == 0 && !issue_d1(sm, tmem, c, b, 0, a.err)) return;
    }
    group_signal(sm, kBarLoad, B_LC0 + b);
  }
}

// ---------------------------------------------------------------- prep role

// 16-byte chunk q of row i of a [64][64] fp32 matrix (chunks XOR-swizzled by row).
__device__ __forceinline__ float4* row_chunk(float* M, int i, int q) {
  return reinterpret_cast<float4*>(M + i * 64 + 4 * (q ^ (i & 7)));
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Warp-level D(16x8) += A(16x8) B(8x8) on tf32 tensor cores, fp32 accumulate.
__device__ __forceinline__ void mma_tf32_16x8x8(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc (16x16 block, two m16n8 fragments) += M1[r1.., c1..] (16x16) * M2[r2.., c2..] (16x16),
// both [64][64] fp32 swizzled tiles in shared memory. Fragment layout of
// m16n8k8: g = lane / 4, t = lane % 4; A: (g, t), (g+8, t), (g, t+4), (g+8, t+4);
// B: (t, g), (t+4, g); C: (g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).
__device__ __forceinline__ void warp_block_mma(float (*acc)[4], const float* M1, int r1, int c1, const float* M2,
                                               int r2, int c2, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 2; ++ks) {
    uint32_t a[4];
    a[0] = to_tf32(M1[sidx(r1 + g, c1 + 8 * ks + t)]);
    a[1] = to_tf32(M1[sidx(r1 + g + 8, c1 + 8 * ks + t)]);
    a[2] = to_tf32(M1[sidx(r1 + g, c1 + 8 * ks + t + 4)]);
    a[3] = to_tf32(M1[sidx(r1 + g + 8, c1 + 8 * ks + t + 4)]);
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t b[2];
      b[0] = to_tf32(M2[sidx(r2 + 8 * ks + t, c2 + 8 * nt + g)]);
      b[1] = to_tf32(M2[sidx(r2 + 8 * ks + t + 4, c2 + 8 * nt + g)]);
      mma_tf32_16x8x8(acc[nt], a, b);
    }
  }
}

// Writes a 16x16 accumulator (two m16n8 fragments) times `sign` into a swizzled tile.
__device__ __forceinline__ void warp_block_store(float* M, int r0, int c0, float (*acc)[4], float sign, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    M[sidx(r0 + g, c0 + 8 * nt + 2 * t)] = sign * acc[nt][0];
    M[sidx(r0 + g, c0 + 8 * nt + 2 * t + 1)] = sign * acc[nt][1];
    M[sidx(r0 + g + 8, c0 + 8 * nt + 2 * t)] = sign * acc[nt][2];
    M[sidx(r0 + g + 8, c0 + 8 * nt + 2 * t + 1)] = sign * acc[nt][3];
  }
}

// T = (I + A)^{-1} for the strictly lower 64x64 A (fp32), in two parts.
//
// solve_local (warps 4 and 5, right after each wrote its 32 rows of A): the two
// 16x16 diagonal blocks of the warp's rows are inverted by forward substitution,
// then merged into the inverse of the warp's 32x32 diagonal block,
// T_10 = -T_11 (A_10 T_00) (or T_32 for warp 5), on tf32 warp MMAs. Only the
// warp's own rows are read, so __syncwarp orders the steps.
//
// Forward substitution by rows, in registers: thread t owns row r = t % 16 of
// block b = t / 16 (its A row), starting from e_r. At step k row k is final; its
// first k+1 entries (the rest are zero) are broadcast by shuffles from lane k of
// the half-warp and every later row subtracts A_rk times it.
__device__ __forceinline__ void solve_local(const Smem& sm, int t) {
  float* A = sm.A();
  float* T = sm.T();
  {
    const int b = t >> 4, r = t & 15, hl = threadIdx.x & 16;
    float arow[16], trow[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 a4 = *row_chunk(A, 16 * b + r, 4 * b + q);
      arow[4 * q + 0] = a4.x; arow[4 * q + 1] = a4.y; arow[4 * q + 2] = a4.z; arow[4 * q + 3] = a4.w;
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) trow[m] = (m == r) ? 1.f : 0.f;
#pragma unroll
    for (int k = 0; k < 15; ++k) {
      const float lk = (k < r) ? arow[k] : 0.f;  // A_rk for the later rows only
#pragma unroll
      for (int m = 0; m <= k; ++m) {
        const float rk = __shfl_sync(0xffffffffu, trow[m], hl | k);
        trow[m] = fmaf(-lk, rk, trow[m]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *row_chunk(T, 16 * b + r, 4 * b + q) =
          make_float4(trow[4 * q + 0], trow[4 * q + 1], trow[4 * q + 2], trow[4 * q + 3]);
  }
  __syncwarp();
  const int wl = t >> 5, lane = t & 31;
  const int i = 2 * wl + 1, j = 2 * wl;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  warp_block_mma(acc, A, 16 * i, 16 * j, T, 16 * j, 16 * j, lane);
  warp_block_store(A, 16 * i, 16 * i, acc, 1.f, lane);  // X = A_ij T_jj parked in A_ii (no longer read)
  __syncwarp();
  float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  warp_block_mma(y, T, 16 * i, 16 * i, A, 16 * i, 16 * i, lane);
  warp_block_store(T, 16 * i, 16 * j, y, -1.f, lane);
}

// solve_merge (all four prep warps, after a barrier): the bottom-left 32x32 block,
// T_BL = -T_bot (A_BL T_top), one 16x16 output block per warp and stage. The
// intermediate Y = A_BL T_top is parked in the four diagonal blocks of A.
__device__ __forceinline__ void solve_merge(const Smem& sm, int t) {
  float* A = sm.A();
  float* T = sm.T();
  const int w = t >> 5, lane = t & 31;
  const int i = 2 + (w >> 1), j = w & 1;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int k = j; k < 2; ++k) warp_block_mma(acc, A, 16 * i, 16 * k, T, 16 * k, 16 * j, lane);  // Y_ij
  const int p = 2 * (i - 2) + j;
  warp_block_store(A, 16 * p, 16 * p, acc, 1.f, lane);
  tc::named_sync(kBarPrep, 128);
  float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int k = 2; k <= i; ++k) {
    const int pk = 2 * (k - 2) + j;
    warp_block_mma(y, T, 16 * i, 16 * k, A, 16 * pk, 16 * pk, lane);  // T_ik Y_kj
  }
  warp_block_store(T, 16 * i, 16 * j, y, -1.f, lane);
  tc::named_sync(kBarPrep, 128);
}

// Columns 32 hq .. 32 hq + 31 of A row t: beta_t 2^(G_t - G_j) x_j for j < t (base-2
// cumulative gates), 16-byte chunks right of the diagonal skipped. The entries with
// j >= t inside the boundary chunk are stored unmasked: the solve masks them itself
// (the forward substitution reads A_rk only for k < r; every other reader takes
// blocks strictly below the diagonal). Products two at a time, rounded as
// (beta 2^dG) x per entry.
__device__ __forceinline__ void a_row_half(float* A, int t, int hq, float bi, float Gi, const float* G,
                                           const float* x) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j0 = 32 * hq + 4 * q;
    const float4 g4 = *reinterpret_cast<const float4*>(G + j0);
    const float2 bb = make_float2(bi, bi);
    const float2 lo = __fmul2_rn(__fmul2_rn(bb, make_float2(exp2_approx(Gi - g4.x), exp2_approx(Gi - g4.y))),
                                 make_float2(x[4 * q + 0], x[4 * q + 1]));
    const float2 hi = __fmul2_rn(__fmul2_rn(bb, make_float2(exp2_approx(Gi - g4.z), exp2_approx(Gi - g4.w))),
                                 make_float2(x[4 * q + 2], x[4 * q + 3]));
    if (j0 < t) *row_chunk(A, t, j0 >> 2) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
}

// Columns 32 hq .. 32 hq + 31 of P row r into the fp16 tile: 2^(G_r - G_i) x_i for
// i <= r; chunks entirely above the diagonal are left as they are (zeros).
__device__ __forceinline__ void p_row_half(uint8_t* p16, int r, int hq, float Gr, const float* G, const float* x) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const float4 g0 = *reinterpret_cast<const float4*>(G + 32 * hq + 8 * cc);
    const float4 g1 = *reinterpret_cast<const float4*>(G + 32 * hq + 8 * cc + 4);
    const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    float v[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int i = 32 * hq + cc * 8 + m;
      v[m] = (i <= r) ? exp2_approx(Gr - gv[m]) * x[cc * 8 + m] : 0.f;
    }
    if (32 * hq + cc * 8 <= r) st_sw128_chunk(p16, r, 4 * hq + cc, v);
  }
}

__device__ void prep_role(const Smem& sm, uint32_t tmem, int nchunks, unsigned int* err) {
  const int t = threadIdx.x - kPrepWarp0 * 32;  // 0..127 == TMEM lane
  const int warp = threadIdx.x >> 5;
  const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  // both P tiles start as zeros: the strictly upper 16-byte chunks are never written
  for (int i = t; i < 2 * P_BUF / 16; i += 128)
    *reinterpret_cast<uint4*>(sm.base + OFF_P16 + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  // so does T: the solve writes only its lower blocks (with zeros above the diagonal
  // inside the 16x16 diagonal blocks), so T's upper triangle stays zero for good
  for (int i = t; i < C * C / 4; i += 128) reinterpret_cast<float4*>(sm.T())[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  tc::named_sync(kBarPrep, 128);
  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    if (!wait_bar(sm, B_L0 + b, (c >> 1) & 1, err)) return;
    if (!wait_bar(sm, B_M1, c & 1, err)) return;
    tc::fence_after_sync();
    const float* vec = sm.vec(c % 3);
    const float* G = vec + V_G;
    if (t < C) {
      // A row t (rows 0-63 of D1): beta_t exp(G_t - G_j) k_t.k_j for j < t; the warp
      // of rows 32-63 also needs the right 32-column half (warp-uniform, as tcgen05.ld
      // is warp-collective). One half is loaded and processed at a time.
      const float Gi = G[t], bi = vec[V_BETA + t];
      const int halves = ((t | 31) > 32) ? 2 : 1;
      for (int hq = 0; hq < halves; ++hq) {
        float x[32];
        tc::tmem_ld16(tl + COL_D1 + 32 * hq, x);
        tc::tmem_ld16(tl + COL_D1 + 32 * hq + 16, x + 16);
        tc::wait_ld();
        a_row_half(sm.A(), t, hq, bi, Gi, G, x);
      }
    } else {
      // P row r (rows 64-127 of D1) into P16[b]; its previous reader (chunk c-2's
      // output MMA) completed before this chunk's D1 MMA, whose completion was waited
      // on. 16-byte chunks entirely above the diagonal keep the zeros written at start.
      const int r = t - C;
      const float Gr = G[r];
      const int halves = ((r | 31) >= 32) ? 2 : 1;
      uint8_t* p16 = sm.base + OFF_P16 + b * P_BUF;
      for (int hq = 0; hq < halves; ++hq) {
        float x[32];
        tc::tmem_ld16(tl + COL_D1 + 32 * hq, x);
        tc::tmem_ld16(tl + COL_D1 + 32 * hq + 16, x + 16);
        tc::wait_ld();
        p_row_half(p16, r, hq, Gr, G, x);
      }
    }
    // this warp's reads of D1 are complete: the next chunk's [K;Q]K^T may overwrite it
    tc::fence_before_sync();
    __syncwarp();
    if ((t & 31) == 0) tc::mbar_arrive(sm.bar(B_E1));
    if (t < C) solve_local(sm, t);  // warps 4 and 5: their own 32x32 diagonal blocks
    tc::named_sync(kBarPrep, 128);
    solve_merge(sm, t);
    // T diag(beta gamma) and T diag(beta) as fp16, once the previous chunk's W/U~
    // MMA has read the old ones
    if (c >= 1 && !wait_bar(sm, B_M2, (c - 1) & 1, err)) return;
    {
      // row i of T times the column scales (T's upper triangle is zero); the row
      // and the scales are loaded up front (independent loads)
      const int mat = t >> 6, i = t & 63;
      const float* colscale = vec + (mat ? V_BETA : V_BG);
      uint8_t* tile = sm.base + (mat ? OFF_TPP : OFF_TP);
      float4 tr[16], cs[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        tr[q] = *row_chunk(sm.T(), i, q);
        cs[q] = *reinterpret_cast<const float4*>(colscale + 4 * q);
      }
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const float4 a0 = tr[2 * cc], a1 = tr[2 * cc + 1], s0 = cs[2 * cc], s1 = cs[2 * cc + 1];
        const float2 p0 = __fmul2_rn(make_float2(a0.x, a0.y), make_float2(s0.x, s0.y));
        const float2 p1 = __fmul2_rn(make_float2(a0.z, a0.w), make_float2(s0.z, s0.w));
        const float2 p2 = __fmul2_rn(make_float2(a1.x, a1.y), make_float2(s1.x, s1.y));
        const float2 p3 = __fmul2_rn(make_float2(a1.z, a1.w), make_float2(s1.z, s1.w));
        const float v[8] = {p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y};
        st_sw128_chunk(tile, i, cc, v);
      }
    }
    group_signal(sm, kBarPrep, B_E2);
  }
}

// ---------------------------------------------------------------- state role

template <typename TIn, typename TOut>
__device__ void state_role(const Smem& sm, const PrefillShape& s, const PrefillArgs& a, const QkvMaps& maps,
                           uint32_t tmem, int h, int64_t bos, int64_t eos, int nchunks, size_t state_off) {
  constexpr bool kTmaLoads = std::is_same<TIn, __nv_bfloat16>::value;
  const int j = threadIdx.x;  // TMEM lane == dv row of S^T
  const int warp = threadIdx.x >> 5;
  const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  TOut* op = static_cast<TOut*>(a.o);
  // outputs of a chunk are staged row-major [64 tokens][128 dv] in the U16/UDD
  // tiles (free between the chunk's last MMA and the next chunk's U epilogue)
  TOut* stage = reinterpret_cast<TOut*>(sm.base + OFF_U16);
  constexpr uint32_t kRowBytes = D * sizeof(TOut);

  // initial state: fp16 TMEM operand = S_0; fp32 TMEM state = gamma_C(0) * S_0
  if (!wait_bar(sm, B_L0, 0, a.err)) return;
  {
    const float gC = sm.vec(0)[V_GAM + C - 1];
    for (int q = 0; q < D / 16; ++q) {
      float v[16];
      if (a.mode == kPrefillTransfer) {  // S_0 = I: row j of S^T is e_j
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = (q * 16 + x == j) ? 1.f : 0.f;
      } else if (a.initial_state) {
        const float4* src = reinterpret_cast<const float4*>(a.initial_state + state_off + (size_t)j * D + q * 16);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float4 f = src[x];
          v[4 * x] = f.x; v[4 * x + 1] = f.y; v[4 * x + 2] = f.z; v[4 * x + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] = 0.f;
      }
      uint32_t hv[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) hv[x] = tc::half2_bits(v[2 * x], v[2 * x + 1]);
      tc::tmem_st8_bits(tl + COL_SH + q * 8, hv);
#pragma unroll
      for (int x = 0; x < 16; ++x) v[x] *= gC;
      tc::tmem_st16(tl + COL_S + q * 16, v);
    }
    tc::wait_st();
  }
  group_signal(sm, kBarState, B_E6A);

  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const float* vec = sm.vec(c % 3);
    const int64_t t0 = bos + (int64_t)c * C;
    const int Lc = (int)((eos - t0) < C ? (eos - t0) : C);
    // E3: W^T -> fp16 tile once the W MMA is done (W16's previous reader, chunk
    // c-1's U MMA, completed before E5 of chunk c-1)
    if (!wait_bar(sm, B_M2, c & 1, a.err)) return;
    tc::fence_after_sync();
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {
      float w[32];
      tc::tmem_ld16(tl + COL_W + hq * 32, w);
      tc::tmem_ld16(tl + COL_W + hq * 32 + 16, w + 16);
      tc::wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) st_sw128_chunk(sm.base + OFF_W16, j, 4 * hq + q, w + 8 * q);
    }
    group_signal(sm, kBarState, B_E3);
    // E5: U^T -> fp16 tiles (after the previous chunk's output stores read the stage)
    if (!wait_bar(sm, B_M3A, c & 1, a.err)) return;
    if (c >= 1) {
      if (j < 32) tc::bulk_wait_read();
      tc::named_sync(kBarState, 128);
    }
    tc::fence_after_sync();
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {
      float u[32];
      tc::tmem_ld16(tl + COL_U + hq * 32, u);
      tc::tmem_ld16(tl + COL_U + hq * 32 + 16, u + 16);
      tc::wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float ud[8];
        {  // U diag(dd), two entries per packed multiply (each rounded as a scalar product)
          const float4 d0 = *reinterpret_cast<const float4*>(vec + V_DD + 32 * hq + 8 * q);
          const float4 d1 = *reinterpret_cast<const float4*>(vec + V_DD + 32 * hq + 8 * q + 4);
          const float2 p0 = __fmul2_rn(make_float2(u[8 * q], u[8 * q + 1]), make_float2(d0.x, d0.y));
          const float2 p1 = __fmul2_rn(make_float2(u[8 * q + 2], u[8 * q + 3]), make_float2(d0.z, d0.w));
          const float2 p2 = __fmul2_rn(make_float2(u[8 * q + 4], u[8 * q + 5]), make_float2(d1.x, d1.y));
          const float2 p3 = __fmul2_rn(make_float2(u[8 * q + 6], u[8 * q + 7]), make_float2(d1.z, d1.w));
          ud[0] = p0.x; ud[1] = p0.y; ud[2] = p1.x; ud[3] = p1.y; ud[4] = p2.x; ud[5] = p2.y; ud[6] = p3.x; ud[7] = p3.y;
        }
        st_sw128_chunk(sm.base + OFF_U16, j, 4 * hq + q, u + 8 * q);
        st_sw128_chunk(sm.base + OFF_UDD, j, 4 * hq + q, ud);
      }
    }
    group_signal(sm, kBarState, B_E5);
    // E6a: new state -> fp16 operand; rescale by the next chunk's gamma_C; final state
    if (!wait_bar(sm, B_M4B, c & 1, a.err)) return;
    tc::fence_after_sync();
    // chunk c's state update was the last reader of tile buffer b: chunk c+2's
    // copies go out now, well before the loader needs them
    if (j == 0) {
      if (kTmaLoads) {
        if (c + 2 < nchunks) issue_tile_loads(sm, maps, b, h, h / (s.H / s.Hqk), t0 + 2 * C, a.mode == kPrefillTransfer);
      } else {
        tc::mbar_arrive(sm.bar(B_FREE0 + b));  // fp32 inputs: the loader refills the buffer itself
      }
    }
    const bool last = (c == nchunks - 1);
    float gnext = 1.f;
    if (!last) {
      if (!wait_bar(sm, B_L0 + (b ^ 1), ((c + 1) >> 1) & 1, a.err)) return;
      gnext = sm.vec((c + 1) % 3)[V_GAM + C - 1];
    }
#pragma unroll
    for (int hq = 0; hq < 4; ++hq) {
      float v[32];
      tc::tmem_ld16(tl + COL_S + hq * 32, v);
      tc::tmem_ld16(tl + COL_S + hq * 32 + 16, v + 16);
      tc::wait_ld();
      if (!last) {
        uint32_t hv[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) hv[x] = tc::half2_bits(v[2 * x], v[2 * x + 1]);
        tc::tmem_st16_bits(tl + COL_SH + hq * 16, hv);
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const float2 p = __fmul2_rn(make_float2(v[x], v[x + 1]), make_float2(gnext, gnext));
          v[x] = p.x;
          v[x + 1] = p.y;
        }
        tc::tmem_st16(tl + COL_S + hq * 32, v);
        tc::tmem_st16(tl + COL_S + hq * 32 + 16, v + 16);
      } else if (a.final_state) {
        float4* dst = reinterpret_cast<float4*>(a.final_state + state_off + (size_t)j * D + hq * 32);
#pragma unroll
        for (int x = 0; x < 8; ++x) dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
      }
    }
    tc::wait_st();
    group_signal(sm, kBarState, B_E6A);
    // E6b: outputs of the chunk -> staging rows -> bulk stores (skipped when the
    // run produces states only)
    if (!wait_bar(sm, B_M4A, c & 1, a.err)) return;
    tc::fence_after_sync();
    if (op == nullptr) {
      tc::fence_before_sync();
      tc::named_sync(kBarState, 128);
      if (j == 0) tc::mbar_arrive(sm.bar(B_E6B));
      continue;
    }
    const float sc = a.scale;
#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {
      float o1[32], o2[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        tc::tmem_ld16(tl + COL_O1 + hq * 32 + q * 16, o1 + 16 * q);
        tc::tmem_ld16(tl + COL_O2 + hq * 32 + q * 16, o2 + 16 * q);
      }
      float4 gm[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) gm[q] = *reinterpret_cast<const float4*>(vec + V_GAM + hq * 32 + 4 * q);
      tc::wait_ld();
      const float2 sc2 = make_float2(sc, sc);  // rows r, r + 1 per packed FMA / multiply
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int r = hq * 32 + 4 * q;
        const float2 a = __fmul2_rn(sc2, __ffma2_rn(make_float2(gm[q].x, gm[q].y),
                                                     make_float2(o1[4 * q], o1[4 * q + 1]),
                                                     make_float2(o2[4 * q], o2[4 * q + 1])));
        const float2 b = __fmul2_rn(sc2, __ffma2_rn(make_float2(gm[q].z, gm[q].w),
                                                     make_float2(o1[4 * q + 2], o1[4 * q + 3]),
                                                     make_float2(o2[4 * q + 2], o2[4 * q + 3])));
        store_out(stage + (r + 0) * D + j, a.x);
        store_out(stage + (r + 1) * D + j, a.y);
        store_out(stage + (r + 2) * D + j, b.x);
        store_out(stage + (r + 3) * D + j, b.y);
      }
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    tc::named_sync(kBarState, 128);
    if (Lc == C) {  // a full chunk: one tensor store of the [64 tokens][128] tile
      if (j == 0) {
        tc::tma_store_3d(&maps.o, 0, h, (int)t0, tc::smem_u32(stage));
        tc::bulk_commit();
      }
    } else if (j < 32) {  // the last, partial chunk: row by row
      for (int r = j; r < Lc; r += 32)
        tc::bulk_store(op + ((size_t)(t0 + r) * s.H + h) * D, tc::smem_u32(stage + r * D), kRowBytes);
      tc::bulk_commit();
    }
    if (j == 0) tc::mbar_arrive(sm.bar(B_E6B));
  }
  if (j < 32) tc::bulk_wait_all();
}

// ---------------------------------------------------------------- mma role

// W^T = K^T T'^T and U~^T = V^T T''^T for chunk buffer b (A MN-major from the token tiles).
__device__ __forceinline__ void issue_m2(const Smem& sm, uint32_t tmem, int b) {
  const uint32_t kq = sm.u32(OFF_KQ + b * KQ_BUF), v16 = sm.u32(OFF_V + b * V_BUF);
  const uint32_t tp = sm.u32(OFF_TP), tpp = sm.u32(OFF_TPP);
  const uint32_t id = tc::idesc_f16(128, 64, 1, 0);
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    tc::mma_f16(tmem + COL_W, tc::sw128_desc(kq + ks * 2048, KQ_HALF, 1024), tc::sw128_desc(tp + ks * 32, 16, 1024),
                id, ks > 0);
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    tc::mma_f16(tmem + COL_U, tc::sw128_desc(v16 + ks * 2048, V_HALF, 1024), tc::sw128_desc(tpp + ks * 32, 16, 1024),
                id, ks > 0);
  tc::mma_commit(sm.bar(B_M2));
}

__device__ void mma_role(const Smem& sm, uint32_t tmem, int nchunks, unsigned int* err) {
  const uint32_t w16 = sm.u32(OFF_W16), u16 = sm.u32(OFF_U16), udd = sm.u32(OFF_UDD);
  const uint32_t p16 = sm.u32(OFF_P16);
  const uint32_t id_u = tc::idesc_f16(128, 64, 0, 1, 1);
  const uint32_t id_o = tc::idesc_f16(128, 64, 0, 0);
  const uint32_t id_s = tc::idesc_f16(128, 128, 0, 1);

  for (int c = 0; c < nchunks; ++c) {
    const int b = c & 1;
    const uint32_t kq = sm.u32(OFF_KQ + b * KQ_BUF);
    // M2: W^T, U~^T of this chunk
    if (!wait_bar(sm, B_E2, c & 1, err)) return;
    if (!wait_bar(sm, B_LC0 + b, (c >> 1) & 1, err)) return;
    tc::fence_after_sync();
    issue_m2(sm, tmem, b);
    // M3a: U^T -= S^T W^T (A = fp16 state from TMEM)
    if (!wait_bar(sm, B_E3, c & 1, err)) return;
    if (!wait_bar(sm, B_E6A, c & 1, err)) return;
    tc::fence_after_sync();
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      tc::mma_f16_ts(tmem + COL_U, tmem + COL_SH + ks * 8, tc::sw128_desc(w16 + ks * 2048, 16384, 1024), id_u, 1);
    tc::mma_commit(sm.bar(B_M3A));
    // M3b: O1 = S^T Q^T (after the previous chunk's outputs were read)
    if (c >= 1 && !wait_bar(sm, B_E6B, (c - 1) & 1, err)) return;
    tc::fence_after_sync();
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t bd = tc::sw128_desc(kq + 8 * 1024 + (ks >> 2) * KQ_HALF + (ks & 3) * 32, 16, 1024);
      tc::mma_f16_ts(tmem + COL_O1, tmem + COL_SH + ks * 8, bd, id_o, ks > 0);
    }
    // M4b: S^T += (U^T diag(dd)) K ; M4a: O2 = U^T P^T
    if (!wait_bar(sm, B_E5, c & 1, err)) return;
    tc::fence_after_sync();
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      tc::mma_f16(tmem + COL_S, tc::sw128_desc(udd + ks * 32, 16, 1024),
                  tc::sw128_desc(kq + ks * 2048, KQ_HALF, 1024), id_s, 1);
    tc::mma_commit(sm.bar(B_M4B));
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      tc::mma_f16(tmem + COL_O2, tc::sw128_desc(u16 + ks * 32, 16, 1024),
                  tc::sw128_desc(p16 + b * P_BUF + ks * 32, 16, 1024), id_o, ks > 0);
    tc::mma_commit(sm.bar(B_M4A));
  }
}

// ---------------------------------------------------------------- kernel

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads, 1)
gdn_prefill_fused_kernel(const PrefillShape s, const PrefillArgs a, const __grid_constant__ QkvMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = tc::align_smem<1024>(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int rank = blockIdx.x / s.H;
  const int h = blockIdx.x - rank * s.H;
  // Longest sequence first: the CTAs of the rank-th longest sequence (ties by
  // index) have the rank-th block indices, so long sequences start in the first
  // wave and the last wave holds short ones. Each CTA ranks the lengths itself
  // (one warp, O(N^2) compares on a shared-memory copy), so only for small N;
  // beyond that the order is the sequence index. Results do not depend on it.
  int n = rank;
  if (s.N > 1 && s.N <= kLptMaxSeqs) {
    int* lens = reinterpret_cast<int*>(sm.A());  // the A tile is free until the first chunk
    for (int i = threadIdx.x; i < s.N; i += blockDim.x) {
      const int32_t l = __ldg(a.cu_seqlens + i + 1) - __ldg(a.cu_seqlens + i);
      lens[i] = l > 0 ? l : 0;
    }
    __syncthreads();
    if (warp == 0) {
      int found = -1;
      for (int i = threadIdx.x; i < s.N; i += 32) {
        const int li = lens[i];
        int r = 0;
        for (int j = 0; j < s.N; ++j) {
          const int lj = lens[j];
          r += (lj > li || (lj == li && j < i)) ? 1 : 0;
        }
        if (r == rank) found = i;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) found = max(found, __shfl_xor_sync(0xffffffffu, found, off));
      if (threadIdx.x == 0) lens[kLptMaxSeqs] = found;
    }
    __syncthreads();
    n = lens[kLptMaxSeqs];
    __syncthreads();  // the A tile is reused below
  }
  int64_t bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, s.total_T, a.err, &bos, &eos)) return;

  const size_t state_off = ((size_t)n * s.H + h) * (size_t)D * D;
  const int nchunks = (int)((eos - bos + C - 1) / C);
  if (nchunks == 0) {  // empty sequence: the state passes through
    if (a.final_state) {
      for (int i = threadIdx.x; i < D * D / 4; i += kThreads) {
        float4 x = a.initial_state ? reinterpret_cast<const float4*>(a.initial_state + state_off)[i]
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.mode == kPrefillTransfer) {  // identity (row r of the K-last layout is e_r)
          const int r = (4 * i) / D, c0 = (4 * i) % D;
          x = make_float4(c0 == r, c0 + 1 == r, c0 + 2 == r, c0 + 3 == r);
        }
        reinterpret_cast<float4*>(a.final_state + state_off)[i] = x;
      }
    }
    return;
  }

  if (warp == kMmaWarp) {
    tc::tmem_alloc(sm.tmem_slot(), TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) tc::mbar_init(sm.bar(i), i == B_E1 ? 4 : 1);
    *sm.abort_flag() = 0;
    sm.loads_issued()[0] = sm.loads_issued()[1] = 0;
    sm.loads_landed()[0] = sm.loads_landed()[1] = 0;
    tc::fence_mbar_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *sm.tmem_slot();

  if (warp < kPrepWarp0) {
    state_role<TIn, TOut>(sm, s, a, maps, tmem, h, bos, eos, nchunks, state_off);
  } else if (warp < kLoadWarp0) {
    prep_role(sm, tmem, nchunks, a.err);
  } else if (warp < kMmaWarp) {
    loader_role<TIn>(sm, s, a, maps, tmem, h, bos, eos, nchunks);
  } else if ((threadIdx.x & 31) == 0) {
    mma_role(sm, tmem, nchunks, a.err);
  }

  // teardown: every role finished (all MMAs were waited on by the state role).
  // After a timeout the roles returned early, so asynchronous work they issued may
  // still be running: each MMA issuer waits for its own MMAs (a commit arrives once
  // every earlier MMA of the thread is done), the output stores of the state warps
  // drain, and outstanding tile copies land, all before TMEM is released and the
  // CTA exits (each wait bounded again).
  if (*sm.abort_flag()) {
    const bool mma_issuer = (warp == kMmaWarp && (threadIdx.x & 31) == 0);
    const bool d1_issuer = (threadIdx.x == kLoadWarp0 * 32);
    if (mma_issuer || d1_issuer) {
      uint64_t* drain = sm.bar(mma_issuer ? B_DRAIN_M : B_DRAIN_L);
      tc::mma_commit(drain);
      tc::mbar_wait(drain, 0, kWaitNs);
    }
    if (threadIdx.x == 0) {
      for (int b = 0; b < 2; ++b)
        for (uint32_t n = sm.loads_landed()[b]; n < sm.loads_issued()[b]; ++n)
          if (!tc::mbar_wait(sm.bar(B_T0 + b), n & 1, kWaitNs)) break;
    }
  }
  if (warp == 0) tc::bulk_wait_all();  // the state warps' output stores (a no-op when none)
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem, TMEM_COLS);
}

template <typename TIn, typename TOut>
gdn_status_t launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("fused prefill: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(gdn_prefill_fused_kernel<TIn, TOut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("fused prefill: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  const unsigned grid = (unsigned)((long long)s.N * s.H);
  QkvMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (std::is_same<TIn, __nv_bfloat16>::value && s.total_T > 0) {
    // q, k as {128, H_qk, total_T} and v as {128, H, total_T} bf16; one box = 64
    // features x 64 tokens of one head
    const uint32_t box[3] = {64, 1, (uint32_t)C};
    const void* src[3] = {a.q, a.k, a.v};
    CUtensorMap* dst[3] = {&maps.q, &maps.k, &maps.v};
    for (int i = 0; i < 3; ++i) {
      const uint64_t heads = (i == 2) ? (uint64_t)s.H : (uint64_t)s.Hqk;
      const uint64_t dims[3] = {(uint64_t)D, heads, (uint64_t)s.total_T};
      const uint64_t strides[2] = {(uint64_t)D * 2, heads * D * 2};
      const gdn_status_t st = make_tensor_map_3d(dst[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, src[i], dims, strides, box,
                                                 "fused prefill");
      if (st != GDN_OK) return st;
    }
  }
  if (a.o != nullptr && s.total_T > 0) {
    constexpr bool kBf16Out = std::is_same<TOut, __nv_bfloat16>::value;
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.H, (uint64_t)s.total_T};
    const uint64_t strides[2] = {(uint64_t)D * sizeof(TOut), (uint64_t)s.H * D * sizeof(TOut)};
    const uint32_t box[3] = {(uint32_t)D, 1, (uint32_t)C};
    const gdn_status_t st =
        make_tensor_map_3d(&maps.o, kBf16Out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.o,
                           dims, strides, box, "fused prefill", CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != GDN_OK) return st;
  }
  gdn_prefill_fused_kernel<TIn, TOut><<<grid, kThreads, SMEM_BYTES, stream>>>(s, a, maps);
  return check_launch("gdn_chunk_prefill (fused)");
}

}  // namespace

gdn_status_t prefill_fused_launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  if ((long long)s.N * s.H >= (1LL << 31)) return fail(GDN_ERR_UNSUPPORTED, "N * H too large");
  if (a.in_dtype == GDN_BF16)
    return a.out_dtype == GDN_BF16 ? launch<__nv_bfloat16, __nv_bfloat16>(s, a, stream)
                                   : launch<__nv_bfloat16, float>(s, a, stream);
  return a.out_dtype == GDN_BF16 ? launch<float, __nv_bfloat16>(s, a, stream)
                                 : launch<float, float>(s, a, stream);
}

}  // namespace gdn
