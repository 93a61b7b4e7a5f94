// Decode step of the gated delta rule / gated delta product over a slot-indexed
// fp32 state pool, updated in place.
//
// Design (B200). The step is HBM-bound: every (slot, head) state of dk x dv fp32
// is read once and written once. The T=1 split-V variant on the FlashInfer PR
// #7156 page ("Cake GDP kernel: shared-memory reduction and direct register
// loads", sections 1-2) streams the state straight into registers; here each
// state instead moves as ONE bulk TMA copy (cp.async.bulk) into a shared-memory
// stage and back out with one bulk store, so the bytes in flight per SM no longer
// depend on how many registers the math needs:
//
//   persistent grid, one CTA per SM, items = (batch row, head) pairs
//   producer warp : per item, slot id, gates and betas (scalar loads issued
//                   before it waits for a free stage), then bulk copies of the
//                   state (64 KiB at dk = 128) and of the item's k, q, v rows into
//                   the stage (2-3 stages), tracked by an mbarrier's transaction
//                   count
//   consumer warps: single token: two threads per state row load its halves from
//                   shared memory into registers, do the arithmetic below and
//                   write the row back, and one consumer thread bulk-stores the
//                   stage to the pool; multi-token: two groups take alternate
//                   items, a thread owning half of two rows, and the producer
//                   stores each finished stage to the pool before refilling it
//
// Arithmetic. Per row j (value column j of S, stored K-last as S^T[j, :]) the
// step is M = T*n_h sub-steps (gate on the first sub-step of each token, then a
// Householder update) and T outputs. Writing the row after sub-step m as
// s_m = Gamma_m s_0 + sum_{l<=m} c_l k_l, every quantity the recurrence needs is
// a dot product of the OLD row s_0 with a key or a query plus per-head Gram
// entries:
//     u_m   = k_m . (gated s) = Gamma_m (k_m . s_0) + sum_{l<m} c_l (k_m . k_l)
//     c_m   = beta_m (v_m[j] - u_m)
//     o_t   = scale (Gamma (q_t . s_0) + sum_{l<=m_t} c_l (q_t . k_l))
//     s_new = Gamma_M s_0 + sum_m c_m k_m
// so one pass over the resident row for all dot products, one partner shuffle,
// an O(M^2) scalar recurrence and one pass for the update. For T = n_h = 1 this
// is u = k.s, c = beta (v - alpha u), s' = alpha s + c k, o = scale (alpha q.s + c q.k).
#pragma once

#include <cstring>

#include "common.cuh"
#include "decode.cuh"
#include "device_once.h"
#include "tcgen05.cuh"
#include "tensor_map.cuh"

namespace gdn {
namespace {

constexpr uint64_t kDecodeWaitNs = 2000000000ull;


// Stage layout for one item (all offsets 16-byte aligned):
//   [state DK x DK fp32][keys M x DK][queries TT x DK][values M x DK][header]
// header: slot (int), alpha[TT], beta[M], gram[M][M], qk[TT][M] (fp32)
//
// Single-token steps copy the state linearly (row j of S^T at j * DK * 4). Multi-
// token steps load and store it as DK/32 tiles of [DK rows][32 fp32] through a
// tensor map with the 128-byte swizzle: tile x holds columns 32x..32x+31, row j
// at j * 128 bytes, its 16-byte chunk c at ((c ^ (j & 7)) * 16). Eight consecutive
// rows then read one chunk index from eight different bank groups while the
// threads of a half-warp read the same key / query chunk (a broadcast).
template <int DK, int TT, int NH, typename TIn, int ROWS = DK>
struct StageLayout {
  static constexpr int M = TT * NH;
  static constexpr bool kSwizzled = M > 1;
  static constexpr uint32_t kAlign = kSwizzled ? 1024 : 128;  // the swizzle follows address bits 4-9
  static constexpr int kRows = ROWS;                           // state rows (value indices) per item
  static constexpr int kParts = DK / ROWS;                     // items per (batch row, head)
  static_assert(!kSwizzled || ROWS == DK, "multi-token steps take whole heads");
  static constexpr uint32_t kState = kRows * DK * 4;
  static constexpr uint32_t kRow = DK * sizeof(TIn);
  static constexpr uint32_t kKeys = kState;
  static constexpr uint32_t kQueries = kKeys + M * kRow;
  static constexpr uint32_t kValues = kQueries + TT * kRow;
  static constexpr uint32_t kHeader = kValues + M * kRow;
  static constexpr uint32_t kAlpha = kHeader + 16;
  static constexpr uint32_t kBeta = kAlpha + 4 * TT;
  static constexpr uint32_t kGram = kBeta + 4 * M;
  static constexpr uint32_t kQK = kGram + 4 * M * M;
  static constexpr uint32_t kBytes = ((kQK + 4 * TT * M) + kAlign - 1) / kAlign * kAlign;
  static constexpr uint32_t kVecBytes = (2 * M + TT) * kRow;
  // consumer groups (items in flight per CTA)
  static constexpr int kGroups = (M > 1) ? 2 : 1;
  // keys and queries as fp32 (one buffer per consumer group, shared by the stages);
  // T = n_h = 1 reads the raw vectors instead and needs none
  static constexpr uint32_t kVecF32 = (M > 1) ? kGroups * (M + TT) * DK * 4 : 0;
  static constexpr int kStages = (3 * kBytes + kVecF32 + 64 + kAlign <= 226 * 1024) ? 3 : 2;
  static constexpr uint32_t kSmem = kStages * kBytes + kVecF32 + 64 + kAlign;  // + barriers + alignment
};

template <typename TIn>
__device__ __forceinline__ void load4_f32(const uint8_t* p, float* out);
template <>
__device__ __forceinline__ void load4_f32<__nv_bfloat16>(const uint8_t* p, float* out) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
}
template <>
__device__ __forceinline__ void load4_f32<float>(const uint8_t* p, float* out) {
  const float4 f = *reinterpret_cast<const float4*>(p);
  out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
}

// Threads per state row of the single-token kernel (2 or 4; its consumer mapping
// supports both). 2 measured best on B200.
template <int TT, int NH>
__host__ __device__ constexpr int threads_per_row() { return 2; }

// Producer (one thread of the last warp): for each item of the CTA, in order, the
// slot id, gates and betas go into the stage header and the state and the item's
// k, q, v rows are bulk-copied into the stage; the stage's full barrier counts the
// bytes. A stage is refilled once its previous item released it (empty barrier).
// With kStores the consumers release a stage as soon as their arithmetic is done
// and the producer writes the stage's state back to the pool (tensor stores of
// the swizzled tiles) before it refills the stage, so the consumers never wait
// for a store to drain.
template <int DK, int TT, int NH, typename TIn, bool kStores, int ROWS = DK>
__device__ __forceinline__ void decode_producer(const DecodeParams& p, const CUtensorMap* pool_map, uint8_t* base,
                                                uint64_t* full, uint64_t* empty) {
  using L = StageLayout<DK, TT, NH, TIn, ROWS>;
  constexpr int M = L::M;
  constexpr int NS = L::kStages;
  const TIn* kp = static_cast<const TIn*>(p.k);
  const TIn* qp = static_cast<const TIn*>(p.q);
  const TIn* vp = static_cast<const TIn*>(p.v);
  // state of the stage's finished item `prev` -> pool
  auto store_stage = [&](int prev, uint8_t* st) {
    const int prev_item = blockIdx.x + prev * gridDim.x;
    const int ph = prev_item - (prev_item / p.H) * p.H;
    const int pslot = *reinterpret_cast<const int*>(st + L::kHeader);
    if (pslot < 0 || !p.update_pool) return;
#pragma unroll
    for (int x = 0; x < DK / 32; ++x)
      tc::tma_store_3d(pool_map, 32 * x, 0, pslot * p.H + ph, tc::smem_u32(st) + x * DK * 128);
    tc::bulk_commit();
  };
  int it = 0;
  int last_fill[NS];  // per stage: the last item filled into it (-1: none)
#pragma unroll
  for (int x = 0; x < NS; ++x) last_fill[x] = -1;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
    const int s = it % NS;
    // the item's scalars are loaded before the stage wait, which hides their latency
    const int bh = item / L::kParts, part = item - bh * L::kParts;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    int slot = __ldg(p.slot_ids + b);
    float gv[TT], bv[M];
#pragma unroll
    for (int t = 0; t < TT; ++t) gv[t] = __ldg(p.g + ((size_t)b * TT + t) * p.H + h);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const int t = m / NH, mm = m - t * NH;
      bv[m] = __ldg(p.beta + (((size_t)b * TT + t) * p.H + h) * NH + mm);
    }
    if (it >= NS && !tc::mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, kDecodeWaitNs)) {
      raise_device_error(p.err, GDN_DEVERR_TIMEOUT);
      break;
    }
    last_fill[s] = it;
    uint8_t* st = base + s * L::kBytes;
    if constexpr (kStores) {
      if (it >= NS) {
        store_stage(it - NS, st);
        tc::bulk_wait_read();  // the stores have read the stage: it may be refilled
      }
    }
    if (slot >= p.num_slots) {
      raise_device_error(p.err, GDN_DEVERR_SLOT_OUT_OF_RANGE);
      slot = -1;
    }
    if (slot < 0) slot = -1;
    *reinterpret_cast<int*>(st + L::kHeader) = slot;
#pragma unroll
    for (int t = 0; t < TT; ++t) reinterpret_cast<float*>(st + L::kAlpha)[t] = expf(gv[t]);
#pragma unroll
    for (int m = 0; m < M; ++m) reinterpret_cast<float*>(st + L::kBeta)[m] = bv[m];
    if (slot < 0) {
      tc::mbar_arrive(&full[s]);
      continue;
    }
    tc::mbar_arrive_expect_tx(&full[s], L::kState + L::kVecBytes);
    const uint32_t sst = tc::smem_u32(st);
    if constexpr (L::kSwizzled) {
#pragma unroll
      for (int x = 0; x < DK / 32; ++x) tc::tma_load_3d(sst + x * DK * 128, pool_map, 32 * x, 0, slot * p.H + h, &full[s]);
    } else {
      tc::bulk_load(sst, p.pool + (((size_t)slot * p.H + h) * DK + (size_t)part * L::kRows) * DK, L::kState,
                    &full[s]);
    }
    const int hq = h / (p.H / p.Hqk);  // the value head's query/key head
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const size_t bth = ((size_t)b * TT + t) * p.H + h;
      const size_t btq = ((size_t)b * TT + t) * p.Hqk + hq;
      tc::bulk_load(sst + L::kKeys + t * NH * L::kRow, kp + btq * NH * DK, NH * L::kRow, &full[s]);
      tc::bulk_load(sst + L::kQueries + t * L::kRow, qp + btq * DK, L::kRow, &full[s]);
      tc::bulk_load(sst + L::kValues + t * NH * L::kRow, vp + bth * NH * DK, NH * L::kRow, &full[s]);
    }
  }
  if constexpr (kStores) {
    // the last items' states: each once its consumers are done with it
    for (int prev = (it > NS ? it - NS : 0); prev < it; ++prev) {
      const int s = prev % NS;
      if (!tc::mbar_wait(&empty[s], (prev / NS) & 1, kDecodeWaitNs)) {
        raise_device_error(p.err, GDN_DEVERR_TIMEOUT);
        break;
      }
      store_stage(prev, base + s * L::kBytes);
    }
    tc::bulk_wait_all();
  }
  // Every fill has landed before the CTA exits: after a timeout some were never
  // consumed. A stage is only refilled after its previous fill was consumed, so
  // waiting for each stage's last fill covers all of them (immediate when consumed).
#pragma unroll
  for (int x = 0; x < NS; ++x)
    if (last_fill[x] >= 0) tc::mbar_wait(&full[x], (last_fill[x] / NS) & 1, kDecodeWaitNs);
}

// Single-token step (T = n_h = 1): 2 threads per state row, all consumers on one item.
// An item is ROWS consecutive state rows (value indices) of one (batch row, head):
// the whole head when there are enough heads to fill the GPU, a part of it (the
// split along V) otherwise. Rows are independent in this step (each needs only the
// head's k, q and its own v entry), so every row gets the same arithmetic in the
// same order whatever ROWS is.
//
// Registers are allocated per scheduler (a quarter of the SM's 64K each, in units
// of 256 per warp). A split head's CTA is small enough that two or more fit in
// shared memory, so its register use is capped at 168 (5,376 per warp, three warps
// per scheduler): at 180 a scheduler holds two warps and one CTA of five warps
// fills the SM.
template <int DK, int TT, int NH, typename TIn, typename TOut, int ROWS>
__global__ void __launch_bounds__(threads_per_row<TT, NH>() * ROWS + 32, 1) __maxnreg__(ROWS < DK ? 168 : 255)
gdn_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap pool_map) {
  using L = StageLayout<DK, TT, NH, TIn, ROWS>;
  static_assert(L::M == 1, "single-token step");
  constexpr int NS = L::kStages;
  constexpr int TPR = threads_per_row<TT, NH>();
  constexpr int kConsumers = TPR * ROWS;
  constexpr int CPH = DK / (4 * TPR);        // float4 chunks per thread's part of a row
  constexpr int RPW = 32 / TPR;              // rows per warp
  constexpr uint32_t kBarConsumers = 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = tc::align_smem<L::kAlign>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + NS * L::kBytes + L::kVecF32);
  uint64_t* empty = full + NS;

  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::fence_mbar_init();
  }
  __syncthreads();

  if (tid >= kConsumers) {
    if (tid == kConsumers) decode_producer<DK, TT, NH, TIn, false, ROWS>(p, &pool_map, base, full, empty);
    return;
  }

  // ---------------- consumers: thread -> (row, part); the parts of a row are lanes
  // that differ in their top bits, so partial sums combine with xor shuffles
  const int lane = tid & 31, warp = tid >> 5;
  const int row = warp * RPW + (lane & (RPW - 1));
  const int half = lane / RPW;  // which part of the row (0..TPR-1)
  TOut* op = static_cast<TOut*>(p.o);
  int it = 0;
  int prev_stage = -1;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
    const int s = it % NS;
    uint8_t* st = base + s * L::kBytes;
    if (!tc::mbar_wait(&full[s], (it / NS) & 1, kDecodeWaitNs)) {
      if (tid == 0) raise_device_error(p.err, GDN_DEVERR_TIMEOUT);
      break;
    }
    const int bh = item / L::kParts, part = item - bh * L::kParts;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int grow = part * ROWS + row;  // the row's value index in the head
    const int slot = *reinterpret_cast<const int*>(st + L::kHeader);
    const float* alpha = reinterpret_cast<const float*>(st + L::kAlpha);
    const float* betas = reinterpret_cast<const float*>(st + L::kBeta);
    if (slot >= 0) {
      // k.s, q.s and the Gram entry q.k in one pass over the half row (the chunk
      // order is rotated by the row, which spreads a warp's loads over the banks)
      float* srow = reinterpret_cast<float*>(st) + (size_t)row * DK + half * (DK / TPR);
      float4 sv[CPH];
#pragma unroll
      for (int c = 0; c < CPH; ++c) sv[c] = reinterpret_cast<const float4*>(srow)[(c + grow) & (CPH - 1)];
      float ks = 0.f, qs = 0.f, qkv = 0.f;
#pragma unroll
      for (int c = 0; c < CPH; ++c) {
        const int e = half * (DK / TPR) + 4 * ((c + grow) & (CPH - 1));
        float wk[4], wq[4];
        load4_f32<TIn>(st + L::kKeys + e * sizeof(TIn), wk);
        load4_f32<TIn>(st + L::kQueries + e * sizeof(TIn), wq);
        ks = fmaf(sv[c].x, wk[0], fmaf(sv[c].y, wk[1], fmaf(sv[c].z, wk[2], fmaf(sv[c].w, wk[3], ks))));
        qs = fmaf(sv[c].x, wq[0], fmaf(sv[c].y, wq[1], fmaf(sv[c].z, wq[2], fmaf(sv[c].w, wq[3], qs))));
        qkv = fmaf(wq[0], wk[0], fmaf(wq[1], wk[1], fmaf(wq[2], wk[2], fmaf(wq[3], wk[3], qkv))));
      }
      ks += __shfl_xor_sync(0xffffffffu, ks, 16);
      qs += __shfl_xor_sync(0xffffffffu, qs, 16);
      qkv += __shfl_xor_sync(0xffffffffu, qkv, 16);
      float rk = 1.f;  // 1 / |k| with the normalisation (the update then adds cm rk k)
      if (p.flags & GDN_QK_L2NORM) {
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int c = 0; c < CPH; ++c) {
          const int e = half * (DK / TPR) + 4 * c;
          float wk[4], wq[4];
          load4_f32<TIn>(st + L::kKeys + e * sizeof(TIn), wk);
          load4_f32<TIn>(st + L::kQueries + e * sizeof(TIn), wq);
          kk = fmaf(wk[0], wk[0], fmaf(wk[1], wk[1], fmaf(wk[2], wk[2], fmaf(wk[3], wk[3], kk))));
          qq = fmaf(wq[0], wq[0], fmaf(wq[1], wq[1], fmaf(wq[2], wq[2], fmaf(wq[3], wq[3], qq))));
        }
        kk += __shfl_xor_sync(0xffffffffu, kk, 16);
        qq += __shfl_xor_sync(0xffffffffu, qq, 16);
        rk = kk > 0.f ? 1.f / sqrtf(kk) : 0.f;
        const float rq = qq > 0.f ? 1.f / sqrtf(qq) : 0.f;
        ks *= rk;
        qs *= rq;
        qkv *= rq * rk;
      }
      const float a = alpha[0];
      const float vj = to_f32(reinterpret_cast<const TIn*>(st + L::kValues)[grow]);
      const float cm = betas[0] * (vj - a * ks);
      const float cmk = cm * rk;
      if (half == 0) store_out(op + ((size_t)b * p.H + h) * DK + grow, p.scale * fmaf(cm, qkv, a * qs));
#pragma unroll
      for (int c = 0; c < CPH; ++c) {
        const int e = half * (DK / TPR) + 4 * ((c + grow) & (CPH - 1));
        float wk[4];
        load4_f32<TIn>(st + L::kKeys + e * sizeof(TIn), wk);
        float4 x = sv[c];
        x.x = fmaf(cmk, wk[0], a * x.x);
        x.y = fmaf(cmk, wk[1], a * x.y);
        x.z = fmaf(cmk, wk[2], a * x.z);
        x.w = fmaf(cmk, wk[3], a * x.w);
        reinterpret_cast<float4*>(srow)[(c + grow) & (CPH - 1)] = x;
      }
    } else {
      // skipped row of the batch: o = 0 (and a zero token state), pool untouched
      if (half == 0) store_out(op + ((size_t)b * p.H + h) * DK + grow, 0.f);
      if (p.token_states) {
        float4* dst = reinterpret_cast<float4*>(p.token_states + (((size_t)b * p.H + h) * DK + grow) * DK +
                                                half * (DK / TPR));
#pragma unroll
        for (int c = 0; c < CPH; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // stage -> pool (one bulk store), and to the token-state buffer when asked (the
    // state after the single token); the previous item's stage is handed back to
    // the producer once its stores have finished reading shared memory
    tc::fence_proxy_async_smem();
    tc::named_sync(kBarConsumers, kConsumers);
    if (tid == 0) {
      const size_t rows_off = ((size_t)h * DK + (size_t)part * ROWS) * DK;
      if (slot >= 0 && p.update_pool)
        tc::bulk_store(p.pool + (size_t)slot * p.H * DK * DK + rows_off, tc::smem_u32(st), L::kState);
      if (slot >= 0 && p.token_states)
        tc::bulk_store(p.token_states + (size_t)b * p.H * DK * DK + rows_off, tc::smem_u32(st), L::kState);
      tc::bulk_commit();
      tc::bulk_wait_read_1();
      if (prev_stage >= 0) tc::mbar_arrive(&empty[prev_stage]);
    }
    prev_stage = s;
  }
  if (tid == 0) tc::bulk_wait_all();
}

// Packed fp32 arithmetic (sm_100): one instruction does two independent fp32 FMAs
// (or products), each rounded like its scalar form, so two state elements advance
// together with the per-element operation sequence of a scalar loop.
__device__ __forceinline__ float2 lo_pair(const float4& x) { return make_float2(x.x, x.y); }
__device__ __forceinline__ float2 hi_pair(const float4& x) { return make_float2(x.z, x.w); }

// One 16-byte chunk (4 columns) of two rows: x <- G x + sum_{m < n_terms} c_m k_m, the
// terms in order m = 0, 1, ...; w points at the chunk's columns of key 0 in the
// [vectors][DK] fp32 buffer, cc0/cc1 hold each row's c_m twice.
template <int DK, int M>
__device__ __forceinline__ void apply_terms(float4& x0, float4& x1, float G, const float2* cc0, const float2* cc1,
                                            const float* w, int n_terms) {
  const float2 gg = make_float2(G, G);
  float2 a0 = __fmul2_rn(gg, lo_pair(x0)), b0 = __fmul2_rn(gg, hi_pair(x0));
  float2 a1 = __fmul2_rn(gg, lo_pair(x1)), b1 = __fmul2_rn(gg, hi_pair(x1));
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if (m >= n_terms) break;
    const float4 wv = *reinterpret_cast<const float4*>(w + m * DK);
    a0 = __ffma2_rn(cc0[m], lo_pair(wv), a0);
    a1 = __ffma2_rn(cc1[m], lo_pair(wv), a1);
    b0 = __ffma2_rn(cc0[m], hi_pair(wv), b0);
    b1 = __ffma2_rn(cc1[m], hi_pair(wv), b1);
  }
  x0 = make_float4(a0.x, a0.y, b0.x, b0.y);
  x1 = make_float4(a1.x, a1.y, b1.x, b1.y);
}

// Multi-token / product step (M = T n_h > 1). Two consumer groups of DK threads
// take the CTA's items alternately (group g its items g, g + 2, ...), so one
// group's phases, which are separated by group barriers, overlap the other's.
// In a group a thread owns one half (16-byte chunks half*DK/8 .. ) of two state
// rows, j and j + DK/2: each key / query chunk it reads from shared memory (a
// broadcast across its half-warp) feeds both rows, which halves the shared-memory
// wavefronts per row against one row per thread. Per item:
//   keys and queries -> fp32 (the group's buffer); the Gram entries k_m.k_l (l < m)
//   and q_t.k_l, one warp per pair; the row pass (all NV dot products of the two
//   old rows, halves combined by one xor shuffle); the scalar recurrence of each
//   row; the update pass s_new = Gamma s_0 + sum_m c_m k_m written back in place;
//   the stage stored to the pool and released.
template <int DK, int TT, int NH, typename TIn, typename TOut, bool kTokenStates>
__global__ void __launch_bounds__(2 * DK + 32, 1)
gdn_decode_multi_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap pool_map) {
  using L = StageLayout<DK, TT, NH, TIn>;
  static_assert(L::M > 1 && L::kGroups == 2, "multi-token step");
  constexpr int M = L::M;
  constexpr int NV = M + TT;                 // vectors dotted with the old rows: keys then queries
  constexpr int NS = L::kStages;
  constexpr int kGroupThreads = DK;          // DK/2 row pairs x 2 halves
  constexpr int kConsumers = 2 * kGroupThreads;
  constexpr int CPH = DK / 8;                // float4 chunks in half a row
  constexpr int kPairsKK = M * (M - 1) / 2;
  constexpr int kPairs = kPairsKK + TT * M;
  constexpr int kGroupWarps = kGroupThreads / 32;
  constexpr int kBatch = 8;                  // Gram pairs per warp reduced together

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = tc::align_smem<L::kAlign>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + NS * L::kBytes + L::kVecF32);
  uint64_t* empty = full + NS;

  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::fence_mbar_init();
  }
  __syncthreads();

  if (tid >= kConsumers) {
    if (tid == kConsumers) decode_producer<DK, TT, NH, TIn, true>(p, &pool_map, base, full, empty);
    return;
  }

  const int grp = tid / kGroupThreads, gt = tid - grp * kGroupThreads;
  const uint32_t bar_id = 1 + grp;
  float* vecf = reinterpret_cast<float*>(base + NS * L::kBytes) + grp * NV * DK;  // [NV][DK] fp32
  const int lane = gt & 31, gw = gt >> 5;
  const int half = lane >> 4;
  const int r0 = gw * 16 + (lane & 15), r1 = r0 + DK / 2;
  // chunk gc of row r sits in tile gc / 8 at the swizzled position (gc % 8) ^ (r % 8);
  // r1 % 8 == r0 % 8, so both rows use the same offsets
  TOut* op = static_cast<TOut*>(p.o);
  for (int it = grp, item = blockIdx.x + grp * gridDim.x; item < p.n_items; it += 2, item += 2 * gridDim.x) {
    const int s = it % NS;
    uint8_t* st = base + s * L::kBytes;
    // The stage's previous item (it - NS) must have been released before this fill
    // is waited for, so that full[s]'s parity names this fill and not the last one.
    if (it >= NS && !tc::mbar_wait(&empty[s], ((it - NS) / NS) & 1, kDecodeWaitNs)) {
      if (gt == 0) raise_device_error(p.err, GDN_DEVERR_TIMEOUT);
      break;
    }
    if (!tc::mbar_wait(&full[s], (it / NS) & 1, kDecodeWaitNs)) {
      if (gt == 0) raise_device_error(p.err, GDN_DEVERR_TIMEOUT);
      break;
    }
    const int b = item / p.H, h = item - (item / p.H) * p.H;
    const int slot = *reinterpret_cast<const int*>(st + L::kHeader);
    const float* alpha = reinterpret_cast<const float*>(st + L::kAlpha);
    const float* betas = reinterpret_cast<const float*>(st + L::kBeta);
    float* gram = reinterpret_cast<float*>(st + L::kGram);
    float* qk = reinterpret_cast<float*>(st + L::kQK);
    if (slot >= 0) {
      // keys and queries of the item -> fp32 once (every FMA below reads them)
      for (int e = gt * 4; e < NV * DK; e += kGroupThreads * 4)
        load4_f32<TIn>(st + L::kKeys + e * sizeof(TIn), vecf + e);
      tc::named_sync(bar_id, kGroupThreads);
      if (p.flags & GDN_QK_L2NORM) {  // every key and query to unit length, in place
        for (int vi = gw; vi < NV; vi += kGroupWarps) {
          float* x = vecf + vi * DK;
          float ss = 0.f;
          for (int e = lane; e < DK; e += 32) ss = fmaf(x[e], x[e], ss);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          const float r = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
          for (int e = lane; e < DK; e += 32) x[e] *= r;
        }
        tc::named_sync(bar_id, kGroupThreads);
      }
      // Gram entries: warp w takes pairs w, w + W, ...; a batch of kBatch pairs has
      // its partial sums reduced together (independent shuffles)
      for (int p0 = gw; p0 < kPairs; p0 += kGroupWarps * kBatch) {
        float gacc[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int pair = p0 + q * kGroupWarps;
          gacc[q] = 0.f;
          if (pair < kPairs) {  // warp-uniform
            int va, vb;
            if (pair < kPairsKK) {
              va = 1;
              int rem = pair;
              while (rem >= va) { rem -= va; ++va; }
              vb = rem;
            } else {
              const int x = pair - kPairsKK;
              va = M + x / M;
              vb = x - (x / M) * M;
            }
            const float* pa = vecf + va * DK;  // the queries follow the keys
            const float* pb = vecf + vb * DK;
            for (int e = lane * 4; e < DK; e += 128) {
              const float4 xa = *reinterpret_cast<const float4*>(pa + e);
              const float4 xb = *reinterpret_cast<const float4*>(pb + e);
              gacc[q] = fmaf(xa.x, xb.x, fmaf(xa.y, xb.y, fmaf(xa.z, xb.z, fmaf(xa.w, xb.w, gacc[q]))));
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
          for (int q = 0; q < kBatch; ++q) gacc[q] += __shfl_xor_sync(0xffffffffu, gacc[q], off);
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < kBatch; ++q) {
            const int pair = p0 + q * kGroupWarps;
            if (pair < kPairsKK) {
              int va = 1, rem = pair;
              while (rem >= va) { rem -= va; ++va; }
              gram[va * M + rem] = gacc[q];
            } else if (pair < kPairs) {
              const int x = pair - kPairsKK;
              qk[(x / M) * M + (x - (x / M) * M)] = gacc[q];
            }
          }
        }
      }
      tc::named_sync(bar_id, kGroupThreads);

      // row pass: dot products of both old rows with every key and query
      const uint8_t* srow0 = st + (size_t)r0 * 128;
      const uint8_t* srow1 = st + (size_t)r1 * 128;
      // (each dot product as two partial sums, over the even and the odd columns,
      // advanced together by packed FMAs and added at the end)
      float2 e0[NV], e1[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) e0[v] = e1[v] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int c = 0; c < CPH; ++c) {
        const int gc = half * CPH + c;
        const uint32_t off = (gc >> 3) * (DK * 128) + (((gc & 7) ^ (r0 & 7)) << 4);
        const float4 x0 = *reinterpret_cast<const float4*>(srow0 + off);
        const float4 x1 = *reinterpret_cast<const float4*>(srow1 + off);
        const float* w = vecf + 4 * gc;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const float4 wv = *reinterpret_cast<const float4*>(w + v * DK);
          e0[v] = __ffma2_rn(lo_pair(x0), lo_pair(wv), e0[v]);
          e1[v] = __ffma2_rn(lo_pair(x1), lo_pair(wv), e1[v]);
          e0[v] = __ffma2_rn(hi_pair(x0), hi_pair(wv), e0[v]);
          e1[v] = __ffma2_rn(hi_pair(x1), hi_pair(wv), e1[v]);
        }
      }
      float d0[NV], d1[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        d0[v] = e0[v].x + e0[v].y;
        d1[v] = e1[v].x + e1[v].y;
      }
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        d0[v] += __shfl_xor_sync(0xffffffffu, d0[v], 16);
        d1[v] += __shfl_xor_sync(0xffffffffu, d1[v], 16);
      }

      // scalar recurrence of both rows (both halves, redundantly); half 0 writes the
      // outputs of row r0, half 1 those of row r1
      float c0[M], c1[M];
      float G = 1.f;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float a = alpha[t];
        G *= a;
#pragma unroll
        for (int l = 0; l < t * NH; ++l) {
          c0[l] *= a;
          c1[l] *= a;
        }
#pragma unroll
        for (int x = 0; x < NH; ++x) {
          const int m = t * NH + x;
          float u0 = G * d0[m], u1 = G * d1[m];
#pragma unroll
          for (int l = 0; l < m; ++l) {
            const float gv = gram[m * M + l];
            u0 = fmaf(c0[l], gv, u0);
            u1 = fmaf(c1[l], gv, u1);
          }
          const TIn* vrow = reinterpret_cast<const TIn*>(st + L::kValues + m * L::kRow);
          c0[m] = betas[m] * (to_f32(vrow[r0]) - u0);
          c1[m] = betas[m] * (to_f32(vrow[r1]) - u1);
        }
        float o0 = G * d0[M + t], o1 = G * d1[M + t];
#pragma unroll
        for (int l = 0; l < (t + 1) * NH; ++l) {
          const float qv = qk[t * M + l];
          o0 = fmaf(c0[l], qv, o0);
          o1 = fmaf(c1[l], qv, o1);
        }
        TOut* orow = op + (((size_t)b * TT + t) * p.H + h) * DK;
        if (half == 0) store_out(orow + r0, p.scale * o0);
        else store_out(orow + r1, p.scale * o1);
        if (kTokenStates) {
          // the state after token t: Gamma_t s_0 + sum_{l <= m_t} c_l k_l (the
          // coefficients as they stand after this token's gate)
          const int n_terms = (t + 1) * NH;  // a constant once the token loop is unrolled
          float* ts0 = p.token_states + ((((size_t)b * TT + t) * p.H + h) * DK + r0) * DK;
          float* ts1 = p.token_states + ((((size_t)b * TT + t) * p.H + h) * DK + r1) * DK;
          float2 cc0[M], cc1[M];
#pragma unroll
          for (int m = 0; m < M; ++m) {
            cc0[m] = make_float2(c0[m], c0[m]);
            cc1[m] = make_float2(c1[m], c1[m]);
          }
#pragma unroll 4
          for (int c = 0; c < CPH; ++c) {
            const int gc = half * CPH + c;
            const uint32_t off = (gc >> 3) * (DK * 128) + (((gc & 7) ^ (r0 & 7)) << 4);
            float4 x0 = *reinterpret_cast<const float4*>(st + (size_t)r0 * 128 + off);
            float4 x1 = *reinterpret_cast<const float4*>(st + (size_t)r1 * 128 + off);
            apply_terms<DK, M>(x0, x1, G, cc0, cc1, vecf + 4 * gc, n_terms);
            reinterpret_cast<float4*>(ts0)[gc] = x0;
            reinterpret_cast<float4*>(ts1)[gc] = x1;
          }
        }
      }

      // update pass: s_new = Gamma s_0 + sum_m c_m k_m, in place (same swizzled chunks)
      uint8_t* wrow0 = st + (size_t)r0 * 128;
      uint8_t* wrow1 = st + (size_t)r1 * 128;
      float2 cc0[M], cc1[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        cc0[m] = make_float2(c0[m], c0[m]);
        cc1[m] = make_float2(c1[m], c1[m]);
      }
#pragma unroll 4
      for (int c = 0; c < CPH; ++c) {
        const int gc = half * CPH + c;
        const uint32_t off = (gc >> 3) * (DK * 128) + (((gc & 7) ^ (r0 & 7)) << 4);
        float4 x0 = *reinterpret_cast<const float4*>(wrow0 + off);
        float4 x1 = *reinterpret_cast<const float4*>(wrow1 + off);
        apply_terms<DK, M>(x0, x1, G, cc0, cc1, vecf + 4 * gc, M);
        *reinterpret_cast<float4*>(wrow0 + off) = x0;
        *reinterpret_cast<float4*>(wrow1 + off) = x1;
      }
    } else {
      // skipped row of the batch: o = 0 (and zero token states), pool untouched
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        TOut* orow = op + (((size_t)b * TT + t) * p.H + h) * DK;
        store_out(orow + (half == 0 ? r0 : r1), 0.f);
        if (kTokenStates) {
          float* ts0 = p.token_states + ((((size_t)b * TT + t) * p.H + h) * DK + r0) * DK;
          float* ts1 = p.token_states + ((((size_t)b * TT + t) * p.H + h) * DK + r1) * DK;
          for (int c = 0; c < CPH; ++c) {
            reinterpret_cast<float4*>(ts0)[half * CPH + c] = make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(ts1)[half * CPH + c] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
    }
    // the stage goes back to the producer, which stores the state to the pool
    // (the writes are made visible to its tensor stores first)
    tc::fence_proxy_async_smem();
    tc::named_sync(bar_id, kGroupThreads);
    if (gt == 0) tc::mbar_arrive(&empty[s]);
  }
}

// The pool as a 3-D fp32 tensor {DK columns, DK rows, num_slots * H states}; a box
// is one 32-column tile of one state, 128-byte swizzled.
template <int DK>
gdn_status_t pool_tensor_map(const DecodeParams& p, CUtensorMap* map) {
  const uint64_t dims[3] = {(uint64_t)DK, (uint64_t)DK, (uint64_t)p.num_slots * (uint64_t)p.H};
  const uint64_t strides[2] = {(uint64_t)DK * 4, (uint64_t)DK * DK * 4};
  const uint32_t box[3] = {32, (uint32_t)DK, 1};
  return make_tensor_map_3d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.pool, dims, strides, box, "gdn_decode");
}

// Multi-token / product step: one CTA per SM, whole heads (with or without the
// per-token states, two instantiations so the plain step carries no extra code).
template <int DK, int TT, int NH, typename TIn, typename TOut, bool kTokenStates>
gdn_status_t launch_multi_k(DecodeParams p, cudaStream_t stream) {
  using L = StageLayout<DK, TT, NH, TIn>;
  // per device: the SM count (grid size) and the shared-memory opt-in
  static PerDeviceOnce once;
  int dev = 0, sm_count = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("gdn_decode: cudaGetDevice: ") + cudaGetErrorString(e));
  const bool ready = run_once_per_device(once, dev, [&](int d, int* sms) {
    e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, d);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn_decode_multi_kernel<DK, TT, NH, TIn, TOut, kTokenStates>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    return e == cudaSuccess;
  }, &sm_count);
  if (!ready)
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("gdn_decode: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  p.n_items = p.B * p.H;
  if (p.n_items == 0) return ok();
  const int grid = p.n_items < sm_count ? p.n_items : sm_count;
  if ((long long)p.num_slots * p.H >= (1LL << 31))
    return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: num_slots * H must be below 2^31 for multi-token steps");
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  const gdn_status_t st = pool_tensor_map<DK>(p, &map);
  if (st != GDN_OK) return st;
  gdn_decode_multi_kernel<DK, TT, NH, TIn, TOut, kTokenStates><<<grid, 2 * DK + 32, L::kSmem, stream>>>(p, map);
  return check_launch("gdn_decode");
}

template <int DK, int TT, int NH, typename TIn, typename TOut>
gdn_status_t launch_multi(DecodeParams p, cudaStream_t stream) {
  return p.token_states ? launch_multi_k<DK, TT, NH, TIn, TOut, true>(p, stream)
                        : launch_multi_k<DK, TT, NH, TIn, TOut, false>(p, stream);
}

// Single-token step with ROWS state rows per item; persistent grid of as many CTAs
// as fit on the device at once (one per SM for whole heads, several for parts).
template <int DK, typename TIn, typename TOut, int ROWS>
gdn_status_t launch_single_rows(DecodeParams p, cudaStream_t stream) {
  using L = StageLayout<DK, 1, 1, TIn, ROWS>;
  constexpr int kThreadsPerCta = threads_per_row<1, 1>() * ROWS + 32;
  auto kernel = gdn_decode_kernel<DK, 1, 1, TIn, TOut, ROWS>;
  static PerDeviceOnce once;  // per device: SMs x resident CTAs, and the shared-memory opt-in
  int dev = 0, slots = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("gdn_decode: cudaGetDevice: ") + cudaGetErrorString(e));
  const bool ready = run_once_per_device(once, dev, [&](int d, int* out) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    // the whole configurable L1/shared split to shared memory, so that several of the
    // smaller CTAs of a split head fit on an SM (the occupancy query below, and the
    // launches, use this carveout)
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreadsPerCta, L::kSmem);
    *out = sms * (per_sm > 0 ? per_sm : 1);
    return e == cudaSuccess;
  }, &slots);
  if (!ready)
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("gdn_decode: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  p.n_items = p.B * p.H * L::kParts;
  if (p.n_items == 0) return ok();
  const int grid = p.n_items < slots ? p.n_items : slots;
  CUtensorMap map;  // unused by the single-token step (linear bulk copies)
  memset(&map, 0, sizeof(map));
  kernel<<<grid, kThreadsPerCta, L::kSmem, stream>>>(p, map);
  return check_launch("gdn_decode");
}

// Parts per head for the single-token step: whole heads when there are at least
// four per SM, else the smallest power-of-two split (rows per part >= 16) that
// reaches four items per SM, so that every SM streams state even at small batch
// (the T=1 split-V idea of the FlashInfer PR #7156 page, introduction).
inline int decode_parts(long long heads, int sm_count, int dk) {
  int parts = 1;
  while (parts * 2 <= dk / 16 && heads * parts < 4LL * sm_count) parts *= 2;
  return parts;
}

template <int DK, typename TIn, typename TOut>
gdn_status_t launch_single(DecodeParams p, cudaStream_t stream) {
  static PerDeviceOnce once;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && !run_once_per_device(once, dev, [&](int d, int* out) {
        e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, d);
        return e == cudaSuccess;
      }, &sms))
    if (e == cudaSuccess) return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: device index too large");
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("gdn_decode: ") + cudaGetErrorString(e));
  switch (decode_parts((long long)p.B * p.H, sms, DK)) {
    case 1: return launch_single_rows<DK, TIn, TOut, DK>(p, stream);
    case 2: if constexpr (DK / 2 >= 16) return launch_single_rows<DK, TIn, TOut, DK / 2>(p, stream); break;
    case 4: if constexpr (DK / 4 >= 16) return launch_single_rows<DK, TIn, TOut, DK / 4>(p, stream); break;
    case 8: if constexpr (DK / 8 >= 16) return launch_single_rows<DK, TIn, TOut, DK / 8>(p, stream); break;
    default: break;
  }
  return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: no split for this head size");
}

template <int DK, int TT, int NH, typename TIn, typename TOut>
gdn_status_t launch_typed(DecodeParams p, cudaStream_t stream) {
  if constexpr (TT == 1 && NH == 1)
    return launch_single<DK, TIn, TOut>(p, stream);
  else
    return launch_multi<DK, TT, NH, TIn, TOut>(p, stream);
}

template <int DK, int TT, int NH>
gdn_status_t launch_dtypes(DecodeParams p, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s) {
  if (in == GDN_BF16) {
    return out == GDN_BF16 ? launch_typed<DK, TT, NH, __nv_bfloat16, __nv_bfloat16>(p, s)
                           : launch_typed<DK, TT, NH, __nv_bfloat16, float>(p, s);
  }
  return out == GDN_BF16 ? launch_typed<DK, TT, NH, float, __nv_bfloat16>(p, s)
                         : launch_typed<DK, TT, NH, float, float>(p, s);
}

template <int DK>
gdn_status_t launch_steps(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out, cudaStream_t s) {
#define GDN_DECODE_CASE(TT_, NH_) \
  if (T == TT_ && nh == NH_) return launch_dtypes<DK, TT_, NH_>(p, in, out, s);
  GDN_DECODE_CASE(1, 1)
  GDN_DECODE_CASE(2, 1)
  GDN_DECODE_CASE(4, 1)
  GDN_DECODE_CASE(8, 1)
  GDN_DECODE_CASE(1, 2)
  GDN_DECODE_CASE(2, 2)
  GDN_DECODE_CASE(4, 2)
  GDN_DECODE_CASE(1, 4)
  GDN_DECODE_CASE(2, 4)
#undef GDN_DECODE_CASE
  return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: (T, n_h) = (" + std::to_string(T) + ", " +
                                       std::to_string(nh) +
                                       ") not built; T in {1,2,4,8}, n_h in {1,2,4}, T*n_h <= 8");
}

}  // namespace
}  // namespace gdn
