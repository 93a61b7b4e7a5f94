// Backward of the prefill: reverse-mode derivatives of the gated delta rule with
// respect to q, k, v, g, beta and the initial state, given the derivatives of a loss
// with respect to the outputs and the final state. The pages give no backward pass;
// this is the chain rule on the two relations of one token (P = I - beta k k^T,
// S~ = alpha S_{t-1}, alpha = exp(g)):
//     S_t = P S~ + beta k v^T,        o_t = scale S_t^T q,
// walked from the last token to the first with D = dL/dS_t:
//     D    += scale q dO^T;           dq = scale S_t dO
//     u     = S~^T k;   w = D^T k;    dv = beta w;   dbeta = w . (v - u)
//     dk    = beta (D (v - u) - S~ w)
//     dg    = <D, S~> - beta (u . w)
//     D    <- alpha (D - beta k w^T)  (dL/dS_{t-1});   dL/dS_0 = D at the end.
// With GDN_QK_L2NORM the relations read k^ = k / |k| and q^ = q / |q| (zero stays
// zero) and the derivatives found for them are mapped back through the
// normalisation, dk = (dk^ - k^ (k^ . dk^)) / |k| (likewise q), a linear map that is
// applied to each CTA's partial sums before they are added up.
//
// Token-sequential SIMT. Every value column j of S (and of D) evolves on its own given
// the token's k, q, v_j, alpha and beta, so one CTA (one warp) takes 1024 / dk columns
// of one (sequence, head) (many small CTAs per SM); value column j is owned by dk / 32
// adjacent lanes, 32 of its dk entries each. The states S_{t-1} the walk needs are recomputed:
//   1. forward over the sequence, writing the state at the start of every chunk of
//      C tokens to the workspace (checkpoints);
//   2. for each chunk, last to first: recompute the chunk's states from its
//      checkpoint into a per-CTA scratch (the state before each of its tokens), then
//      walk its tokens backwards reading S_{t-1} from there (a thread reads back only
//      what it wrote, so no barrier orders the scratch).
// Per token the sums over columns of dq and dk go through shared memory (each thread
// writes its partial products, then each thread adds dk / 32 consecutive entries over
// the CTA's columns); dg and dbeta are warp reductions. All four are accumulated
// with fp32 atomics (vector atomics for dq and dk) into zeroed outputs, so the column
// blocks of a head and the value heads that share a q/k head add up.
// Latency: the tokens' k, q, gates and the CTA's columns of v and dO are copied into
// a shared-memory ring by cp.async several positions ahead of their use (the order
// in which the three passes visit the tokens is fixed, so an incremental cursor
// walks it without divisions); in the backward walk S_t is the previous token's
// S_{t-1} (kept in registers) and the next S_{t-1} is fetched from the scratch into
// shared memory by cp.async while the current token computes (each thread copies and
// reads only its own entries). Dot products over a thread's entries use four partial
// sums, which shortens their dependency chains.
#include <string>

#include "device_once.h"
#include "prefill.cuh"

namespace gdn {
namespace {

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* d_o;
  const float* g;
  const float* beta;
  const int32_t* cu;
  const float* init;
  const float* d_fin;
  float* dq;
  float* dk;
  float* dv;
  float* dg;
  float* dbeta;
  float* d_init;
  float* ckpt;     // [H][ck_slots][D][D]
  float* scratch;  // [N * H][C + 1][D][D] (each CTA its own columns' rows)
  size_t ck_slots;
  int64_t total_T;
  int N, H, Hqk, C;
  float scale;
  int l2norm;
  unsigned int* err;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  size_t ck_slots, scratch_off, bytes;
};

// Sequence n's checkpoints take slots bos / C + n ... (+ ceil(len / C)), which never
// overlap the next sequence's and stay below total_T / C + N + 1.
BwdLayout bwd_layout(int N, int64_t total_T, int H, int D, int C) {
  BwdLayout L;
  const size_t st = (size_t)D * D * sizeof(float);
  L.ck_slots = (size_t)(total_T / C) + (size_t)N + 1;
  L.scratch_off = align256((size_t)H * L.ck_slots * st);
  L.bytes = L.scratch_off + (size_t)N * H * (size_t)(C + 1) * st;
  return L;
}

// entries of a state column held by one thread; a column takes D / kBwdPer lanes
constexpr int kBwdPer = 32;
template <int D>
constexpr int bwd_tpc() { return D / kBwdPer; }

// value columns per CTA: one warp per CTA (32 / (D / kBwdPer) columns), so many small
// CTAs share an SM and a barrier spans one warp
template <int D>
constexpr int bwd_cols() { return 32 / bwd_tpc<D>(); }

// Shared-memory stride of one column in the [columns][D entries] buffers, padded so
// that the eight lanes of a quarter warp (8 / tpc columns of tpc 16-byte pieces each)
// store to distinct banks: consecutive columns start 4 tpc banks apart.
template <int D>
constexpr int bwd_col_stride() { return D + 4 * bwd_tpc<D>(); }

template <int D>
constexpr int bwd_threads() { return bwd_cols<D>() * bwd_tpc<D>(); }

// The kernel visits its tokens in a fixed order of 3 len positions: the forward
// sweep, then for each chunk from the last its tokens forward (recompute) and
// backward (walk). Each position's k, q, g, beta and the CTA's columns of v and dO
// are copied, in the input dtype, into a ring of kRing shared-memory slots by cp.async
// kRing - 1 positions ahead of their use.
constexpr int kRing = 8;

template <int D, typename TIn>
struct BwdSlot {
  static constexpr int kVec = D * (int)sizeof(TIn);               // bytes of k (and of q)
  static constexpr int kOwn = bwd_cols<D>() * (int)sizeof(TIn);   // bytes of the CTA's columns of v (of dO)
  static constexpr int kOwnPad = (kOwn + 15) / 16 * 16;
  static constexpr int kQ = kVec;
  static constexpr int kV = 2 * kVec;
  static constexpr int kDO = kV + kOwnPad;
  static constexpr int kG = kDO + kOwnPad;  // g, then beta (fp32)
  static constexpr int kBytes = kG + 16;
  static_assert(kVec % 16 == 0 && (kOwn == 4 || kOwn == 8 || kOwn % 16 == 0), "cp.async sizes");
};

template <int D, typename TIn>
constexpr size_t bwd_smem_bytes() {
  // the token ring, then (fp32) the column partials of dq and dk and the prefetched
  // S_{t-1}, [columns][stride] each
  return (size_t)kRing * BwdSlot<D, TIn>::kBytes + 3 * (size_t)bwd_cols<D>() * bwd_col_stride<D>() * sizeof(float);
}

template <int N>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  if constexpr (N == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(d), "l"(src), "n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// N = 1, 2 or 4 consecutive fp32 entries (aligned to N) from shared memory, and their
// addition to global memory by one vector atomic
template <int N>
__device__ __forceinline__ void ld_vec(const float* p, float* out) {
  if constexpr (N == 4) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
  } else if constexpr (N == 2) {
    const float2 f = *reinterpret_cast<const float2*>(p);
    out[0] = f.x; out[1] = f.y;
  } else {
    out[0] = *p;
  }
}
template <int N>
__device__ __forceinline__ void atomic_add_vec(float* p, const float* v) {
  if constexpr (N == 4) {
    atomicAdd(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
  } else if constexpr (N == 2) {
    atomicAdd(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
  } else {
    atomicAdd(p, v[0]);
  }
}

// entries x, x + 1 of a register array as one packed pair, and back
__device__ __forceinline__ float2 pr(const float* a, int x) { return make_float2(a[x], a[x + 1]); }
__device__ __forceinline__ void put(float* a, int x, float2 v) {
  a[x] = v.x;
  a[x + 1] = v.y;
}

// four consecutive entries of a token vector in shared memory, as fp32
__device__ __forceinline__ float4 ld4_f32(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4_f32(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

template <int D, typename TIn>
__global__ void __launch_bounds__(bwd_threads<D>())
gdn_prefill_backward_kernel(const BwdArgs a) {
  constexpr int TPC = bwd_tpc<D>();  // threads per state column
  constexpr int kBwdCols = bwd_cols<D>();
  constexpr int NT = kBwdCols * TPC;
  constexpr int EPT = D / NT;  // consecutive dk entries of dq and dk per thread
  static_assert(NT * EPT == D && NT == 32 && TPC * kBwdPer == D, "one warp, whole vectors");
  constexpr int PER = kBwdPer;  // entries of the column per thread
  constexpr int NP = PER / 4;   // 16-byte pieces per thread
  constexpr int RS = bwd_col_stride<D>();
  using SL = BwdSlot<D, TIn>;
  extern __shared__ __align__(16) uint8_t bsm[];
  uint8_t* ring = bsm;                                                    // [kRing][slot]
  float* red_q = reinterpret_cast<float*>(bsm + kRing * SL::kBytes);      // [kBwdCols][RS]
  float* red_k = red_q + kBwdCols * RS;
  float* sp_buf = red_k + kBwdCols * RS;  // [kBwdCols][RS]: the next S_{t-1}, each thread its own entries
  const bool l2 = a.l2norm != 0;

  const int tid = threadIdx.x;
  constexpr int kBlocks = D / kBwdCols;   // column blocks per head
  const int cb = blockIdx.x % kBlocks;
  const int item = blockIdx.x / kBlocks;  // (sequence, head)
  const int lcol = tid / TPC, part = tid % TPC;
  const int col = cb * kBwdCols + lcol;
  // this thread's entries of column col: the 16-byte pieces part, part + TPC, ...,
  // i.e. entries 4 (part + TPC y) + z, y < NP, z < 4 (local index x = 4 y + z)
  auto piece = [&](int y) { return 4 * (part + TPC * y); };
  const int n = item / a.H, h = item - n * a.H;
  const int hq = h / (a.H / a.Hqk);
  int64_t bos, eos;
  if (!seq_bounds(a.cu, n, a.total_T, a.err, &bos, &eos)) return;
  const int64_t len = eos - bos;
  const int nck = (int)((len + a.C - 1) / a.C);
  const size_t SS = (size_t)D * D;
  const size_t state_off = ((size_t)n * a.H + h) * SS + (size_t)col * D;
  float* ck = a.ckpt + ((size_t)h * a.ck_slots + (size_t)(bos / a.C) + n) * SS + (size_t)col * D;
  float* scr = a.scratch + (size_t)item * (size_t)(a.C + 1) * SS + (size_t)col * D;
  float* spb = sp_buf + lcol * RS;

  // The issue cursor: the token of the next position to copy, walked through the
  // visiting order one position at a time (phase 0 forward sweep, 1 recompute of
  // chunk [ct0, ct1), 2 its walk, 3 past the end), and the ring slot it goes to.
  int64_t ct = bos, ct0 = 0, ct1 = 0;
  int cc = 0, cphase = len > 0 ? 0 : 3, islot = 0;
  auto cursor_next = [&]() {
    if (cphase == 0) {
      if (++ct == eos) {
        cc = nck - 1;
        ct0 = bos + (int64_t)cc * a.C;
        ct1 = eos;
        ct = ct0;
        cphase = 1;
      }
    } else if (cphase == 1) {
      if (++ct == ct1) {
        ct = ct1 - 1;
        cphase = 2;
      }
    } else if (cphase == 2) {
      if (ct == ct0) {
        if (--cc < 0) {
          cphase = 3;
        } else {
          ct1 = ct0;
          ct0 -= a.C;
          ct = ct0;
          cphase = 1;
        }
      } else {
        --ct;
      }
    }
    islot = islot + 1 == kRing ? 0 : islot + 1;
  };
  // copies of the cursor's position into its slot, as one cp.async group (empty past
  // the end); the cursor moves on
  auto issue = [&]() {
    if (cphase != 3) {
      const int64_t t = ct;
      uint8_t* sl = ring + islot * SL::kBytes;
      const size_t th = (size_t)t * a.H + h, tq = (size_t)t * a.Hqk + hq;
      const char* kr = static_cast<const char*>(a.k) + tq * SL::kVec;
      const char* qr = static_cast<const char*>(a.q) + tq * SL::kVec;
      constexpr int n16 = SL::kVec / 16;
      for (int c = tid; c < 2 * n16; c += NT) cp_async<16>(sl + 16 * c, c < n16 ? kr + 16 * c : qr + 16 * (c - n16));
      const size_t own = (th * D + (size_t)cb * kBwdCols) * sizeof(TIn);
      const char* vr = static_cast<const char*>(a.v) + own;
      const char* dr = static_cast<const char*>(a.d_o) + own;
      if constexpr (SL::kOwn >= 16) {
        constexpr int m16 = SL::kOwn / 16;
        for (int c = tid; c < 2 * m16; c += NT) {
          const int r = c < m16 ? c : c - m16;
          cp_async<16>(sl + (c < m16 ? SL::kV : SL::kDO) + 16 * r, (c < m16 ? vr : dr) + 16 * r);
        }
      } else {
        if (tid < 2) cp_async<SL::kOwn>(sl + (tid == 0 ? SL::kV : SL::kDO), tid == 0 ? vr : dr);
      }
      if (tid == NT - 1) cp_async<4>(sl + SL::kG, a.g + th);
      if (tid == NT - 2) cp_async<4>(sl + SL::kG + 4, a.beta + th);
    }
    cp_async_commit();
    cursor_next();
  };
  int rslot = 0;  // the slot of the position being computed
  auto take_slot = [&]() -> const uint8_t* {
    const uint8_t* sl = ring + rslot * SL::kBytes;
    rslot = rslot + 1 == kRing ? 0 : rslot + 1;
    return sl;
  };
  // this thread's entries of the slot's k (or q) vector
  auto load_tok = [&](const uint8_t* v, float* out) {
    const TIn* e = reinterpret_cast<const TIn*>(v);
#pragma unroll
    for (int y = 0; y < NP; ++y) {
      const float4 f = ld4_f32(e + piece(y));
      out[4 * y] = f.x; out[4 * y + 1] = f.y; out[4 * y + 2] = f.z; out[4 * y + 3] = f.w;
    }
  };
  // 1 / |x| from this thread's entries, summed over the column's lanes (1 without the
  // normalisation; zero stays zero)
  auto inv_norm = [&](const float* x) {
    if (!l2) return 1.f;
    // four partial sums (entries 0, 1, 2, 3 mod 4: shorter dependency chains), as two
    // packed pairs
    float2 sa = make_float2(0.f, 0.f), sb = sa;
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
      sa = __ffma2_rn(pr(x, i), pr(x, i), sa);
      sb = __ffma2_rn(pr(x, i + 2), pr(x, i + 2), sb);
    }
    float ss = (sa.x + sa.y) + (sb.x + sb.y);
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    return ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
  };
  // one token forward on this thread's entries of column col (as the forward kernel;
  // the update adds c k with c = beta (v_j - alpha (k^ . S_j)) / |k|)
  auto advance = [&](float* st, const uint8_t* sl) {
    const float alpha = expf(*reinterpret_cast<const float*>(sl + SL::kG));
    const float beta = *reinterpret_cast<const float*>(sl + SL::kG + 4);
    const float vj = to_f32(reinterpret_cast<const TIn*>(sl + SL::kV)[lcol]);
    float kv[PER];
    load_tok(sl, kv);
    const float rk = inv_norm(kv);
    float2 ua = make_float2(0.f, 0.f), ub = ua;
#pragma unroll
    for (int x = 0; x < PER; x += 4) {
      ua = __ffma2_rn(pr(kv, x), pr(st, x), ua);
      ub = __ffma2_rn(pr(kv, x + 2), pr(st, x + 2), ub);
    }
    float u = (ua.x + ua.y) + (ub.x + ub.y);
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
    const float c = beta * (vj - alpha * (u * rk)) * rk;
    const float2 a2 = make_float2(alpha, alpha), c2 = make_float2(c, c);
#pragma unroll
    for (int x = 0; x < PER; x += 2) put(st, x, __ffma2_rn(a2, pr(st, x), __fmul2_rn(c2, pr(kv, x))));
  };
  // a state column's entries of this thread from / to memory (p = the column's base)
  auto load_vec = [&](const float* v, float* out) {
#pragma unroll
    for (int y = 0; y < NP; ++y) {
      const float4 f = *reinterpret_cast<const float4*>(v + piece(y));
      out[4 * y] = f.x; out[4 * y + 1] = f.y; out[4 * y + 2] = f.z; out[4 * y + 3] = f.w;
    }
  };
  auto store_state = [&](float* p, const float* st) {
#pragma unroll
    for (int y = 0; y < NP; ++y)
      *reinterpret_cast<float4*>(p + piece(y)) = make_float4(st[4 * y], st[4 * y + 1], st[4 * y + 2], st[4 * y + 3]);
  };
  auto prefetch_state = [&](const float* p) {  // this thread's entries -> sp_buf, asynchronously
#pragma unroll
    for (int y = 0; y < NP; ++y) cp_async<16>(spb + piece(y), p + piece(y));
  };
  // Every step p commits two groups: [the S_{t-1} of the next step when that is a walk
  // step, else none], then [position p + kRing - 1]. At step p, position p's group is
  // followed by 2 (kRing - 2) newer ones, a walk step's S_{t-1} by one. The slot
  // refilled at step p is step p - 1's, which every thread has left at the barrier.
  constexpr int kWaitSweep = 2 * (kRing - 2);
  for (int i = 0; i < kRing - 1; ++i) {
    cp_async_commit();
    issue();
  }

  // 1. forward with a checkpoint at the start of every chunk
  {
    float st[PER];
    if (a.init) {
      load_vec(a.init + state_off, st);
    } else {
#pragma unroll
      for (int x = 0; x < PER; ++x) st[x] = 0.f;
    }
    float* ckp = ck;  // the next checkpoint
    int in_chunk = 0;
    for (int64_t t = bos; t < eos; ++t) {
      cp_async_wait<kWaitSweep>();
      __syncthreads();
      if (in_chunk == 0) {
        store_state(ckp, st);
        ckp += SS;
      }
      in_chunk = in_chunk + 1 == a.C ? 0 : in_chunk + 1;
      cp_async_commit();
      issue();
      advance(st, take_slot());
    }
  }

  // 2. chunks last to first
  float Dm[PER];  // dL/dS_t, this thread's entries
  if (a.d_fin) {
    load_vec(a.d_fin + state_off, Dm);
  } else {
#pragma unroll
    for (int x = 0; x < PER; ++x) Dm[x] = 0.f;
  }
  for (int c = nck - 1; c >= 0; --c) {
    const int64_t t0 = bos + (int64_t)c * a.C;
    const int64_t t1 = (t0 + a.C < eos) ? t0 + a.C : eos;
    float sc[PER];  // S_t of the token being walked
    // recompute: scratch slot x = the state before token t0 + x
    load_vec(ck + (size_t)c * SS, sc);
    for (int64_t t = t0; t < t1; ++t) {
      cp_async_wait<kWaitSweep>();
      __syncthreads();
      store_state(scr + (size_t)(t - t0) * SS, sc);
      if (t + 1 == t1) prefetch_state(scr + (size_t)(t - t0) * SS);  // the first walk step's S_{t-1}
      cp_async_commit();
      issue();
      advance(sc, take_slot());
    }
    // walk: sc = S_t, its S_{t-1} waits in sp_buf
    for (int64_t t = t1 - 1; t >= t0; --t) {
      cp_async_wait<1>();
      __syncthreads();
      const uint8_t* sl = take_slot();
      const float vj = to_f32(reinterpret_cast<const TIn*>(sl + SL::kV)[lcol]);
      const float dOj = to_f32(reinterpret_cast<const TIn*>(sl + SL::kDO)[lcol]);
      const float alpha = expf(*reinterpret_cast<const float*>(sl + SL::kG));
      const float beta = *reinterpret_cast<const float*>(sl + SL::kG + 4);
      const size_t th = (size_t)t * a.H + h, tq = (size_t)t * a.Hqk + hq;
      // column j's terms of dq (S_t dO) first: S_t is not needed after them
      float* rowq = red_q + lcol * RS;
      float* rowk = red_k + lcol * RS;
      const float2 do2 = make_float2(dOj, dOj);
#pragma unroll
      for (int y = 0; y < NP; ++y) {
        const float2 lo = __fmul2_rn(pr(sc, 4 * y), do2), hi = __fmul2_rn(pr(sc, 4 * y + 2), do2);
        *reinterpret_cast<float4*>(rowq + piece(y)) = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      float sp[PER];  // S_{t-1}
      load_vec(spb, sp);
      if (t - 1 >= t0) prefetch_state(scr + (size_t)(t - 1 - t0) * SS);
      cp_async_commit();
      issue();
      float kv[PER];
      load_tok(sl, kv);
      const float rk = inv_norm(kv);
      // D += scale q dO^T
      float rq;
      {
        float qv[PER];
        load_tok(sl + SL::kQ, qv);
        rq = inv_norm(qv);
        const float sr = a.scale * rq;
        const float2 sr2 = make_float2(sr, sr);
#pragma unroll
        for (int x = 0; x < PER; x += 2) put(Dm, x, __ffma2_rn(__fmul2_rn(sr2, pr(qv, x)), do2, pr(Dm, x)));
      }
      // u = S~^T k (S~ = alpha S_{t-1}), w = D^T k, column j
      float2 pua = make_float2(0.f, 0.f), pub = pua, pwa = pua, pwb = pua;
#pragma unroll
      for (int x = 0; x < PER; x += 4) {
        pua = __ffma2_rn(pr(kv, x), pr(sp, x), pua);
        pub = __ffma2_rn(pr(kv, x + 2), pr(sp, x + 2), pub);
        pwa = __ffma2_rn(pr(kv, x), pr(Dm, x), pwa);
        pwb = __ffma2_rn(pr(kv, x + 2), pr(Dm, x + 2), pwb);
      }
      float pu = (pua.x + pua.y) + (pub.x + pub.y), pw = (pwa.x + pwa.y) + (pwb.x + pwb.y);
#pragma unroll
      for (int off = 1; off < TPC; off <<= 1) {
        pu += __shfl_xor_sync(0xffffffffu, pu, off);
        pw += __shfl_xor_sync(0xffffffffu, pw, off);
      }
      const float u = alpha * pu * rk, w = pw * rk, vmu = vj - u;
      // column j's terms of dk (D (v - u) - S~ w) and of dg
      const float2 al2 = make_float2(alpha, alpha), vmu2 = make_float2(vmu, vmu), nw2 = make_float2(-w, -w);
      float2 ga = make_float2(0.f, 0.f), gb = ga;
#pragma unroll
      for (int y = 0; y < NP; ++y) {
        const int x = 4 * y;
        const float2 s0 = __fmul2_rn(al2, pr(sp, x)), s1 = __fmul2_rn(al2, pr(sp, x + 2));  // S~ entries
        const float2 k0 = __ffma2_rn(pr(Dm, x), vmu2, __fmul2_rn(s0, nw2));
        const float2 k1 = __ffma2_rn(pr(Dm, x + 2), vmu2, __fmul2_rn(s1, nw2));
        ga = __ffma2_rn(pr(Dm, x), s0, ga);
        gb = __ffma2_rn(pr(Dm, x + 2), s1, gb);
        *reinterpret_cast<float4*>(rowk + piece(y)) = make_float4(k0.x, k0.y, k1.x, k1.y);
      }
      float sdg = (ga.x + ga.y) + (gb.x + gb.y);
      float sdb = 0.f;
      if (part == 0) {
        sdg -= beta * u * w;
        sdb = w * vmu;
        a.dv[th * D + col] = beta * w;
      }
      // dL/dS_{t-1}; S_{t-1} becomes the next token's S_t
      const float bw = beta * w * rk;
      const float2 nbw2 = make_float2(-bw, -bw);
#pragma unroll
      for (int x = 0; x < PER; x += 2) put(Dm, x, __fmul2_rn(al2, __ffma2_rn(nbw2, pr(kv, x), pr(Dm, x))));
#pragma unroll
      for (int x = 0; x < PER; ++x) sc[x] = sp[x];
      // dg and dbeta over the CTA's columns (every lane ends with the sums)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sdg += __shfl_xor_sync(0xffffffffu, sdg, off);
        sdb += __shfl_xor_sync(0xffffffffu, sdb, off);
      }
      __syncthreads();  // the column partials of dq and dk are written
      {  // entries i0 .. i0 + EPT - 1 of dq and of dk over this CTA's columns
        const int i0 = EPT * tid;
        float gq[EPT], gk[EPT];  // this CTA's part of dq^, dk^
#pragma unroll
        for (int e = 0; e < EPT; ++e) gq[e] = gk[e] = 0.f;
#pragma unroll 8
        for (int j = 0; j < kBwdCols; ++j) {
          float xq[EPT], xk[EPT];
          ld_vec<EPT>(red_q + j * RS + i0, xq);
          ld_vec<EPT>(red_k + j * RS + i0, xk);
#pragma unroll
          for (int e = 0; e < EPT; ++e) {
            gq[e] += xq[e];
            gk[e] += xk[e];
          }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          gq[e] *= a.scale;
          gk[e] *= beta;
        }
        if (l2) {  // through the normalisation: (g - x^ (x^ . g)) / |x|
          const TIn* ke = reinterpret_cast<const TIn*>(sl);
          const TIn* qe = reinterpret_cast<const TIn*>(sl + SL::kQ);
          float pk = 0.f, pq = 0.f;
#pragma unroll
          for (int e = 0; e < EPT; ++e) {
            pk = fmaf(to_f32(ke[i0 + e]) * rk, gk[e], pk);
            pq = fmaf(to_f32(qe[i0 + e]) * rq, gq[e], pq);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            pk += __shfl_xor_sync(0xffffffffu, pk, off);
            pq += __shfl_xor_sync(0xffffffffu, pq, off);
          }
#pragma unroll
          for (int e = 0; e < EPT; ++e) {
            gk[e] = (gk[e] - to_f32(ke[i0 + e]) * rk * pk) * rk;
            gq[e] = (gq[e] - to_f32(qe[i0 + e]) * rq * pq) * rq;
          }
        }
        atomic_add_vec<EPT>(a.dq + tq * D + i0, gq);
        atomic_add_vec<EPT>(a.dk + tq * D + i0, gk);
      }
      if (tid == 0) {
        atomicAdd(a.dg + th, sdg);
        atomicAdd(a.dbeta + th, sdb);
      }
    }
  }
  if (a.d_init) store_state(a.d_init + state_off, Dm);
}

template <int D, typename TIn>
gdn_status_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  auto kernel = gdn_prefill_backward_kernel<D, TIn>;
  constexpr size_t smem = bwd_smem_bytes<D, TIn>();
  static PerDeviceOnce once;  // the shared-memory opt-in applies to the current device only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(GDN_ERR_CUDA, std::string("prefill backward: cudaGetDevice: ") + cudaGetErrorString(e));
  if (!run_once_per_device(once, dev, [&](int, int*) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        return e == cudaSuccess;
      }))
    return fail(e != cudaSuccess ? GDN_ERR_CUDA : GDN_ERR_UNSUPPORTED,
                std::string("prefill backward: setup: ") + (e != cudaSuccess ? cudaGetErrorString(e) : "device index too large"));
  kernel<<<(unsigned)((long long)a.N * a.H * (D / bwd_cols<D>())), bwd_threads<D>(), smem, stream>>>(a);
  return check_launch("gdn_chunk_prefill_backward");
}

}  // namespace
}  // namespace gdn

using gdn::fail;

namespace {

gdn_status_t bwd_check_shape(int N, int64_t total_T, int H, int dk, int dv, int chunk) {
  if (N < 0 || total_T < 0 || H < 1 || chunk < 1)
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: need N >= 0, total_T >= 0, H >= 1, chunk >= 1");
  if (dk != dv || (dk != 32 && dk != 64 && dk != 128))
    return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_backward: dk == dv in {32, 64, 128}");
  if (chunk > 4096) return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_backward: chunk <= 4096");
  if ((long long)N * H * (dk * dk / (32 * gdn::kBwdPer)) >= (1LL << 31))  // column blocks per head: dk / cols
    return fail(GDN_ERR_UNSUPPORTED, "gdn_chunk_prefill_backward: N * H too large");
  return gdn::ok();
}

bool ptr_ok(const void* p) { return p != nullptr && gdn::aligned16(p); }

}  // namespace

extern "C" gdn_status_t gdn_chunk_prefill_backward_workspace_size(int N, int64_t total_T, int H, int dk, int dv,
                                                                  int chunk, size_t* bytes) {
  if (!bytes) return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward_workspace_size: bytes is NULL");
  const gdn_status_t st = bwd_check_shape(N, total_T, H, dk, dv, chunk);
  if (st != GDN_OK) return st;
  *bytes = gdn::bwd_layout(N, total_T, H, dk, chunk).bytes;
  return gdn::ok();
}

extern "C" gdn_status_t gdn_chunk_prefill_backward(
    const void* q, const void* k, const void* v, const float* g, const float* beta, const int32_t* cu_seqlens, int N,
    int64_t total_T, const float* initial_state, const void* d_o, const float* d_final_state, float* d_q, float* d_k,
    float* d_v, float* d_g, float* d_beta, float* d_initial_state, int H, int H_qk, int dk, int dv, int chunk,
    float scale, uint32_t flags, gdn_dtype_t in_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  gdn_status_t st = bwd_check_shape(N, total_T, H, dk, dv, chunk);
  if (st != GDN_OK) return st;
  if (H_qk < 1 || H % H_qk != 0)
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: H must be a positive multiple of H_qk");
  if ((flags & ~(uint32_t)GDN_QK_L2NORM) != 0) return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: unknown flags");
  if (!(in_dtype == GDN_BF16 || in_dtype == GDN_F32))
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: unknown dtype");
  if (N == 0) return gdn::ok();
  if (cu_seqlens == nullptr) return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: cu_seqlens is NULL");
  if (total_T > 0 && (!ptr_ok(q) || !ptr_ok(k) || !ptr_ok(v) || !ptr_ok(d_o) || g == nullptr || beta == nullptr ||
                      !ptr_ok(d_q) || !ptr_ok(d_k) || d_v == nullptr || d_g == nullptr || d_beta == nullptr))
    return fail(GDN_ERR_INVALID_ARG,
                "gdn_chunk_prefill_backward: q, k, v, d_o, d_q, d_k must be non-NULL and 16-byte aligned; "
                "g, beta, d_v, d_g, d_beta non-NULL");
  if ((initial_state && !ptr_ok(initial_state)) || (d_final_state && !ptr_ok(d_final_state)) ||
      (d_initial_state && !ptr_ok(d_initial_state)))
    return fail(GDN_ERR_INVALID_ARG, "gdn_chunk_prefill_backward: state pointers must be 16-byte aligned");
  const gdn::BwdLayout L = gdn::bwd_layout(N, total_T, H, dk, chunk);
  if (workspace == nullptr || workspace_bytes < L.bytes || !gdn::aligned16(workspace))
    return fail(GDN_ERR_WORKSPACE, "gdn_chunk_prefill_backward: workspace missing, misaligned or smaller than "
                                   "gdn_chunk_prefill_backward_workspace_size");
  unsigned int* err = nullptr;
  st = gdn::device_error_word(&err);
  if (st != GDN_OK) return st;
  cudaStream_t s = gdn::as_stream(stream);
  if (total_T > 0) {
    const size_t qk_bytes = (size_t)total_T * H_qk * dk * sizeof(float);
    const size_t gb_bytes = (size_t)total_T * H * sizeof(float);
    cudaError_t e = cudaMemsetAsync(d_q, 0, qk_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_k, 0, qk_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_g, 0, gb_bytes, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_beta, 0, gb_bytes, s);
    if (e != cudaSuccess)
      return fail(GDN_ERR_CUDA, std::string("gdn_chunk_prefill_backward: clearing the outputs: ") +
                                    cudaGetErrorString(e));
  }
  gdn::BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.d_o = d_o; a.g = g; a.beta = beta; a.cu = cu_seqlens;
  a.init = initial_state; a.d_fin = d_final_state;
  a.dq = d_q; a.dk = d_k; a.dv = d_v; a.dg = d_g; a.dbeta = d_beta; a.d_init = d_initial_state;
  a.ckpt = static_cast<float*>(workspace);
  a.scratch = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + L.scratch_off);
  a.ck_slots = L.ck_slots;
  a.total_T = total_T; a.N = N; a.H = H; a.Hqk = H_qk; a.C = chunk; a.scale = scale;
  a.l2norm = (flags & GDN_QK_L2NORM) != 0; a.err = err;
  const bool bf = in_dtype == GDN_BF16;
  switch (dk) {
    case 32: return bf ? gdn::launch_bwd<32, __nv_bfloat16>(a, s) : gdn::launch_bwd<32, float>(a, s);
    case 64: return bf ? gdn::launch_bwd<64, __nv_bfloat16>(a, s) : gdn::launch_bwd<64, float>(a, s);
    default: return bf ? gdn::launch_bwd<128, __nv_bfloat16>(a, s) : gdn::launch_bwd<128, float>(a, s);
  }
}
