// Decode step of the gated delta rule / gated delta product over a slot-indexed
// fp32 state pool, updated in place.
//
// Design (B200). The step is HBM-bound: every (slot, head) state of dk x dv fp32
// is read once and written once. Following the T=1 split-V variant of the
// FlashInfer PR #7156 page ("Cake GDP kernel: shared-memory reduction and direct
// register loads", sections 1-2), the state is streamed straight from HBM into
// registers with 16-byte vector loads (no shared-memory staging), and the value
// dimension is split across CTAs so that small batches still fill the 148 SMs.
//
// Mapping. State rows are K-last rows S^T[j, :] (one value column j of S, dk
// contiguous fp32). A group of LPR lanes shares one row: lane `sub` holds the
// float4 chunks sub, sub+LPR, sub+2*LPR, ... so that each warp-wide load covers
// LPR*16 contiguous bytes of 32/LPR rows. Each thread owns R rows.
//
// Arithmetic. Per row j the step is M = T*n_h sub-steps (gate on the first
// sub-step of each token, then a Householder update) and T outputs. Writing the
// row after sub-step m as s_m = Gamma_m s_0 + sum_{l<=m} c_l k_l, every quantity
// the recurrence needs is a dot product of the OLD row s_0 with a key or a query
// plus per-head Gram entries:
//     u_m   = k_m . (gated s) = Gamma_m (k_m . s_0) + sum_{l<m} c_l (k_m . k_l)
//     c_m   = beta_m (v_m[j] - u_m)
//     o_t   = scale (Gamma (q_t . s_0) + sum_{l<=m_t} c_l (q_t . k_l))
//     s_new = Gamma_M s_0 + sum_m c_m k_m
// so one pass of FMAs over the resident row, one shuffle reduction of all M + T
// dot products, a scalar recurrence of O(M^2) per row, and one pass of FMAs for
// the update. For T = n_h = 1 this is u = k.s, c = beta (v - alpha u),
// s' = alpha s + c k, o = scale (alpha q.s + c q.k).
#include "common.cuh"

namespace gdn {
namespace {

constexpr int kDecodeThreads = 128;

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
  int B, H, dv, num_slots;
  int row_blocks;  // CTAs per (b, h)
  float scale;
};

template <typename TIn>
__device__ __forceinline__ float ld_in(const TIn* p) { return to_f32(*p); }

// DK: head key dim; LPR: lanes per row; R: rows per thread; TT tokens, NH keys per token.
template <int DK, int LPR, int R, int TT, int NH, typename TIn, typename TOut>
__global__ void __launch_bounds__(kDecodeThreads, (TT * NH + TT > 2) ? 3 : 4)
gdn_decode_kernel(const DecodeParams p) {
  constexpr int M = TT * NH;            // sub-steps
  constexpr int NV = M + TT;            // vectors dotted with the old row: keys then queries
  constexpr int CPL = DK / (4 * LPR);   // float4 chunks per lane per row
  constexpr int SLOTS = 32 / LPR;       // row slots per warp
  constexpr int WARPS = kDecodeThreads / 32;
  constexpr int RPC = WARPS * SLOTS * R;  // rows per CTA
  static_assert(CPL >= 1 && DK % (4 * LPR) == 0, "bad DK/LPR");

  __shared__ __align__(16) float s_vec[NV][DK];   // k_1..k_M, q_1..q_T (fp32)
  __shared__ float s_vals[M][RPC];                // v_m[j] for this CTA's rows
  __shared__ float s_gram[M][M];                  // k_m . k_l
  __shared__ float s_qk[TT][M];                   // q_t . k_l
  __shared__ float s_beta[M];
  __shared__ float s_alpha[TT];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int sub = lane % LPR;
  const int slot_in_warp = lane / LPR;

  const int bh = blockIdx.x / p.row_blocks;
  const int rb = blockIdx.x - bh * p.row_blocks;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int row0 = rb * RPC;

  const TIn* qp = static_cast<const TIn*>(p.q);
  const TIn* kp = static_cast<const TIn*>(p.k);
  const TIn* vp = static_cast<const TIn*>(p.v);
  TOut* op = static_cast<TOut*>(p.o);

  const int slot = __ldg(p.slot_ids + b);
  if (slot < 0 || slot >= p.num_slots) {
    if (slot >= p.num_slots && tid == 0 && rb == 0) raise_device_error(p.err, GDN_DEVERR_SLOT_OUT_OF_RANGE);
    for (int i = tid; i < TT * RPC; i += kDecodeThreads) {
      const int t = i / RPC, j = row0 + (i - t * RPC);
      if (j < p.dv) store_out(op + (((size_t)b * TT + t) * p.H + h) * p.dv + j, 0.f);
    }
    return;
  }

  // 1) Stream this thread's state rows HBM -> registers first, so the loads are
  //    in flight while the per-head vectors are staged and the Gram is built.
  float* state = p.pool + ((size_t)slot * p.H + h) * (size_t)p.dv * DK;
  int rows[R];
  bool live[R];  // rows past dv (small dv, last row block) are computed on zeros, never stored
  float4 s[R][CPL];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    rows[r] = row0 + (warp * R + r) * SLOTS + slot_in_warp;
    live[r] = rows[r] < p.dv;
    const float4* src = reinterpret_cast<const float4*>(state + (size_t)rows[r] * DK);
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      s[r][c] = live[r] ? __ldcs(src + c * LPR + sub) : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // 2) Stage keys and queries of this (b, h) as fp32, the values of this CTA's
  //    rows, beta and the gates.
  {
    constexpr int kChunks = NV * DK / 8;
    for (int i = tid; i < kChunks; i += kDecodeThreads) {
      const int vec = i / (DK / 8);
      const int e = (i - vec * (DK / 8)) * 8;
      const TIn* src;
      if (vec < M) {
        const int t = vec / NH, m = vec - t * NH;
        src = kp + ((((size_t)b * TT + t) * p.H + h) * NH + m) * DK + e;
      } else {
        const int t = vec - M;
        src = qp + (((size_t)b * TT + t) * p.H + h) * DK + e;
      }
      float tmp[8];
      load8_f32(src, tmp);
#pragma unroll
      for (int x = 0; x < 8; ++x) s_vec[vec][e + x] = tmp[x];
    }
    for (int i = tid; i < M * RPC; i += kDecodeThreads) {
      const int m = i / RPC, jj = i - m * RPC;
      const int t = m / NH, mm = m - t * NH;
      s_vals[m][jj] = (row0 + jj < p.dv)
          ? ld_in(vp + ((((size_t)b * TT + t) * p.H + h) * NH + mm) * p.dv + row0 + jj)
          : 0.f;
    }
    if (tid < M) {
      const int t = tid / NH, mm = tid - t * NH;
      s_beta[tid] = __ldg(p.beta + (((size_t)b * TT + t) * p.H + h) * NH + mm);
    }
    if (tid >= 32 && tid < 32 + TT) {
      const int t = tid - 32;
      s_alpha[t] = expf(__ldg(p.g + ((size_t)b * TT + t) * p.H + h));
    }
  }
  __syncthreads();

  // 3) Per-head Gram entries k_m.k_l (l < m) and q_t.k_l, one warp per pair.
  {
    constexpr int kPairsKK = M * (M - 1) / 2;
    constexpr int kPairs = kPairsKK + TT * M;
    for (int pair = warp; pair < kPairs; pair += WARPS) {
      int a, c;
      if (pair < kPairsKK) {
        a = 1;
        int rem = pair;
        while (rem >= a) { rem -= a; ++a; }
        c = rem;  // (a, c) with c < a
      } else {
        const int x = pair - kPairsKK;
        a = M + x / M;  // query index into s_vec
        c = x - (x / M) * M;
      }
      float acc = 0.f;
      for (int e = lane; e < DK; e += 32) acc = fmaf(s_vec[a][e], s_vec[c][e], acc);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) {
        if (pair < kPairsKK) s_gram[a][c] = acc;
        else s_qk[a - M][c] = acc;
      }
    }
  }
  __syncthreads();

  // 4) Dot products of the old rows with every key and query.
  float dots[NV][R];
#pragma unroll
  for (int vec = 0; vec < NV; ++vec)
#pragma unroll
    for (int r = 0; r < R; ++r) dots[vec][r] = 0.f;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
#pragma unroll
    for (int vec = 0; vec < NV; ++vec) {
      const float4 w = *reinterpret_cast<const float4*>(&s_vec[vec][(c * LPR + sub) * 4]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float a = dots[vec][r];
        a = fmaf(s[r][c].x, w.x, a);
        a = fmaf(s[r][c].y, w.y, a);
        a = fmaf(s[r][c].z, w.z, a);
        a = fmaf(s[r][c].w, w.w, a);
        dots[vec][r] = a;
      }
    }
  }
#pragma unroll
  for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
    for (int vec = 0; vec < NV; ++vec)
#pragma unroll
      for (int r = 0; r < R; ++r) dots[vec][r] += __shfl_xor_sync(0xffffffffu, dots[vec][r], off);

  // 5) Scalar recurrence per row (every lane of the row group, redundantly).
  float coef[R][M];
  float gam[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int jj = rows[r] - row0;
    float G = 1.f;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float a = s_alpha[t];
      G *= a;
#pragma unroll
      for (int l = 0; l < t * NH; ++l) coef[r][l] *= a;
#pragma unroll
      for (int x = 0; x < NH; ++x) {
        const int m = t * NH + x;
        float u = G * dots[m][r];
#pragma unroll
        for (int l = 0; l < m; ++l) u = fmaf(coef[r][l], s_gram[m][l], u);
        coef[r][m] = s_beta[m] * (s_vals[m][jj] - u);
      }
      float out = G * dots[M + t][r];
#pragma unroll
      for (int l = 0; l < (t + 1) * NH; ++l) out = fmaf(coef[r][l], s_qk[t][l], out);
      if (live[r] && sub == (t % LPR))
        store_out(op + (((size_t)b * TT + t) * p.H + h) * p.dv + rows[r], p.scale * out);
    }
    gam[r] = G;
  }

  // 6) s_new = Gamma s_0 + sum_m c_m k_m, written back in place.
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      s[r][c].x *= gam[r];
      s[r][c].y *= gam[r];
      s[r][c].z *= gam[r];
      s[r][c].w *= gam[r];
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float4 w = *reinterpret_cast<const float4*>(&s_vec[m][(c * LPR + sub) * 4]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        s[r][c].x = fmaf(coef[r][m], w.x, s[r][c].x);
        s[r][c].y = fmaf(coef[r][m], w.y, s[r][c].y);
        s[r][c].z = fmaf(coef[r][m], w.z, s[r][c].z);
        s[r][c].w = fmaf(coef[r][m], w.w, s[r][c].w);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (!live[r]) continue;
    float4* dst = reinterpret_cast<float4*>(state + (size_t)rows[r] * DK);
#pragma unroll
    for (int c = 0; c < CPL; ++c) __stcs(dst + c * LPR + sub, s[r][c]);
  }
}

template <int DK, int TT, int NH, typename TIn, typename TOut>
gdn_status_t launch_typed(DecodeParams p, cudaStream_t stream) {
  constexpr int LPR = 4;
  constexpr int R = (TT * NH + TT > 2) ? 1 : 2;  // 32 or 64 state floats per thread
  constexpr int RPC = (kDecodeThreads / 32) * (32 / LPR) * R;
  p.row_blocks = (p.dv + RPC - 1) / RPC;
  const long long grid = (long long)p.B * p.H * p.row_blocks;
  if (grid == 0) return ok();
  gdn_decode_kernel<DK, LPR, R, TT, NH, TIn, TOut><<<(unsigned)grid, kDecodeThreads, 0, stream>>>(p);
  return check_launch("gdn_decode");
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
gdn_status_t launch_steps(DecodeParams p, int T, int nh, gdn_dtype_t in, gdn_dtype_t out,
                          cudaStream_t s) {
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

gdn_status_t decode_launch(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, float* pool, int num_slots, const int32_t* slot_ids,
                           void* o, int B, int T, int H, int dk, int dv, int nh, float scale,
                           gdn_dtype_t in, gdn_dtype_t out, unsigned int* err, cudaStream_t stream) {
  DecodeParams p{q, k, v, g, beta, pool, slot_ids, o, err, B, H, dv, num_slots, 0, scale};
  switch (dk) {
    case 32: return launch_steps<32>(p, T, nh, in, out, stream);
    case 64: return launch_steps<64>(p, T, nh, in, out, stream);
    case 128: return launch_steps<128>(p, T, nh, in, out, stream);
    default: return fail(GDN_ERR_UNSUPPORTED, "gdn_decode: dk must be 32, 64 or 128");
  }
}

}  // namespace gdn
