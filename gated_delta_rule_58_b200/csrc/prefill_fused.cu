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
// Every product is written with the value dimension (dv = 128) or the key
// dimension on the MMA's M side, so all MMAs are M = 128 (cta_group::1) with
// fp16 operands in 128-byte-swizzled shared memory and fp32 accumulators in
// TMEM. fp16 (10-bit mantissa) keeps the result within the 2e-3 tolerance where
// bf16 operands do not; bf16 inputs are converted on load. The decay factors
// exp(G_i - G_j) are taken on differences of cumulative gates (the cumulative
// decay idiom of the FlashInfer PR #6291 page, section 2), never as a ratio.
//
// The local-state / transfer view of the same chunk step (S_{c+1} = M_c S_c +
// H_c, FlashInfer PR #3866 page, section 2) is what this kernel evaluates
// without materialising M_c or H_c: H_c = K~^T U~ and -K~^T W S_c are the two
// halves of the accumulate into the state.
#include "prefill.cuh"
#include "tcgen05.cuh"

namespace gdn {
namespace {

constexpr int C = 64;      // chunk
constexpr int D = 128;     // dk = dv
constexpr int kThreads = 128;
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded MMA waits: 2 s

// Shared memory map (bytes from a 1024-aligned base). fp16 operand tiles use the
// SWIZZLE_128B canonical layouts (see tcgen05.cuh).
constexpr uint32_t OFF_KQ = 0;          // [2 dk halves][128 rows: K tokens 0-63, Q tokens 64-127][64] fp16
constexpr uint32_t KQ_HALF = 16384;
constexpr uint32_t OFF_V = 32768;       // [2 dv halves][64 tokens][64] fp16
constexpr uint32_t V_HALF = 8192;
constexpr uint32_t OFF_S16 = 49152;     // S^T [2 dk halves][128 dv rows][64] fp16 (K-major A)
constexpr uint32_t S16_HALF = 16384;
constexpr uint32_t OFF_W16 = 81920;     // W^T [128 dk rows][64 tokens] fp16 (MN-major B)
constexpr uint32_t OFF_U16 = 98304;     // U^T [128 dv rows][64 tokens] fp16 (K-major A)
constexpr uint32_t OFF_UDD = 114688;    // U^T diag(exp(G_C - G_i)), same layout
constexpr uint32_t OFF_TP = 131072;     // T diag(beta gamma)  [64 rows][64] fp16 (K-major B)
constexpr uint32_t OFF_TPP = 139264;    // T diag(beta)        [64 rows][64] fp16
constexpr uint32_t OFF_P16 = 147456;    // P                   [64 rows][64] fp16
constexpr int LDA = C + 1;              // padded fp32 row stride
constexpr uint32_t OFF_A = 155648;      // A fp32 [64][65]
constexpr uint32_t OFF_T = OFF_A + C * LDA * 4;   // T fp32 [64][65]
constexpr uint32_t OFF_X = OFF_T + C * LDA * 4;   // 3 x 16x16 fp32 scratch
constexpr uint32_t OFF_VEC = OFF_X + 3 * 256 * 4; // G, gamma, dd, beta, beta*gamma (5 x 64 fp32)
constexpr uint32_t OFF_BAR = OFF_VEC + 5 * C * 4; // mbarrier, TMEM base, abort flag
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment

// TMEM columns (fp32 accumulators, 128 lanes)
constexpr uint32_t COL_S = 0;     // S^T: lane = dv row, 128 columns = dk
constexpr uint32_t COL_D1 = 128;  // [K;Q] K^T: lanes 0-63 K K^T, 64-127 Q K^T
constexpr uint32_t COL_W = 192;   // W^T: lane = dk, column = token
constexpr uint32_t COL_U = 256;   // U~^T then U^T: lane = dv, column = token
constexpr uint32_t COL_O1 = 320;  // S^T Q^T
constexpr uint32_t COL_O2 = 384;  // U^T P^T
constexpr uint32_t TMEM_COLS = 512;

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Writes 8 fp32 values as fp16 into 16-byte chunk `chunk` of row `row` of a
// swizzled tile at byte address `tile` (8-row groups 1024 bytes apart).
__device__ __forceinline__ void st_sw128_chunk(uint8_t* tile, uint32_t row, uint32_t chunk, const float* v) {
  uint4 u;
  u.x = pack_half2(v[0], v[1]);
  u.y = pack_half2(v[2], v[3]);
  u.z = pack_half2(v[4], v[5]);
  u.w = pack_half2(v[6], v[7]);
  *reinterpret_cast<uint4*>(tile + tc::sw128_offset(row, chunk, 1024)) = u;
}

struct Smem {
  uint8_t* base;
  __device__ float* A() const { return reinterpret_cast<float*>(base + OFF_A); }
  __device__ float* T() const { return reinterpret_cast<float*>(base + OFF_T); }
  __device__ float* X() const { return reinterpret_cast<float*>(base + OFF_X); }
  __device__ float* G() const { return reinterpret_cast<float*>(base + OFF_VEC); }
  __device__ float* gam() const { return G() + C; }
  __device__ float* dd() const { return G() + 2 * C; }
  __device__ float* beta() const { return G() + 3 * C; }
  __device__ float* bg() const { return G() + 4 * C; }
  __device__ uint64_t* bar() const { return reinterpret_cast<uint64_t*>(base + OFF_BAR); }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + OFF_BAR + 8); }
  __device__ int* abort_flag() const { return reinterpret_cast<int*>(base + OFF_BAR + 12); }
  __device__ uint32_t u32(uint32_t off) const { return tc::smem_u32(base + off); }
};

// Thread 0 waits for the committed MMAs; everyone then learns whether they finished.
__device__ __forceinline__ bool wait_mma(const Smem& sm, uint32_t& phase, unsigned int* err) {
  if (threadIdx.x == 0) {
    if (!tc::mbar_wait(sm.bar(), phase, kWaitNs)) {
      *sm.abort_flag() = 1;
      raise_device_error(err, GDN_DEVERR_TIMEOUT);
    }
  }
  phase ^= 1u;
  __syncthreads();
  tc::fence_after_sync();
  return *sm.abort_flag() == 0;
}

// Barrier after threads wrote operand tiles (generic proxy) and/or touched TMEM,
// before the MMA issuer reads them.
__device__ __forceinline__ void publish_to_mma() {
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
}

template <typename TIn>
__device__ __forceinline__ void load_chunk(const Smem& sm, const PrefillShape& s, const PrefillArgs& a, int h,
                                           int64_t t0, int Lc) {
  const int tid = threadIdx.x;
  if (tid < C) {
    float gv = 0.f, bv = 0.f;
    if (tid < Lc) {
      const size_t th = (size_t)(t0 + tid) * s.H + h;
      gv = __ldg(a.g + th);
      bv = __ldg(a.beta + th);
    }
    sm.G()[tid] = gv;
    sm.beta()[tid] = bv;
  }
  const TIn* srcs[3] = {static_cast<const TIn*>(a.k), static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.v)};
#pragma unroll 4
  for (int i = tid; i < 3 * C * 16; i += kThreads) {
    const int mat = i / (C * 16);
    const int rem = i - mat * (C * 16);
    const int row = rem >> 4;
    const int ch = rem & 15;  // 8-element chunk of the 128-wide row
    float v8[8];
    if (row < Lc) {
      load8_f32(srcs[mat] + ((size_t)(t0 + row) * s.H + h) * D + ch * 8, v8);
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) v8[x] = 0.f;
    }
    uint8_t* tile;
    uint32_t r;
    if (mat == 2) {
      tile = sm.base + OFF_V + (ch >> 3) * V_HALF;
      r = row;
    } else {
      tile = sm.base + OFF_KQ + (ch >> 3) * KQ_HALF;
      r = row + (mat == 1 ? C : 0);
    }
    st_sw128_chunk(tile, r, ch & 7, v8);
  }
  __syncthreads();
  if (tid < 32) {
    // inclusive cumulative sum of the chunk's log gates (two per lane)
    const float x0 = sm.G()[2 * tid], x1 = sm.G()[2 * tid + 1];
    float pre = x0 + x1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, pre, off);
      if (tid >= off) pre += y;
    }
    __syncwarp();
    sm.G()[2 * tid] = pre - x1;
    sm.G()[2 * tid + 1] = pre;
    __syncwarp();
    const float Gc = __shfl_sync(0xffffffffu, pre, 31);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = 2 * tid + e;
      const float Gi = e ? pre : pre - x1;
      const float gm = __expf(Gi);
      sm.gam()[i] = gm;
      sm.dd()[i] = __expf(Gc - Gi);
      sm.bg()[i] = sm.beta()[i] * gm;
    }
  }
  publish_to_mma();
}

// T = (I + A)^{-1} for the strictly lower 64x64 A in shared memory (fp32):
// 16x16 diagonal blocks by forward substitution, then the off-diagonal blocks
// by diagonals: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj.
__device__ __forceinline__ void solve_unit_lower(const Smem& sm) {
  const int tid = threadIdx.x;
  float* A = sm.A();
  float* T = sm.T();
  float* X = sm.X();
  if (tid < C) {
    const int b = tid >> 4, c = tid & 15;
    float t[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < r; ++k) acc = fmaf(A[(16 * b + r) * LDA + 16 * b + k], t[k], acc);
      t[r] = (r < c) ? 0.f : ((r == c) ? 1.f : -acc);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) T[(16 * b + r) * LDA + 16 * b + c] = t[r];
  }
  __syncthreads();
  for (int d = 1; d < 4; ++d) {
    const int nb = 4 - d;
    for (int o = threadIdx.x; o < nb * 256; o += kThreads) {
      const int bi = o >> 8, i = d + bi, j = i - d, r = (o >> 4) & 15, cc = o & 15;
      float acc = 0.f;
      for (int k = j; k < i; ++k) {
#pragma unroll
        for (int m = 0; m < 16; ++m)
          acc = fmaf(A[(16 * i + r) * LDA + 16 * k + m], T[(16 * k + m) * LDA + 16 * j + cc], acc);
      }
      X[bi * 256 + r * 16 + cc] = acc;
    }
    __syncthreads();
    for (int o = threadIdx.x; o < nb * 256; o += kThreads) {
      const int bi = o >> 8, i = d + bi, j = i - d, r = (o >> 4) & 15, cc = o & 15;
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) acc = fmaf(T[(16 * i + r) * LDA + 16 * i + m], X[bi * 256 + m * 16 + cc], acc);
      T[(16 * i + r) * LDA + 16 * j + cc] = -acc;
    }
    __syncthreads();
  }
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads, 1)
gdn_prefill_fused_kernel(const PrefillShape s, const PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int n = blockIdx.x / s.H;
  const int h = blockIdx.x - n * s.H;
  int64_t bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, s.total_T, a.err, &bos, &eos)) return;

  const size_t state_off = ((size_t)n * s.H + h) * (size_t)D * D;
  const int64_t L = eos - bos;
  const int nchunks = (int)((L + C - 1) / C);
  if (nchunks == 0) {  // empty sequence: the state passes through
    if (a.final_state) {
      for (int i = tid; i < D * D / 4; i += kThreads) {
        const float4 x = a.initial_state ? reinterpret_cast<const float4*>(a.initial_state + state_off)[i]
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(a.final_state + state_off)[i] = x;
      }
    }
    return;
  }

  if (warp == 0) {
    tc::tmem_alloc(sm.tmem_slot(), TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(sm.bar(), 1);
    tc::fence_mbar_init();
    *sm.abort_flag() = 0;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *sm.tmem_slot();
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lane quarter
  uint32_t phase = 0;

  const uint32_t kq = sm.u32(OFF_KQ), v16 = sm.u32(OFF_V), s16 = sm.u32(OFF_S16), w16 = sm.u32(OFF_W16);
  const uint32_t u16 = sm.u32(OFF_U16), udd = sm.u32(OFF_UDD), tp = sm.u32(OFF_TP), tpp = sm.u32(OFF_TPP);
  const uint32_t p16 = sm.u32(OFF_P16);

  // ---- initial state: row j = tid of S^T into TMEM (fp32) and S16 (fp16)
  {
    const int j = tid;
    for (int q = 0; q < D / 16; ++q) {
      float v[16];
      if (a.initial_state) {
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
      tc::tmem_st16(tl + COL_S + q * 16, v);
      uint8_t* tile = sm.base + OFF_S16 + (q >> 2) * S16_HALF;
      st_sw128_chunk(tile, j, (q & 3) * 2, v);
      st_sw128_chunk(tile, j, (q & 3) * 2 + 1, v + 8);
    }
    tc::wait_st();
  }
  publish_to_mma();

  const TOut* dummy = nullptr;
  (void)dummy;
  TOut* op = static_cast<TOut*>(a.o);

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = bos + (int64_t)c * C;
    const int Lc = (int)((eos - t0) < C ? (eos - t0) : C);

    // P0: inputs of the chunk -> fp16 tiles; cumulative gates
    load_chunk<TIn>(sm, s, a, h, t0, Lc);

    // P1: [K;Q] K^T -> TMEM D1 (M=128 rows K then Q, N=64, K=dk)
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t id = tc::idesc_f16(128, 64, 0, 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * KQ_HALF + (ks & 3) * 32;
        tc::mma_f16(tmem + COL_D1, tc::sw128_desc(kq + off, 16, 1024), tc::sw128_desc(kq + off, 16, 1024), id,
                    ks > 0);
      }
      tc::mma_commit(sm.bar());
    }
    if (!wait_mma(sm, phase, a.err)) break;

    // P2: A (fp32) from the K K^T rows, P (fp16) from the Q K^T rows
    {
      float x[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tc::tmem_ld16(tl + COL_D1 + q * 16, x + 16 * q);
      tc::wait_ld();
      const float* G = sm.G();
      if (tid < C) {
        const int i = tid;
        const float Gi = G[i], bi = sm.beta()[i];
        float* Arow = sm.A() + i * LDA;
#pragma unroll
        for (int j = 0; j < C; ++j) Arow[j] = (j < i) ? bi * __expf(Gi - G[j]) * x[j] : 0.f;
      } else {
        const int r = tid - C;
        const float Gr = G[r];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float v[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int i = cc * 8 + m;
            v[m] = (i <= r) ? __expf(Gr - G[i]) * x[i] : 0.f;
          }
          st_sw128_chunk(sm.base + OFF_P16, r, cc, v);
        }
      }
    }
    __syncthreads();

    // P3: T = (I + A)^{-1}; T diag(beta gamma) and T diag(beta) as fp16 B operands
    solve_unit_lower(sm);
    {
      const int mat = tid >> 6, i = tid & 63;
      const float* colscale = mat ? sm.beta() : sm.bg();
      uint8_t* tile = sm.base + (mat ? OFF_TPP : OFF_TP);
      const float* Trow = sm.T() + i * LDA;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        float v[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int j = cc * 8 + m;
          v[m] = (j <= i) ? Trow[j] * colscale[j] : 0.f;
        }
        st_sw128_chunk(tile, i, cc, v);
      }
    }
    publish_to_mma();

    // P4: W^T = K^T T'^T and U~^T = V^T T''^T (A MN-major from the token tiles)
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t id = tc::idesc_f16(128, 64, 1, 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        tc::mma_f16(tmem + COL_W, tc::sw128_desc(kq + ks * 2048, KQ_HALF, 1024),
                    tc::sw128_desc(tp + ks * 32, 16, 1024), id, ks > 0);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        tc::mma_f16(tmem + COL_U, tc::sw128_desc(v16 + ks * 2048, V_HALF, 1024),
                    tc::sw128_desc(tpp + ks * 32, 16, 1024), id, ks > 0);
      }
      tc::mma_commit(sm.bar());
    }
    if (!wait_mma(sm, phase, a.err)) break;

    // P5: W^T -> fp16 MN-major B tile; scale the resident state by gamma_C
    {
      const int i = tid;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float w[16];
        tc::tmem_ld16(tl + COL_W + q * 16, w);
        tc::wait_ld();
        st_sw128_chunk(sm.base + OFF_W16, i, 2 * q, w);
        st_sw128_chunk(sm.base + OFF_W16, i, 2 * q + 1, w + 8);
      }
      const float gC = sm.gam()[C - 1];
#pragma unroll
      for (int q = 0; q < D / 16; ++q) {
        float v[16];
        tc::tmem_ld16(tl + COL_S + q * 16, v);
        tc::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) v[x] *= gC;
        tc::tmem_st16(tl + COL_S + q * 16, v);
      }
      tc::wait_st();
    }
    publish_to_mma();

    // P6: U^T = U~^T - S^T W^T (accumulate with negated A); O1 = S^T Q^T
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t idu = tc::idesc_f16(128, 64, 0, 1, 1);
      const uint32_t ido = tc::idesc_f16(128, 64, 0, 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = tc::sw128_desc(s16 + (ks >> 2) * S16_HALF + (ks & 3) * 32, 16, 1024);
        tc::mma_f16(tmem + COL_U, ad, tc::sw128_desc(w16 + ks * 2048, 16384, 1024), idu, 1);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = tc::sw128_desc(s16 + (ks >> 2) * S16_HALF + (ks & 3) * 32, 16, 1024);
        const uint64_t bd = tc::sw128_desc(kq + 8 * 1024 + (ks >> 2) * KQ_HALF + (ks & 3) * 32, 16, 1024);
        tc::mma_f16(tmem + COL_O1, ad, bd, ido, ks > 0);
      }
      tc::mma_commit(sm.bar());
    }
    if (!wait_mma(sm, phase, a.err)) break;

    // P7: U^T -> fp16 A tiles (plain and decayed to the chunk end)
    {
      const int j = tid;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float u[16], ud[16];
        tc::tmem_ld16(tl + COL_U + q * 16, u);
        tc::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) ud[x] = u[x] * sm.dd()[q * 16 + x];
        st_sw128_chunk(sm.base + OFF_U16, j, 2 * q, u);
        st_sw128_chunk(sm.base + OFF_U16, j, 2 * q + 1, u + 8);
        st_sw128_chunk(sm.base + OFF_UDD, j, 2 * q, ud);
        st_sw128_chunk(sm.base + OFF_UDD, j, 2 * q + 1, ud + 8);
      }
    }
    publish_to_mma();

    // P8: O2 = U^T P^T; S^T += (U^T diag(dd)) K
    if (tid == 0) {
      tc::fence_after_sync();
      const uint32_t ido = tc::idesc_f16(128, 64, 0, 0);
      const uint32_t ids = tc::idesc_f16(128, 128, 0, 1);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_f16(tmem + COL_O2, tc::sw128_desc(u16 + ks * 32, 16, 1024),
                    tc::sw128_desc(p16 + ks * 32, 16, 1024), ido, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        tc::mma_f16(tmem + COL_S, tc::sw128_desc(udd + ks * 32, 16, 1024),
                    tc::sw128_desc(kq + ks * 2048, KQ_HALF, 1024), ids, 1);
      tc::mma_commit(sm.bar());
    }
    if (!wait_mma(sm, phase, a.err)) break;

    // P9: outputs of the chunk; new state -> fp16 operand (and fp32 final state)
    {
      const int j = tid;
      const float sc = a.scale;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float o1[16], o2[16];
        tc::tmem_ld16(tl + COL_O1 + q * 16, o1);
        tc::tmem_ld16(tl + COL_O2 + q * 16, o2);
        tc::wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const int r = q * 16 + x;
          if (r < Lc)
            store_out(op + ((size_t)(t0 + r) * s.H + h) * D + j, sc * fmaf(sm.gam()[r], o1[x], o2[x]));
        }
      }
      const bool last = (c == nchunks - 1);
#pragma unroll
      for (int q = 0; q < D / 16; ++q) {
        float v[16];
        tc::tmem_ld16(tl + COL_S + q * 16, v);
        tc::wait_ld();
        uint8_t* tile = sm.base + OFF_S16 + (q >> 2) * S16_HALF;
        st_sw128_chunk(tile, j, (q & 3) * 2, v);
        st_sw128_chunk(tile, j, (q & 3) * 2 + 1, v + 8);
        if (last && a.final_state) {
          float4* dst = reinterpret_cast<float4*>(a.final_state + state_off + (size_t)j * D + q * 16);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
        }
      }
    }
    publish_to_mma();
  }

  // teardown: every MMA has completed (each phase waited), TMEM can be released
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, TMEM_COLS);
}

template <typename TIn, typename TOut>
gdn_status_t launch(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    const cudaError_t e = cudaFuncSetAttribute(gdn_prefill_fused_kernel<TIn, TOut>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess)
      return fail(GDN_ERR_CUDA, std::string("fused prefill: cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    configured = true;
  }
  const unsigned grid = (unsigned)((long long)s.N * s.H);
  gdn_prefill_fused_kernel<TIn, TOut><<<grid, kThreads, SMEM_BYTES, stream>>>(s, a);
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
