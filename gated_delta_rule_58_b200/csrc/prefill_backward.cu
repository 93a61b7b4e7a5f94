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
// writes its 32 partial products, then each of the dk threads adds two entries over
// the CTA's columns); dg and dbeta are block reductions. All four are accumulated
// with fp32 atomics into zeroed outputs, so the column blocks of a head and the value
// heads that share a q/k head add up.
// Latency: the next token's k, q, v, dO and gates are loaded into registers while
// the current token computes; in the backward walk S_t is the previous token's
// S_{t-1} (kept in registers) and the next S_{t-1} is fetched from the scratch into
// shared memory by cp.async while the current token computes (each thread copies and
// reads only its own entries).
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

// value columns per CTA: one warp per CTA (1024 / dk columns of dk / 32 lanes each),
// so many small CTAs share an SM and a barrier spans one warp
template <int D>
constexpr int bwd_cols() { return 1024 / D; }

// Shared-memory stride of one column in the [columns][D entries] buffers, padded so
// that the eight lanes of a quarter warp (two columns x four 16-byte pieces) store to
// distinct banks.
template <int D>
constexpr int bwd_col_stride() { return D + 16; }

template <int D>
constexpr int bwd_threads() { return bwd_cols<D>() * (D / 32); }
template <int D>
constexpr int bwd_warps() { return (bwd_threads<D>() + 31) / 32; }

template <int D>
constexpr size_t bwd_smem_bytes() {
  // token vectors [2][k, q, v, dO][D], gates [2][alpha, beta], column partials of dq
  // and dk and the prefetched S_{t-1} ([columns][stride] each), scalar partials
  // [warps][2], per-warp partial squared norms of k and q [2][warps][2] and partial
  // projections [warps][2]; bwd_cols * D / 32 threads
  return (8 * D + 4 + 3 * bwd_cols<D>() * bwd_col_stride<D>() + 8 * bwd_warps<D>()) * sizeof(float);
}

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

template <int D, typename TIn>
__global__ void __launch_bounds__(bwd_threads<D>())
gdn_prefill_backward_kernel(const BwdArgs a) {
  constexpr int TPC = D / 32;  // threads per state column
  constexpr int kBwdCols = bwd_cols<D>();
  constexpr int NT = kBwdCols * TPC;
  constexpr int EPT = D / NT;  // dk entries of the token vectors per thread
  static_assert(NT * EPT == D && NT % 32 == 0, "whole warps, whole vectors");
  constexpr int PER = 32;      // entries of the column per thread
  constexpr int NP = PER / 4;  // 16-byte pieces per thread
  constexpr int NW = NT / 32;
  constexpr int RS = bwd_col_stride<D>();
  extern __shared__ __align__(16) float bsm[];
  float* tok = bsm;                       // [2][4][D]
  float* gates = tok + 8 * D;             // [2][2]
  float* red_q = gates + 4;               // [kBwdCols][RS]
  float* red_k = red_q + kBwdCols * RS;
  float* sp_buf = red_k + kBwdCols * RS;  // [kBwdCols][RS]: the next S_{t-1}, each thread its own entries
  float* red_s = sp_buf + kBwdCols * RS;  // [NW][2]
  float* nrm = red_s + 2 * NW;            // [2][NW][2]: partial |k|^2, |q|^2 of a buffer's token
  float* jred = nrm + 4 * NW;             // [NW][2]: partial k^ . dk^, q^ . dq^
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
  const int nck = (int)((eos - bos + a.C - 1) / a.C);
  const size_t SS = (size_t)D * D;
  const size_t state_off = ((size_t)n * a.H + h) * SS + (size_t)col * D;
  float* ck = a.ckpt + ((size_t)h * a.ck_slots + (size_t)(bos / a.C) + n) * SS + (size_t)col * D;
  float* scr = a.scratch + (size_t)item * (size_t)(a.C + 1) * SS + (size_t)col * D;
  float* spb = sp_buf + lcol * RS;
  const TIn* qp = static_cast<const TIn*>(a.q);
  const TIn* kp = static_cast<const TIn*>(a.k);
  const TIn* vp = static_cast<const TIn*>(a.v);
  const TIn* dop = static_cast<const TIn*>(a.d_o);

  // A token's k, q, v, dO and gates are
  // fetched into registers, then committed to shared-memory buffer `buf` (two
  // buffers: the barrier of the token in between orders every read of a buffer
  // before its refill).
  // (thread tid holds entries tid + NT e, e < EPT)
  float fk[EPT], fq[EPT], fv[EPT], fdo[EPT], fg = 0.f, fb = 0.f;
  auto fetch = [&](int64_t t) {
    const size_t th = (size_t)t * a.H + h, tq = (size_t)t * a.Hqk + hq;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int i = tid + NT * e;
      fk[e] = to_f32(kp[tq * D + i]);
      fq[e] = to_f32(qp[tq * D + i]);
      fv[e] = to_f32(vp[th * D + i]);
      fdo[e] = to_f32(dop[th * D + i]);
    }
    if (tid == 0) {
      fg = a.g[th];
      fb = a.beta[th];
    }
  };
  auto commit = [&](int buf) {
    float* tb = tok + buf * 4 * D;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int i = tid + NT * e;
      tb[i] = fk[e];
      tb[D + i] = fq[e];
      tb[2 * D + i] = fv[e];
      tb[3 * D + i] = fdo[e];
    }
    if (tid == 0) {
      gates[2 * buf] = expf(fg);
      gates[2 * buf + 1] = fb;
    }
    if (l2) {  // per-warp partial squared norms
      float kk = 0.f, qq = 0.f;
#pragma unroll
      for (int e = 0; e < EPT; ++e) {
        kk = fmaf(fk[e], fk[e], kk);
        qq = fmaf(fq[e], fq[e], qq);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
      }
      if ((tid & 31) == 0) {
        nrm[(buf * NW + (tid >> 5)) * 2] = kk;
        nrm[(buf * NW + (tid >> 5)) * 2 + 1] = qq;
      }
    }
  };
  // 1 / |k| and 1 / |q| of the token in buffer `buf` (1 without the normalisation)
  auto inv_norms = [&](int buf, float* rk, float* rq) {
    *rk = 1.f;
    *rq = 1.f;
    if (l2) {
      float kk = 0.f, qq = 0.f;
      for (int wi = 0; wi < NW; ++wi) {
        kk += nrm[(buf * NW + wi) * 2];
        qq += nrm[(buf * NW + wi) * 2 + 1];
      }
      *rk = kk > 0.f ? 1.f / sqrtf(kk) : 0.f;
      *rq = qq > 0.f ? 1.f / sqrtf(qq) : 0.f;
    }
  };
  // this thread's entries of a D-vector in shared memory
  auto load_vec = [&](const float* v, float* out) {
#pragma unroll
    for (int y = 0; y < NP; ++y) {
      const float4 f = *reinterpret_cast<const float4*>(v + piece(y));
      out[4 * y] = f.x; out[4 * y + 1] = f.y; out[4 * y + 2] = f.z; out[4 * y + 3] = f.w;
    }
  };
  // one token forward on this thread's entries of column col (as the forward kernel;
  // the update adds c k with c = beta (v_j - alpha (k^ . S_j)) / |k|)
  auto advance = [&](float* st, int buf) {
    const float* tb = tok + buf * 4 * D;
    const float alpha = gates[2 * buf], beta = gates[2 * buf + 1];
    float rk, rq;
    inv_norms(buf, &rk, &rq);
    float kv[PER];
    load_vec(tb, kv);
    float u = 0.f;
#pragma unroll
    for (int x = 0; x < PER; ++x) u = fmaf(kv[x], st[x], u);
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
    const float c = beta * (tb[2 * D + col] - alpha * (u * rk)) * rk;
#pragma unroll
    for (int x = 0; x < PER; ++x) st[x] = fmaf(alpha, st[x], c * kv[x]);
  };
  // a state column's entries of this thread from / to memory (p = the column's base)
  auto load_state = [&](const float* p, float* st) {
#pragma unroll
    for (int y = 0; y < NP; ++y) {
      const float4 f = *reinterpret_cast<const float4*>(p + piece(y));
      st[4 * y] = f.x; st[4 * y + 1] = f.y; st[4 * y + 2] = f.z; st[4 * y + 3] = f.w;
    }
  };
  auto store_state = [&](float* p, const float* st) {
#pragma unroll
    for (int y = 0; y < NP; ++y)
      *reinterpret_cast<float4*>(p + piece(y)) = make_float4(st[4 * y], st[4 * y + 1], st[4 * y + 2], st[4 * y + 3]);
  };
  auto prefetch_state = [&](const float* p) {  // this thread's entries -> sp_buf, asynchronously
#pragma unroll
    for (int y = 0; y < NP; ++y) cp_async16(spb + piece(y), p + piece(y));
  };

  // 1. forward with a checkpoint at the start of every chunk
  int it = 0;  // staged tokens so far (buffer parity)
  {
    float st[PER];
    if (a.init) {
      load_state(a.init + state_off, st);
    } else {
#pragma unroll
      for (int x = 0; x < PER; ++x) st[x] = 0.f;
    }
    if (bos < eos) fetch(bos);
    for (int64_t t = bos; t < eos; ++t) {
      const int buf = (it++) & 1;
      commit(buf);
      if (t + 1 < eos) fetch(t + 1);
      __syncthreads();
      if ((t - bos) % a.C == 0) store_state(ck + (size_t)((t - bos) / a.C) * SS, st);
      advance(st, buf);
    }
  }

  // 2. chunks last to first
  float Dm[PER];  // dL/dS_t, this thread's entries
  if (a.d_fin) {
    load_state(a.d_fin + state_off, Dm);
  } else {
#pragma unroll
    for (int x = 0; x < PER; ++x) Dm[x] = 0.f;
  }
  for (int c = nck - 1; c >= 0; --c) {
    const int64_t t0 = bos + (int64_t)c * a.C;
    const int64_t t1 = (t0 + a.C < eos) ? t0 + a.C : eos;
    float sc[PER];  // S_t of the token being walked
    {
      // scratch slot x = the state before token t0 + x
      load_state(ck + (size_t)c * SS, sc);
      fetch(t0);
      for (int64_t t = t0; t < t1; ++t) {
        const int buf = (it++) & 1;
        commit(buf);
        if (t + 1 < t1) fetch(t + 1);
        __syncthreads();
        store_state(scr + (size_t)(t - t0) * SS, sc);
        advance(sc, buf);
      }
    }
    // sc = the state after the chunk's last token; its S_{t-1} goes into sp_buf
    prefetch_state(scr + (size_t)(t1 - 1 - t0) * SS);
    fetch(t1 - 1);
    for (int64_t t = t1 - 1; t >= t0; --t) {
      const int buf = (it++) & 1;
      commit(buf);
      if (t - 1 >= t0) fetch(t - 1);
      __syncthreads();
      const float* tb = tok + buf * 4 * D;
      const float vj = tb[2 * D + col], dOj = tb[3 * D + col];
      const float alpha = gates[2 * buf], beta = gates[2 * buf + 1];
      float rk, rq;
      inv_norms(buf, &rk, &rq);
      const size_t th = (size_t)t * a.H + h, tq = (size_t)t * a.Hqk + hq;
      // column j's terms of dq (S_t dO) first: S_t is not needed after them
      float* rowq = red_q + lcol * RS;
      float* rowk = red_k + lcol * RS;
#pragma unroll
      for (int y = 0; y < NP; ++y)
        *reinterpret_cast<float4*>(rowq + piece(y)) = make_float4(sc[4 * y] * dOj, sc[4 * y + 1] * dOj,
                                                                sc[4 * y + 2] * dOj, sc[4 * y + 3] * dOj);
      float sp[PER];  // S_{t-1}
      cp_async_wait_all();
      load_vec(spb, sp);
      if (t - 1 >= t0) prefetch_state(scr + (size_t)(t - 1 - t0) * SS);
      // D += scale q dO^T
      {
        float qv[PER];
        load_vec(tb + D, qv);
#pragma unroll
        for (int x = 0; x < PER; ++x) Dm[x] = fmaf(a.scale * rq * qv[x], dOj, Dm[x]);
      }
      float kv[PER];
      load_vec(tb, kv);
      // u = S~^T k (S~ = alpha S_{t-1}), w = D^T k, column j
      float pu = 0.f, pw = 0.f;
#pragma unroll
      for (int x = 0; x < PER; ++x) {
        pu = fmaf(kv[x], sp[x], pu);
        pw = fmaf(kv[x], Dm[x], pw);
      }
#pragma unroll
      for (int off = 1; off < TPC; off <<= 1) {
        pu += __shfl_xor_sync(0xffffffffu, pu, off);
        pw += __shfl_xor_sync(0xffffffffu, pw, off);
      }
      const float u = alpha * pu * rk, w = pw * rk, vmu = vj - u;
      // column j's terms of dk (D (v - u) - S~ w) and of dg
      float sdg = 0.f;
#pragma unroll
      for (int y = 0; y < NP; ++y) {
        float kk[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) {
          const int x = 4 * y + z;
          const float stl = alpha * sp[x];
          kk[z] = Dm[x] * vmu - stl * w;
          sdg = fmaf(Dm[x], stl, sdg);
        }
        *reinterpret_cast<float4*>(rowk + piece(y)) = make_float4(kk[0], kk[1], kk[2], kk[3]);
      }
      float sdb = 0.f;
      if (part == 0) {
        sdg -= beta * u * w;
        sdb = w * vmu;
        a.dv[th * D + col] = beta * w;
      }
      // dL/dS_{t-1}; S_{t-1} becomes the next token's S_t
      const float bw = beta * w * rk;
#pragma unroll
      for (int x = 0; x < PER; ++x) {
        Dm[x] = alpha * (Dm[x] - bw * kv[x]);
        sc[x] = sp[x];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sdg += __shfl_xor_sync(0xffffffffu, sdg, off);
        sdb += __shfl_xor_sync(0xffffffffu, sdb, off);
      }
      if ((tid & 31) == 0) {
        red_s[2 * (tid >> 5)] = sdg;
        red_s[2 * (tid >> 5) + 1] = sdb;
      }
      __syncthreads();
      {  // entries tid + NT e of dq and of dk over this CTA's columns
        float gq[EPT], gk[EPT];  // this CTA's part of dq^, dk^
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          const int i = tid + NT * e;
          float sq = 0.f, sk = 0.f;
#pragma unroll 8
          for (int j = 0; j < kBwdCols; ++j) {
            sq += red_q[j * RS + i];
            sk += red_k[j * RS + i];
          }
          gq[e] = a.scale * sq;
          gk[e] = beta * sk;
        }
        if (l2) {  // through the normalisation: (g - x^ (x^ . g)) / |x|
          float pk = 0.f, pq = 0.f;
#pragma unroll
          for (int e = 0; e < EPT; ++e) {
            const int i = tid + NT * e;
            pk = fmaf(tb[i] * rk, gk[e], pk);
            pq = fmaf(tb[D + i] * rq, gq[e], pq);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            pk += __shfl_xor_sync(0xffffffffu, pk, off);
            pq += __shfl_xor_sync(0xffffffffu, pq, off);
          }
          if ((tid & 31) == 0) {
            jred[2 * (tid >> 5)] = pk;
            jred[2 * (tid >> 5) + 1] = pq;
          }
          __syncthreads();
          float dotk = 0.f, dotq = 0.f;
          for (int wi = 0; wi < NW; ++wi) {
            dotk += jred[2 * wi];
            dotq += jred[2 * wi + 1];
          }
#pragma unroll
          for (int e = 0; e < EPT; ++e) {
            const int i = tid + NT * e;
            gk[e] = (gk[e] - tb[i] * rk * dotk) * rk;
            gq[e] = (gq[e] - tb[D + i] * rq * dotq) * rq;
          }
        }
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          atomicAdd(a.dq + tq * D + tid + NT * e, gq[e]);
          atomicAdd(a.dk + tq * D + tid + NT * e, gk[e]);
        }
      }
      if (tid == 0) {
        float g_sum = 0.f, b_sum = 0.f;
        for (int wi = 0; wi < NW; ++wi) {
          g_sum += red_s[2 * wi];
          b_sum += red_s[2 * wi + 1];
        }
        atomicAdd(a.dg + th, g_sum);
        atomicAdd(a.dbeta + th, b_sum);
      }
    }
  }
  if (a.d_init) store_state(a.d_init + state_off, Dm);
}

template <int D, typename TIn>
gdn_status_t launch_bwd(const BwdArgs& a, cudaStream_t stream) {
  auto kernel = gdn_prefill_backward_kernel<D, TIn>;
  constexpr size_t smem = bwd_smem_bytes<D>();
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
  if ((long long)N * H * (dk * dk / 1024) >= (1LL << 31))  // column blocks: dk / (1024 / dk) per head
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
