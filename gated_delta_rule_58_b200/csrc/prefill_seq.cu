// Token-sequential prefill (SIMT): one CTA per (sequence, head), the state held
// in registers across the whole sequence. Used for small head dims (dk = dv in
// {32, 64}, e.g. the fp32 tiny workload) and as the always-available GPU path;
// the chunk size does not change its arithmetic.
//
// Mapping: value column j of S (row j of the K-last state S^T) is owned by TPC =
// dk / 32 adjacent lanes, each holding 32 of its dk entries. Per token every
// column needs only k, q, v_j, alpha and beta:
//     u_j = k . S[:, j]                      (lane partials + shuffle reduction)
//     S[:, j] <- alpha S[:, j] + beta k (v_j - alpha u_j)
//     o_j = scale * q . S[:, j]
// which is S_t = alpha (I - beta k k^T) S_{t-1} + beta k v^T column by column.
// k, q, v of the token are staged in double-buffered shared memory (one barrier
// per token). With GDN_QK_L2NORM, k and q are used divided by their Euclidean
// norms, which the TPC lanes of a column reduce from their own 32 entries.
#include "prefill.cuh"

namespace gdn {
namespace {

template <int D, typename TIn, typename TOut>
__global__ void __launch_bounds__(D * (D / 32))
gdn_prefill_sequential_kernel(const PrefillShape s, const PrefillArgs a) {
  constexpr int TPC = D / 32;        // threads per state column
  constexpr int NT = D * TPC;        // threads per CTA
  constexpr int PER = D / TPC;       // = 32 entries of the column per thread
  __shared__ __align__(16) float s_k[2][D];
  __shared__ __align__(16) float s_q[2][D];
  __shared__ float s_v[2][D];
  __shared__ float s_ab[2][2];       // alpha, beta

  const int tid = threadIdx.x;
  const int col = tid / TPC;         // value index j
  const int part = tid % TPC;        // which 32 entries of the column
  const int n = blockIdx.x / s.H;
  const int h = blockIdx.x - n * s.H;
  const int hq = h / (s.H / s.Hqk);  // the value head's query/key head
  const bool l2 = (a.flags & GDN_QK_L2NORM) != 0;
  int64_t bos, eos;
  if (!seq_bounds(a.cu_seqlens, n, s.total_T, a.err, &bos, &eos)) return;

  const size_t state_off = ((size_t)n * s.H + h) * (size_t)D * D + (size_t)col * D + part * PER;
  float st[PER];
  if (a.initial_state) {
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
      const float4 x = *reinterpret_cast<const float4*>(a.initial_state + state_off + i);
      st[i] = x.x; st[i + 1] = x.y; st[i + 2] = x.z; st[i + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) st[i] = 0.f;
  }

  const TIn* qp = static_cast<const TIn*>(a.q);
  const TIn* kp = static_cast<const TIn*>(a.k);
  const TIn* vp = static_cast<const TIn*>(a.v);
  TOut* op = static_cast<TOut*>(a.o);

  for (int64_t t = bos; t < eos; ++t) {
    const int buf = (int)(t - bos) & 1;
    const size_t th = (size_t)t * s.H + h;       // v, g, beta, o
    const size_t tq = (size_t)t * s.Hqk + hq;    // q, k
    for (int i = tid; i < D; i += NT) {
      s_k[buf][i] = to_f32(kp[tq * D + i]);
      s_q[buf][i] = to_f32(qp[tq * D + i]);
      s_v[buf][i] = to_f32(vp[th * D + i]);
    }
    if (tid == 0) {
      s_ab[buf][0] = expf(a.g[th]);
      s_ab[buf][1] = a.beta[th];
    }
    __syncthreads();
    const float alpha = s_ab[buf][0], beta = s_ab[buf][1];
    const float* kv = s_k[buf] + part * PER;
    const float* qv = s_q[buf] + part * PER;
    float rk = 1.f, rq = 1.f;  // 1 / |k|, 1 / |q| with the normalisation
    if (l2) {
      float kk = 0.f, qq = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        kk = fmaf(kv[i], kv[i], kk);
        qq = fmaf(qv[i], qv[i], qq);
      }
#pragma unroll
      for (int off = 1; off < TPC; off <<= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
      }
      rk = kk > 0.f ? 1.f / sqrtf(kk) : 0.f;
      rq = qq > 0.f ? 1.f / sqrtf(qq) : 0.f;
    }
    float u = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) u = fmaf(kv[i], st[i], u);
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
    const float c = beta * (s_v[buf][col] - alpha * (u * rk)) * rk;  // the update adds c k
    float o = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      st[i] = fmaf(alpha, st[i], c * kv[i]);
      o = fmaf(qv[i], st[i], o);
    }
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) o += __shfl_xor_sync(0xffffffffu, o, off);
    if (part == 0) store_out(op + th * D + col, a.scale * (o * rq));
  }

  if (a.final_state) {
#pragma unroll
    for (int i = 0; i < PER; i += 4)
      *reinterpret_cast<float4*>(a.final_state + state_off + i) =
          make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
  }
}

template <int D, typename TIn>
gdn_status_t launch_out(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  const unsigned grid = (unsigned)((long long)s.N * s.H);
  if (a.out_dtype == GDN_BF16)
    gdn_prefill_sequential_kernel<D, TIn, __nv_bfloat16><<<grid, D * (D / 32), 0, stream>>>(s, a);
  else
    gdn_prefill_sequential_kernel<D, TIn, float><<<grid, D * (D / 32), 0, stream>>>(s, a);
  return check_launch("gdn_chunk_prefill (sequential)");
}

template <int D>
gdn_status_t launch_in(const PrefillShape& s, const PrefillArgs& a, cudaStream_t stream) {
  return a.in_dtype == GDN_BF16 ? launch_out<D, __nv_bfloat16>(s, a, stream)
                                : launch_out<D, float>(s, a, stream);
}

}  // namespace

gdn_status_t prefill_sequential_launch(const PrefillShape& s, const PrefillArgs& a,
                                       cudaStream_t stream) {
  if ((long long)s.N * s.H >= (1LL << 31)) return fail(GDN_ERR_UNSUPPORTED, "N * H too large");
  switch (s.dk) {
    case 32: return launch_in<32>(s, a, stream);
    case 64: return launch_in<64>(s, a, stream);
    case 128: return launch_in<128>(s, a, stream);
    default: return fail(GDN_ERR_UNSUPPORTED, "sequential prefill: dk must be 32, 64 or 128");
  }
}

}  // namespace gdn
