/*
 * Gated delta rule: plain, sequential, fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library. The CUDA library never
 * links, calls or includes anything from here, and this file includes nothing
 * from the CUDA sources.
 *
 * What it computes (per sequence or slot, per head, tokens in order):
 *
 *   gated delta rule (Yang, Kautz, Hatamizadeh, "Gated Delta Networks:
 *   Improving Mamba2 with Delta Rule", ICLR 2025, eq. for the gated delta
 *   update):
 *       S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *       o_t = scale * S_t^T q_t,          alpha_t = exp(g_t),
 *   with S_t of shape dk x dv.
 *
 *   gated delta product (the multi-Householder variant named by the kernel
 *   family cake_gated_delta_product_mtp on the FlashInfer PR #7156 page,
 *   "Cake GDP kernel: shared-memory reduction and direct register loads",
 *   introduction): per token one gate, then n_h Householder updates in order
 *   j = 1..n_h, then one output:
 *       S <- alpha_t S
 *       S <- (I - beta_{t,j} k_{t,j} k_{t,j}^T) S + beta_{t,j} k_{t,j} v_{t,j}^T
 *       o_t = scale * S^T q_t
 *   With n_h = 1 this is the gated delta rule above, since
 *   (I - b k k^T)(a S) = a (I - b k k^T) S.
 *
 * Heads (grouped value attention): q and k may have fewer heads (H_qk) than
 * v, g, beta, o and the state (H, a multiple of H_qk). Value head h then reads
 * query/key head h / (H / H_qk): consecutive value heads share one q/k head, the
 * grouping of repeating each q/k head H / H_qk times in place. H_qk = H is the
 * plain one-to-one case. With l2norm set, q and k are first scaled to unit
 * Euclidean length per token (per q/k head and, for k, per Householder), in
 * fp64; a zero vector stays zero.
 *
 * Storage: states are kept K-last, i.e. S^T row-major [dv][dk], the layout the
 * FlashInfer PR #7156 page (section 1) indexes as state + row + k_col and the
 * FlashInfer PR #3866 page (section 2, accumulate_state_fragment) contracts over
 * the second index. Everything here is fp64; inputs arrive as fp64 copies of the
 * exact values the GPU reads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ---- the three steps of one token, on one head, state St = S^T [dv][dk] ---- */

/* S <- alpha S */
static void apply_gate(double* St, double alpha, int dk, int dv) {
  for (int j = 0; j < dv; ++j)
    for (int i = 0; i < dk; ++i) St[(size_t)j * dk + i] *= alpha;
}

/* S <- (I - beta k k^T) S + beta k v^T, one column S[:, j] (= row j of St) at a
 * time: p = k^T S[:, j];  S[:, j] <- S[:, j] - beta k p + beta k v_j. */
static void apply_householder(double* St, const double* k, const double* v, double beta,
                              int dk, int dv) {
  for (int j = 0; j < dv; ++j) {
    double* col = St + (size_t)j * dk;
    double p = 0.0;
    for (int i = 0; i < dk; ++i) p += k[i] * col[i];
    for (int i = 0; i < dk; ++i) col[i] = col[i] - beta * k[i] * p + beta * k[i] * v[j];
  }
}

/* o = scale * S^T q */
static void emit_output(const double* St, const double* q, double scale, double* o,
                        int dk, int dv) {
  for (int j = 0; j < dv; ++j) {
    const double* col = St + (size_t)j * dk;
    double acc = 0.0;
    for (int i = 0; i < dk; ++i) acc += col[i] * q[i];
    o[j] = scale * acc;
  }
}

/* q/k of one token, optionally scaled to unit length (into `buf`) */
static const double* maybe_unit(const double* x, int n, int l2norm, double* buf) {
  if (!l2norm) return x;
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
  for (int i = 0; i < n; ++i) buf[i] = x[i] * inv;
  return buf;
}

/* ---- a tiny work queue over independent (sequence or slot, head) pairs ---- */

typedef struct {
  int n_items;
  int next;
  pthread_mutex_t lock;
  void (*fn)(void* ctx, int item);
  void* ctx;
} queue_t;

static void* worker(void* arg) {
  queue_t* q = (queue_t*)arg;
  for (;;) {
    pthread_mutex_lock(&q->lock);
    int item = q->next++;
    pthread_mutex_unlock(&q->lock);
    if (item >= q->n_items) break;
    q->fn(q->ctx, item);
  }
  return NULL;
}

static int run_items(int n_items, int nthreads, void (*fn)(void*, int), void* ctx) {
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n_items) nthreads = n_items > 0 ? n_items : 1;
  queue_t q;
  q.n_items = n_items;
  q.next = 0;
  q.fn = fn;
  q.ctx = ctx;
  pthread_mutex_init(&q.lock, NULL);
  if (nthreads == 1) {
    worker(&q);
  } else {
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &q);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  pthread_mutex_destroy(&q.lock);
  return nthreads;
}

/* ---- prefill: packed varlen sequences ---- */

typedef struct {
  const double *q, *k, *v, *g, *beta;
  const int64_t* cu;
  int H, Hqk, dk, dv, l2norm;
  double scale;
  const double* init;
  double* o;
  double* fin;
} prefill_ctx;

static void prefill_item(void* vctx, int item) {
  prefill_ctx* c = (prefill_ctx*)vctx;
  const int H = c->H, Hqk = c->Hqk, dk = c->dk, dv = c->dv;
  const int n = item / H, h = item % H;
  const int hq = h / (H / Hqk); /* the value head's query/key head */
  const size_t ssz = (size_t)dk * dv;
  double* St = (double*)malloc(ssz * sizeof(double));
  double* buf = (double*)malloc(2 * (size_t)dk * sizeof(double));
  if (c->init)
    memcpy(St, c->init + ((size_t)n * H + h) * ssz, ssz * sizeof(double));
  else
    memset(St, 0, ssz * sizeof(double));
  for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
    const size_t th = (size_t)t * H + h;   /* v, g, beta, o */
    const size_t tq = (size_t)t * Hqk + hq; /* q, k */
    const double* kt = maybe_unit(c->k + tq * dk, dk, c->l2norm, buf);
    const double* qt = maybe_unit(c->q + tq * dk, dk, c->l2norm, buf + dk);
    apply_gate(St, exp(c->g[th]), dk, dv);
    apply_householder(St, kt, c->v + th * dv, c->beta[th], dk, dv);
    emit_output(St, qt, c->scale, c->o + th * dv, dk, dv);
  }
  if (c->fin) memcpy(c->fin + ((size_t)n * H + h) * ssz, St, ssz * sizeof(double));
  free(buf);
  free(St);
}

/*
 * q, k: [total_T, Hqk, dk]; v: [total_T, H, dv]; g, beta: [total_T, H];
 * cu_seqlens: [N + 1] (cu[0] = 0, non-decreasing); init: [N, H, dv, dk] or NULL
 * (zero state); o: [total_T, H, dv]; final_state: [N, H, dv, dk] or NULL.
 * H must be a multiple of Hqk; l2norm != 0 normalises q and k per token.
 * Returns the number of threads used, or a negative value on bad arguments.
 */
int gdn_oracle_prefill(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, const int64_t* cu_seqlens, int N, int H, int Hqk,
                       int dk, int dv, double scale, int l2norm, const double* init, double* o,
                       double* final_state, int nthreads) {
  if (N < 0 || H <= 0 || Hqk <= 0 || H % Hqk != 0 || dk <= 0 || dv <= 0 || !cu_seqlens) return -1;
  if (cu_seqlens[0] != 0) return -1;
  for (int n = 0; n < N; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
  prefill_ctx c = {q, k, v, g, beta, cu_seqlens, H, Hqk, dk, dv, l2norm, scale, init, o, final_state};
  return run_items(N * H, nthreads, prefill_item, &c);
}

/* ---- decode: slot-indexed state pool, updated in place ---- */

typedef struct {
  const double *q, *k, *v, *g, *beta;
  double* pool;
  int num_slots;
  const int32_t* slot_ids;
  double* o;
  int T, H, Hqk, dk, dv, nh, l2norm;
  double scale;
  double* token_states; /* [B, T, H, dv, dk] or NULL */
} decode_ctx;

static void decode_item(void* vctx, int item) {
  decode_ctx* c = (decode_ctx*)vctx;
  const int H = c->H, Hqk = c->Hqk, T = c->T, dk = c->dk, dv = c->dv, nh = c->nh;
  const int b = item / H, h = item % H;
  const int hq = h / (H / Hqk); /* the value head's query/key head */
  const int slot = c->slot_ids[b];
  if (slot < 0 || slot >= c->num_slots) {
    for (int t = 0; t < T; ++t) {
      memset(c->o + (((size_t)b * T + t) * H + h) * dv, 0, (size_t)dv * sizeof(double));
      if (c->token_states)
        memset(c->token_states + (((size_t)b * T + t) * H + h) * (size_t)dk * dv, 0,
               (size_t)dk * dv * sizeof(double));
    }
    return;
  }
  double* St = c->pool + ((size_t)slot * H + h) * (size_t)dk * dv;
  double* buf = (double*)malloc(2 * (size_t)dk * sizeof(double));
  for (int t = 0; t < T; ++t) {
    const size_t bth = ((size_t)b * T + t) * H + h;   /* v, g, beta, o */
    const size_t btq = ((size_t)b * T + t) * Hqk + hq; /* q, k */
    apply_gate(St, exp(c->g[bth]), dk, dv);
    for (int m = 0; m < nh; ++m) {
      const size_t km = bth * nh + m;
      const double* kt = maybe_unit(c->k + (btq * nh + m) * dk, dk, c->l2norm, buf);
      apply_householder(St, kt, c->v + km * dv, c->beta[km], dk, dv);
    }
    emit_output(St, maybe_unit(c->q + btq * dk, dk, c->l2norm, buf + dk), c->scale, c->o + bth * dv, dk, dv);
    if (c->token_states) /* the state after token t (speculative-verify rollback point) */
      memcpy(c->token_states + bth * (size_t)dk * dv, St, (size_t)dk * dv * sizeof(double));
  }
  free(buf);
}

/*
 * q: [B, T, Hqk, dk]; k: [B, T, Hqk, nh, dk]; v: [B, T, H, nh, dv]; g: [B, T, H];
 * beta: [B, T, H, nh]; pool: [num_slots, H, dv, dk], updated in place for the
 * slots named by slot_ids[B] (a negative or out-of-range id leaves the pool
 * untouched and writes zeros to that row of o); o: [B, T, H, dv]. H must be a
 * multiple of Hqk; l2norm != 0 normalises q and every k per token. token_states
 * [B, T, H, dv, dk] (or NULL) receives the state after each token (zeros for a
 * skipped row).
 * Returns the number of threads used, or a negative value on bad arguments.
 */
int gdn_oracle_decode(const double* q, const double* k, const double* v, const double* g,
                      const double* beta, double* pool, int num_slots, const int32_t* slot_ids,
                      double* o, int B, int T, int H, int Hqk, int dk, int dv, int nh, double scale,
                      int l2norm, double* token_states, int nthreads) {
  if (B < 0 || T <= 0 || H <= 0 || Hqk <= 0 || H % Hqk != 0 || dk <= 0 || dv <= 0 || nh <= 0 ||
      num_slots < 0)
    return -1;
  decode_ctx c = {q, k, v, g, beta, pool, num_slots, slot_ids, o, T, H, Hqk, dk, dv, nh, l2norm, scale,
                  token_states};
  return run_items(B * H, nthreads, decode_item, &c);
}

/* ---- prefill backward: reverse-mode derivatives of the gated delta rule ----
 *
 * For a loss L with upstream derivatives dO_t = dL/do_t and dS_T = dL/dS_T (the
 * final state), the token recurrence is walked backwards with D = dL/dS_t, written
 * out from the chain rule on the two relations of each token (P = I - beta k k^T,
 * S~ = alpha S_{t-1}):
 *     S_t = P S~ + beta k v^T,        o_t = scale S_t^T q.
 * Per token, last to first:
 *     D    += scale q dO^T                          (o_t reads S_t)
 *     dq    = scale S_t dO
 *     u     = S~^T k,   w = D^T k
 *     dv    = beta w
 *     dbeta = w . (v - u)
 *     dk    = beta (D (v - u) - S~ w)
 *     dg    = <D, S~> - beta (u . w)                 (alpha = exp(g): dg = alpha dL/dalpha)
 *     D    <- alpha (D - beta k w^T)                 (= alpha P D, dL/dS_{t-1})
 * and dL/dS_0 = D at the end. Every state S_t is kept from a forward pass first.
 * With l2norm the relations read the unit vectors k^ = k / |k|, q^ = q / |q| (a zero
 * vector stays zero); the walk above gives the derivatives for k^ and q^, and the
 * chain rule through the normalisation maps them to dk = (dk^ - k^ (k^ . dk^)) / |k|
 * (zero for a zero vector), likewise for q. Scope: one Householder per token.
 */

typedef struct {
  const double *q, *k, *v, *g, *beta;
  const int64_t* cu;
  int H, Hqk, dk, dv, l2norm;
  double scale;
  const double *init, *d_o, *d_fin;
  double *dq, *dkk, *dvv, *dg, *dbeta, *d_init;
} backward_ctx;

/* the derivative for x from the one for x^ = x / |x|: (d - x^ (x^ . d)) / |x| */
static void unit_backward(const double* x, double* d, int n) {
  double ss = 0.0, dot = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  if (!(ss > 0.0)) {
    for (int i = 0; i < n; ++i) d[i] = 0.0;
    return;
  }
  const double inv = 1.0 / sqrt(ss);
  for (int i = 0; i < n; ++i) dot += x[i] * inv * d[i];
  for (int i = 0; i < n; ++i) d[i] = (d[i] - x[i] * inv * dot) * inv;
}

static void backward_item(void* vctx, int item) {
  backward_ctx* c = (backward_ctx*)vctx;
  const int H = c->H, Hqk = c->Hqk, dk = c->dk, dv = c->dv;
  const int n = item / H, h = item % H;
  const int hq = h / (H / Hqk);
  const size_t ssz = (size_t)dk * dv;
  const int64_t t0 = c->cu[n], T = c->cu[n + 1] - c->cu[n];
  /* states S_0 .. S_T, each S^T [dv][dk] */
  double* states = (double*)malloc((size_t)(T + 1) * ssz * sizeof(double));
  double* Dt = (double*)malloc(ssz * sizeof(double));
  double* u = (double*)malloc((size_t)dv * sizeof(double));
  double* w = (double*)malloc((size_t)dv * sizeof(double));
  double* unit = (double*)malloc(2 * (size_t)dk * sizeof(double));  /* k^, q^ of a token */
  if (c->init)
    memcpy(states, c->init + ((size_t)n * H + h) * ssz, ssz * sizeof(double));
  else
    memset(states, 0, ssz * sizeof(double));
  for (int64_t t = 0; t < T; ++t) {
    const size_t th = (size_t)(t0 + t) * H + h, tq = (size_t)(t0 + t) * Hqk + hq;
    double* St = states + (size_t)(t + 1) * ssz;
    memcpy(St, states + (size_t)t * ssz, ssz * sizeof(double));
    apply_gate(St, exp(c->g[th]), dk, dv);
    apply_householder(St, maybe_unit(c->k + tq * dk, dk, c->l2norm, unit), c->v + th * dv, c->beta[th], dk, dv);
  }
  if (c->d_fin)
    memcpy(Dt, c->d_fin + ((size_t)n * H + h) * ssz, ssz * sizeof(double));
  else
    memset(Dt, 0, ssz * sizeof(double));
  for (int64_t t = T - 1; t >= 0; --t) {
    const size_t th = (size_t)(t0 + t) * H + h, tq = (size_t)(t0 + t) * Hqk + hq;
    const double* q = maybe_unit(c->q + tq * dk, dk, c->l2norm, unit + dk);
    const double* k = maybe_unit(c->k + tq * dk, dk, c->l2norm, unit);
    const double* v = c->v + th * dv;
    const double* dO = c->d_o + th * dv;
    const double alpha = exp(c->g[th]), beta = c->beta[th];
    const double* St = states + (size_t)(t + 1) * ssz;  /* S_t */
    const double* Sp = states + (size_t)t * ssz;        /* S_{t-1} */
    double* dq = c->dq + th * dk;                       /* per value head */
    double* dkv = c->dkk + th * dk;
    /* D += scale q dO^T;  dq = scale S_t dO */
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i) Dt[(size_t)j * dk + i] += c->scale * q[i] * dO[j];
    for (int i = 0; i < dk; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dv; ++j) acc += St[(size_t)j * dk + i] * dO[j];
      dq[i] = c->scale * acc;
    }
    /* u = S~^T k, w = D^T k */
    for (int j = 0; j < dv; ++j) {
      double pu = 0.0, pw = 0.0;
      for (int i = 0; i < dk; ++i) {
        pu += alpha * Sp[(size_t)j * dk + i] * k[i];
        pw += Dt[(size_t)j * dk + i] * k[i];
      }
      u[j] = pu;
      w[j] = pw;
    }
    double db = 0.0, uw = 0.0, ds = 0.0;
    for (int j = 0; j < dv; ++j) {
      c->dvv[th * dv + j] = beta * w[j];
      db += w[j] * (v[j] - u[j]);
      uw += u[j] * w[j];
    }
    c->dbeta[th] = db;
    for (int i = 0; i < dk; ++i) {
      double a = 0.0, b = 0.0;
      for (int j = 0; j < dv; ++j) {
        a += Dt[(size_t)j * dk + i] * (v[j] - u[j]);
        b += alpha * Sp[(size_t)j * dk + i] * w[j];
      }
      dkv[i] = beta * (a - b);
    }
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i) ds += Dt[(size_t)j * dk + i] * alpha * Sp[(size_t)j * dk + i];
    c->dg[th] = ds - beta * uw;
    /* D <- alpha (D - beta k w^T) */
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i)
        Dt[(size_t)j * dk + i] = alpha * (Dt[(size_t)j * dk + i] - beta * k[i] * w[j]);
    if (c->l2norm) { /* through the normalisation, from the raw vectors */
      unit_backward(c->q + tq * dk, dq, dk);
      unit_backward(c->k + tq * dk, dkv, dk);
    }
  }
  if (c->d_init) memcpy(c->d_init + ((size_t)n * H + h) * ssz, Dt, ssz * sizeof(double));
  free(unit);
  free(w);
  free(u);
  free(Dt);
  free(states);
}

/*
 * Inputs as for gdn_oracle_prefill (l2norm != 0: q and k normalised per token), plus
 * d_o [total_T, H, dv] and d_final_state
 * [N, H, dv, dk] or NULL (zero). Outputs: dq, dk [total_T, H, dk] per VALUE head
 * (the caller sums the heads that share a q/k head), dv [total_T, H, dv], dg and
 * dbeta [total_T, H], d_initial_state [N, H, dv, dk] or NULL.
 * Returns the number of threads used, or a negative value on bad arguments.
 */
int gdn_oracle_prefill_backward(const double* q, const double* k, const double* v, const double* g,
                                const double* beta, const int64_t* cu_seqlens, int N, int H, int Hqk,
                                int dk, int dv, double scale, int l2norm, const double* init, const double* d_o,
                                const double* d_final_state, double* dq, double* dk_out, double* dv_out,
                                double* dg, double* dbeta, double* d_init, int nthreads) {
  if (N < 0 || H <= 0 || Hqk <= 0 || H % Hqk != 0 || dk <= 0 || dv <= 0 || !cu_seqlens || !d_o) return -1;
  if (cu_seqlens[0] != 0) return -1;
  for (int n = 0; n < N; ++n)
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
  backward_ctx c = {q, k, v, g, beta, cu_seqlens, H, Hqk, dk, dv, l2norm, scale, init, d_o, d_final_state,
                    dq, dk_out, dv_out, dg, dbeta, d_init};
  return run_items(N * H, nthreads, backward_item, &c);
}
