"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each test names what fixes the expected value: exact rational brute force over
explicit update matrices, a hand-derived closed form, an algebraic invariant, an
independent chunked (WY) form, or an identity between the oracle's entry points.
Shapes use dk != dv wherever a transposed state could hide.
"""
import functools
import math
import os
from fractions import Fraction as Fr

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_58_b200 import inputs
from tests.chunked_ref import prefill_chunked

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _rand_prefill(rng, T, H, dk, dv, g_lo=0.01, g_hi=0.5):
    q = _unit(rng.standard_normal((T, H, dk)))
    k = _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -rng.uniform(g_lo, g_hi, (T, H))
    return q, k, v, g, beta


def _prefill(lib):
    return functools.partial(oracle.prefill, lib=lib)


def _decode(lib):
    return functools.partial(oracle.decode, lib=lib)


PIN_CHECKS = []  # filled at the end of the module: every check_* function


def _relerr(x, r):
    return np.abs(x - r).max() / max(np.abs(r).max(), 1e-300)


# ---------------------------------------------------------------- golden fixture

def _read_fixture(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()])
    return vals


def check_hand_two_token_fixture(lib=None):
    fx = _read_fixture("hand_two_tokens.txt")
    k = fx["k"].reshape(2, 1, 2)
    v = fx["v"].reshape(2, 1, 2)
    q = fx["q"].reshape(2, 1, 2)
    beta = fx["beta"].reshape(2, 1)
    g = np.log(fx["alpha"]).reshape(2, 1)
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, [0, 2], None, scale=1.0)
    np.testing.assert_allclose(o.reshape(-1), fx["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fin.reshape(-1), fx["final_state_kv_last"], rtol=0, atol=1e-14)


def test_hand_two_token_fixture():
    check_hand_two_token_fixture()


# ---------------------------------------------------------------- exact rationals

def _frac_mat(rows, cols, rng, den=8):
    return [[Fr(int(rng.integers(-den, den + 1)), den) for _ in range(cols)] for _ in range(rows)]


def _mm(a, b):
    return [[sum(a[i][t] * b[t][j] for t in range(len(b))) for j in range(len(b[0]))]
            for i in range(len(a))]


def _madd(a, b):
    return [[a[i][j] + b[i][j] for j in range(len(a[0]))] for i in range(len(a))]


def _outer(x, y):
    return [[xi * yj for yj in y] for xi in x]


def _eye(n):
    return [[Fr(int(i == j)) for j in range(n)] for i in range(n)]


def _householder(k, beta):
    kk = _outer(k, k)
    n = len(k)
    return [[(Fr(int(i == j)) - beta * kk[i][j]) for j in range(n)] for i in range(n)]


def _scal(a, s):
    return [[s * x for x in row] for row in a]


def check_exact_rational_brute_force_gdn(lib=None):
    """S_T = (A_T..A_1) S0 + sum_t (A_T..A_{t+1}) B_t with A_t = alpha_t (I - beta_t k_t k_t^T),
    B_t = beta_t k_t v_t^T, built as explicit matrices in exact rationals; o_t = scale S_t^T q_t."""
    rng = _rng(1)
    dk, dv, T = 3, 4, 6
    S0 = _frac_mat(dk, dv, rng)
    ks = [[Fr(int(rng.integers(-4, 5)), 4) for _ in range(dk)] for _ in range(T)]
    vs = [[Fr(int(rng.integers(-6, 7)), 3) for _ in range(dv)] for _ in range(T)]
    qs = [[Fr(int(rng.integers(-4, 5)), 2) for _ in range(dk)] for _ in range(T)]
    betas = [Fr(int(rng.integers(0, 9)), 8) for _ in range(T)]
    alphas = [Fr(int(rng.integers(1, 9)), 8) for _ in range(T)]
    scale = Fr(1, 3)
    A = [_scal(_householder(ks[t], betas[t]), alphas[t]) for t in range(T)]
    B = [_scal(_outer(ks[t], vs[t]), betas[t]) for t in range(T)]
    S_t, outs = [], []
    for t in range(T):
        # closed form for the state after token t, from the explicit products
        prod = _eye(dk)
        for s in range(t, -1, -1):
            prod = _mm(prod, A[s])
        S = _mm(prod, S0)
        for s in range(t + 1):
            tail = _eye(dk)
            for r in range(t, s, -1):
                tail = _mm(tail, A[r])
            S = _madd(S, _mm(tail, B[s]))
        S_t.append(S)
        outs.append([scale * sum(S[i][j] * qs[t][i] for i in range(dk)) for j in range(dv)])
    f = lambda m: np.array([[float(x) for x in row] for row in m])
    q = f(qs).reshape(T, 1, dk)
    k = f(ks).reshape(T, 1, dk)
    v = f(vs).reshape(T, 1, dv)
    beta = np.array([float(b) for b in betas]).reshape(T, 1)
    g = np.log(np.array([float(a) for a in alphas])).reshape(T, 1)
    init = f(S0).T.reshape(1, 1, dv, dk)
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, [0, T], init, scale=float(scale))
    exp_o = f(outs).reshape(T, 1, dv)
    exp_S = f(S_t[-1]).T.reshape(1, 1, dv, dk)
    assert _relerr(o, exp_o) < 1e-13
    assert _relerr(fin, exp_S) < 1e-13


def test_exact_rational_brute_force_gdn():
    check_exact_rational_brute_force_gdn()


def check_exact_rational_brute_force_gdp(lib=None):
    """Gated delta product: per token one gate alpha_t, then n_h Householder updates in order,
    then one output. Explicit affine maps per token in exact rationals."""
    rng = _rng(2)
    dk, dv, T, nh = 3, 2, 3, 2
    S0 = _frac_mat(dk, dv, rng)
    ks = [[[Fr(int(rng.integers(-4, 5)), 4) for _ in range(dk)] for _ in range(nh)] for _ in range(T)]
    vs = [[[Fr(int(rng.integers(-6, 7)), 3) for _ in range(dv)] for _ in range(nh)] for _ in range(T)]
    qs = [[Fr(int(rng.integers(-4, 5)), 2) for _ in range(dk)] for _ in range(T)]
    betas = [[Fr(int(rng.integers(0, 9)), 8) for _ in range(nh)] for _ in range(T)]
    alphas = [Fr(int(rng.integers(1, 9)), 8) for _ in range(T)]
    scale = Fr(1, 2)
    S = S0
    outs = []
    for t in range(T):
        S = _scal(S, alphas[t])
        for j in range(nh):
            S = _madd(_mm(_householder(ks[t][j], betas[t][j]), S),
                      _scal(_outer(ks[t][j], vs[t][j]), betas[t][j]))
        outs.append([scale * sum(S[i][c] * qs[t][i] for i in range(dk)) for c in range(dv)])
    f = lambda m: np.array(m, dtype=object).astype(float)
    q = f(qs).reshape(1, T, 1, dk)
    k = f(ks).reshape(1, T, 1, nh, dk)
    v = f(vs).reshape(1, T, 1, nh, dv)
    beta = f(betas).reshape(1, T, 1, nh)
    g = np.log(f(alphas)).reshape(1, T, 1)
    pool = np.zeros((3, 1, dv, dk))
    pool[2, 0] = f(S0).T
    o, new_pool, _ = _decode(lib)(q, k, v, g, beta, pool, np.array([2], np.int32),
                                   scale=float(scale))
    assert _relerr(o.reshape(T, dv), f(outs)) < 1e-13
    assert _relerr(new_pool[2, 0], f(S).T) < 1e-13
    assert np.array_equal(new_pool[:2], pool[:2])


def test_exact_rational_brute_force_gdp():
    check_exact_rational_brute_force_gdp()


# ---------------------------------------------------------------- closed forms / invariants

def check_beta0_alpha1_leaves_state(lib=None):
    rng = _rng(3)
    T, H, dk, dv = 9, 2, 5, 7
    q, k, v, _, _ = _rand_prefill(rng, T, H, dk, dv)
    init = rng.standard_normal((1, H, dv, dk))
    o, fin, _ = _prefill(lib)(q, k, v, np.zeros((T, H)), np.zeros((T, H)), [0, T], init)
    assert np.array_equal(fin, init)
    exp_o = np.einsum("hji,thi->thj", init[0], q) / np.sqrt(dk)
    assert _relerr(o, exp_o) < 1e-13


def test_beta0_alpha1_leaves_state():
    check_beta0_alpha1_leaves_state()


def check_alpha0_gives_rank_one_write(lib=None):
    rng = _rng(4)
    T, H, dk, dv = 5, 2, 4, 6
    q, k, v, _, beta = _rand_prefill(rng, T, H, dk, dv)
    init = rng.standard_normal((1, H, dv, dk))
    g = np.full((T, H), -np.inf)
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, [0, T], init)
    exp_fin = beta[-1][:, None, None] * np.einsum("hj,hi->hji", v[-1], k[-1])
    assert _relerr(fin[0], exp_fin) < 1e-14
    qk = np.einsum("thi,thi->th", q, k)
    exp_o = (beta * qk)[..., None] * v / np.sqrt(dk)
    assert _relerr(o, exp_o) < 1e-13


def test_alpha0_gives_rank_one_write():
    check_alpha0_gives_rank_one_write()


def check_single_token_from_zero(lib=None):
    rng = _rng(5)
    H, dk, dv = 3, 6, 4
    q, k, v, g, beta = _rand_prefill(rng, 1, H, dk, dv)
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, [0, 1], None, scale=0.25)
    exp_fin = beta[0][:, None, None] * np.einsum("hj,hi->hji", v[0], k[0])
    assert _relerr(fin[0], exp_fin) < 1e-14
    exp_o = 0.25 * (beta[0] * np.einsum("hi,hi->h", q[0], k[0]))[:, None] * v[0]
    assert _relerr(o[0], exp_o) < 1e-13


def test_single_token_from_zero():
    check_single_token_from_zero()


def check_unit_key_overwrites_one_row(lib=None):
    """k = e_i, beta = 1, alpha = 1: S[i, :] := v, every other row of S untouched (exactly)."""
    rng = _rng(6)
    dk, dv, i = 5, 3, 2
    init = rng.standard_normal((1, 1, dv, dk))
    k = np.zeros((1, 1, dk))
    k[0, 0, i] = 1.0
    v = rng.standard_normal((1, 1, dv))
    q = rng.standard_normal((1, 1, dk))
    o, fin, _ = _prefill(lib)(q, k, v, np.zeros((1, 1)), np.ones((1, 1)), [0, 1], init)
    exp = init.copy()
    exp[0, 0, :, i] = v[0, 0]
    assert np.array_equal(fin, exp)


def test_unit_key_overwrites_one_row():
    check_unit_key_overwrites_one_row()


def check_householder_reflection_preserves_norm(lib=None):
    """beta = 2, |k| = 1, alpha = 1, v = 0: each step is a reflection, Frobenius norm kept."""
    rng = _rng(7)
    T, dk, dv = 12, 8, 5
    k = _unit(rng.standard_normal((T, 1, dk)))
    init = rng.standard_normal((1, 1, dv, dk))
    _, fin, _ = _prefill(lib)(np.zeros((T, 1, dk)), k, np.zeros((T, 1, dv)), np.zeros((T, 1)),
                               np.full((T, 1), 2.0), [0, T], init)
    assert abs(np.linalg.norm(fin) - np.linalg.norm(init)) < 1e-12 * np.linalg.norm(init)
    assert _relerr(fin, init) > 1e-3  # and the state did change


def test_householder_reflection_preserves_norm():
    check_householder_reflection_preserves_norm()


def check_contraction_norm_bound(lib=None):
    """beta in [0,1], |k| = 1: |S_t|_F <= alpha_t |S_{t-1}|_F + beta_t |v_t|."""
    rng = _rng(8)
    T, dk, dv = 20, 6, 4
    q, k, v, g, beta = _rand_prefill(rng, T, 1, dk, dv, 0.0, 0.3)
    S = rng.standard_normal((1, 1, dv, dk))
    for t in range(T):
        sl = slice(t, t + 1)
        _, S_new, _ = _prefill(lib)(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, 1], S)
        bound = np.exp(g[t, 0]) * np.linalg.norm(S) + beta[t, 0] * np.linalg.norm(v[t, 0])
        assert np.linalg.norm(S_new) <= bound * (1 + 1e-12)
        S = S_new


def test_contraction_norm_bound():
    check_contraction_norm_bound()


# ---------------------------------------------------------------- chunked form

@pytest.mark.parametrize("chunk,g_lo,g_hi", [(16, 0.01, 0.5), (64, 0.0, 0.01), (64, 0.01, 0.5),
                                             (32, 0.0, 0.0)])
def test_chunked_form_equals_sequential(chunk, g_lo, g_hi):
    rng = _rng(9)
    lens = [70, 128, 1, 0, 200]
    H, dk, dv = 2, 16, 12
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta = _rand_prefill(rng, int(cu[-1]), H, dk, dv, g_lo, g_hi)
    init = rng.standard_normal((len(lens), H, dv, dk)) * 0.1
    o_ref, f_ref, _ = oracle.prefill(q, k, v, g, beta, cu, init)
    for transfer in (False, True):
        o, f = prefill_chunked(q, k, v, g, beta, cu, init, chunk=chunk, use_transfer=transfer)
        assert _relerr(o, o_ref) < 1e-10
        assert _relerr(f, f_ref) < 1e-10


# ---------------------------------------------------------------- identities between entry points

def test_gdp_with_one_householder_is_gdn():
    rng = _rng(10)
    B, T, H, dk, dv = 2, 5, 3, 6, 4
    q, k, v, g, beta = (np.stack(x) for x in zip(*[_rand_prefill(rng, T, H, dk, dv) for _ in range(B)]))
    pool = rng.standard_normal((4, H, dv, dk))
    slots = np.array([3, 1], np.int32)
    o_d, pool_d, _ = oracle.decode(q, k[:, :, :, None], v[:, :, :, None], g, beta[..., None],
                                   pool, slots)
    for b in range(B):
        o_p, f_p, _ = oracle.prefill(q[b], k[b], v[b], g[b], beta[b], [0, T],
                                     pool[slots[b]][None])
        assert np.array_equal(o_d[b], o_p)
        assert np.array_equal(pool_d[slots[b]], f_p[0])


def check_gdp_equals_gdn_over_flattened_substeps(lib=None):
    """n_h Householders under one gate == GDN over T*n_h sub-steps with log-gates (g_t, 0, ..)
    and the token's output read at its last sub-step."""
    rng = _rng(11)
    T, H, dk, dv, nh = 4, 2, 5, 3, 3
    q = _unit(rng.standard_normal((1, T, H, dk)))
    k = _unit(rng.standard_normal((1, T, H, nh, dk)))
    v = rng.standard_normal((1, T, H, nh, dv))
    beta = rng.uniform(0, 1, (1, T, H, nh))
    g = -rng.uniform(0.01, 0.5, (1, T, H))
    pool = rng.standard_normal((1, H, dv, dk))
    o_d, pool_d, _ = _decode(lib)(q, k, v, g, beta, pool, np.array([0], np.int32))
    kf = k[0].transpose(0, 2, 1, 3).reshape(T * nh, H, dk)
    vf = v[0].transpose(0, 2, 1, 3).reshape(T * nh, H, dv)
    bf = beta[0].transpose(0, 2, 1).reshape(T * nh, H)
    gf = np.zeros((T, nh, H))
    gf[:, 0] = g[0]
    gf = gf.reshape(T * nh, H)
    qf = np.repeat(q[0], nh, axis=0)
    o_p, f_p, _ = _prefill(lib)(qf, kf, vf, gf, bf, [0, T * nh], pool)
    assert np.array_equal(o_p[nh - 1::nh], o_d[0])
    assert np.array_equal(f_p, pool_d)


def test_gdp_equals_gdn_over_flattened_substeps():
    check_gdp_equals_gdn_over_flattened_substeps()


def test_decode_T_times_equals_prefill():
    rng = _rng(12)
    T, H, dk, dv = 7, 2, 8, 6
    q, k, v, g, beta = _rand_prefill(rng, T, H, dk, dv)
    pool = rng.standard_normal((2, H, dv, dk))
    o_p, f_p, _ = oracle.prefill(q, k, v, g, beta, [0, T], pool[1:])
    cur = pool
    for t in range(T):
        o_t, cur, _ = oracle.decode(q[t][None, None], k[t][None, None, :, None],
                                    v[t][None, None, :, None], g[t][None, None],
                                    beta[t][None, None, :, None], cur, np.array([1], np.int32))
        assert np.array_equal(o_t[0, 0], o_p[t])
    assert np.array_equal(cur[1], f_p[0])
    assert np.array_equal(cur[0], pool[0])


def test_prefill_resume_from_final_state():
    rng = _rng(13)
    T1, T2, H, dk, dv = 11, 6, 2, 5, 4
    q, k, v, g, beta = _rand_prefill(rng, T1 + T2, H, dk, dv)
    init = rng.standard_normal((1, H, dv, dk))
    o_all, f_all, _ = oracle.prefill(q, k, v, g, beta, [0, T1 + T2], init)
    a, b = slice(0, T1), slice(T1, T1 + T2)
    o1, f1, _ = oracle.prefill(q[a], k[a], v[a], g[a], beta[a], [0, T1], init)
    o2, f2, _ = oracle.prefill(q[b], k[b], v[b], g[b], beta[b], [0, T2], f1)
    assert np.array_equal(np.concatenate([o1, o2]), o_all)
    assert np.array_equal(f2, f_all)


def test_varlen_equals_separate_calls_and_empty_sequence():
    rng = _rng(14)
    lens = [5, 0, 9, 1]
    H, dk, dv = 2, 4, 3
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta = _rand_prefill(rng, int(cu[-1]), H, dk, dv)
    init = rng.standard_normal((len(lens), H, dv, dk))
    o, fin, _ = oracle.prefill(q, k, v, g, beta, cu, init)
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        o_n, f_n, _ = oracle.prefill(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, L], init[n:n + 1])
        assert np.array_equal(o[sl], o_n)
        assert np.array_equal(fin[n], f_n[0])
    assert np.array_equal(fin[1], init[1])  # empty sequence: state passes through


def test_decode_negative_slot_and_untouched_slots():
    rng = _rng(15)
    B, H, dk, dv = 3, 2, 4, 5
    q, k, v, g, beta = (np.stack(x) for x in zip(*[_rand_prefill(rng, 1, H, dk, dv) for _ in range(B)]))
    pool = rng.standard_normal((6, H, dv, dk))
    slots = np.array([4, -1, 0], np.int32)
    o, new_pool, _ = oracle.decode(q, k[:, :, :, None], v[:, :, :, None], g, beta[..., None], pool, slots)
    assert np.all(o[1] == 0)
    for s in (1, 2, 3, 5):
        assert np.array_equal(new_pool[s], pool[s])
    assert not np.array_equal(new_pool[4], pool[4])


def test_oracle_consumes_generator_inputs_exactly():
    """The oracle sees the generator's bf16 values upcast exactly (no renormalisation)."""
    inp = inputs.prefill_inputs([33], 2, 16, 8, seed=0)
    q64 = oracle.f64(inp.q)
    assert np.array_equal(q64, inp.q.to(torch.float64).numpy())
    o, fin, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state)
    o2, fin2 = prefill_chunked(oracle.f64(inp.q), oracle.f64(inp.k), oracle.f64(inp.v),
                               oracle.f64(inp.g), oracle.f64(inp.beta), [0, 33],
                               oracle.f64(inp.initial_state), chunk=16)
    assert _relerr(o, o2) < 1e-10 and _relerr(fin, fin2) < 1e-10


def test_oracle_threads_do_not_change_results():
    rng = _rng(16)
    lens = [40, 17, 3]
    H, dk, dv = 3, 8, 8
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, g, beta = _rand_prefill(rng, int(cu[-1]), H, dk, dv)
    o1, f1, n1 = oracle.prefill(q, k, v, g, beta, cu, None, nthreads=1)
    o4, f4, n4 = oracle.prefill(q, k, v, g, beta, cu, None, nthreads=4)
    assert n1 == 1 and n4 == 4
    assert np.array_equal(o1, o4) and np.array_equal(f1, f4)


def test_oracle_rejects_bad_cu_seqlens():
    q = np.zeros((4, 1, 2))
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, np.zeros((4, 1)), np.zeros((4, 1)), [0, 3, 2, 4])
    with pytest.raises(ValueError):
        oracle.prefill(q, q, q, np.zeros((4, 1)), np.zeros((4, 1)), [1, 4])


# ---------------------------------------------------------------- grouped heads, q/k normalisation

def check_grouped_heads_equal_repeated_qk_heads(lib=None):
    """H value heads over H_qk q/k heads (value head h reads q/k head h // (H // H_qk))
    give exactly the results of the one-to-one call whose q/k heads are repeated in
    place H // H_qk times; prefill and (multi-Householder) decode."""
    rng = _rng(31)
    T, Hqk, r, dk, dv = 9, 2, 3, 4, 3
    H = Hqk * r
    q = _unit(rng.standard_normal((T, Hqk, dk)))
    k = _unit(rng.standard_normal((T, Hqk, dk)))
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -rng.uniform(0.0, 0.3, (T, H))
    init = 0.1 * rng.standard_normal((2, H, dv, dk))
    cu = [0, 4, T]
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, cu, init, scale=0.7)
    o1, fin1, _ = _prefill(lib)(np.repeat(q, r, axis=1), np.repeat(k, r, axis=1), v, g, beta, cu, init, scale=0.7)
    assert np.array_equal(o, o1) and np.array_equal(fin, fin1)
    B, TT, nh, slots = 2, 2, 2, 3
    qd = _unit(rng.standard_normal((B, TT, Hqk, dk)))
    kd = _unit(rng.standard_normal((B, TT, Hqk, nh, dk)))
    vd = rng.standard_normal((B, TT, H, nh, dv))
    bd = 1 / (1 + np.exp(-rng.standard_normal((B, TT, H, nh))))
    gd = -rng.uniform(0.0, 0.3, (B, TT, H))
    pool = 0.1 * rng.standard_normal((slots, H, dv, dk))
    sid = np.array([2, 0], np.int32)
    od, pd, _ = _decode(lib)(qd, kd, vd, gd, bd, pool, sid, scale=0.7)
    od1, pd1, _ = _decode(lib)(np.repeat(qd, r, axis=2), np.repeat(kd, r, axis=2), vd, gd, bd, pool, sid, scale=0.7)
    assert np.array_equal(od, od1) and np.array_equal(pd, pd1)


def check_l2norm_is_scale_invariant(lib=None):
    """With the q/k normalisation on, positive per-token scalings of q and k change
    nothing (up to rounding), and the result equals the plain recurrence on q and k
    normalised beforehand; prefill and decode."""
    rng = _rng(32)
    T, H, dk, dv = 7, 2, 5, 3
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -rng.uniform(0.0, 0.3, (T, H))
    init = 0.1 * rng.standard_normal((1, H, dv, dk))
    sq = rng.uniform(0.1, 10.0, (T, H, 1))
    sk = rng.uniform(0.1, 10.0, (T, H, 1))
    o, fin, _ = _prefill(lib)(q, k, v, g, beta, [0, T], init, scale=0.5, l2norm=True)
    o2, fin2, _ = _prefill(lib)(q * sq, k * sk, v, g, beta, [0, T], init, scale=0.5, l2norm=True)
    o3, fin3, _ = _prefill(lib)(_unit(q), _unit(k), v, g, beta, [0, T], init, scale=0.5)
    for x, y in ((o, o2), (fin, fin2), (o, o3), (fin, fin3)):
        assert _relerr(x, y) < 1e-13
    # the normalisation matters: un-normalised keys give a different state
    o4, _, _ = _prefill(lib)(q * sq, k * sk, v, g, beta, [0, T], init, scale=0.5)
    assert _relerr(o4, o) > 1e-3
    B, TT, nh = 2, 2, 2
    qd = rng.standard_normal((B, TT, H, dk))
    kd = rng.standard_normal((B, TT, H, nh, dk))
    vd = rng.standard_normal((B, TT, H, nh, dv))
    bd = 1 / (1 + np.exp(-rng.standard_normal((B, TT, H, nh))))
    gd = -rng.uniform(0.0, 0.3, (B, TT, H))
    pool = 0.1 * rng.standard_normal((2, H, dv, dk))
    sid = np.array([1, 0], np.int32)
    od, pd, _ = _decode(lib)(qd, kd, vd, gd, bd, pool, sid, scale=0.5, l2norm=True)
    od2, pd2, _ = _decode(lib)(qd * 3.0, kd * rng.uniform(0.1, 10.0, (B, TT, H, nh, 1)), vd, gd, bd, pool, sid,
                               scale=0.5, l2norm=True)
    od3, pd3, _ = _decode(lib)(_unit(qd), _unit(kd), vd, gd, bd, pool, sid, scale=0.5)
    for x, y in ((od, od2), (pd, pd2), (od, od3), (pd, pd3)):
        assert _relerr(x, y) < 1e-13


def test_grouped_heads_equal_repeated_qk_heads():
    check_grouped_heads_equal_repeated_qk_heads()


def test_l2norm_is_scale_invariant():
    check_l2norm_is_scale_invariant()


def test_oracle_rejects_head_counts_that_do_not_divide():
    rng = _rng(33)
    q = rng.standard_normal((3, 2, 4))
    v = rng.standard_normal((3, 3, 4))
    with pytest.raises(ValueError):
        oracle.prefill(q, q, v, np.zeros((3, 3)), np.ones((3, 3)), [0, 3])


# ---------------------------------------------------------------- per-token states (speculative verify)

def check_token_states_are_prefix_decodes(lib=None):
    """The state recorded after token t equals the pool state left by a decode of
    the first t + 1 tokens alone (bitwise: the same arithmetic), the last one equals
    the final pool state, and restoring the state after token t and decoding the
    remaining tokens reproduces the full step (the rollback use)."""
    rng = _rng(34)
    B, T, H, nh, dk, dv, slots = 3, 4, 2, 2, 4, 3, 5
    q = _unit(rng.standard_normal((B, T, H, dk)))
    k = _unit(rng.standard_normal((B, T, H, nh, dk)))
    v = rng.standard_normal((B, T, H, nh, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, nh))))
    g = -rng.uniform(0.0, 0.4, (B, T, H))
    pool = 0.1 * rng.standard_normal((slots, H, dv, dk))
    sid = np.array([4, -1, 1], np.int32)
    o, fin, _, ts = _decode(lib)(q, k, v, g, beta, pool, sid, scale=0.6, token_states=True)
    for b in (0, 2):
        assert np.array_equal(ts[b, T - 1], fin[sid[b]])
    assert not ts[1].any()
    for t in range(T):
        _, pre, _ = _decode(lib)(q[:, :t + 1], k[:, :t + 1], v[:, :t + 1], g[:, :t + 1], beta[:, :t + 1],
                                 pool, sid, scale=0.6)
        for b in (0, 2):
            assert np.array_equal(ts[b, t], pre[sid[b]])
    t = 1
    rolled = pool.copy()
    for b in (0, 2):
        rolled[sid[b]] = ts[b, t]
    o2, fin2, _ = _decode(lib)(q[:, t + 1:], k[:, t + 1:], v[:, t + 1:], g[:, t + 1:], beta[:, t + 1:],
                               rolled, sid, scale=0.6)
    assert _relerr(o2[[0, 2]], o[[0, 2], t + 1:]) < 1e-14 and _relerr(fin2, fin) < 1e-14


def test_token_states_are_prefix_decodes():
    check_token_states_are_prefix_decodes()


# ---------------------------------------------------------------- affine in the start state (context parallelism)

def check_prefill_is_affine_in_the_initial_state(lib=None):
    """A sequence's final state is affine in its start state, S_end = M S_0 + H,
    with H the final state from a zero start and M (K-last: M^T) the final state
    from the identity with the values set to zero; and running slice after slice
    equals composing the slices' (M, H) pairs (what context parallelism exchanges).
    Pinned against direct oracle runs from arbitrary start states."""
    rng = _rng(35)
    T, H, d = 23, 2, 4
    q, k, v, g, beta = _rand_prefill(rng, T, H, d, d, 0.0, 0.3)
    pref = _prefill(lib)
    ident = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()

    def pair(sl):
        _, Ht, _ = pref(q[sl], k[sl], v[sl], g[sl], beta[sl], [0, sl.stop - sl.start], None, scale=0.5)
        _, Mt, _ = pref(q[sl], k[sl], np.zeros_like(v[sl]), g[sl], beta[sl], [0, sl.stop - sl.start], ident,
                        scale=0.5)
        return Mt[0], Ht[0]  # K-last: [H, dv, dk] and [H, dk, dk]

    S0 = 0.1 * rng.standard_normal((1, H, d, d))
    Mt, Ht = pair(slice(0, T))
    _, fin, _ = pref(q, k, v, g, beta, [0, T], S0, scale=0.5)
    assert _relerr(np.einsum("hij,hjk->hik", S0[0], Mt) + Ht, fin[0]) < 1e-13
    # slices of 7, 9 and 7 tokens, composed in order from S0
    S = S0[0]
    for sl in (slice(0, 7), slice(7, 16), slice(16, T)):
        Mt, Ht = pair(sl)
        S = np.einsum("hij,hjk->hik", S, Mt) + Ht
    assert _relerr(S, fin[0]) < 1e-13


def test_prefill_is_affine_in_the_initial_state():
    check_prefill_is_affine_in_the_initial_state()


# ---------------------------------------------------------------- backward (reverse-mode derivatives)

def _backward_case(seed, l2norm=False):
    """Three sequences (one empty), two value heads over one q/k head, dk != dv, an
    initial state, upstream derivatives R (outputs) and Q (final state) of the loss
    L = sum(R * o) + sum(Q * S_final). Keys are unit vectors, except with l2norm,
    where keys and queries have norms in (0.5, 2) and are normalised by the method."""
    rng = _rng(seed)
    lens, H, Hqk, dk, dv = [4, 0, 3], 2, 1, 3, 2
    T = sum(lens)
    q = rng.standard_normal((T, Hqk, dk))
    k = _unit(rng.standard_normal((T, Hqk, dk)))
    if l2norm:
        k = k * rng.uniform(0.5, 2.0, (T, Hqk, 1))
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -rng.uniform(0.05, 0.6, (T, H))
    init = rng.standard_normal((len(lens), H, dv, dk)) * 0.5
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    R = rng.standard_normal((T, H, dv))
    Q = rng.standard_normal((len(lens), H, dv, dk))
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=init), cu, R, Q


def _loss(lib, x, cu, R, Q, l2norm=False):
    o, fin, _ = oracle.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, x["initial_state"], scale=0.7,
                               lib=lib, l2norm=l2norm)
    return float((R * o).sum() + (Q * fin).sum())


def check_backward_matches_central_differences(lib=None):
    """Every derivative of the backward pass against central finite differences of
    the oracle's forward (fp64, step 1e-6) on every input entry, without and with the
    q/k normalisation."""
    for l2norm in (False, True):
        x, cu, R, Q = _backward_case(40, l2norm)
        d = oracle.prefill_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, R, x["initial_state"], Q,
                                    scale=0.7, lib=lib, l2norm=l2norm)
        names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", initial_state="d_initial_state")
        eps = 1e-6
        for name, gname in names.items():
            fd = np.zeros_like(x[name])
            for idx in np.ndindex(x[name].shape):
                xp = {kk: vv.copy() for kk, vv in x.items()}
                xm = {kk: vv.copy() for kk, vv in x.items()}
                xp[name][idx] += eps
                xm[name][idx] -= eps
                fd[idx] = (_loss(lib, xp, cu, R, Q, l2norm) - _loss(lib, xm, cu, R, Q, l2norm)) / (2 * eps)
            assert _relerr(d[gname], fd) < 1e-6, (l2norm, name, _relerr(d[gname], fd))


def check_backward_matches_autograd_of_a_plain_torch_forward(lib=None):
    """The derivatives against torch.autograd through a plain fp64 PyTorch forward
    of the recurrence written here (gate, Householder write, output per token), with
    the q/k normalisation."""
    import torch
    x, cu, R, Q = _backward_case(41, l2norm=True)
    tx = {kk: torch.tensor(vv, requires_grad=True) for kk, vv in x.items()}
    H, Hqk = x["v"].shape[1], x["q"].shape[1]
    loss = torch.zeros((), dtype=torch.float64)
    for n in range(len(cu) - 1):
        for h in range(H):
            hq = h // (H // Hqk)
            S = tx["initial_state"][n, h].T  # dk x dv
            for t in range(int(cu[n]), int(cu[n + 1])):
                kt, qt, vt = tx["k"][t, hq], tx["q"][t, hq], tx["v"][t, h]
                kt, qt = kt / torch.linalg.vector_norm(kt), qt / torch.linalg.vector_norm(qt)
                S = torch.exp(tx["g"][t, h]) * S
                S = S - tx["beta"][t, h] * torch.outer(kt, kt @ S) + tx["beta"][t, h] * torch.outer(kt, vt)
                loss = loss + (torch.tensor(R[t, h]) * (0.7 * (S.T @ qt))).sum()
            loss = loss + (torch.tensor(Q[n, h]) * S.T).sum()
    loss.backward()
    d = oracle.prefill_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], cu, R, x["initial_state"], Q, scale=0.7,
                                lib=lib, l2norm=True)
    names = dict(q="dq", k="dk", v="dv", g="dg", beta="dbeta", initial_state="d_initial_state")
    for name, gname in names.items():
        ref = tx[name].grad.numpy()
        assert _relerr(d[gname], ref) < 1e-12, (name, _relerr(d[gname], ref))


def test_backward_matches_central_differences():
    check_backward_matches_central_differences()


def test_backward_matches_autograd_of_a_plain_torch_forward():
    check_backward_matches_autograd_of_a_plain_torch_forward()


PIN_CHECKS.extend(v for k, v in sorted(globals().items()) if k.startswith("check_"))
