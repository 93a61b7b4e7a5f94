"""Independent fp64 chunked (WY / UT) form of the gated delta rule, test-only.

Used to pin the chunk algebra that the GPU prefill relies on against the
token-sequential oracle: both must agree to ~1e-10 in fp64. Per chunk of C
tokens with start state S0 (dk x dv), cumulative log gate G_r = sum_{i<=r} g_i,
gamma_r = exp(G_r):

    A_ij  = beta_i exp(G_i - G_j) k_i^T k_j            (j < i, else 0)
    T     = (I + A)^{-1}
    W     = T diag(beta * gamma) K                      (C x dk)
    U~    = T diag(beta) V                              (C x dv)
    U     = U~ - W S0                                   (the corrected values)
    O     = scale [diag(gamma) Q S0 + (L o exp(G_r - G_i) o Q K^T) U]
    S_C   = gamma_C S0 + K~^T U,   K~ = diag(exp(G_C - G_i)) K

and the affine transfer form S_C = M S0 + H with M = gamma_C I - K~^T W,
H = K~^T U~ (the transfer and local state objects of the chunk/context-parallel
fixup on the FlashInfer PR #3866 page, section 2).
"""
import numpy as np


def chunk_step(S0, q, k, v, g, beta, scale):
    C = k.shape[0]
    G = np.cumsum(g)
    gam = np.exp(G)
    D = np.exp(G[:, None] - G[None, :])
    A = np.tril(beta[:, None] * D * (k @ k.T), -1)
    T = np.linalg.inv(np.eye(C) + A)
    W = T @ ((beta * gam)[:, None] * k)
    Ut = T @ (beta[:, None] * v)
    U = Ut - W @ S0
    P = np.tril(D * (q @ k.T))
    O = scale * (gam[:, None] * (q @ S0) + P @ U)
    Kt = np.exp(G[-1] - G)[:, None] * k
    S = gam[-1] * S0 + Kt.T @ U
    M = gam[-1] * np.eye(k.shape[1]) - Kt.T @ W
    Hc = Kt.T @ Ut
    return O, S, M, Hc


def prefill_chunked(q, k, v, g, beta, cu_seqlens, initial_state=None, chunk=64, scale=None,
                    use_transfer=False):
    """Chunked fp64 prefill. Shapes as the oracle: q,k [T,H,dk], v [T,H,dv],
    g,beta [T,H], states [N,H,dv,dk] (K-last). With use_transfer the state is
    passed by S <- M S + H instead of the direct update."""
    q, k, v, g, beta = (np.asarray(a, np.float64) for a in (q, k, v, g, beta))
    cu = [int(x) for x in cu_seqlens]
    total, H, dk = q.shape
    dv = v.shape[-1]
    N = len(cu) - 1
    scale = 1.0 / np.sqrt(dk) if scale is None else scale
    o = np.zeros((total, H, dv))
    fin = np.zeros((N, H, dv, dk))
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if initial_state is None else \
                np.asarray(initial_state[n, h], np.float64).T.copy()
            for c0 in range(cu[n], cu[n + 1], chunk):
                c1 = min(c0 + chunk, cu[n + 1])
                sl = slice(c0, c1)
                O, S_next, M, Hc = chunk_step(S, q[sl, h], k[sl, h], v[sl, h], g[sl, h],
                                              beta[sl, h], scale)
                o[sl, h] = O
                S = M @ S + Hc if use_transfer else S_next
            fin[n, h] = S.T
    return o, fin
