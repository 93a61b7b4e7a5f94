"""fp64 CPU oracle for the gated delta rule (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library and its Python binding
never import it. The arithmetic lives in ``gdn_oracle.c`` (plain sequential fp64
loops, one token at a time; see its header for the definition it follows); this
module only compiles it with gcc, converts arrays to fp64 and marshals pointers.

Parity pins: the oracle is checked, in ``tests/test_oracle_pins.py``, against
exact rational brute force (explicit products of the per-token update matrices),
closed forms (single token, alpha = 0, key overwrite), invariants (beta = 0 and
alpha = 1 leave S unchanged; Householder reflection preserves the Frobenius
norm; the norm bound of a contraction), an independent fp64 chunked (WY) form,
and decode/prefill/varlen consistency identities.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into oracle/libgdn_oracle.so with gcc (-O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-D_POSIX_C_SOURCE=200809L",
               "-o", _LIB_PATH, _SRC, "-lm", "-lpthread"]
        subprocess.check_call(cmd)
    return _LIB_PATH


def load_library(path: str):
    """Load an oracle build from an explicit path (used by the mutation tests)."""
    lib = ctypes.CDLL(path)
    _declare(lib)
    return lib


def _declare(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gdn_oracle_prefill.restype = ctypes.c_int
    lib.gdn_oracle_prefill.argtypes = [dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, ctypes.c_int, dp, dp, dp, ctypes.c_int]
    lib.gdn_oracle_prefill_backward.restype = ctypes.c_int
    lib.gdn_oracle_prefill_backward.argtypes = [dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_double, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                                ctypes.c_int]
    lib.gdn_oracle_decode.restype = ctypes.c_int
    lib.gdn_oracle_decode.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int,
                                      ctypes.POINTER(ctypes.c_int32), dp,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, dp, ctypes.c_int]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            _declare(lib)
            _lib = lib
    return _lib


def f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or torch tensor (bf16/fp32 upcast exactly)."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def prefill(q, k, v, g, beta, cu_seqlens, initial_state=None, scale=None, nthreads=0, lib=None,
            l2norm=False):
    """Sequential fp64 prefill over packed sequences.

    q, k: [total_T, H_qk, dk] (H a multiple of H_qk; value head h reads q/k head
    h // (H // H_qk)); v: [total_T, H, dv]; g, beta: [total_T, H];
    cu_seqlens: [N + 1]; initial_state: [N, H, dv, dk] or None (zero state).
    l2norm: scale q and k to unit length per token (in fp64) before use.
    Returns (o [total_T, H, dv], final_state [N, H, dv, dk], threads_used), fp64.
    """
    lib = lib or _load()
    q, k, v, g, beta = (f64(a) for a in (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(f64(cu_seqlens), dtype=np.int64))
    init = f64(initial_state)
    total_T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu.shape[0] - 1
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    o = np.zeros((total_T, H, dv), np.float64)
    fin = np.zeros((N, H, dv, dk), np.float64)
    rc = lib.gdn_oracle_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                _ptr(cu, ctypes.c_int64), N, H, Hqk, dk, dv, float(scale), int(bool(l2norm)),
                                _ptr(init), _ptr(o), _ptr(fin), int(nthreads))
    if rc < 0:
        raise ValueError("gdn_oracle_prefill: bad arguments")
    return o, fin, rc


def prefill_backward(q, k, v, g, beta, cu_seqlens, d_o, initial_state=None, d_final_state=None, scale=None,
                     nthreads=0, lib=None, l2norm=False):
    """Reverse-mode derivatives of `prefill` (one Householder per token; with l2norm,
    through the per-token q/k normalisation), fp64, token by token (see gdn_oracle.c).

    d_o: [total_T, H, dv]; d_final_state: [N, H, dv, dk] or None (zero).
    Returns dict(dq [total_T, H_qk, dk], dk [total_T, H_qk, dk], dv [total_T, H, dv],
    dg [total_T, H], dbeta [total_T, H], d_initial_state [N, H, dv, dk]). The q/k
    derivatives of value heads that share a q/k head are summed.
    """
    lib = lib or _load()
    q, k, v, g, beta, d_o = (f64(a) for a in (q, k, v, g, beta, d_o))
    cu = np.ascontiguousarray(np.asarray(f64(cu_seqlens), dtype=np.int64))
    init, dfin = f64(initial_state), f64(d_final_state)
    total_T, Hqk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu.shape[0] - 1
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    dq = np.zeros((total_T, H, dk), np.float64)
    dkk = np.zeros((total_T, H, dk), np.float64)
    dvv = np.zeros((total_T, H, dv), np.float64)
    dg = np.zeros((total_T, H), np.float64)
    db = np.zeros((total_T, H), np.float64)
    dinit = np.zeros((N, H, dv, dk), np.float64)
    rc = lib.gdn_oracle_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu, ctypes.c_int64),
                                         N, H, Hqk, dk, dv, float(scale), int(bool(l2norm)), _ptr(init), _ptr(d_o),
                                         _ptr(dfin),
                                         _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db), _ptr(dinit),
                                         int(nthreads))
    if rc < 0:
        raise ValueError("gdn_oracle_prefill_backward: bad arguments")
    grp = H // Hqk
    return dict(dq=dq.reshape(total_T, Hqk, grp, dk).sum(2), dk=dkk.reshape(total_T, Hqk, grp, dk).sum(2),
                dv=dvv, dg=dg, dbeta=db, d_initial_state=dinit)


def decode(q, k, v, g, beta, pool, slot_ids, scale=None, nthreads=0, lib=None, copy_pool=True,
           l2norm=False, token_states=False):
    """Sequential fp64 decode over a slot-indexed pool (the pool copy is updated).

    q: [B, T, H_qk, dk]; k: [B, T, H_qk, nh, dk]; v: [B, T, H, nh, dv]; g: [B, T, H];
    beta: [B, T, H, nh]; pool: [num_slots, H, dv, dk]; slot_ids: [B].
    Returns (o [B, T, H, dv], new_pool, threads_used), fp64. With copy_pool=False an
    fp64 C-contiguous numpy pool is updated in place (no copy). With token_states=True
    returns (o, new_pool, threads_used, states [B, T, H, dv, dk]): the state after
    each token (the rollback points of a speculative verification).
    """
    lib = lib or _load()
    q, k, v, g, beta = (f64(a) for a in (q, k, v, g, beta))
    if copy_pool or not (isinstance(pool, np.ndarray) and pool.dtype == np.float64
                         and pool.flags.c_contiguous):
        pool = f64(pool).copy()
    slots = np.ascontiguousarray(np.asarray(f64(slot_ids), dtype=np.int32))
    B, T, Hqk, dk = q.shape
    H, nh, dv = v.shape[2], v.shape[3], v.shape[4]
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    o = np.zeros((B, T, H, dv), np.float64)
    ts = np.zeros((B, T, H, dv, dk), np.float64) if token_states else None
    rc = lib.gdn_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(pool),
                               pool.shape[0], _ptr(slots, ctypes.c_int32), _ptr(o),
                               B, T, H, Hqk, dk, dv, nh, float(scale), int(bool(l2norm)), _ptr(ts),
                               int(nthreads))
    if rc < 0:
        raise ValueError("gdn_oracle_decode: bad arguments")
    if token_states:
        return o, pool, rc, ts
    return o, pool, rc
