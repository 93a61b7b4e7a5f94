"""ctypes binding of libgdn.so (include/gdn.h). Argument marshalling only.

Every compute step runs in the CUDA library; this module turns torch tensors
into device pointers and sizes, passes the current CUDA stream, and raises
GdnError on a non-OK status. There is no CPU fallback: if libgdn.so is missing
the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdn.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "gdn.h")

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_WORKSPACE = 3
GDN_ERR_CUDA = 4
GDN_ERR_DEVICE_DATA = 5

GDN_BF16 = 0
GDN_F32 = 1

GDN_PREFILL_AUTO = 0
GDN_PREFILL_FUSED = 1
GDN_PREFILL_TRANSFER = 2
GDN_PREFILL_SEQUENTIAL = 3

GDN_QK_L2NORM = 0x1

GDN_DEVERR_SLOT_OUT_OF_RANGE = 0x1
GDN_DEVERR_BAD_CU_SEQLENS = 0x2
GDN_DEVERR_TIMEOUT = 0x4

_lib = None
_lock = threading.Lock()


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"gdn status {status}: {message}")
        self.status = status


def declared_functions(header: str = HEADER):
    """Names of the functions include/gdn.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_58_b200.build` "
                    "(the library has no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                     ctypes.c_size_t)
            L.gdn_decode.restype = i32
            u32 = ctypes.c_uint32
            L.gdn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                     f32, u32, i32, i32, vp]
            L.gdn_decode_mtp.restype = i32
            L.gdn_decode_mtp.argtypes = [vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                         i32, f32, u32, i32, i32, i32, vp]
            L.gdn_chunk_prefill_workspace_size.restype = sz
            L.gdn_chunk_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
            L.gdn_chunk_prefill.restype = i32
            L.gdn_chunk_prefill.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, i32, i32,
                                            i32, f32, u32, i32, i32, i32, vp, sz, vp]
            L.gdn_chunk_prefill_static_scratch.restype = i32
            L.gdn_chunk_prefill_static_scratch.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, i32,
                                                           i32, i32, i32, i32, f32, u32, i32, i32, vp]
            L.gdn_last_error.restype = ctypes.c_char_p
            L.gdn_last_error.argtypes = []
            L.gdn_get_device_error.restype = i32
            L.gdn_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
            L.gdn_cp_local_state.restype = i32
            L.gdn_cp_local_state.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, i32, i32, i32, i32, i32, u32,
                                             i32, vp, sz, vp]
            L.gdn_cp_local_state_workspace_size.restype = i32
            L.gdn_cp_local_state_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32,
                                                            ctypes.POINTER(ctypes.c_size_t)]
            L.gdn_cp_finish.restype = i32
            L.gdn_cp_finish.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, i32, i32, i32, i32, i32, f32, u32,
                                        i32, i32, vp, sz, vp]
            L.gdn_cp_combine.restype = i32
            L.gdn_cp_combine.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
            L.gdn_chunk_prefill_backward_workspace_size.restype = i32
            L.gdn_chunk_prefill_backward_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32,
                                                                    ctypes.POINTER(ctypes.c_size_t)]
            L.gdn_chunk_prefill_backward.restype = i32
            L.gdn_chunk_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp, vp, vp, vp,
                                                     vp, vp, i32, i32, i32, i32, i32, f32, u32, i32, vp, sz, vp]
            L.gdn_selftest_wait_timeout.restype = i32
            L.gdn_selftest_wait_timeout.argtypes = [u32, vp]
            L.gdn_version.restype = ctypes.c_char_p
            L.gdn_version.argtypes = []
            _lib = L
    return _lib


def gdn_last_error() -> str:
    return lib().gdn_last_error().decode()


def gdn_version() -> str:
    return lib().gdn_version().decode()


def _check(status: int):
    if status != GDN_OK:
        raise GdnError(status, gdn_last_error())


def gdn_get_device_error() -> int:
    """Read and clear the sticky device error word (synchronises the device)."""
    flags = ctypes.c_uint32(0)
    st = lib().gdn_get_device_error(ctypes.byref(flags))
    if st not in (GDN_OK, GDN_ERR_DEVICE_DATA):
        _check(st)
    return int(flags.value)


def gdn_cp_local_state_workspace_size(N, total_T, H, dk, dv, chunk=64) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().gdn_cp_local_state_workspace_size(N, total_T, H, dk, dv, chunk, ctypes.byref(out)))
    return int(out.value)


def gdn_cp_local_state(q, k, v, g, beta, cu_seqlens, local_state, transfer, chunk=64, stream=None, l2norm=False,
                       workspace=None):
    """Context parallelism, step 1 (see include/gdn.h): the slice's local state H and
    transfer M^T, both [N,H,dv,dk] fp32 K-last. `workspace` (uint8 CUDA tensor) is
    allocated through torch when None (pass one with a raw stream handle)."""
    import torch
    total_T, H_qk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu_seqlens.numel() - 1
    if workspace is None:
        if stream is not None and not isinstance(stream, torch.cuda.Stream):
            raise ValueError("gdn_cp_local_state: pass `workspace` when `stream` is a raw handle")
        need = gdn_cp_local_state_workspace_size(N, total_T, H, dk, dv, chunk)
        ctx = torch.cuda.stream(stream) if stream is not None else _nullcontext()
        with ctx:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check(lib().gdn_cp_local_state(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, total_T,
                                    _ptr(local_state), _ptr(transfer), H, H_qk, dk, dv, chunk,
                                    GDN_QK_L2NORM if l2norm else 0, _dtype_code(q), _ptr(workspace),
                                    workspace.numel(), _stream_ptr(stream, q.device)))


def gdn_cp_finish(q, k, v, g, beta, cu_seqlens, o, workspace, start_state=None, final_state=None, chunk=64,
                  scale=None, stream=None, l2norm=False):
    """Context parallelism, step 4 (see include/gdn.h): the slice's outputs and final
    state from the rank's start state, reusing the segments that gdn_cp_local_state
    left in `workspace` (the same slice, shapes and workspace)."""
    total_T, H_qk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu_seqlens.numel() - 1
    if scale is None:
        scale = dk ** -0.5
    _check(lib().gdn_cp_finish(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, total_T,
                               _ptr(start_state), _ptr(final_state), _ptr(o), H, H_qk, dk, dv, chunk, float(scale),
                               GDN_QK_L2NORM if l2norm else 0, _dtype_code(q), _dtype_code(o), _ptr(workspace),
                               workspace.numel(), _stream_ptr(stream, q.device)))
    return o


def gdn_cp_combine(local_states, transfers, rank, start_state, initial_state=None, stream=None):
    """Context parallelism, step 3: rank `rank`'s start state [N,H,dv,dk] from the
    rank-major pairs [ranks,N,H,dv,dk] of ranks 0..rank-1 and the initial state."""
    ranks, N, H, dv, dk = local_states.shape
    _check(lib().gdn_cp_combine(_ptr(local_states), _ptr(transfers), ranks, rank, N, H, dk, dv, _ptr(initial_state),
                                _ptr(start_state), _stream_ptr(stream, start_state.device)))


def gdn_selftest_wait_timeout(wait_us: int, stream=None):
    """Enqueue the bounded-wait self-test kernel (see include/gdn.h); afterwards
    gdn_get_device_error() reports GDN_DEVERR_TIMEOUT."""
    _check(lib().gdn_selftest_wait_timeout(int(wait_us), stream))


# ---------------------------------------------------------------- torch marshalling

def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream, device):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def gdn_decode(q, k, v, g, beta, state_pool, slot_ids, o, scale=None, stream=None, l2norm=False):
    """One decode step (see include/gdn.h). Shapes:
    q [B,T,H_qk,dk], k [B,T,H_qk,n_h,dk], v [B,T,H,n_h,dv], g [B,T,H], beta [B,T,H,n_h],
    state_pool [num_slots,H,dv,dk] fp32 (updated in place), slot_ids [B] int32, o [B,T,H,dv].
    l2norm: normalise q and k per token inside the kernel (GDN_QK_L2NORM)."""
    B, T, H_qk, dk = q.shape
    H, n_h, dv = v.shape[2], k.shape[3], v.shape[4]
    if scale is None:
        scale = dk ** -0.5
    st = lib().gdn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                          state_pool.shape[0], _ptr(slot_ids), _ptr(o), B, T, H, H_qk, dk, dv, n_h,
                          float(scale), GDN_QK_L2NORM if l2norm else 0, _dtype_code(q), _dtype_code(o),
                          _stream_ptr(stream, q.device))
    _check(st)
    return o


def gdn_decode_mtp(q, k, v, g, beta, state_pool, slot_ids, o, token_states, update_pool=True, scale=None,
                   stream=None, l2norm=False):
    """gdn_decode that also writes the state after every token into token_states
    [B,T,H,dv,dk] fp32 (the rollback points of a speculative verification); with
    update_pool=False the pool is only read. Other shapes as gdn_decode."""
    B, T, H_qk, dk = q.shape
    H, n_h, dv = v.shape[2], k.shape[3], v.shape[4]
    if scale is None:
        scale = dk ** -0.5
    st = lib().gdn_decode_mtp(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                              state_pool.shape[0], _ptr(slot_ids), _ptr(o), _ptr(token_states), B, T, H, H_qk,
                              dk, dv, n_h, float(scale), GDN_QK_L2NORM if l2norm else 0, 1 if update_pool else 0,
                              _dtype_code(q), _dtype_code(o), _stream_ptr(stream, q.device))
    _check(st)
    return o


def gdn_chunk_prefill_workspace_size(N, total_T, H, dk, dv, chunk, algo=GDN_PREFILL_AUTO) -> int:
    n = lib().gdn_chunk_prefill_workspace_size(N, total_T, H, dk, dv, chunk, algo)
    if n == ctypes.c_size_t(-1).value:
        raise GdnError(GDN_ERR_INVALID_ARG, gdn_last_error())
    return int(n)


def gdn_chunk_prefill(q, k, v, g, beta, cu_seqlens, o, initial_state=None, final_state=None,
                      chunk=64, scale=None, algo=GDN_PREFILL_AUTO, workspace=None, stream=None, l2norm=False):
    """Chunked varlen prefill (see include/gdn.h). Shapes: q,k [total_T,H_qk,dk], v [total_T,H,dv],
    g,beta [total_T,H] fp32, cu_seqlens [N+1] int32 (device), initial/final_state [N,H,dv,dk] fp32,
    o [total_T,H,dv]. `workspace` is a uint8 CUDA tensor; when None one of the required size is
    allocated through torch for this call, on `stream` when one is given, so torch orders any
    reuse of that memory after the call's kernels; a raw stream handle needs an explicit
    `workspace`. l2norm: normalise q and k per token inside the kernels."""
    import torch
    total_T, H_qk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu_seqlens.numel() - 1
    if scale is None:
        scale = dk ** -0.5
    need = gdn_chunk_prefill_workspace_size(N, total_T, H, dk, dv, chunk, algo)
    if workspace is None and need > 0:
        if stream is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        elif isinstance(stream, torch.cuda.Stream):
            with torch.cuda.stream(stream):  # the caching allocator orders reuse on this stream
                workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        else:
            raise ValueError("gdn_chunk_prefill: pass `workspace` when `stream` is a raw handle")
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() if workspace is not None else 0
    st = lib().gdn_chunk_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N,
                                 total_T, _ptr(initial_state), _ptr(final_state), _ptr(o), H, H_qk, dk, dv,
                                 chunk, float(scale), GDN_QK_L2NORM if l2norm else 0, _dtype_code(q),
                                 _dtype_code(o), algo, ws_ptr, ws_bytes, _stream_ptr(stream, q.device))
    _check(st)
    return o


def gdn_chunk_prefill_backward_workspace_size(N, total_T, H, dk, dv, chunk=64) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().gdn_chunk_prefill_backward_workspace_size(N, total_T, H, dk, dv, chunk, ctypes.byref(out)))
    return int(out.value)


def gdn_chunk_prefill_backward(q, k, v, g, beta, cu_seqlens, d_o, initial_state=None, d_final_state=None,
                               chunk=64, scale=None, workspace=None, stream=None, grads=None, l2norm=False):
    """Derivatives of a loss with respect to the prefill's inputs (see include/gdn.h),
    given d_o [total_T,H,dv] (q's dtype) and d_final_state [N,H,dv,dk] fp32 or None.
    Returns dict(dq, dk [total_T,H_qk,dk], dv [total_T,H,dv], dg, dbeta [total_T,H],
    d_initial_state [N,H,dv,dk]), fp32; `grads` may pass these tensors in. The
    workspace (uint8 CUDA tensor) is allocated through torch when None. l2norm: the
    forward normalised q and k per token (GDN_QK_L2NORM)."""
    import torch
    total_T, H_qk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu_seqlens.numel() - 1
    if scale is None:
        scale = dk ** -0.5
    dev = q.device
    if d_o.dtype != q.dtype:
        raise TypeError("gdn_chunk_prefill_backward: d_o must have q's dtype")
    if grads is None:
        f = dict(dtype=torch.float32, device=dev)
        grads = dict(dq=torch.empty((total_T, H_qk, dk), **f), dk=torch.empty((total_T, H_qk, dk), **f),
                     dv=torch.empty((total_T, H, dv), **f), dg=torch.empty((total_T, H), **f),
                     dbeta=torch.empty((total_T, H), **f), d_initial_state=torch.empty((N, H, dv, dk), **f))
    need = gdn_chunk_prefill_backward_workspace_size(N, total_T, H, dk, dv, chunk)
    if workspace is None:
        if stream is not None and not isinstance(stream, torch.cuda.Stream):
            raise ValueError("gdn_chunk_prefill_backward: pass `workspace` when `stream` is a raw handle")
        ctx = torch.cuda.stream(stream) if stream is not None else _nullcontext()
        with ctx:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = lib().gdn_chunk_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, total_T, _ptr(initial_state),
        _ptr(d_o), _ptr(d_final_state), _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
        _ptr(grads["dg"]), _ptr(grads["dbeta"]), _ptr(grads.get("d_initial_state")), H, H_qk, dk, dv, chunk,
        float(scale), GDN_QK_L2NORM if l2norm else 0, _dtype_code(q), _ptr(workspace), workspace.numel(),
        _stream_ptr(stream, dev))
    _check(st)
    return grads


def _nullcontext():
    import contextlib
    return contextlib.nullcontext()


def gdn_chunk_prefill_static_scratch(q, k, v, g, beta, cu_seqlens, o, initial_state=None, final_state=None,
                                     chunk=64, scale=None, stream=None, l2norm=False):
    """Transfer prefill whose scratch is the library's own 32 MiB device array, for
    callers that cannot allocate device memory at call time (see include/gdn.h).
    Same shapes as gdn_chunk_prefill; nothing is allocated, here or in the library."""
    total_T, H_qk, dk = q.shape
    H, dv = v.shape[1], v.shape[-1]
    N = cu_seqlens.numel() - 1
    if scale is None:
        scale = dk ** -0.5
    st = lib().gdn_chunk_prefill_static_scratch(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), N, total_T, _ptr(initial_state),
        _ptr(final_state), _ptr(o), H, H_qk, dk, dv, chunk, float(scale), GDN_QK_L2NORM if l2norm else 0,
        _dtype_code(q), _dtype_code(o), _stream_ptr(stream, q.device))
    _check(st)
    return o
