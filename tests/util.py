"""Comparison helpers shared by the GPU parity tests.

With GDN_PARITY_LOG set to a file path, every comparison appends one JSON line
(what, normwise relative error, max abs error, tolerance) to that file."""
import json
import os

import numpy as np
import torch

# Normwise tolerance for fp32 results: max|x - r| / max|r|.
TOL = 2e-3


def relerr(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = max(float(np.abs(ref).max()), 1e-30) if ref.size else 1.0
    return float(np.abs(x - ref).max() / denom) if ref.size else 0.0


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, np.float64)


def assert_close(x, ref, tol=TOL, what=""):
    """fp32 result: normwise relative error <= tol. bf16 result: additionally each
    element within one bf16 ulp of the reference plus tol * max|ref| (the output's
    own rounding is up to half an ulp)."""
    is_bf16 = isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16
    xa, ra = to64(x), to64(ref)
    assert xa.shape == ra.shape, (what, xa.shape, ra.shape)
    if not ra.size:
        return
    scale = max(float(np.abs(ra).max()), 1e-30)
    log = os.environ.get("GDN_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"what": what, "relerr": relerr(xa, ra), "max_abs": float(np.abs(xa - ra).max()),
                                "tol": tol, "bf16": is_bf16, "n": int(ra.size)}) + "\n")
    if is_bf16:
        ulp = np.maximum(np.abs(ra), 1e-38)
        ulp = 2.0 ** (np.floor(np.log2(ulp)) - 7)
        bound = ulp + tol * scale
        bad = np.abs(xa - ra) > bound
        assert not bad.any(), f"{what}: {int(bad.sum())} bf16 elements off; max err {np.abs(xa - ra).max():.3e}"
    else:
        e = relerr(xa, ra)
        assert e <= tol, f"{what}: normwise relative error {e:.3e} > {tol}"


_CACHE = {}


def cached(key, fn):
    """fn() once per test process under `key` (the oracle's full-size results and
    the inputs they were computed from are reused by several tests)."""
    if key not in _CACHE:
        _CACHE[key] = fn()
    return _CACHE[key]
