"""Seeded synthetic inputs for the gated delta rule workloads.

This module is shared by the tests, the benchmark and the CPU oracle runs. It
only draws random numbers and shapes them; it holds none of the recurrence's
arithmetic. Every tensor is drawn from one ``torch.Generator`` seeded per call,
in a fixed order (documented on each function), on the device the caller names.
The same seed gives different values on CPU and CUDA generators; the GPU path and
the oracle therefore always consume the same materialised tensors (copied between
devices), never two independent draws.

Distributions follow the workload definitions of the gated delta rule
benchmarks (decode, chunked prefill, varlen prefill, gated delta product):

* q, k ~ N(0, 1) per element, then L2-normalised per token (and per Householder
  key) in fp32, then rounded to the input dtype (bf16 round-to-nearest-even).
* v ~ N(0, 1), rounded to the input dtype.
* beta = sigmoid(N(0, 1)) in fp32.
* g = -U(lo, hi) in fp32 (log-space gate, alpha = exp(g)); default (0.01, 0.5).
* recurrent states ~ N(0, 0.1^2) in fp32 (std 0.1), stored K-last [.., dv, dk].
* decode slot ids: the first B entries of a seeded permutation of the pool.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

DEFAULT_G_RANGE = (0.01, 0.5)


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    """L2-normalise the last axis in fp32 (input recipe: normalised q and k)."""
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True).clamp_min(1e-30)


def _draw_normal(shape, gen, device) -> torch.Tensor:
    return torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32)


def _draw_gate(shape, gen, device, g_range) -> torch.Tensor:
    lo, hi = float(g_range[0]), float(g_range[1])
    u = torch.rand(tuple(shape), generator=gen, device=device, dtype=torch.float32)
    return -(lo + (hi - lo) * u)


def _draw_beta(shape, gen, device) -> torch.Tensor:
    return torch.sigmoid(_draw_normal(shape, gen, device))


@dataclasses.dataclass
class DecodeInputs:
    q: torch.Tensor          # [B, T, H, dk] in dtype
    k: torch.Tensor          # [B, T, H, n_h, dk] in dtype
    v: torch.Tensor          # [B, T, H, n_h, dv] in dtype
    g: torch.Tensor          # [B, T, H] fp32
    beta: torch.Tensor       # [B, T, H, n_h] fp32
    pool: torch.Tensor       # [num_slots, H, dv, dk] fp32
    slot_ids: torch.Tensor   # [B] int32
    scale: float


def decode_inputs(B: int, T: int, H: int, dk: int, dv: int, n_h: int, num_slots: int,
                  seed: int = 0, dtype=torch.bfloat16, device="cpu",
                  g_range=DEFAULT_G_RANGE, state_std: float = 0.1, H_qk: Optional[int] = None,
                  normalize_qk: bool = True) -> DecodeInputs:
    """Inputs of one (multi-token, multi-Householder) decode step. q and k have
    H_qk heads (default H); with normalize_qk=False they are left as N(0, 1) draws
    (for the in-kernel normalisation).

    Draw order: q, k, v, beta, g, pool, slot permutation.
    """
    if B > num_slots:
        raise ValueError("B must not exceed num_slots (slot ids are distinct)")
    H_qk = H if H_qk is None else H_qk
    unit = _unit_rows if normalize_qk else (lambda x: x)
    gen = _gen(seed, device)
    q = unit(_draw_normal((B, T, H_qk, dk), gen, device)).to(dtype)
    k = unit(_draw_normal((B, T, H_qk, n_h, dk), gen, device)).to(dtype)
    v = _draw_normal((B, T, H, n_h, dv), gen, device).to(dtype)
    beta = _draw_beta((B, T, H, n_h), gen, device)
    g = _draw_gate((B, T, H), gen, device, g_range)
    pool = _draw_normal((num_slots, H, dv, dk), gen, device) * state_std
    perm = torch.randperm(num_slots, generator=gen, device=device)
    slot_ids = perm[:B].to(torch.int32)
    return DecodeInputs(q, k, v, g, beta, pool, slot_ids, 1.0 / float(dk) ** 0.5)


@dataclasses.dataclass
class PrefillInputs:
    q: torch.Tensor                    # [total_T, H, dk] in dtype
    k: torch.Tensor                    # [total_T, H, dk] in dtype
    v: torch.Tensor                    # [total_T, H, dv] in dtype
    g: torch.Tensor                    # [total_T, H] fp32
    beta: torch.Tensor                 # [total_T, H] fp32
    cu_seqlens: torch.Tensor           # [N + 1] int32
    initial_state: Optional[torch.Tensor]  # [N, H, dv, dk] fp32 or None
    scale: float

    @property
    def seqlens(self):
        c = self.cu_seqlens.cpu().tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def varlen_lengths(n: int, lo: int, hi: int, seed: int = 0) -> list:
    """n sequence lengths ~ U{lo..hi} (inclusive), from a CPU generator so that
    shapes never depend on the device."""
    gen = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def prefill_inputs(seqlens: Sequence[int], H: int, dk: int, dv: int, seed: int = 0,
                   dtype=torch.bfloat16, device="cpu", g_range=DEFAULT_G_RANGE,
                   with_initial_state: bool = True, state_std: float = 0.1, H_qk: Optional[int] = None,
                   normalize_qk: bool = True) -> PrefillInputs:
    """Packed varlen prefill inputs for sequences of the given lengths. q and k have
    H_qk heads (default H); with normalize_qk=False they are left as N(0, 1) draws.

    Draw order: q, k, v, beta, g, initial state.
    """
    seqlens = [int(x) for x in seqlens]
    total = sum(seqlens)
    H_qk = H if H_qk is None else H_qk
    unit = _unit_rows if normalize_qk else (lambda x: x)
    gen = _gen(seed, device)
    q = unit(_draw_normal((total, H_qk, dk), gen, device)).to(dtype)
    k = unit(_draw_normal((total, H_qk, dk), gen, device)).to(dtype)
    v = _draw_normal((total, H, dv), gen, device).to(dtype)
    beta = _draw_beta((total, H), gen, device)
    g = _draw_gate((total, H), gen, device, g_range)
    init = None
    if with_initial_state:
        init = _draw_normal((len(seqlens), H, dv, dk), gen, device) * state_std
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    if seqlens:
        cu[1:] = torch.tensor(seqlens, dtype=torch.int64).cumsum(0).to(torch.int32)
    return PrefillInputs(q, k, v, g, beta, cu.to(device), init, 1.0 / float(dk) ** 0.5)


# ---------------------------------------------------------------------------
# The five benchmark workloads (shapes and distributions), by name.
# ---------------------------------------------------------------------------

def tiny_prefill(device="cpu", seed=0) -> PrefillInputs:
    """B=1, H=2, T=64, dk=dv=32, fp32 inputs, zero initial state (chunk 16)."""
    return prefill_inputs([64], 2, 32, 32, seed=seed, dtype=torch.float32, device=device,
                          with_initial_state=False)


def decode_b64_h32(device="cpu", seed=0) -> DecodeInputs:
    """T=1 decode: B=64, H=32, dk=dv=128, pool of 256 slots."""
    return decode_inputs(64, 1, 32, 128, 128, 1, 256, seed=seed, device=device)


def prefill_b4_t8192_h16(device="cpu", seed=0) -> PrefillInputs:
    """Chunked prefill: 4 sequences of 8192 tokens, H=16, dk=dv=128 (chunk 64)."""
    return prefill_inputs([8192] * 4, 16, 128, 128, seed=seed, device=device)


def varlen32_h32(device="cpu", seed=0) -> PrefillInputs:
    """Varlen prefill: 32 sequences, lengths ~U{64..16384}, H=32, dk=dv=128."""
    return prefill_inputs(varlen_lengths(32, 64, 16384, seed), 32, 128, 128, seed=seed,
                          device=device)


def longseq_b1_t65536_h4(device="cpu", seed=0) -> PrefillInputs:
    """Low-parallelism prefill: 1 sequence of 65536 tokens, H=4, dk=dv=128."""
    return prefill_inputs([65536], 4, 128, 128, seed=seed, device=device)


def gdp_b128_h32_t4_nh2(device="cpu", seed=0) -> DecodeInputs:
    """Gated delta product decode: B=128, H=32, T=4, n_h=2, pool of 512 slots."""
    return decode_inputs(128, 4, 32, 128, 128, 2, 512, seed=seed, device=device)
