"""Prefill backward (gdn_chunk_prefill_backward) against the fp64 oracle's
reverse-mode pass on the same seeded inputs: every derivative (q, k, v, g, beta,
initial state), element by element within the normwise tolerance."""
import pytest
import torch

import oracle
import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import inputs
from tests.util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _upstream(inp, seed, dtype):
    gen = torch.Generator().manual_seed(seed)
    T, H, dv = inp.v.shape
    N = inp.cu_seqlens.numel() - 1
    d_o = torch.randn((T, H, dv), generator=gen).to(dtype)
    d_fin = torch.randn((N, H, dv, inp.q.shape[-1]), generator=gen) * 0.1
    return d_o, d_fin


def _run(inp, d_o, d_fin, chunk, l2norm=False):
    dev = [x.to(DEV) if x is not None else None
           for x in (inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state, d_o, d_fin)]
    q, k, v, g, beta, cu, init, do, dfin = dev
    out = gdn.gdn_chunk_prefill_backward(q, k, v, g, beta, cu, do, initial_state=init, d_final_state=dfin,
                                         chunk=chunk, scale=inp.scale, l2norm=l2norm)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error() == 0
    return out


def _check(inp, d_o, d_fin, chunk, what, l2norm=False):
    out = _run(inp, d_o, d_fin, chunk, l2norm)
    ref = oracle.prefill_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, d_o, inp.initial_state,
                                  d_fin, scale=inp.scale, l2norm=l2norm)
    for name in ("dq", "dk", "dv", "dg", "dbeta", "d_initial_state"):
        assert_close(out[name], ref[name], what=f"{what} {name}")


@pytest.mark.parametrize("chunk", [1, 16, 64])
@pytest.mark.parametrize("g_range", [(0.01, 0.5), (0.0, 0.01)])
def test_backward_varlen_grouped_heads_bf16(chunk, g_range):
    inp = inputs.prefill_inputs([200, 0, 65, 130], 4, 128, 128, seed=90, g_range=g_range, H_qk=2)
    d_o, d_fin = _upstream(inp, 91, torch.bfloat16)
    _check(inp, d_o, d_fin, chunk, f"bwd chunk={chunk} g={g_range}")


@pytest.mark.parametrize("d", [32, 64])
def test_backward_small_heads_fp32(d):
    inp = inputs.prefill_inputs([97, 33], 3, d, d, seed=92 + d, dtype=torch.float32, g_range=(0.0, 0.05))
    d_o, d_fin = _upstream(inp, 93, torch.float32)
    _check(inp, d_o, d_fin, 16, f"bwd d={d}")


def test_backward_without_initial_or_final_state_and_chunk_beyond_the_sequence():
    inp = inputs.prefill_inputs([70, 3], 2, 128, 128, seed=94, g_range=(0.0, 0.02), with_initial_state=False)
    d_o, _ = _upstream(inp, 95, torch.bfloat16)
    _check(inp, d_o, None, 256, "bwd no states")


def test_backward_long_sequence_weak_decay():
    inp = inputs.prefill_inputs([4096], 2, 128, 128, seed=96, g_range=(0.0, 0.002))
    d_o, d_fin = _upstream(inp, 97, torch.bfloat16)
    _check(inp, d_o, d_fin, 64, "bwd long")


def test_backward_leaves_no_trace_between_calls():
    """Two calls in a row on reused memory: dv and the initial-state derivative,
    written directly, are bitwise equal; dq, dk, dg and dbeta, summed over column
    blocks with fp32 atomics in whatever order they arrive, agree to rounding."""
    inp = inputs.prefill_inputs([150, 40], 2, 128, 128, seed=98, g_range=(0.0, 0.05))
    d_o, d_fin = _upstream(inp, 99, torch.bfloat16)
    a = _run(inp, d_o, d_fin, 32)
    b = _run(inp, d_o, d_fin, 32)
    for name in ("dv", "d_initial_state"):
        assert torch.equal(a[name], b[name]), name
    for name in ("dq", "dk", "dg", "dbeta"):
        err = (a[name] - b[name]).abs().max() / b[name].abs().max()
        assert err < 1e-5, (name, float(err))


@pytest.mark.parametrize("chunk", [16, 64])
def test_backward_through_the_qk_normalisation(chunk):
    """Raw (unnormalised) q and k with GDN_QK_L2NORM, grouped heads, varlen."""
    inp = inputs.prefill_inputs([180, 0, 77], 4, 128, 128, seed=100, g_range=(0.0, 0.05), H_qk=2,
                                normalize_qk=False)
    d_o, d_fin = _upstream(inp, 101, torch.bfloat16)
    _check(inp, d_o, d_fin, chunk, f"bwd l2norm chunk={chunk}", l2norm=True)


def test_backward_through_the_qk_normalisation_small_heads_fp32():
    inp = inputs.prefill_inputs([90, 41], 2, 64, 64, seed=102, dtype=torch.float32, g_range=(0.0, 0.05),
                                normalize_qk=False)
    d_o, d_fin = _upstream(inp, 103, torch.float32)
    _check(inp, d_o, d_fin, 16, "bwd l2norm d=64", l2norm=True)


@pytest.mark.parametrize("chunk", [3, 7])
def test_backward_odd_checkpoint_intervals_one_shared_qk_head(chunk):
    """Checkpoint intervals that divide no sequence length (the staging order then has
    a short last chunk), all value heads on one q/k head, d=64 bf16."""
    inp = inputs.prefill_inputs([50, 1, 64, 33], 3, 64, 64, seed=104 + chunk, g_range=(0.0, 0.1), H_qk=1)
    d_o, d_fin = _upstream(inp, 105, torch.bfloat16)
    _check(inp, d_o, d_fin, chunk, f"bwd chunk={chunk} H_qk=1")


def test_backward_fp32_inputs_full_head_size():
    inp = inputs.prefill_inputs([129, 64, 5], 2, 128, 128, seed=106, dtype=torch.float32, g_range=(0.0, 0.05))
    d_o, d_fin = _upstream(inp, 107, torch.float32)
    _check(inp, d_o, d_fin, 5, "bwd fp32 d=128 chunk=5")


def test_backward_full_size_bench_workload_sampled_heads():
    """The bench's backward workload (B=4 x 8192, H=16, bf16, checkpoints every 16
    tokens) in the launch configuration the bench times; three (sequence, head) pairs,
    each its own chain (H_qk = H), against the oracle run on that pair alone."""
    import bench
    inp, d_o, d_fin, chunk, _ = bench.backward_inputs("backward", torch.device(DEV), 0)
    assert inp.q.shape[1] == inp.v.shape[1]
    out = gdn.gdn_chunk_prefill_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, d_o,
                                         initial_state=inp.initial_state, d_final_state=d_fin, chunk=chunk,
                                         scale=inp.scale)
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error() == 0
    cu = inp.cu_seqlens.cpu().tolist()
    for n, h in ((0, 0), (1, 7), (3, 15)):
        a, b = cu[n], cu[n + 1]

        def tok(x):
            return x[a:b, h:h + 1].cpu()

        def state(x):
            return x[n:n + 1, h:h + 1].cpu()

        ref = oracle.prefill_backward(tok(inp.q), tok(inp.k), tok(inp.v), tok(inp.g), tok(inp.beta),
                                      torch.tensor([0, b - a], dtype=torch.int32), tok(d_o),
                                      state(inp.initial_state), state(d_fin), scale=inp.scale)
        got = {name: tok(out[name]) for name in ("dq", "dk", "dv", "dg", "dbeta")}
        got["d_initial_state"] = state(out["d_initial_state"])
        for name in ref:
            assert_close(got[name], ref[name], what=f"bwd full size n={n} h={h} {name}")
