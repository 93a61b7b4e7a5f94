"""GPU parity of gdn_chunk_prefill against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import inputs
from tests.util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"

SEQ = gdn.GDN_PREFILL_SEQUENTIAL


def run_prefill(inp, algo, chunk=64, out_dtype=torch.float32, with_final=True, alias=False,
                workspace=None):
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    g, beta, cu = inp.g.to(DEV), inp.beta.to(DEV), inp.cu_seqlens.to(DEV)
    total, H, dk = q.shape
    dv = v.shape[-1]
    N = cu.numel() - 1
    init = inp.initial_state.to(DEV).clone() if inp.initial_state is not None else None
    o = torch.full((total, H, dv), float("nan"), dtype=out_dtype, device=DEV)
    fin = None
    if with_final:
        fin = init if (alias and init is not None) else torch.full((N, H, dv, dk), float("nan"), device=DEV)
    gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, o, initial_state=init, final_state=fin, chunk=chunk,
                          scale=inp.scale, algo=algo, workspace=workspace)
    torch.cuda.synchronize()
    return o, fin


def oracle_prefill(inp):
    o, fin, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                               inp.initial_state, scale=inp.scale)
    return o, fin


def check(inp, algo, chunk=64, what="", **kw):
    o, fin = run_prefill(inp, algo, chunk=chunk, **kw)
    o_ref, f_ref = oracle_prefill(inp)
    assert_close(o, o_ref, what=f"{what} o")
    if fin is not None:
        assert_close(fin, f_ref, what=f"{what} final state")
    return o, fin


def test_tiny_fp32_sequential():
    """B=1, H=2, T=64, dk=dv=32, fp32 inputs, zero initial state, chunk 16."""
    inp = inputs.tiny_prefill()
    check(inp, gdn.GDN_PREFILL_AUTO, chunk=16, what="tiny")
    check(inp, SEQ, chunk=16, what="tiny seq", out_dtype=torch.bfloat16)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_sequential_varlen_shapes(d):
    lens = [1, 0, 63, 64, 65, 130]
    inp = inputs.prefill_inputs(lens, 3, d, d, seed=d)
    check(inp, SEQ, what=f"seq d={d}")


def test_sequential_no_initial_state_and_alias():
    inp = inputs.prefill_inputs([50, 7], 2, 64, 64, seed=4, with_initial_state=False)
    check(inp, SEQ, what="no init")
    inp2 = inputs.prefill_inputs([50, 7], 2, 64, 64, seed=5)
    check(inp2, SEQ, what="alias", alias=True)


def test_sequential_weak_decay_long():
    inp = inputs.prefill_inputs([1000], 2, 128, 128, seed=6, g_range=(0.0, 0.01))
    check(inp, SEQ, what="weak decay")


def test_bad_cu_seqlens_flagged():
    inp = inputs.prefill_inputs([10, 10], 1, 32, 32, seed=7)
    gdn.gdn_get_device_error()
    inp.cu_seqlens[1] = 25  # > total
    run_prefill(inp, SEQ)
    assert gdn.gdn_get_device_error() & gdn.GDN_DEVERR_BAD_CU_SEQLENS


# ---------------------------------------------------------------- fused tensor-core path

FUSED = gdn.GDN_PREFILL_FUSED


@pytest.mark.parametrize("g_range", [(0.01, 0.5), (0.0, 0.01), (0.0, 0.0)])
def test_fused_varlen_edges(g_range):
    """Lengths around the chunk size, an empty and a one-token sequence; weak and zero
    decay make the state passing between chunks visible in the outputs."""
    lens = [1, 0, 63, 64, 65, 130, 200, 7]
    inp = inputs.prefill_inputs(lens, 3, 128, 128, seed=21, g_range=g_range)
    check(inp, FUSED, what=f"fused {g_range}")


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fused_dtypes(in_dtype, out_dtype):
    inp = inputs.prefill_inputs([300, 65], 2, 128, 128, seed=22, dtype=in_dtype, g_range=(0.0, 0.05))
    check(inp, FUSED, what="fused dtypes", out_dtype=out_dtype)


def test_fused_no_initial_state_and_alias():
    inp = inputs.prefill_inputs([129, 64], 2, 128, 128, seed=23, with_initial_state=False)
    check(inp, FUSED, what="fused no init")
    inp2 = inputs.prefill_inputs([129, 64], 2, 128, 128, seed=24, g_range=(0.0, 0.02))
    check(inp2, FUSED, what="fused alias", alias=True)


def test_fused_resume_equals_one_call():
    """prefill(T1) then prefill(T2, init=final) equals prefill(T1 + T2), on the GPU."""
    inp = inputs.prefill_inputs([320], 2, 128, 128, seed=25, g_range=(0.0, 0.01))
    o_all, f_all = run_prefill(inp, FUSED)
    a = inputs.PrefillInputs(inp.q[:192], inp.k[:192], inp.v[:192], inp.g[:192], inp.beta[:192],
                             torch.tensor([0, 192], dtype=torch.int32), inp.initial_state, inp.scale)
    o1, f1 = run_prefill(a, FUSED)
    b = inputs.PrefillInputs(inp.q[192:], inp.k[192:], inp.v[192:], inp.g[192:], inp.beta[192:],
                             torch.tensor([0, 128], dtype=torch.int32), f1.cpu(), inp.scale)
    o2, f2 = run_prefill(b, FUSED)
    assert_close(torch.cat([o1, o2]), o_all, tol=1e-5, what="resume o")
    assert_close(f2, f_all, tol=1e-5, what="resume state")


def test_fused_varlen_bitwise_equals_single_sequence_calls():
    lens = [100, 37, 256]
    inp = inputs.prefill_inputs(lens, 2, 128, 128, seed=26, g_range=(0.0, 0.02))
    o, fin = run_prefill(inp, FUSED)
    cu = inp.cu_seqlens.tolist()
    for n in range(len(lens)):
        sl = slice(cu[n], cu[n + 1])
        one = inputs.PrefillInputs(inp.q[sl], inp.k[sl], inp.v[sl], inp.g[sl], inp.beta[sl],
                                   torch.tensor([0, lens[n]], dtype=torch.int32),
                                   inp.initial_state[n:n + 1], inp.scale)
        o_n, f_n = run_prefill(one, FUSED)
        assert torch.equal(o_n, o[sl]) and torch.equal(f_n[0], fin[n])
    o2, fin2 = run_prefill(inp, FUSED)
    assert torch.equal(o, o2) and torch.equal(fin, fin2)  # deterministic


@pytest.mark.parametrize("nseq", [64, 70])
def test_fused_many_sequences_launch_order(nseq):
    """The fused kernel launches the longest sequences first when there are at most
    64 of them and in index order beyond; both must give the oracle's results, and
    a sequence's results must not depend on its neighbours (ties and empty
    sequences included)."""
    rng = np.random.default_rng(nseq)
    lens = [int(x) for x in rng.integers(0, 200, size=nseq)]
    lens[3] = lens[5] = 150  # a tie
    lens[7] = 0
    inp = inputs.prefill_inputs(lens, 2, 128, 128, seed=40 + nseq, g_range=(0.0, 0.05))
    o, fin = check(inp, FUSED, what=f"{nseq} sequences")
    cu = inp.cu_seqlens.tolist()
    for n in (3, 5, 7, nseq - 1):
        sl = slice(cu[n], cu[n + 1])
        one = inputs.PrefillInputs(inp.q[sl], inp.k[sl], inp.v[sl], inp.g[sl], inp.beta[sl],
                                   torch.tensor([0, lens[n]], dtype=torch.int32),
                                   inp.initial_state[n:n + 1], inp.scale)
        o_n, f_n = run_prefill(one, FUSED)
        assert torch.equal(o_n, o[sl]) and torch.equal(f_n[0], fin[n])


def test_fused_b4_t8192_h16_full_size():
    """Chunked prefill at the benchmark size (B=4 x 8192, H=16), every (sequence, head)."""
    inp = inputs.prefill_b4_t8192_h16()
    check(inp, FUSED, what="B4 T8192 H16", out_dtype=torch.bfloat16)


def _sampled_pairs_check(inp, algo, pairs, chunk=64):
    o, fin = run_prefill(inp, algo, chunk=chunk, out_dtype=torch.bfloat16)
    cu = inp.cu_seqlens.tolist()
    for n, h in pairs:
        sl = slice(cu[n], cu[n + 1])
        L = cu[n + 1] - cu[n]
        o_r, f_r, _ = oracle.prefill(inp.q[sl, h:h + 1], inp.k[sl, h:h + 1], inp.v[sl, h:h + 1],
                                     inp.g[sl, h:h + 1], inp.beta[sl, h:h + 1], [0, L],
                                     inp.initial_state[n:n + 1, h:h + 1], scale=inp.scale)
        assert_close(o[sl, h:h + 1], o_r, what=f"pair ({n},{h}) o")
        assert_close(fin[n:n + 1, h:h + 1], f_r, what=f"pair ({n},{h}) state")


def test_fused_varlen32_h32_sampled():
    """Varlen 32 sequences x H=32 at full size; the oracle checks a seeded sample of
    (sequence, head) pairs, including the longest and the shortest sequence."""
    inp = inputs.varlen32_h32(device=DEV)
    lens = inp.seqlens
    longest, shortest = int(np.argmax(lens)), int(np.argmin(lens))
    rng = np.random.default_rng(0)
    pairs = [(longest, 0), (shortest, 31)] + [(int(rng.integers(32)), int(rng.integers(32))) for _ in range(4)]
    _sampled_pairs_check(inp, FUSED, pairs)


# ---------------------------------------------------------------- transfer (chunk-parallel fixup) path

TRANSFER = gdn.GDN_PREFILL_TRANSFER


@pytest.mark.parametrize("g_range", [(0.01, 0.5), (0.0, 0.01), (0.0, 0.0)])
def test_transfer_varlen_edges(g_range):
    lens = [1, 0, 63, 64, 65, 130, 200, 7]
    inp = inputs.prefill_inputs(lens, 3, 128, 128, seed=31, g_range=g_range)
    check(inp, TRANSFER, what=f"transfer {g_range}")


def test_transfer_no_initial_state_and_alias():
    inp = inputs.prefill_inputs([129, 0, 64], 2, 128, 128, seed=32, with_initial_state=False)
    check(inp, TRANSFER, what="transfer no init")
    inp2 = inputs.prefill_inputs([400, 64], 2, 128, 128, seed=33, g_range=(0.0, 0.02))
    check(inp2, TRANSFER, what="transfer alias", alias=True)


def test_transfer_multi_chunk_segments_weak_decay():
    """20000 tokens x 8 heads: segments of several chunks (G > 1) and a long fixup chain."""
    inp = inputs.prefill_inputs([20000], 8, 128, 128, seed=34, g_range=(0.0, 0.02))
    check(inp, TRANSFER, what="transfer long weak decay")


def test_transfer_matches_fused():
    inp = inputs.prefill_inputs([3000, 500, 1], 4, 128, 128, seed=35, g_range=(0.0, 0.05))
    o_f, f_f = run_prefill(inp, FUSED)
    o_t, f_t = run_prefill(inp, TRANSFER)
    assert_close(o_t, o_f, what="transfer vs fused o")
    assert_close(f_t, f_f, what="transfer vs fused state")


def test_transfer_b1_t65536_h4_full_size():
    """Low-parallelism prefill at the benchmark size (B=1 x 65536, H=4), every head."""
    inp = inputs.longseq_b1_t65536_h4()
    check(inp, TRANSFER, what="B1 T65536 H4", out_dtype=torch.bfloat16)

