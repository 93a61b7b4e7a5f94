"""GPU parity of gdn_chunk_prefill against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import inputs
from tests.util import assert_close, cached

pytestmark = pytest.mark.gpu
DEV = "cuda"

SEQ = gdn.GDN_PREFILL_SEQUENTIAL


def run_prefill(inp, algo, chunk=64, out_dtype=torch.float32, with_final=True, alias=False,
                workspace=None, l2norm=False):
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    g, beta, cu = inp.g.to(DEV), inp.beta.to(DEV), inp.cu_seqlens.to(DEV)
    total, dk = q.shape[0], q.shape[2]
    H, dv = v.shape[1], v.shape[-1]
    N = cu.numel() - 1
    init = inp.initial_state.to(DEV).clone() if inp.initial_state is not None else None
    o = torch.full((total, H, dv), float("nan"), dtype=out_dtype, device=DEV)
    fin = None
    if with_final:
        fin = init if (alias and init is not None) else torch.full((N, H, dv, dk), float("nan"), device=DEV)
    gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, o, initial_state=init, final_state=fin, chunk=chunk,
                          scale=inp.scale, algo=algo, workspace=workspace, l2norm=l2norm)
    torch.cuda.synchronize()
    return o, fin


def oracle_prefill(inp, l2norm=False):
    o, fin, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens,
                               inp.initial_state, scale=inp.scale, l2norm=l2norm)
    return o, fin


def check(inp, algo, chunk=64, what="", **kw):
    o, fin = run_prefill(inp, algo, chunk=chunk, **kw)
    o_ref, f_ref = oracle_prefill(inp, l2norm=kw.get("l2norm", False))
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


def _full_size(name):
    """The named benchmark workload and its oracle results, computed once per process."""
    def make():
        inp = getattr(inputs, name)()
        return inp, oracle_prefill(inp)
    return cached(name, make)


@pytest.mark.parametrize("algo", [gdn.GDN_PREFILL_AUTO, FUSED])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_b4_t8192_h16_full_size(algo, out_dtype):
    """Chunked prefill at the benchmark size (B=4 x 8192, H=16), every (sequence, head);
    fp32 outputs are held to the 2e-3 normwise bar directly."""
    inp, (o_ref, f_ref) = _full_size("prefill_b4_t8192_h16")
    o, fin = run_prefill(inp, algo, out_dtype=out_dtype)
    assert_close(o, o_ref, what=f"B4 T8192 H16 o ({out_dtype})")
    assert_close(fin, f_ref, what=f"B4 T8192 H16 final state ({out_dtype})")


@pytest.mark.parametrize("algo", [gdn.GDN_PREFILL_AUTO, FUSED])
def test_varlen32_h32_every_pair(algo):
    """Varlen 32 sequences x H=32 at full size (lengths ~U[64, 16384]), every
    (sequence, head) against the oracle: fp32 outputs at 2e-3 normwise, bf16 outputs
    element-wise, final states at 2e-3. The oracle runs one sequence at a time."""
    inp = cached("varlen32_h32", inputs.varlen32_h32)
    o32, fin = run_prefill(inp, algo, out_dtype=torch.float32)
    o16, fin16 = run_prefill(inp, algo, out_dtype=torch.bfloat16)
    assert torch.equal(fin, fin16)  # the state path does not depend on the output dtype
    cu = inp.cu_seqlens.tolist()
    for n in range(len(cu) - 1):
        sl = slice(cu[n], cu[n + 1])
        L = cu[n + 1] - cu[n]
        o_r, f_r, _ = oracle.prefill(inp.q[sl], inp.k[sl], inp.v[sl], inp.g[sl], inp.beta[sl], [0, L],
                                     inp.initial_state[n:n + 1], scale=inp.scale)
        assert_close(o32[sl], o_r, what=f"varlen seq {n} (L={L}) o fp32")
        assert_close(o16[sl], o_r, what=f"varlen seq {n} (L={L}) o bf16")
        assert_close(fin[n:n + 1], f_r, what=f"varlen seq {n} (L={L}) state")


def _poisoned(inp, n, value):
    """A copy of the packed inputs with every token of sequence n set to `value`
    (q, k, v; g and beta too)."""
    cu = inp.cu_seqlens.tolist()
    sl = slice(cu[n], cu[n + 1])
    out = inputs.PrefillInputs(inp.q.clone(), inp.k.clone(), inp.v.clone(), inp.g.clone(), inp.beta.clone(),
                               inp.cu_seqlens.clone(), inp.initial_state.clone(), inp.scale)
    for t in (out.q, out.k, out.v, out.g, out.beta):
        t[sl] = value
    return out


@pytest.mark.parametrize("algo", [FUSED, gdn.GDN_PREFILL_TRANSFER])
@pytest.mark.parametrize("value", [float("nan"), 1.0e5, float("inf")])
def test_neighbour_data_cannot_leak_into_a_sequence(algo, value):
    """The last, partial chunk of a sequence is loaded together with the first tokens
    of the next sequence. Whatever those tokens hold (NaN, inf, or a value beyond the
    fp16 range), the sequence's outputs and final state must be bitwise those of a
    call with clean neighbours."""
    lens = [100, 37, 256, 65]
    inp = inputs.prefill_inputs(lens, 2, 128, 128, seed=27, g_range=(0.0, 0.02))
    o_ref, f_ref = run_prefill(inp, algo)
    cu = inp.cu_seqlens.tolist()
    for bad in (1, 2, 3):  # poison sequence `bad`; sequence bad-1 ends in a partial chunk
        o, fin = run_prefill(_poisoned(inp, bad, value), algo)
        good = bad - 1
        sl = slice(cu[good], cu[good + 1])
        assert torch.equal(o[sl], o_ref[sl]), f"sequence {good} outputs changed by its neighbour ({value})"
        assert torch.equal(fin[good], f_ref[good]), f"sequence {good} state changed by its neighbour ({value})"
        for other in range(len(lens)):
            if other != bad:
                slo = slice(cu[other], cu[other + 1])
                assert torch.equal(o[slo], o_ref[slo]) and torch.equal(fin[other], f_ref[other])


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


@pytest.mark.parametrize("algo,out_dtype", [(gdn.GDN_PREFILL_AUTO, torch.float32),
                                             (gdn.GDN_PREFILL_AUTO, torch.bfloat16),
                                             (FUSED, torch.float32)])
def test_b1_t65536_h4_full_size(algo, out_dtype):
    """Low-parallelism prefill at the benchmark size (B=1 x 65536, H=4), every head;
    AUTO takes the transfer (chunk-parallel fixup) path here."""
    inp, (o_ref, f_ref) = _full_size("longseq_b1_t65536_h4")
    o, fin = run_prefill(inp, algo, out_dtype=out_dtype)
    assert_close(o, o_ref, what=f"B1 T65536 H4 o ({out_dtype})")
    assert_close(fin, f_ref, what=f"B1 T65536 H4 final state ({out_dtype})")


# ---------------------------------------------------------------- grouped q/k heads, q/k normalisation

@pytest.mark.parametrize("algo", [FUSED, TRANSFER, SEQ])
@pytest.mark.parametrize("l2norm", [False, True])
def test_grouped_heads_varlen(algo, l2norm):
    """8 value heads over 2 q/k heads, lengths around the chunk size; with the
    normalisation q and k are un-normalised N(0, 1) draws."""
    lens = [1, 0, 63, 64, 65, 130, 200, 7]
    inp = inputs.prefill_inputs(lens, 8, 128, 128, seed=51, g_range=(0.0, 0.05), H_qk=2,
                                normalize_qk=not l2norm)
    check(inp, algo, what=f"GVA algo={algo} l2={l2norm}", l2norm=l2norm)


@pytest.mark.parametrize("in_dtype", [torch.bfloat16, torch.float32])
def test_l2norm_fused_input_dtypes(in_dtype):
    inp = inputs.prefill_inputs([300, 65], 4, 128, 128, seed=52, dtype=in_dtype, g_range=(0.0, 0.05),
                                H_qk=4, normalize_qk=False)
    check(inp, FUSED, what=f"l2 fused {in_dtype}", l2norm=True)


def test_grouped_heads_hv32_hqk8_l2norm():
    """32 value heads over 8 q/k heads with the normalisation, a few sequences of
    several chunks (fused and transfer)."""
    inp = inputs.prefill_inputs([1000, 333, 64], 32, 128, 128, seed=53, H_qk=8, normalize_qk=False)
    check(inp, FUSED, what="GVA Hv32 Hqk8 fused", l2norm=True)
    check(inp, TRANSFER, what="GVA Hv32 Hqk8 transfer", l2norm=True)


def test_l2norm_neighbour_cannot_leak():
    """With the normalisation the partial chunk's padded rows are zeroed before the
    norms are taken: a NaN neighbour leaves the sequence bitwise unchanged."""
    lens = [100, 37]
    inp = inputs.prefill_inputs(lens, 2, 128, 128, seed=54, normalize_qk=False)
    o_ref, f_ref = run_prefill(inp, FUSED, l2norm=True)
    o, fin = run_prefill(_poisoned(inp, 1, float("nan")), FUSED, l2norm=True)
    assert torch.equal(o[:100], o_ref[:100]) and torch.equal(fin[0], f_ref[0])
