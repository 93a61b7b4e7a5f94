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
