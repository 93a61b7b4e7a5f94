"""The allocation-free prefill entry point (gdn_chunk_prefill_static_scratch).

It serves callers that cannot allocate device memory when they call, e.g. a
plugin whose host framework owns every device allocation, or a serving engine
that reserved the whole device for its own pool: the transfer prefill's scratch
lives in a fixed 32 MiB array inside the library instead of a caller workspace.
This file is collected last so that a failure here never hides another test.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import _lib, inputs
from tests.util import assert_close

STATIC_SCRATCH_BYTES = 32 << 20


def _run(inp, fn, **kw):
    dev = "cuda"
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    total, H, dk = q.shape
    N = inp.cu_seqlens.numel() - 1
    o = torch.full((total, H, v.shape[-1]), float("nan"), dtype=torch.float32, device=dev)
    fin = torch.full((N, H, v.shape[-1], dk), float("nan"), device=dev)
    init = inp.initial_state.to(dev) if inp.initial_state is not None else None
    fn(q, k, v, inp.g.to(dev), inp.beta.to(dev), inp.cu_seqlens.to(dev), o,
       initial_state=init, final_state=fin, chunk=64, scale=inp.scale, **kw)
    torch.cuda.synchronize()
    return o, fin


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_and_oracle():
    """Calls in a row through the C ABI, each checked against gdn_chunk_prefill with a
    caller workspace and against the fp64 oracle (2e-3 normwise on fp32 outputs and
    final states). The cases: varlen with an empty sequence; no initial state; the
    long single sequence B=1 x 65536, H=4, whose scratch (about 25 MiB) comes close
    to the 32 MiB limit; then the first case again, over scratch that now holds the
    long call's data, which must give the same result as its first call."""
    import oracle
    cases = [inputs.prefill_inputs([700, 0, 300, 65], 2, 128, 128, seed=41, g_range=(0.0, 0.05)),
             inputs.prefill_inputs([130, 64], 3, 128, 128, seed=42, g_range=(0.01, 0.5),
                                   with_initial_state=False),
             inputs.longseq_b1_t65536_h4()]
    first = None
    for i, inp in enumerate(cases):
        total, H = inp.q.shape[0], inp.q.shape[1]
        need = gdn.gdn_chunk_prefill_workspace_size(inp.cu_seqlens.numel() - 1, total, H, 128, 128, 64,
                                                    gdn.GDN_PREFILL_TRANSFER)
        assert need <= STATIC_SCRATCH_BYTES
        o_ws, f_ws = _run(inp, gdn.gdn_chunk_prefill, algo=gdn.GDN_PREFILL_TRANSFER)
        o, f = _run(inp, gdn.gdn_chunk_prefill_static_scratch)
        assert_close(o, o_ws, what=f"case {i}: static scratch o vs workspace entry point")
        assert_close(f, f_ws, what=f"case {i}: static scratch state vs workspace entry point")
        o_r, f_r, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state,
                                     scale=inp.scale)
        assert_close(o, o_r, what=f"case {i}: static scratch o vs oracle")
        assert_close(f, f_r, what=f"case {i}: static scratch state vs oracle")
        if i == 0:
            first = (o, f)
    o, f = _run(cases[0], gdn.gdn_chunk_prefill_static_scratch)
    assert_close(o, first[0], what="repeat call o")
    assert_close(f, first[1], what="repeat call state")


def test_static_scratch_rejects_shapes_beyond_its_size():
    """A shape whose transfer workspace exceeds the 32 MiB scratch is refused on the
    host (GDN_ERR_WORKSPACE) before any CUDA call."""
    L = _lib.lib()
    fake = 0x10000  # never dereferenced: the size check fails first
    N, total, H = 1, 65536, 16
    need = gdn.gdn_chunk_prefill_workspace_size(N, total, H, 128, 128, 64, gdn.GDN_PREFILL_TRANSFER)
    assert need > STATIC_SCRATCH_BYTES
    st = L.gdn_chunk_prefill_static_scratch(fake, fake, fake, fake, fake, fake, N, total, None, None, fake,
                                            H, H, 128, 128, 64, 0.1, 0, gdn.GDN_BF16, gdn.GDN_BF16, None)
    assert st == gdn.GDN_ERR_WORKSPACE
    assert "static scratch" in gdn.gdn_last_error()
