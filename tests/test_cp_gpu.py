"""Context-parallel prefill with the library's kernels, ranks emulated one after
another in one process on one GPU (nothing waits on another rank: the exchange is
the stacking of the ranks' pairs). Each rank's slice: gdn_cp_local_state, then
gdn_cp_combine over the earlier ranks' pairs, then gdn_cp_finish (or
gdn_chunk_prefill) from that start state. The assembled outputs and the last rank's final state are compared
with the oracle over whole sequences."""
import pytest
import torch

import oracle
import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import inputs
from tests.cp_slices import rank_slice, slice_bounds
from tests.util import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _emulate(inp, ranks, l2norm=False, out_dtype=torch.float32, finish=True):
    lengths = inp.seqlens
    N, H, dk = len(lengths), inp.v.shape[1], inp.q.shape[-1]
    bounds = slice_bounds(lengths, ranks)
    slices = [rank_slice(inp, bounds, r) for r in range(ranks)]
    loc = torch.empty((ranks, N, H, 128, 128), device=DEV)
    tr = torch.empty_like(loc)
    wss = []
    for r, ((q, k, v, g, beta), cu, _) in enumerate(slices):
        ws = torch.empty(max(gdn.gdn_cp_local_state_workspace_size(N, q.shape[0], H, 128, 128), 1), dtype=torch.uint8,
                         device=DEV)
        wss.append(ws)
        gdn.gdn_cp_local_state(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), cu.to(DEV), loc[r], tr[r],
                               l2norm=l2norm, workspace=ws)
    o = torch.full((inp.q.shape[0], H, 128), float("nan"), dtype=out_dtype, device=DEV)
    fin = None
    init = inp.initial_state.to(DEV) if inp.initial_state is not None else None
    for r, ((q, k, v, g, beta), cu, idx) in enumerate(slices):
        start = torch.empty((N, H, 128, 128), device=DEV)
        gdn.gdn_cp_combine(loc, tr, r, start, initial_state=init)
        o_r = torch.empty((q.shape[0], H, 128), dtype=out_dtype, device=DEV)
        fin = torch.empty((N, H, 128, 128), device=DEV)
        if finish:
            gdn.gdn_cp_finish(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), cu.to(DEV), o_r, wss[r],
                              start_state=start, final_state=fin, scale=inp.scale, l2norm=l2norm)
        else:
            gdn.gdn_chunk_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), cu.to(DEV), o_r,
                                  initial_state=start, final_state=fin, scale=inp.scale, l2norm=l2norm)
        o[idx.to(DEV)] = o_r
    torch.cuda.synchronize()
    return o, fin


@pytest.mark.parametrize("ranks", [1, 2, 4])
@pytest.mark.parametrize("g_range", [(0.01, 0.5), (0.0, 0.01)])
def test_cp_emulated_ranks_against_oracle(ranks, g_range):
    inp = inputs.prefill_inputs([3000, 333, 64, 0, 1000], 4, 128, 128, seed=80, g_range=g_range)
    o, fin = _emulate(inp, ranks)
    o_r, f_r, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state,
                                 scale=inp.scale)
    assert_close(o, o_r, what=f"cp ranks={ranks} o")
    assert_close(fin, f_r, what=f"cp ranks={ranks} final state")


def test_cp_one_long_sequence_grouped_heads_l2norm():
    """One 16384-token sequence over 4 ranks, 8 value heads over 2 q/k heads, with
    the normalisation and no initial state."""
    inp = inputs.prefill_inputs([16384], 8, 128, 128, seed=81, g_range=(0.0, 0.02), H_qk=2, normalize_qk=False,
                                with_initial_state=False)
    o, fin = _emulate(inp, 4, l2norm=True, out_dtype=torch.bfloat16)
    o_r, f_r, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, None, scale=inp.scale,
                                 l2norm=True)
    assert_close(o, o_r, what="cp long o")
    assert_close(fin, f_r, what="cp long final state")


def test_cp_single_rank_is_the_transfer_prefill_bitwise():
    """One rank: the combine copies the initial state and the finish is the transfer
    prefill of the whole batch."""
    inp = inputs.prefill_inputs([700, 65], 2, 128, 128, seed=82, g_range=(0.0, 0.05))
    o, fin = _emulate(inp, 1)
    o2 = torch.empty_like(o)
    fin2 = torch.empty_like(fin)
    gdn.gdn_chunk_prefill(inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV), inp.g.to(DEV), inp.beta.to(DEV),
                          inp.cu_seqlens.to(DEV), o2, initial_state=inp.initial_state.to(DEV), final_state=fin2,
                          scale=inp.scale, algo=gdn.GDN_PREFILL_TRANSFER)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(fin, fin2)


def test_cp_finish_equals_the_transfer_prefill_of_the_slice_bitwise():
    """gdn_cp_finish reuses gdn_cp_local_state's segments: its outputs and final state
    are bitwise those of gdn_chunk_prefill with GDN_PREFILL_TRANSFER on the slice."""
    inp = inputs.prefill_inputs([5000, 777], 4, 128, 128, seed=83, g_range=(0.0, 0.05))
    dev = [x.to(DEV) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state)]
    q, k, v, g, beta, cu, init = dev
    N, H = 2, 4
    ws = torch.empty(gdn.gdn_cp_local_state_workspace_size(N, q.shape[0], H, 128, 128), dtype=torch.uint8, device=DEV)
    loc = torch.empty((N, H, 128, 128), device=DEV)
    tr = torch.empty_like(loc)
    gdn.gdn_cp_local_state(q, k, v, g, beta, cu, loc, tr, workspace=ws)
    o1 = torch.empty((q.shape[0], H, 128), dtype=torch.bfloat16, device=DEV)
    f1 = torch.empty((N, H, 128, 128), device=DEV)
    gdn.gdn_cp_finish(q, k, v, g, beta, cu, o1, ws, start_state=init, final_state=f1, scale=inp.scale)
    o2 = torch.empty_like(o1)
    f2 = torch.empty_like(f1)
    gdn.gdn_chunk_prefill(q, k, v, g, beta, cu, o2, initial_state=init, final_state=f2, scale=inp.scale,
                          algo=gdn.GDN_PREFILL_TRANSFER)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)
    # the pair is the slice's composition: S_end^T = S_0^T M^T + H^T (fp32)
    comp = torch.einsum("nhij,nhjk->nhik", init, tr) + loc
    assert_close(comp, f2, tol=1e-4, what="local state and transfer compose to the final state")


def test_cp_plain_prefill_path_still_matches():
    inp = inputs.prefill_inputs([3000, 333, 64, 0, 1000], 4, 128, 128, seed=84, g_range=(0.0, 0.01))
    o, fin = _emulate(inp, 2, finish=False)
    o_r, f_r, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state,
                                 scale=inp.scale)
    assert_close(o, o_r, what="cp plain o")
    assert_close(fin, f_r, what="cp plain final state")


def _gpu_rank_main(rank, ranks, port, lengths, out):
    """One rank of cp_chunk_prefill (the library driver and kernels) on cuda:0; the
    ranks share the GPU as separate processes, which only exchange through a gloo
    all-gather between launches (no kernel waits on another process)."""
    import datetime
    import os
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from gated_delta_rule_58_b200 import inputs as inp_mod
    from gated_delta_rule_58_b200.cp import cp_chunk_prefill
    from tests.cp_slices import rank_slice as rs, slice_bounds as sb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ranks, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        inp = inp_mod.prefill_inputs(lengths, 4, 128, 128, seed=86, g_range=(0.0, 0.02), H_qk=2)
        (q, k, v, g, beta), cu, idx = rs(inp, sb(lengths, ranks), rank)
        q, k, v, g, beta, cu = (x.cuda() for x in (q, k, v, g, beta, cu))
        o = torch.empty((q.shape[0], 4, 128), dtype=torch.float32, device="cuda")
        fin = torch.empty((len(lengths), 4, 128, 128), device="cuda")
        cp_chunk_prefill(q, k, v, g, beta, cu, o, initial_state=inp.initial_state.cuda(), final_state=fin,
                         scale=inp.scale)
        torch.cuda.synchronize()
        out[rank] = (idx.numpy(), o.cpu().numpy(), fin.cpu().numpy())
    finally:
        dist.destroy_process_group()


def test_cp_driver_over_two_processes_on_one_gpu():
    import socket
    import numpy as np
    import torch.multiprocessing as mp
    lengths = [2000, 130, 0, 700]
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_gpu_rank_main, args=(2, port, lengths, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    inp = inputs.prefill_inputs(lengths, 4, 128, 128, seed=86, g_range=(0.0, 0.02), H_qk=2)
    o_ref, f_ref, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state,
                                     scale=inp.scale)
    o = np.zeros_like(o_ref)
    for r in range(2):
        idx, o_r, _ = res[r]
        o[idx] = o_r
    assert_close(o, o_ref, what="cp driver o")
    assert_close(res[1][2], f_ref, what="cp driver final state")
