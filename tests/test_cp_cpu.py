"""Context-parallel prefill across ranks, the rank logic on the CPU: two and three
gloo ranks, each holding a slice of every sequence, exchange their (local state,
transfer) pairs and prefill their slices (gated_delta_rule_58_b200.cp). The
library's kernels are replaced by the fp64 oracle here (a local state is the
oracle's final state from zero, a transfer its final state from the identity with
zero values, the combine folds the pairs of the earlier ranks); the slices'
outputs and the last rank's final state must equal the oracle run over whole
sequences."""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    import oracle

    def local_state(q, k, v, g, beta, cu, chunk, l2norm):
        N, H, dk = cu.numel() - 1, v.shape[1], q.shape[-1]
        _, Ht, _ = oracle.prefill(q, k, v, g, beta, cu, None, scale=0.3, l2norm=l2norm)
        ident = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
        zero_v = torch.zeros(v.shape[0], H, dk, dtype=torch.float64)
        _, Mt, _ = oracle.prefill(q, k, zero_v, g, beta, cu, ident, scale=0.3, l2norm=l2norm)
        return torch.from_numpy(Ht), torch.from_numpy(Mt), None

    def combine(all_loc, all_tr, rank, initial_state):
        # the library's combine takes contiguous rank-major arrays
        assert all_loc.is_contiguous() and all_tr.is_contiguous()
        S = torch.zeros_like(all_loc[0]) if initial_state is None else initial_state.clone()
        for r in range(rank):
            S = torch.einsum("nhij,nhjk->nhik", S, all_tr[r]) + all_loc[r]
        return S

    def prefill(q, k, v, g, beta, cu, o, start, final_state, chunk, scale, l2norm, ctx):
        o_, f_, _ = oracle.prefill(q, k, v, g, beta, cu, start, scale=0.3, l2norm=l2norm)
        o.copy_(torch.from_numpy(o_))
        final_state.copy_(torch.from_numpy(f_))

    return types.SimpleNamespace(local_state=local_state, combine=combine, prefill=prefill)


def _rank_main(rank, ranks, port, lengths, l2norm, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from gated_delta_rule_58_b200 import inputs
    from gated_delta_rule_58_b200.cp import cp_chunk_prefill
    from tests.cp_slices import rank_slice, slice_bounds
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ranks)
    try:
        inp = inputs.prefill_inputs(lengths, 3, 4, 3, seed=5, g_range=(0.0, 0.2), H_qk=3,
                                    normalize_qk=not l2norm)
        bounds = slice_bounds(lengths, ranks)
        (q, k, v, g, beta), cu, idx = rank_slice(inp, bounds, rank)
        o = torch.zeros((q.shape[0], 3, 3), dtype=torch.float64)
        fin = torch.zeros((len(lengths), 3, 3, 4), dtype=torch.float64)
        init = inp.initial_state.double()
        cp_chunk_prefill(q, k, v, g, beta, cu, o, initial_state=init, final_state=fin, l2norm=l2norm,
                         ops=_oracle_ops())
        out[rank] = (idx.numpy(), o.numpy(), fin.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ranks,l2norm", [(2, False), (3, True)])
def test_cp_prefill_over_gloo_ranks_equals_whole_sequences(ranks, l2norm):
    import oracle
    from gated_delta_rule_58_b200 import inputs
    lengths = [29, 0, 7, 40]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(ranks, _free_port(), lengths, l2norm, out), nprocs=ranks, join=True,
                           start_method="spawn")
        res = dict(out)
    inp = inputs.prefill_inputs(lengths, 3, 4, 3, seed=5, g_range=(0.0, 0.2), H_qk=3, normalize_qk=not l2norm)
    o_ref, f_ref, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.initial_state,
                                     scale=0.3, l2norm=l2norm)
    o = np.zeros_like(o_ref)
    for r in range(ranks):
        idx, o_r, _ = res[r]
        o[idx] = o_r
    assert np.abs(o - o_ref).max() <= 1e-12 * max(np.abs(o_ref).max(), 1.0)
    fin_last = res[ranks - 1][2]
    assert np.abs(fin_last - f_ref).max() <= 1e-12 * np.abs(f_ref).max()
