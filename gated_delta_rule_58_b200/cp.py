"""Context-parallel chunked prefill across the ranks of a torch.distributed group.

Each rank holds a consecutive slice of the tokens of every sequence (rank 0 the
first tokens), packed as a varlen batch with its own cu_seqlens. The steps (see
the context-parallelism block of include/gdn.h):

  1. the slice's local state H and transfer M (library kernels);
  2. one all-gather of (H, M) over the group, in rank order;
  3. this rank's start state from the pairs of the ranks before it (library kernel);
  4. the slice's outputs from that start state, reusing step 1's segments (library
     kernels: gdn_cp_finish).

Only step 2 communicates; this module does the orchestration and the collective
and none of the method's arithmetic. `ops` replaces the library calls of steps 1,
3 and 4 (used by the CPU tests of the rank logic, which run without a GPU); its
local_state returns (H, M, context) and its prefill receives that context.
"""
from __future__ import annotations

import types

import torch


def _library_ops():
    from . import _lib

    def local_state(q, k, v, g, beta, cu, chunk, l2norm):
        N, H, total_T = cu.numel() - 1, v.shape[1], q.shape[0]
        dk, dv = q.shape[-1], v.shape[-1]
        loc = torch.empty((N, H, dv, dk), dtype=torch.float32, device=q.device)
        tr = torch.empty_like(loc)
        ws = torch.empty(max(_lib.gdn_cp_local_state_workspace_size(N, total_T, H, dk, dv, chunk), 1),
                         dtype=torch.uint8, device=q.device)
        _lib.gdn_cp_local_state(q, k, v, g, beta, cu, loc, tr, chunk=chunk, l2norm=l2norm, workspace=ws)
        return loc, tr, ws

    def combine(all_loc, all_tr, rank, initial_state):
        start = torch.empty(all_loc.shape[1:], dtype=torch.float32, device=all_loc.device)
        _lib.gdn_cp_combine(all_loc, all_tr, rank, start, initial_state=initial_state)
        return start

    def prefill(q, k, v, g, beta, cu, o, start, final_state, chunk, scale, l2norm, ctx):
        _lib.gdn_cp_finish(q, k, v, g, beta, cu, o, ctx, start_state=start, final_state=final_state, chunk=chunk,
                           scale=scale, l2norm=l2norm)

    return types.SimpleNamespace(local_state=local_state, combine=combine, prefill=prefill)


def cp_chunk_prefill(q, k, v, g, beta, cu_seqlens, o, initial_state=None, final_state=None, group=None,
                     chunk=64, scale=None, l2norm=False, ops=None):
    """Prefill this rank's slice of every sequence given the slices of the other
    ranks of `group` (all ranks call this together). initial_state [N,H,dv,dk] is
    the sequences' start state (the same on every rank, or None); final_state
    receives the state at the end of this rank's slice (on the last rank: the
    sequences' final state). Returns o."""
    import torch.distributed as dist
    ops = ops or _library_ops()
    rank = dist.get_rank(group)
    ranks = dist.get_world_size(group)
    loc, tr, ctx = ops.local_state(q, k, v, g, beta, cu_seqlens, chunk, l2norm)
    # this rank's (H, M) as one flat buffer, so that a single all-gather carries both
    pair = torch.cat((loc.contiguous().view(-1), tr.contiguous().view(-1)))
    parts = [torch.empty_like(pair) for _ in range(ranks)]
    dist.all_gather(parts, pair, group=group)
    gathered = torch.stack(parts)  # rank-major [ranks, |H| + |M|]
    all_loc = gathered[:, :loc.numel()].reshape((ranks,) + tuple(loc.shape)).contiguous()
    all_tr = gathered[:, loc.numel():].reshape((ranks,) + tuple(tr.shape)).contiguous()
    start = ops.combine(all_loc, all_tr, rank, initial_state)
    ops.prefill(q, k, v, g, beta, cu_seqlens, o, start, final_state, chunk, scale, l2norm, ctx)
    return o
