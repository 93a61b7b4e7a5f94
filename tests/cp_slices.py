"""Helpers of the context-parallel tests: slicing a packed varlen batch into the
per-rank slices (consecutive token ranges of every sequence) and putting outputs
back together. Pure indexing, no arithmetic of the method."""
import torch


def slice_bounds(lengths, ranks):
    """For every sequence, the token offsets where each rank's slice starts and
    ends (uneven splits and empty slices included)."""
    out = []
    for L in lengths:
        cuts = [(L * r) // ranks for r in range(ranks + 1)]
        if ranks > 1 and L > 3:  # make the split uneven
            cuts[1] = max(0, cuts[1] - L // 7)
        out.append(cuts)
    return out


def rank_slice(inp, bounds, rank):
    """The packed inputs (q, k, v, g, beta) and cu_seqlens of one rank."""
    cu = inp.cu_seqlens.tolist()
    idx, lens = [], []
    for n, cuts in enumerate(bounds):
        a, b = cu[n] + cuts[rank], cu[n] + cuts[rank + 1]
        idx.append(torch.arange(a, b))
        lens.append(b - a)
    idx = torch.cat(idx) if idx else torch.zeros(0, dtype=torch.long)
    cus = torch.zeros(len(lens) + 1, dtype=torch.int32)
    if lens:
        cus[1:] = torch.tensor(lens).cumsum(0).to(torch.int32)
    return [t[idx] for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)], cus, idx
