"""The prefill backward's token staging, modelled on the CPU.

The kernel (csrc/prefill_backward.cu) visits the tokens of a sequence in a fixed
order: the forward sweep, then for each chunk from the last its tokens forward
(recompute) and backward (walk). It copies each position into a ring of kRing
shared-memory slots kRing - 1 positions ahead, walking that order with an
incremental cursor, and waits with cp.async.wait_group: every step commits two
groups, [the next walk step's S_{t-1} or nothing] then [the ring position], so a
sweep step waits for all but the newest 2 (kRing - 2) groups and a walk step for all
but the newest one. This model replays the cursor and the group accounting and
checks that every step finds its own position (and, in the walk, its S_{t-1})
complete and that a slot is refilled only after the step that read it."""
import os
import random
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ring_size():
    with open(os.path.join(ROOT, "gated_delta_rule_58_b200", "csrc", "prefill_backward.cu")) as f:
        m = re.search(r"constexpr int kRing = (\d+);", f.read())
    assert m, "kRing not found"
    return int(m.group(1))


def _visiting_order(bos, length, C):
    """(token, kind) per position; kind F forward sweep, R recompute, W walk."""
    eos, nck = bos + length, (length + C - 1) // C
    order = [(t, "F") for t in range(bos, eos)]
    for c in range(nck - 1, -1, -1):
        t0, t1 = bos + c * C, min(bos + (c + 1) * C, eos)
        order += [(t, "R") for t in range(t0, t1)]
        order += [(t, "W") for t in range(t1 - 1, t0 - 1, -1)]
    return order


def _cursor(bos, length, C, count):
    """The kernel's issue cursor: phase 0 forward, 1 recompute, 2 walk, 3 past the end."""
    eos, nck = bos + length, (length + C - 1) // C
    ct, ct0, ct1, cc, ph = bos, 0, 0, 0, (0 if length > 0 else 3)
    out = []
    for _ in range(count):
        out.append(ct if ph != 3 else None)
        if ph == 0:
            ct += 1
            if ct == eos:
                cc = nck - 1
                ct0, ct1 = bos + cc * C, eos
                ct, ph = ct0, 1
        elif ph == 1:
            ct += 1
            if ct == ct1:
                ct, ph = ct1 - 1, 2
        elif ph == 2:
            if ct == ct0:
                cc -= 1
                if cc < 0:
                    ph = 3
                else:
                    ct1, ct0 = ct0, ct0 - C
                    ct, ph = ct0, 1
            else:
                ct -= 1
    return out


def _check(bos, length, C, R):
    order = _visiting_order(bos, length, C)
    P = len(order)
    assert P == 3 * length
    assert _cursor(bos, length, C, P + R) == [t for t, _ in order] + [None] * R
    groups = []  # commit order; wait_group N completes all but the newest N
    for i in range(R - 1):
        groups += [("state", None), ("ring", i)]
    done, n_done = set(), 0
    holder = {i % R: i for i in range(R - 1)}  # slot -> position it holds
    for p in range(P):
        kind = order[p][1]
        n = 1 if kind == "W" else 2 * (R - 2)
        done.update(groups[n_done:len(groups) - n])
        n_done = max(n_done, len(groups) - n)
        assert ("ring", p) in done and holder[p % R] == p, (bos, length, C, p)
        if kind == "W":
            assert ("state", p) in done, (bos, length, C, p)
        nxt_walk = p + 1 < P and order[p + 1][1] == "W"
        groups.append(("state", p + 1 if nxt_walk else None))
        q = p + R - 1
        if q < P:
            assert q % R == (p - 1) % R and (p == 0 or holder[q % R] == p - 1)
            holder[q % R] = q
        groups.append(("ring", q))


def test_cursor_and_group_accounting():
    R = _ring_size()
    assert R >= 3
    cases = [(0, 0, 16), (0, 1, 1), (0, 1, 16), (5, 16, 16), (0, 17, 16), (3, 64, 64), (7, 65, 64), (0, 3, 256),
             (0, 8192, 16)]
    rng = random.Random(1)
    cases += [(rng.randint(0, 100), rng.randint(1, 300), rng.choice([1, 2, 3, 16, 32, 64, 100])) for _ in range(150)]
    for c in cases:
        _check(*c, R)
