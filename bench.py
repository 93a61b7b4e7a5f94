"""Benchmark of the gated delta rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--parts ...]

Headline (one JSON line on rank 0): the T=1 decode step on B=64 sequences x
H=32 heads, dk=dv=128, fp32 state pool of 256 slots, as state GB/s (state bytes
read + written per second). A step is one decode launch over one batch; steps
rotate over 4 disjoint slot sets of the 512 MiB pool so that each step reads
state that is not in the 126 MB L2. The other workloads (chunked prefill
B=4 x 8192 x H=16; varlen prefill 32 seqs x H=32; long sequence B=1 x 65536 x
H=4; gated delta product B=128 x T=4 x n_h=2; tiny fp32) are measured in the
same run and reported under "parts".

With torchrun (N > 1) every rank runs the same per-GPU workload on its own
device (weak scaling, no collective on the data path); times are the max over
ranks. `--impl reference` times the fp64 CPU oracle on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN decode state GB/s (% of 8 TB/s); chunked prefill tokens/s (% roofline)"
NOMINAL_HBM_GBS = 8000.0
# fp32 FMA peak of a B200 from its unit counts: 148 SMs x 128 fp32 lanes x 2 flops at
# the 1965 MHz maximum SM clock (TFLOP/s); the roofline of SIMT fp32 arithmetic
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------- environment

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup():
    """One process per GPU under torchrun (env RANK/LOCAL_RANK/WORLD_SIZE/MASTER_*).
    NCCL on GPUs; gloo when CUDA is absent (the CPU-only reference arm and tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        timeout = datetime.timedelta(seconds=120)
        if cuda:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif cuda:
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self._stop = threading.Event()
        self._th = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.rows.append([x.strip() for x in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._th = threading.Thread(target=self._run, daemon=True)
        self._th.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._th.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if len(r) > 5 + i and r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def source_code(text: str) -> str:
    """The code of a C++/CUDA source: // and /* */ comments, trailing blanks and
    empty lines removed, so an edit of comments alone keeps the hash."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", l).rstrip() for l in text.splitlines())
    return "\n".join(l for l in lines if l)


def source_sha(*rel_paths) -> str:
    h = hashlib.sha256()
    for p in rel_paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(source_code(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(part_key: str):
    """DRAM bytes (read + write) per launch of the part's dominant kernel (for the
    transfer prefill: of all library kernels of one step) from the committed ncu
    capture, or None when a source file it names has changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(part_key)
    if not e or e.get("source_sha") != source_sha(*e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- timing helpers

def time_launches(fn, steps, warmup, ws, stream=None):
    """Runs fn(i) warmup times, then `steps` times bracketed by barrier + synchronize;
    returns (max-over-ranks total ms, list of per-launch ms from CUDA events)."""
    stream = stream or torch.cuda.current_stream()
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        evs[i][0].record(stream)
        fn(warmup + i)
        evs[i][1].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    total = max_over_ranks(start.elapsed_time(stop), ws)
    per = [a.elapsed_time(b) for a, b in evs]
    return total, per


def time_graph(fn, steps, warmup, ws):
    """Runs fn(i) `warmup` times eagerly, captures `steps` calls into one CUDA graph,
    replays it once untimed, then times one replay bracketed by barrier + synchronize.
    Returns the max-over-ranks total ms of the K timed steps."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cap):
        for i in range(steps):
            fn(warmup + i)
    graph.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start.record(stream)
    graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    total = max_over_ranks(start.elapsed_time(stop), ws)
    del graph
    return total


# ---------------------------------------------------------------- decode workloads

DECODE_CFGS = {
    "decode": dict(B=64, T=1, H=32, d=128, nh=1, slots=256,
                   name="decode T=1, B=64, H=32, dk=dv=128, fp32 pool of 256 slots, bf16 q/k/v"),
    # small batches: the T=1 step splits each head's state rows over several CTAs
    "decode_b1": dict(B=1, T=1, H=32, d=128, nh=1, slots=512,
                      name="decode T=1, B=1, H=32, dk=dv=128, fp32 pool of 512 slots (split along V)"),
    "decode_b4": dict(B=4, T=1, H=32, d=128, nh=1, slots=512,
                      name="decode T=1, B=4, H=32, dk=dv=128, fp32 pool of 512 slots (split along V)"),
    "decode_b16": dict(B=16, T=1, H=32, d=128, nh=1, slots=512,
                       name="decode T=1, B=16, H=32, dk=dv=128, fp32 pool of 512 slots (split along V)"),
    "gdp": dict(B=128, T=4, H=32, d=128, nh=2, slots=512,
                name="gated delta product decode, B=128, H=32, T=4, n_h=2, dk=dv=128, pool of 512 slots"),
}


def decode_bytes(c):
    """Algorithmic HBM bytes of one decode step: state read + write, q/k/v (bf16),
    g and beta (fp32), o (bf16), slot ids."""
    B, T, H, d, nh = c["B"], c["T"], c["H"], c["d"], c["nh"]
    heads = B * H
    state = 2 * heads * d * d * 4
    qkv = heads * T * (d + nh * d + nh * d) * 2
    gb = heads * T * (1 + nh) * 4
    o = heads * T * d * 2
    return state, state + qkv + gb + o + B * 4


def e2e_decode(gdn, inp, pool, o, slot_sets, nsets, steps, warmup, ws, state_b):
    """End to end through the public API with host buffers: every step copies its
    inputs (q, k, v, g, beta, slot ids) from pinned host memory, runs gdn_decode and
    reads o back to pinned host memory, all inside the timed region. As a serving
    loop would, the copies run on their own streams with double-buffered device
    buffers, so step i+1's inputs travel while step i computes; events order each
    step's copies, its kernel and the reuse of its buffers."""
    names = ("q", "k", "v", "g", "beta")
    srcs = [getattr(inp, n) for n in names] + [slot_sets[0]]

    def packed(device, pin):
        """One byte buffer holding every input of a step (256-byte aligned
        segments) and tensor views into it, so a step's inputs move in one copy."""
        offs, off = [], 0
        for t in srcs:
            offs.append(off)
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.empty(off, dtype=torch.uint8, device=device, pin_memory=pin)
        views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, srcs)]
        return buf, views

    host = []  # one pinned pack per slot set (never written inside the timed loop)
    for ss in slot_sets:
        hb, hv = packed("cpu", True)
        for v_, t in zip(hv, srcs[:-1] + [ss]):
            v_.copy_(t.cpu())
        host.append(hb)
    dev = [packed(pool.device, False) for _ in range(2)]
    obuf = [torch.empty_like(o) for _ in range(2)]
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in srcs)
    d2h = o.numel() * o.element_size()
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, kern_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def step(i):
        j = i % 2
        if used[j]:
            s_in.wait_event(kern_done[j])   # step i-2's kernel no longer reads these inputs
        with torch.cuda.stream(s_in):
            dev[j][0].copy_(host[i % nsets], non_blocking=True)  # all inputs of the step in one copy
            in_ready[j].record(s_in)
        compute.wait_event(in_ready[j])
        if used[j]:
            compute.wait_event(out_done[j])  # step i-2's outputs were read back
        q, k, v, g, beta, slots = dev[j][1]
        gdn.gdn_decode(q, k, v, g, beta, pool, slots, obuf[j], scale=inp.scale, stream=compute)
        kern_done[j].record(compute)
        s_out.wait_event(kern_done[j])
        with torch.cuda.stream(s_out):
            o_host[j].copy_(obuf[j], non_blocking=True)
            out_done[j].record(s_out)
        used[j] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    start.record(compute)
    for i in range(steps):
        step(warmup + i)
    compute.wait_event(out_done[(warmup + steps - 1) % 2])  # the last read-back is inside the region
    stop.record(compute)
    torch.cuda.synchronize()
    barrier(ws)
    e_ms = max_over_ranks(start.elapsed_time(stop), ws) / steps
    return {"value": state_b / (e_ms * 1e-3) / 1e9 * ws, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
            "method": "per step: one pinned H2D copy of all inputs (q, k, v, g, beta, slot ids), gdn_decode, "
                      "D2H of o; copies on two side streams, double-buffered, overlapping the previous "
                      "step's kernel"}


def bench_decode(key, steps, warmup, ws, rank, peaks, e2e=True):
    import gated_delta_rule_58_b200 as gdn
    from gated_delta_rule_58_b200 import inputs
    c = DECODE_CFGS[key]
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = inputs.decode_inputs(c["B"], c["T"], c["H"], c["d"], c["d"], c["nh"], c["slots"],
                               seed=rank, device=dev)
    nsets = c["slots"] // c["B"]
    perm = torch.randperm(c["slots"], generator=torch.Generator().manual_seed(rank)).to(torch.int32)
    slot_sets = [perm[i * c["B"]:(i + 1) * c["B"]].to(dev) for i in range(nsets)]
    o = torch.empty((c["B"], c["T"], c["H"], c["d"]), dtype=torch.bfloat16, device=dev)
    pool = inp.pool

    def step(i):
        gdn.gdn_decode(inp.q, inp.k, inp.v, inp.g, inp.beta, pool, slot_sets[i % nsets], o, scale=inp.scale)

    # the steps are replayed as one CUDA graph (launch overhead off the GPU's path);
    # the eager per-launch timing is reported beside it
    total_ms = time_graph(step, steps, warmup, ws)
    eager_total, per = time_launches(step, min(steps, 200), warmup, ws)
    state_b, alg_b = decode_bytes(c)
    ms = total_ms / steps
    res = {
        "workload": c["name"],
        "ms_per_step": ms,
        "state_gbs": state_b / (ms * 1e-3) / 1e9 * ws,
        "launch_ms_mean": ms,
        "eager_ms_per_step": eager_total / min(steps, 200),
        "eager_launch_ms_mean": statistics.fmean(per),
        "launches_per_step": 1,
        "alg_bytes_per_launch": alg_b,
        "state_bytes_per_launch": state_b,
        "timing": "CUDA graph of the timed steps, one kernel per step",
    }
    if e2e:
        res["e2e"] = e2e_decode(gdn, inp, pool, o, slot_sets, nsets, steps, warmup, ws, state_b)
    achieved = alg_b / (res["launch_ms_mean"] * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    res["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                       "frac": achieved / peak,
                       "traffic": ncu_traffic(key)}
    res["pct_of_8tbs_state"] = res["state_gbs"] / ws / NOMINAL_HBM_GBS * 100
    return res


# ---------------------------------------------------------------- prefill workloads

def prefill_cfg(key, device, seed):
    from gated_delta_rule_58_b200 import inputs
    if key == "prefill":
        return inputs.prefill_b4_t8192_h16(device=device, seed=seed), 64, \
            "chunked prefill, B=4 x T=8192, H=16, dk=dv=128, chunk 64, bf16 q/k/v, fp32 initial state"
    if key == "varlen":
        return inputs.varlen32_h32(device=device, seed=seed), 64, \
            "varlen prefill, 32 seqs L~U[64,16384], H=32, dk=dv=128, chunk 64"
    if key == "longseq":
        return inputs.longseq_b1_t65536_h4(device=device, seed=seed), 64, \
            "low-parallelism prefill, B=1 x T=65536, H=4, dk=dv=128, chunk 64"
    if key == "tiny":
        return inputs.tiny_prefill(device=device, seed=seed), 16, \
            "tiny prefill, B=1, H=2, T=64, dk=dv=32, fp32, chunk 16"
    raise KeyError(key)


def prefill_alg_bytes(inp):
    total, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    N = inp.cu_seqlens.numel() - 1
    es = inp.q.element_size()
    per_tok = H * ((2 * dk + dv) * es + 8 + dv * 2)
    states = N * H * dk * dv * 4 * (2 if inp.initial_state is not None else 1)
    return total * per_tok + states


def prefill_flops(inp, chunk):
    """Algorithmic flops of the chunked form per (sequence, head) chunk, summed."""
    total, H, d = inp.q.shape
    lens = inp.seqlens
    f = 0
    for L in lens:
        full, rem = divmod(L, chunk)
        for C in [chunk] * full + ([rem] if rem else []):
            f += 5 * 2 * C * C * d + 3 * 2 * C * d * d + 2 * C ** 3 // 3
    return f * H


def bench_prefill(key, steps, warmup, ws, rank, peaks, algo=None):
    import gated_delta_rule_58_b200 as gdn
    dev = torch.device("cuda", torch.cuda.current_device())
    inp, chunk, name = prefill_cfg(key, dev, rank)
    algo = gdn.GDN_PREFILL_AUTO if algo is None else algo
    total, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    N = inp.cu_seqlens.numel() - 1
    o = torch.empty((total, H, dv), dtype=torch.bfloat16, device=dev)
    fin = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    ws_bytes = gdn.gdn_chunk_prefill_workspace_size(N, total, H, dk, dv, chunk, algo)
    work = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    def step(i):
        gdn.gdn_chunk_prefill(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, o,
                              initial_state=inp.initial_state, final_state=fin, chunk=chunk,
                              scale=inp.scale, algo=algo, workspace=work)

    total_ms, per = time_launches(step, steps, warmup, ws)
    ms = total_ms / steps
    alg_b = prefill_alg_bytes(inp)
    flops = prefill_flops(inp, chunk)
    t = ms * 1e-3
    hbm_t = alg_b / (peaks["hbm_gbs"] * 1e9)
    tc_t = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if hbm_t >= tc_t else "tensor"
    res = {
        "workload": name,
        "algo": {0: "auto", 1: "fused", 2: "transfer", 3: "sequential"}[algo],
        "ms_per_step": ms,
        "tokens_per_s": total / t * ws,
        "roofline": {"bound": bound,
                     "achieved": alg_b / t / 1e9 if bound == "hbm" else flops / t / 1e12,
                     "peak": peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"],
                     "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                     "frac": max(hbm_t, tc_t) / t,
                     "traffic": ncu_traffic(key)},
        "pct_of_nominal_roofline": max(alg_b / (NOMINAL_HBM_GBS * 1e9), flops / 2.25e15) / t * 100,
        "alg_bytes": alg_b,
        "flops": flops,
        "workspace_bytes": ws_bytes,
    }
    del inp, o, fin, work
    torch.cuda.empty_cache()
    return res


def backward_alg_flops(inp):
    """Algorithmic fp32 flops of one backward step, per token and value head and per
    entry of the dk x dv state: one forward step to regain S_t (u = S~^T k and the
    update, 2 FMAs) and the reverse step (D += q dO^T, the terms S_t dO of dq, w = D^T k,
    D (v - u) and S~ w of dk, <D, S~> of dg, D <- alpha (D - beta k w^T): 7.5 FMAs) =
    19 flops. The recomputation of the states from checkpoints is not counted."""
    total, _, dk = inp.q.shape
    H, dv = inp.v.shape[1], inp.v.shape[-1]
    return 19.0 * total * H * dk * dv


def backward_alg_bytes(inp):
    """Algorithmic HBM bytes of one backward step: q, k, v and d_o read (input dtype),
    g and beta read, dq, dk, dv, dg, dbeta written (fp32), and per (sequence, head) the
    initial state and the final-state derivative read and the initial-state
    derivative written (fp32)."""
    total, Hqk, dk = inp.q.shape
    H, dv = inp.v.shape[1], inp.v.shape[-1]
    N = inp.cu_seqlens.numel() - 1
    es = inp.q.element_size()
    per_tok = Hqk * 2 * dk * (es + 4) + H * (2 * dv * es + 8 + dv * 4 + 8)
    return total * per_tok + 3 * N * H * dk * dv * 4


def backward_inputs(key, device, seed):
    """The backward part runs on the chunked-prefill workload with seeded upstream
    derivatives d_o (bf16, N(0, 1)) and d_final_state (fp32, N(0, 0.1^2))."""
    inp, _, name = prefill_cfg("prefill", device, seed)
    # checkpoints every 16 tokens: a chunk's recomputed states (16 x 64 KiB per head)
    # then stay in L2 between their write and their read
    chunk = 16
    gen = torch.Generator(device=device).manual_seed(seed + 7)
    total, H, dv = inp.v.shape
    N = inp.cu_seqlens.numel() - 1
    d_o = torch.randn((total, H, dv), generator=gen, device=device).to(inp.q.dtype)
    d_fin = torch.randn((N, H, dv, inp.q.shape[-1]), generator=gen, device=device) * 0.1
    return inp, d_o, d_fin, chunk, ("prefill backward (dq, dk, dv, dg, dbeta, d_initial_state), checkpoints every "
                                     "16 tokens, " + name)


def bench_backward(key, steps, warmup, ws, rank, peaks):
    import gated_delta_rule_58_b200 as gdn
    dev = torch.device("cuda", torch.cuda.current_device())
    inp, d_o, d_fin, chunk, name = backward_inputs(key, dev, rank)
    total, Hqk, dk = inp.q.shape
    H, dv = inp.v.shape[1], inp.v.shape[-1]
    N = inp.cu_seqlens.numel() - 1
    f = dict(dtype=torch.float32, device=dev)
    grads = dict(dq=torch.empty((total, Hqk, dk), **f), dk=torch.empty((total, Hqk, dk), **f),
                 dv=torch.empty((total, H, dv), **f), dg=torch.empty((total, H), **f),
                 dbeta=torch.empty((total, H), **f), d_initial_state=torch.empty((N, H, dv, dk), **f))
    ws_bytes = gdn.gdn_chunk_prefill_backward_workspace_size(N, total, H, dk, dv, chunk)
    work = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(i):
        gdn.gdn_chunk_prefill_backward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, d_o,
                                       initial_state=inp.initial_state, d_final_state=d_fin, chunk=chunk,
                                       scale=inp.scale, workspace=work, grads=grads)

    total_ms, per = time_launches(step, steps, warmup, ws)
    ms = total_ms / steps
    t = ms * 1e-3
    alg_b = backward_alg_bytes(inp)
    alg_f = backward_alg_flops(inp)
    # the arithmetic, not the memory, bounds this step: its flops take about 11x as
    # long at the fp32 peak as its bytes at the copy peak
    achieved = alg_f / t / 1e12
    res = {
        "workload": name,
        "algo": "token-sequential with chunk checkpoints",
        "ms_per_step": ms,
        "tokens_per_s": total / t * ws,
        "roofline": {"bound": "alu", "achieved": achieved, "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
                     "frac": achieved / FP32_SIMT_TFLOPS, "traffic": ncu_traffic(key),
                     "peak_source": "148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz"},
        "hbm_frac": alg_b / t / 1e9 / peaks["hbm_gbs"],
        "pct_of_nominal_roofline": alg_b / (NOMINAL_HBM_GBS * 1e9) / t * 100,
        "alg_flops": alg_f,
        "alg_bytes": alg_b,
        "workspace_bytes": ws_bytes,
    }
    del inp, d_o, d_fin, grads, work
    torch.cuda.empty_cache()
    return res


CP_RANKS = 4


def bench_cp(key, steps, warmup, peaks):
    """Context-parallel prefill of the low-parallelism workload (B=1 x 65536, H=4)
    over CP_RANKS ranks, emulated one after another on this GPU (no kernel waits on
    another rank; the exchange, an all-gather of the (local state, transfer) pairs,
    is a device copy here). Each rank's slice is a contiguous quarter of the
    sequence; its device time (local state and transfer, combine, finish of the
    slice) is timed with CUDA events, and the part reports the maximum over ranks:
    the step time CP_RANKS GPUs would need with a free exchange."""
    import gated_delta_rule_58_b200 as gdn
    dev = torch.device("cuda", torch.cuda.current_device())
    inp, chunk, name = prefill_cfg("longseq", dev, 0)
    T, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    R = CP_RANKS
    cuts = [T * r // R for r in range(R + 1)]
    sl = []
    for r in range(R):
        a, b = cuts[r], cuts[r + 1]
        cu = torch.tensor([0, b - a], dtype=torch.int32, device=dev)
        sl.append([x[a:b].contiguous() for x in (inp.q, inp.k, inp.v, inp.g, inp.beta)] + [cu])
    loc = torch.empty((R, 1, H, dv, dk), device=dev)
    tr = torch.empty_like(loc)
    start = torch.empty((R, 1, H, dv, dk), device=dev)
    o = torch.empty((T, H, dv), dtype=torch.bfloat16, device=dev)
    fin = torch.empty((1, H, dv, dk), device=dev)
    gathered = torch.empty((2, R, 1, H, dv, dk), device=dev)
    ws_cp = [torch.empty(gdn.gdn_cp_local_state_workspace_size(1, cuts[r + 1] - cuts[r], H, dk, dv, chunk),
                         dtype=torch.uint8, device=dev) for r in range(R)]

    def rank_step(r):
        q, k, v, g, beta, cu = sl[r]
        gdn.gdn_cp_local_state(q, k, v, g, beta, cu, loc[r], tr[r], chunk=chunk, workspace=ws_cp[r])
        gathered[0].copy_(loc)  # stands in for the all-gather
        gathered[1].copy_(tr)
        gdn.gdn_cp_combine(gathered[0], gathered[1], r, start[r], initial_state=inp.initial_state)
        gdn.gdn_cp_finish(q, k, v, g, beta, cu, o[cuts[r]:cuts[r + 1]], ws_cp[r], start_state=start[r],
                          final_state=fin, chunk=chunk, scale=inp.scale)

    for _ in range(warmup):
        for r in range(R):
            rank_step(r)
    torch.cuda.synchronize()
    per_rank = []
    for r in range(R):
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_.record()
        for _ in range(steps):
            rank_step(r)
        e_.record()
        torch.cuda.synchronize()
        per_rank.append(s_.elapsed_time(e_) / steps)
    ms = max(per_rank)
    alg_b = prefill_alg_bytes(inp)
    exchange = 2 * R * H * dv * dk * 4
    achieved = alg_b / (ms * 1e-3) / 1e9
    res = {
        "workload": f"context-parallel prefill over {R} ranks emulated on one GPU, {name}",
        "algo": "per rank: local state and transfer over segments (fused kernel, two folds in one fixup launch), "
                "combine (fixup scan), finish (fixup scan from the start state, output pass over the segments)",
        "ms_per_step": ms,
        "ms_per_rank": per_rank,
        "tokens_per_s": T / (ms * 1e-3),
        "exchange_bytes_per_rank": exchange,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"] * R, "unit": "GB/s",
                     "frac": achieved / (peaks["hbm_gbs"] * R), "traffic": ncu_traffic(key),
                     "note": f"peak = {R} GPUs' copy bandwidth; not a multi-GPU measurement"},
        "alg_bytes": alg_b,
    }
    del sl, loc, tr, start, o, fin, gathered, ws_cp, inp
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

class OracleDecode:
    """The fp64 CPU oracle on a decode workload, timed on the host cores. A sample is
    the first `rows` batch rows of one full step (all heads), so its cost is bounded."""

    def __init__(self, key, seed=0):
        import oracle
        from gated_delta_rule_58_b200 import inputs
        self.oracle = oracle
        self.c = DECODE_CFGS[key]
        c = self.c
        inp = inputs.decode_inputs(c["B"], c["T"], c["H"], c["d"], c["d"], c["nh"], c["slots"], seed=seed)
        self.args = [oracle.f64(x) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
        self.pool = oracle.f64(inp.pool)
        self.slots = inp.slot_ids
        self.scale = inp.scale
        self.threads = 0

    def step(self, rows):
        """One oracle call on `rows` batch rows; returns its wall time in seconds."""
        sub = [a[:rows] for a in self.args]
        t0 = time.perf_counter()
        _, self.pool, self.threads = self.oracle.decode(*sub, self.pool, self.slots[:rows], scale=self.scale,
                                                        copy_pool=False)
        return time.perf_counter() - t0

    def state_bytes(self, rows):
        c = self.c
        return 2 * rows * c["H"] * c["d"] * c["d"] * 4

    def rows_for(self, seconds):
        """Batch rows whose oracle step takes about `seconds` (at least one row)."""
        B = self.c["B"]
        t_full = self.step(B)
        return B if t_full <= seconds else max(1, int(B * seconds / t_full))


def oracle_decode_rate(key, budget_s=10.0, seed=0):
    """cpu_baseline: the oracle on the decode workload for about budget_s; returns
    state GB/s-equivalent, threads used and the sample description."""
    od = OracleDecode(key, seed)
    rows = od.rows_for(budget_s / 10)
    n, dt = 0, 0.0
    while dt < budget_s:
        dt += od.step(rows)
        n += 1
    return (od.state_bytes(rows) * n / dt / 1e9, od.threads,
            f"{n} oracle steps of {rows} of {od.c['B']} batch rows x {od.c['H']} heads ({od.c['name']}), "
            f"{dt:.1f} s")


def oracle_prefill_rate(key, budget_s=4.0, seed=0):
    """cpu_baseline of a prefill part: the fp64 oracle on the first L tokens of every
    sequence of the workload (all heads), L chosen from a short calibration run so
    the timed call takes about budget_s. Returns tokens/s (a token = all H heads of
    one position, as in the GPU metric), the threads used and the sample."""
    import numpy as np
    import oracle
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"  # the sample is copied to the host
    inp, _, name = prefill_cfg(key, gen_dev, seed)
    cu = inp.cu_seqlens.tolist()
    N = len(cu) - 1
    H = inp.q.shape[1]
    longest = max(cu[n + 1] - cu[n] for n in range(N))

    def sample(L):
        lens = [min(L, cu[n + 1] - cu[n]) for n in range(N)]
        idx = torch.cat([torch.arange(cu[n], cu[n] + lens[n]) for n in range(N)])
        new_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        idx_dev = idx.to(inp.q.device)
        args = [oracle.f64(t[idx_dev]) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
        return args, new_cu, int(new_cu[-1])

    init = oracle.f64(inp.initial_state)

    def timed(L, reps=1):
        args, new_cu, tokens = sample(L)
        t0 = time.perf_counter()
        for _ in range(reps):
            _, _, threads = oracle.prefill(*args, new_cu, init, scale=inp.scale)
        return time.perf_counter() - t0, threads, tokens * reps

    L = min(64, longest)
    dt, threads, tokens = timed(L)
    reps = 1
    if L < longest:
        L = max(L, min(longest, int(L * budget_s / max(dt, 1e-3)) // 64 * 64))
        dt, threads, tokens = timed(L)
    else:  # the whole workload is short: repeat it
        reps = max(1, int(budget_s / max(dt, 1e-4)))
        dt, threads, tokens = timed(L, reps)
    note = f" ({N * H} (sequence, head) chains: at most {N * H} threads)" if N * H < 16 else ""
    rep = f", {reps} calls" if reps > 1 else ""
    return (tokens / dt, threads,
            f"oracle on the first {L} tokens of each of the {N} sequences x {H} heads "
            f"({tokens // reps} tokens{rep}) of '{name}', {dt:.1f} s{note}")


def oracle_backward_rate(key, budget_s=4.0, seed=0):
    """cpu_baseline of the backward part: the fp64 oracle's backward on the first L
    tokens of every sequence (all heads), L sized from a calibration call so the timed
    call takes about budget_s. Returns tokens/s, threads used and the sample."""
    import numpy as np
    import oracle
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp, d_o, d_fin, _, name = backward_inputs(key, gen_dev, seed)
    cu = inp.cu_seqlens.tolist()
    N = len(cu) - 1
    H = inp.v.shape[1]
    longest = max(cu[n + 1] - cu[n] for n in range(N))

    def timed(L):
        lens = [min(L, cu[n + 1] - cu[n]) for n in range(N)]
        idx = torch.cat([torch.arange(cu[n], cu[n] + lens[n]) for n in range(N)]).to(inp.q.device)
        new_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        args = [oracle.f64(t[idx]) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
        t0 = time.perf_counter()
        oracle.prefill_backward(*args, new_cu, oracle.f64(d_o[idx]), oracle.f64(inp.initial_state),
                                oracle.f64(d_fin), scale=inp.scale)
        return time.perf_counter() - t0, int(new_cu[-1])

    L = min(16, longest)
    dt, tokens = timed(L)
    L = max(L, min(longest, int(L * budget_s / max(dt, 1e-3))))
    dt, tokens = timed(L)
    threads = min(os.cpu_count() or 1, N * H)
    return (tokens / dt, threads,
            f"oracle backward on the first {L} tokens of each of the {N} sequences x {H} heads "
            f"({tokens} tokens) of '{name}', {dt:.1f} s")


def run_reference(args, ws, rank):
    """The reference arm: the fp64 CPU oracle on the headline workload, on rank 0 only.
    Each step is a bounded sample (the first rows of the batch, all heads), sized so the
    whole run takes about --reference-seconds (two minutes) whatever --steps/--warmup are."""
    if rank != 0:
        return
    steps, warmup = args.steps, args.warmup
    od = OracleDecode("decode")
    per_step = args.reference_seconds / (steps + warmup)
    rows = od.rows_for(per_step)
    for _ in range(warmup):
        od.step(rows)
    t = sum(od.step(rows) for _ in range(steps))
    value = od.state_bytes(rows) * steps / t / 1e9
    c = od.c
    sample = (f"each step: the oracle on {rows} of {c['B']} batch rows x {c['H']} heads of one decode "
              f"step; {steps} timed steps in {t:.3f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
        "steps": steps, "warmup": warmup, "ms_per_step": t / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": c["name"], "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": od.threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--parts", default="gdp,decode_b1,decode_b4,decode_b16,prefill,varlen,longseq,tiny,backward,cp",
                    help="comma list of extra workloads to measure ('none' for none)")
    ap.add_argument("--part-steps", type=int, default=5,
                    help="timed steps of each prefill part (decode parts: 20 times this, at least 20)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="wall-time budget of the --impl reference run")
    ap.add_argument("--prefill-algo", default=None, help="force fused|transfer|sequential for the parts")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    ws, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import gated_delta_rule_58_b200 as gdn
    gdn.lib()  # fails loudly if the CUDA library is missing
    peaks, peak_src = load_peaks()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    vis_list = [x for x in vis.split(",") if x]
    gpu_index = vis_list[local] if local < len(vis_list) else str(local)

    with ClockSampler(gpu_index) as clk:
        with torch.cuda.nvtx.range("decode"):  # NVTX ranges let ncu select one workload
            head = bench_decode("decode", args.steps, args.warmup, ws, rank, peaks)
        parts = []
        algo = None
        if args.prefill_algo:
            algo = {"fused": gdn.GDN_PREFILL_FUSED, "transfer": gdn.GDN_PREFILL_TRANSFER,
                    "sequential": gdn.GDN_PREFILL_SEQUENTIAL}[args.prefill_algo]
        for key in [p for p in args.parts.split(",") if p and p != "none"]:
            torch.cuda.nvtx.range_push(key)
            try:
                if key in DECODE_CFGS:
                    r = bench_decode(key, max(args.part_steps * 20, 20), args.warmup, ws, rank, peaks,
                                     e2e=False)
                    r["metric"] = "GDP decode state GB/s" if key == "gdp" else "decode state GB/s"
                elif key == "backward":
                    r = bench_backward(key, max(args.part_steps // 2, 1), 3, ws, rank, peaks)
                    r["metric"] = "backward tokens/s"
                elif key == "cp":
                    r = bench_cp(key, args.part_steps, 3, peaks)
                    r["metric"] = "prefill tokens/s (max over emulated ranks)"
                else:
                    r = bench_prefill(key, args.part_steps, 3, ws, rank, peaks, algo=algo)
                    r["metric"] = "prefill tokens/s"
                r["key"] = key
            except Exception as e:  # a part that is not supported is reported, not fatal
                r = {"key": key, "error": f"{type(e).__name__}: {e}"}
            torch.cuda.nvtx.range_pop()
            parts.append(r)

    if ws > 1:
        import torch.distributed as dist
        dist.barrier()

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and ws == 1:
            v, threads, sample = oracle_decode_rate("decode", budget_s=10.0)
            cpu = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample}
            for r in parts:  # every part gets the oracle's rate in the part's own unit
                if "error" in r:
                    continue
                if r["key"] in DECODE_CFGS:
                    v, threads, sample = oracle_decode_rate(r["key"], budget_s=2.0 if r["key"] != "gdp" else 4.0)
                    r["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                         "sample": sample}
                elif r["key"] == "cp":
                    v, threads, sample = oracle_prefill_rate("longseq", budget_s=4.0)
                    r["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                         "sample": sample}
                elif r["key"] == "backward":
                    v, threads, sample = oracle_backward_rate(r["key"], budget_s=4.0)
                    r["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                         "sample": sample}
                else:
                    v, threads, sample = oracle_prefill_rate(r["key"], budget_s=4.0)
                    r["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                         "sample": sample}
        clocks = clk.summary()
        line = {
            "metric": METRIC,
            "value": head["state_gbs"],
            "unit": "GB/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": head["workload"],
                       "timing": head["timing"],
                       "eager_ms_per_step": head["eager_ms_per_step"],
                       "l2": "inputs larger than L2: steps rotate over 4 disjoint 64-slot sets of a 512 MiB pool",
                       "parallelism": f"dp{ws} (independent sequences per GPU)",
                       "pct_of_8tbs_state": head["pct_of_8tbs_state"],
                       "peaks": peak_src},
            "roofline": head["roofline"],
            "cpu_baseline": cpu,
            "e2e": head.get("e2e"),
            "gpu_launches": args.steps,
            "clocks": clocks,
            "parts": parts,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
