"""GPU parity of gdn_decode (gated delta rule T=1 and the gated delta product)
against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import inputs
from tests.util import assert_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(inp, out_dtype=torch.bfloat16, l2norm=False):
    pool = inp.pool.to(DEV).clone()
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    g, beta = inp.g.to(DEV), inp.beta.to(DEV)
    slots = inp.slot_ids.to(DEV)
    B, T, H = v.shape[:3]
    o = torch.empty((B, T, H, v.shape[-1]), dtype=out_dtype, device=DEV)
    gdn.gdn_decode(q, k, v, g, beta, pool, slots, o, scale=inp.scale, l2norm=l2norm)
    torch.cuda.synchronize()
    return o, pool


def _check_against_oracle(inp, o, pool, what, l2norm=False):
    o_ref, pool_ref, _ = oracle.decode(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.pool, inp.slot_ids,
                                       scale=inp.scale, l2norm=l2norm)
    assert_close(o, o_ref, what=f"{what} o")
    used = sorted(set(int(s) for s in inp.slot_ids.tolist() if 0 <= s < inp.pool.shape[0]))
    assert_close(pool[used], pool_ref[used], what=f"{what} state")
    untouched = [s for s in range(inp.pool.shape[0]) if s not in used]
    assert torch.equal(pool[untouched].cpu(), inp.pool[untouched]), "untouched slots changed"


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_b64_h32_full_size(out_dtype):
    """T=1 decode at the benchmark size: B=64, H=32, dk=dv=128, 256 slots, every head
    checked; fp32 outputs are held to the 2e-3 normwise bar directly."""
    inp = inputs.decode_b64_h32()
    o, pool = _run(inp, out_dtype=out_dtype)
    _check_against_oracle(inp, o, pool, f"decode B64 H32 ({out_dtype})")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gdp_b128_h32_t4_nh2_full_size(out_dtype):
    """Gated delta product at the benchmark size: B=128, H=32, T=4, n_h=2, 512 slots."""
    inp = inputs.gdp_b128_h32_t4_nh2()
    o, pool = _run(inp, out_dtype=out_dtype)
    _check_against_oracle(inp, o, pool, f"GDP B128 T4 nh2 ({out_dtype})")


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("T,nh", [(1, 1), (2, 1), (4, 1), (8, 1), (1, 2), (2, 2), (4, 2), (1, 4), (2, 4)])
def test_decode_shapes(d, T, nh):
    inp = inputs.decode_inputs(5, T, 3, d, d, nh, 9, seed=d + 10 * T + nh)
    o, pool = _run(inp, out_dtype=torch.float32)
    _check_against_oracle(inp, o, pool, f"d={d} T={T} nh={nh}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_input_dtypes(dtype):
    inp = inputs.decode_inputs(7, 2, 4, 128, 128, 2, 10, seed=3, dtype=dtype)
    for out in (torch.float32, torch.bfloat16):
        o, pool = _run(inp, out_dtype=out)
        _check_against_oracle(inp, o, pool, f"in={dtype} out={out}")


@pytest.mark.parametrize("T,nh,dtype", [(4, 2, torch.float32), (8, 1, torch.bfloat16), (4, 2, torch.bfloat16)])
def test_multi_token_many_items_per_cta(T, nh, dtype):
    """Several items per CTA (B*H = 151*3 over at most 148 CTAs), so both consumer
    groups cycle through the stages more than once, with skipped rows in between;
    fp32 inputs and T=8 run with two stages, bf16 T=4 n_h=2 with three."""
    inp = inputs.decode_inputs(151, T, 3, 128, 128, nh, 160, seed=21 + T + nh, dtype=dtype)
    inp.slot_ids[5] = -1
    inp.slot_ids[77] = -1
    o, pool = _run(inp, out_dtype=torch.float32)
    assert torch.all(o[5] == 0) and torch.all(o[77] == 0)
    _check_against_oracle(inp, o, pool, f"many items T={T} nh={nh} {dtype}")
    assert gdn.gdn_get_device_error() == 0


def test_decode_weak_and_zero_decay():
    for g_range in ((0.0, 0.0), (0.0, 0.01)):
        inp = inputs.decode_inputs(8, 4, 4, 128, 128, 2, 16, seed=5, g_range=g_range)
        o, pool = _run(inp, out_dtype=torch.float32)
        _check_against_oracle(inp, o, pool, f"g_range={g_range}")


def test_decode_alpha_zero():
    """g = -inf (alpha = 0): the old state is dropped exactly."""
    inp = inputs.decode_inputs(4, 1, 2, 128, 128, 1, 6, seed=6)
    inp.g.fill_(float("-inf"))
    o, pool = _run(inp, out_dtype=torch.float32)
    _check_against_oracle(inp, o, pool, "alpha=0")
    s = int(inp.slot_ids[0])
    exp = inp.beta[0, 0, 0, 0] * torch.outer(inp.v[0, 0, 0, 0].float(), inp.k[0, 0, 0, 0].float())
    assert torch.allclose(pool[s, 0].cpu(), exp, rtol=1e-6, atol=1e-7)


def test_negative_slot_skips_row():
    inp = inputs.decode_inputs(4, 2, 2, 64, 64, 1, 8, seed=7)
    inp.slot_ids[1] = -1
    o, pool = _run(inp, out_dtype=torch.float32)
    assert torch.all(o[1] == 0)
    _check_against_oracle(inp, o, pool, "negative slot")
    assert gdn.gdn_get_device_error() == 0


def test_out_of_range_slot_is_flagged_and_skipped():
    inp = inputs.decode_inputs(3, 1, 2, 128, 128, 1, 6, seed=8)
    gdn.gdn_get_device_error()  # clear
    inp.slot_ids[2] = 6  # == num_slots
    o, pool = _run(inp, out_dtype=torch.float32)
    assert torch.all(o[2] == 0)
    flags = gdn.gdn_get_device_error()
    assert flags & gdn.GDN_DEVERR_SLOT_OUT_OF_RANGE
    assert gdn.gdn_get_device_error() == 0  # read clears
    _check_against_oracle(inp, o, pool, "slot out of range")


def test_decode_deterministic_and_permutation_equivariant():
    inp = inputs.decode_b64_h32(seed=11)
    o1, p1 = _run(inp)
    o2, p2 = _run(inp)
    assert torch.equal(o1, o2) and torch.equal(p1, p2)
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(0))
    inp_p = inputs.DecodeInputs(inp.q[perm], inp.k[perm], inp.v[perm], inp.g[perm], inp.beta[perm],
                                inp.pool, inp.slot_ids[perm], inp.scale)
    o3, p3 = _run(inp_p)
    assert torch.equal(o3, o1[perm.to(DEV)]) and torch.equal(p3, p1)


def test_decode_T_steps_equal_sequential_prefill_on_gpu():
    """Decode applied token by token == the sequential GPU prefill over the same tokens."""
    T, H, d = 6, 2, 64
    pin = inputs.prefill_inputs([T], H, d, d, seed=12)
    pool = torch.zeros((2, H, d, d), device=DEV)
    pool[1] = pin.initial_state[0].to(DEV)
    slots = torch.tensor([1], dtype=torch.int32, device=DEV)
    outs = []
    for t in range(T):
        o = torch.empty((1, 1, H, d), device=DEV)
        gdn.gdn_decode(pin.q[t][None, None].to(DEV), pin.k[t][None, None, :, None].to(DEV),
                       pin.v[t][None, None, :, None].to(DEV), pin.g[t][None, None].to(DEV),
                       pin.beta[t][None, None, :, None].to(DEV), pool, slots, o, scale=pin.scale)
        outs.append(o[0, 0])
    o_p = torch.empty((T, H, d), device=DEV)
    fin = torch.empty((1, H, d, d), device=DEV)
    gdn.gdn_chunk_prefill(pin.q.to(DEV), pin.k.to(DEV), pin.v.to(DEV), pin.g.to(DEV),
                          pin.beta.to(DEV), pin.cu_seqlens.to(DEV), o_p,
                          initial_state=pin.initial_state.to(DEV), final_state=fin, chunk=16,
                          scale=pin.scale, algo=gdn.GDN_PREFILL_SEQUENTIAL)
    assert_close(torch.stack(outs), o_p, tol=1e-5, what="decode vs prefill o")
    assert_close(pool[1], fin[0], tol=1e-5, what="decode vs prefill state")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_split_v_small_batch_bitwise_equals_whole_heads(B):
    """With few heads the T=1 step splits each head's state rows over several items
    (the split along V). Each row gets the same arithmetic in the same order, so the
    first B batch rows of a B=64 x H=32 step (whole heads per item) must come out
    bitwise identical when they are run alone (split heads)."""
    inp = inputs.decode_b64_h32(seed=13)
    o_full, p_full = _run(inp, out_dtype=torch.float32)
    sub = inputs.DecodeInputs(inp.q[:B], inp.k[:B], inp.v[:B], inp.g[:B], inp.beta[:B], inp.pool,
                              inp.slot_ids[:B], inp.scale)
    o, p = _run(sub, out_dtype=torch.float32)
    used = sub.slot_ids.long().to(DEV)
    assert torch.equal(o, o_full[:B])
    assert torch.equal(p[used], p_full[used])
    _check_against_oracle(sub, o, p, f"split-V B={B}")


def test_split_v_b1_h4_against_oracle():
    """B=1, H=4: four heads, each split into parts of 16 state rows."""
    for out_dtype in (torch.float32, torch.bfloat16):
        inp = inputs.decode_inputs(1, 1, 4, 128, 128, 1, 3, seed=14)
        o, pool = _run(inp, out_dtype=out_dtype)
        _check_against_oracle(inp, o, pool, f"split-V B=1 H=4 ({out_dtype})")


# ---------------------------------------------------------------- grouped q/k heads, q/k normalisation

@pytest.mark.parametrize("l2norm", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_heads_b64_hv32_hqk8(l2norm, out_dtype):
    """T=1 decode with 32 value heads over 8 q/k heads (each q/k head shared by four
    value heads), B=64, 256 slots; with the in-kernel normalisation q and k are
    un-normalised N(0, 1) draws."""
    inp = inputs.decode_inputs(64, 1, 32, 128, 128, 1, 256, seed=15, H_qk=8, normalize_qk=not l2norm)
    o, pool = _run(inp, out_dtype=out_dtype, l2norm=l2norm)
    _check_against_oracle(inp, o, pool, f"GVA B64 Hv32 Hqk8 l2={l2norm} ({out_dtype})", l2norm=l2norm)


@pytest.mark.parametrize("T,nh", [(4, 2), (2, 1), (1, 4)])
@pytest.mark.parametrize("l2norm", [False, True])
def test_grouped_heads_multi_token(T, nh, l2norm):
    inp = inputs.decode_inputs(9, T, 8, 128, 128, nh, 12, seed=16 + T, H_qk=2, normalize_qk=not l2norm)
    o, pool = _run(inp, out_dtype=torch.float32, l2norm=l2norm)
    _check_against_oracle(inp, o, pool, f"GVA T={T} nh={nh} l2={l2norm}", l2norm=l2norm)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_grouped_heads_split_v_l2norm(d):
    """Few heads (the split along V) with one q/k head for all value heads and the
    normalisation on."""
    inp = inputs.decode_inputs(2, 1, 4, d, d, 1, 5, seed=17 + d, H_qk=1, normalize_qk=False)
    o, pool = _run(inp, out_dtype=torch.float32, l2norm=True)
    _check_against_oracle(inp, o, pool, f"GVA split-V d={d}", l2norm=True)


def test_l2norm_of_normalised_inputs_changes_little():
    """On inputs that are already unit vectors (in bf16) the normalisation only
    corrects their bf16 rounding of the norm."""
    inp = inputs.decode_inputs(8, 1, 4, 128, 128, 1, 10, seed=18)
    o1, p1 = _run(inp, out_dtype=torch.float32)
    o2, p2 = _run(inp, out_dtype=torch.float32, l2norm=True)
    assert_close(o2, o1, tol=5e-3, what="l2norm on unit inputs")


# ---------------------------------------------------------------- per-token states (speculative verify)

def _run_mtp(inp, update_pool, out_dtype=torch.float32, l2norm=False):
    pool = inp.pool.to(DEV).clone()
    q, k, v = inp.q.to(DEV), inp.k.to(DEV), inp.v.to(DEV)
    B, T, H = v.shape[:3]
    dk = q.shape[-1]
    o = torch.empty((B, T, H, v.shape[-1]), dtype=out_dtype, device=DEV)
    ts = torch.full((B, T, H, v.shape[-1], dk), float("nan"), device=DEV)
    gdn.gdn_decode_mtp(q, k, v, inp.g.to(DEV), inp.beta.to(DEV), pool, inp.slot_ids.to(DEV), o, ts,
                       update_pool=update_pool, scale=inp.scale, l2norm=l2norm)
    torch.cuda.synchronize()
    return o, pool, ts


@pytest.mark.parametrize("T,nh", [(4, 2), (2, 1), (1, 1), (8, 1), (1, 4)])
@pytest.mark.parametrize("update_pool", [True, False])
def test_mtp_token_states_against_oracle(T, nh, update_pool):
    """The state after every token (and the outputs) against the oracle; a skipped
    batch row gets zero states; with update_pool=False the pool is bitwise untouched."""
    inp = inputs.decode_inputs(6, T, 4, 128, 128, nh, 9, seed=60 + T + nh)
    inp.slot_ids[2] = -1
    o, pool, ts = _run_mtp(inp, update_pool)
    o_ref, pool_ref, _, ts_ref = oracle.decode(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.pool, inp.slot_ids,
                                               scale=inp.scale, token_states=True)
    assert_close(o, o_ref, what=f"mtp T={T} nh={nh} o")
    assert_close(ts, ts_ref, what=f"mtp T={T} nh={nh} token states")
    assert torch.all(ts[2] == 0)
    used = sorted(int(x) for x in inp.slot_ids.tolist() if x >= 0)
    if update_pool:
        assert_close(pool[used], pool_ref[used], what=f"mtp T={T} nh={nh} pool")
        assert torch.equal(ts[[b for b in range(6) if b != 2], T - 1].cpu(),
                           pool[[int(inp.slot_ids[b]) for b in range(6) if b != 2]].cpu())
    else:
        assert torch.equal(pool.cpu(), inp.pool)


def test_mtp_rollback_round_trip():
    """Verify 4 draft tokens without committing, accept 2: restoring the state after
    token 1 and decoding tokens 2-3 gives the full step's outputs and final state."""
    inp = inputs.decode_inputs(16, 4, 8, 128, 128, 2, 20, seed=64, g_range=(0.0, 0.05))
    o_full, pool_full = _run(inp, out_dtype=torch.float32)
    o, pool, ts = _run_mtp(inp, update_pool=False)
    assert_close(o, o_full, tol=1e-6, what="mtp outputs vs decode")
    rolled = pool.clone()
    slots = inp.slot_ids.long().to(DEV)
    rolled[slots] = ts[:, 1]
    rest = inputs.DecodeInputs(inp.q[:, 2:].contiguous(), inp.k[:, 2:].contiguous(), inp.v[:, 2:].contiguous(),
                               inp.g[:, 2:].contiguous(), inp.beta[:, 2:].contiguous(), rolled.cpu(),
                               inp.slot_ids, inp.scale)
    o2, pool2 = _run(rest, out_dtype=torch.float32)
    assert_close(o2, o_full[:, 2:], tol=1e-5, what="rollback outputs")
    assert_close(pool2[slots], pool_full[slots], tol=1e-5, what="rollback final state")


def test_mtp_split_v_grouped_l2norm():
    """T=1 with few heads (split along V), grouped q/k heads and the normalisation."""
    inp = inputs.decode_inputs(2, 1, 4, 128, 128, 1, 5, seed=65, H_qk=2, normalize_qk=False)
    o, pool, ts = _run_mtp(inp, update_pool=True, l2norm=True)
    o_ref, pool_ref, _, ts_ref = oracle.decode(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.pool, inp.slot_ids,
                                               scale=inp.scale, token_states=True, l2norm=True)
    assert_close(o, o_ref, what="mtp split-V o")
    assert_close(ts, ts_ref, what="mtp split-V token states")


def test_bounded_wait_gives_up_reports_timeout_and_the_context_stays_usable():
    """A bounded in-kernel wait on a barrier that nothing completes gives up after
    its limit, the device error word reports GDN_DEVERR_TIMEOUT (read and cleared
    once), and later calls on the same context still give the oracle's results."""
    gdn.gdn_get_device_error()  # clear
    gdn.gdn_selftest_wait_timeout(2000)  # 2 ms
    assert gdn.gdn_get_device_error() & gdn.GDN_DEVERR_TIMEOUT
    assert gdn.gdn_get_device_error() == 0
    inp = inputs.decode_inputs(3, 2, 2, 64, 64, 2, 5, seed=70)
    o, pool = _run(inp, out_dtype=torch.float32)
    _check_against_oracle(inp, o, pool, "after a timeout")
    assert gdn.gdn_get_device_error() == 0
