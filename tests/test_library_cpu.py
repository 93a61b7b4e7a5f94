"""The C-ABI library loads on a machine without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes

import pytest

import gated_delta_rule_58_b200 as gdn
from gated_delta_rule_58_b200 import _lib


@pytest.fixture(scope="module")
def L():
    from gated_delta_rule_58_b200 import build
    build.build()
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    names = _lib.declared_functions()
    assert {"gdn_decode", "gdn_chunk_prefill", "gdn_chunk_prefill_workspace_size",
            "gdn_last_error", "gdn_get_device_error", "gdn_version"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libgdn.so does not export {n}"


def test_version(L):
    assert "sm_100a" in gdn.gdn_version()


FAKE = 0x10000  # an aligned, never-dereferenced address: validation fails before any use


def _decode(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, pool=FAKE, num_slots=4, slots=FAKE, o=FAKE,
             B=2, T=1, H=2, Hqk=None, dk=128, dv=128, nh=1, scale=0.1, flags=0, din=0, dout=0, stream=None)
    a.update(kw)
    hqk = a["H"] if a["Hqk"] is None else a["Hqk"]
    return L.gdn_decode(a["q"], a["k"], a["v"], a["g"], a["beta"], a["pool"], a["num_slots"], a["slots"],
                        a["o"], a["B"], a["T"], a["H"], hqk, a["dk"], a["dv"], a["nh"], a["scale"], a["flags"],
                        a["din"], a["dout"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48, dv=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=128, dv=64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(nh=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(din=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(pool=FAKE + 4), gdn.GDN_ERR_INVALID_ARG),
    (dict(slots=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=4, Hqk=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hqk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(flags=0x2), gdn.GDN_ERR_INVALID_ARG),
])
def test_decode_rejects_on_host(L, kw, status):
    assert _decode(L, **kw) == status
    assert gdn.gdn_last_error() != ""


def test_decode_empty_batch_is_ok_without_gpu(L):
    assert _decode(L, B=0, q=None, k=None, v=None) == gdn.GDN_OK


def test_workspace_size_queries(L):
    ws = gdn.gdn_chunk_prefill_workspace_size
    assert ws(4, 32768, 16, 128, 128, 64, gdn.GDN_PREFILL_SEQUENTIAL) == 0
    assert ws(1, 64, 2, 32, 32, 16, gdn.GDN_PREFILL_AUTO) == 0
    with pytest.raises(gdn.GdnError):
        ws(1, 64, 2, 48, 48, 16, gdn.GDN_PREFILL_AUTO)
    with pytest.raises(gdn.GdnError):
        ws(1, 64, 2, 128, 128, 32, gdn.GDN_PREFILL_FUSED)
    assert L.gdn_chunk_prefill_workspace_size(-1, 0, 1, 32, 32, 16, 0) == ctypes.c_size_t(-1).value



def test_prefill_raw_stream_handle_needs_an_explicit_workspace(L):
    """With a raw stream handle the binding cannot tie a workspace it allocates to
    that stream, so it refuses before allocating or launching anything."""
    import torch
    q = torch.empty((128, 4, 128), dtype=torch.bfloat16)
    g = torch.empty((128, 4))
    cu = torch.tensor([0, 128], dtype=torch.int32)
    assert gdn.gdn_chunk_prefill_workspace_size(1, 128, 4, 128, 128, 64, gdn.GDN_PREFILL_TRANSFER) > 0
    with pytest.raises(ValueError, match="raw handle"):
        gdn.gdn_chunk_prefill(q, q, q, g, g, cu, q, algo=gdn.GDN_PREFILL_TRANSFER, stream=12345)

def _prefill(L, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, N=1, total=64, init=None, fin=FAKE,
             o=FAKE, H=2, Hqk=None, dk=32, dv=32, chunk=16, scale=0.1, flags=0, din=1, dout=1, algo=0, ws=None,
             wsb=0, stream=None)
    a.update(kw)
    hqk = a["H"] if a["Hqk"] is None else a["Hqk"]
    return L.gdn_chunk_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["total"],
                               a["init"], a["fin"], a["o"], a["H"], hqk, a["dk"], a["dv"], a["chunk"],
                               a["scale"], a["flags"], a["din"], a["dout"], a["algo"], a["ws"], a["wsb"],
                               a["stream"])


def test_auto_choice_between_fused_and_transfer():
    """AUTO follows the chunk-step cost model: transfer for few long chains, fused
    when the pairs fill the GPU or the sequences are too short to pay for three
    passes. The choice shows in the workspace query (0 for fused)."""
    ws = gdn.gdn_chunk_prefill_workspace_size
    A, T = gdn.GDN_PREFILL_AUTO, gdn.GDN_PREFILL_TRANSFER
    for shape in [(1, 65536, 4), (1, 16384, 8), (2, 32768, 8), (1, 8192, 16)]:
        N, total, H = shape
        assert ws(N, total, H, 128, 128, 64, A) == ws(N, total, H, 128, 128, 64, T) > 0, shape
    for shape in [(4, 32768, 16), (8, 8192, 8), (32, 263000, 32), (1, 2048, 1), (0, 0, 4)]:
        N, total, H = shape
        assert ws(N, total, H, 128, 128, 64, A) == 0, shape


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48, dv=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(total=-5), gdn.GDN_ERR_INVALID_ARG),
    (dict(chunk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=FAKE + 2), gdn.GDN_ERR_INVALID_ARG),
    (dict(init=FAKE + 8), gdn.GDN_ERR_INVALID_ARG),
    (dict(algo=9), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=128, dv=128, chunk=32, algo=gdn.GDN_PREFILL_FUSED), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dout=5), gdn.GDN_ERR_INVALID_ARG),
    (dict(H=4, Hqk=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(Hqk=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(flags=0x10), gdn.GDN_ERR_INVALID_ARG),
])
def test_prefill_rejects_on_host(L, kw, status):
    assert _prefill(L, **kw) == status
    assert gdn.gdn_last_error() != ""


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _lib.lib()


def test_selftest_wait_rejects_bad_limits_on_host(L):
    assert L.gdn_selftest_wait_timeout(0, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_selftest_wait_timeout(10000001, None) == gdn.GDN_ERR_INVALID_ARG


def test_cp_entry_points_reject_on_host(L):
    st = L.gdn_cp_combine(FAKE, FAKE, 2, 2, 1, 2, 128, 128, None, FAKE, None)  # rank >= ranks
    assert st == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_cp_combine(FAKE, FAKE, 2, 1, 1, 2, 64, 64, None, FAKE, None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_cp_combine(None, None, 2, 1, 1, 2, 128, 128, None, FAKE, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_cp_local_state(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, FAKE, FAKE, 2, 2, 128, 128, 32, 0,
                                gdn.GDN_BF16, FAKE, 1 << 40, None) == gdn.GDN_ERR_UNSUPPORTED  # chunk 32
    assert L.gdn_cp_local_state(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, None, FAKE, 2, 2, 128, 128, 64, 0,
                                gdn.GDN_BF16, FAKE, 1 << 40, None) == gdn.GDN_ERR_INVALID_ARG
    size = ctypes.c_size_t(0)
    assert L.gdn_cp_local_state_workspace_size(1, 64, 2, 128, 128, 64, ctypes.byref(size)) == gdn.GDN_OK
    assert size.value > 0
    assert L.gdn_cp_local_state(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, FAKE, FAKE, 2, 2, 128, 128, 64, 0,
                                gdn.GDN_BF16, FAKE, size.value - 1, None) == gdn.GDN_ERR_WORKSPACE
    assert L.gdn_cp_local_state(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 64, FAKE, FAKE, 2, 2, 128, 128, 64, 0,
                                gdn.GDN_BF16, None, size.value, None) == gdn.GDN_ERR_WORKSPACE


def test_backward_entry_points_reject_on_host(L):
    size = ctypes.c_size_t(0)
    assert L.gdn_chunk_prefill_backward_workspace_size(2, 100, 4, 128, 128, 64, ctypes.byref(size)) == gdn.GDN_OK
    # 4 heads x (100 // 64 + 2 + 1) checkpoints + 2 x 4 x 65 scratch states of 64 KiB
    assert size.value >= (4 * 4 + 2 * 4 * 65) * 128 * 128 * 4
    assert L.gdn_chunk_prefill_backward_workspace_size(2, 100, 4, 128, 64, 64, ctypes.byref(size)) == \
        gdn.GDN_ERR_UNSUPPORTED  # dk != dv
    assert L.gdn_chunk_prefill_backward_workspace_size(2, 100, 4, 96, 96, 64, ctypes.byref(size)) == \
        gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_chunk_prefill_backward_workspace_size(2, 100, 4, 128, 128, 0, ctypes.byref(size)) == \
        gdn.GDN_ERR_INVALID_ARG

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, N=2, T=100, init=None, d_o=FAKE, dfin=None,
                 dq=FAKE, dk_=FAKE, dv_=FAKE, dg=FAKE, db=FAKE, dinit=None, H=4, Hqk=2, dk=128, dv=128, chunk=64,
                 scale=0.1, flags=0, dt=gdn.GDN_BF16, ws=FAKE, wsb=1 << 40, stream=None)
        a.update(kw)
        return L.gdn_chunk_prefill_backward(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["T"],
                                            a["init"], a["d_o"], a["dfin"], a["dq"], a["dk_"], a["dv_"], a["dg"],
                                            a["db"], a["dinit"], a["H"], a["Hqk"], a["dk"], a["dv"], a["chunk"],
                                            a["scale"], a["flags"], a["dt"], a["ws"], a["wsb"], a["stream"])
    assert call(flags=0x80) == gdn.GDN_ERR_INVALID_ARG  # unknown flag
    assert call(Hqk=3) == gdn.GDN_ERR_INVALID_ARG
    assert call(d_o=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(dq=FAKE + 4) == gdn.GDN_ERR_INVALID_ARG  # misaligned
    assert call(wsb=16) == gdn.GDN_ERR_WORKSPACE
    assert call(ws=None) == gdn.GDN_ERR_WORKSPACE
    assert call(N=0) == gdn.GDN_OK  # nothing to do, nothing launched


def test_cp_finish_rejects_on_host(L):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu=FAKE, N=1, T=64, start=None, fin=None, o=FAKE, H=2,
                 Hqk=2, dk=128, dv=128, chunk=64, scale=0.1, flags=0, dt=gdn.GDN_BF16, odt=gdn.GDN_BF16, ws=FAKE,
                 wsb=1 << 40, stream=None)
        a.update(kw)
        return L.gdn_cp_finish(a["q"], a["k"], a["v"], a["g"], a["beta"], a["cu"], a["N"], a["T"], a["start"],
                               a["fin"], a["o"], a["H"], a["Hqk"], a["dk"], a["dv"], a["chunk"], a["scale"],
                               a["flags"], a["dt"], a["odt"], a["ws"], a["wsb"], a["stream"])
    assert call(chunk=32) == gdn.GDN_ERR_UNSUPPORTED      # the segment passes need chunk 64
    assert call(dk=64, dv=64) == gdn.GDN_ERR_UNSUPPORTED
    assert call(Hqk=3) == gdn.GDN_ERR_INVALID_ARG
    assert call(cu=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(o=FAKE + 8) == gdn.GDN_ERR_INVALID_ARG     # misaligned output
    assert call(odt=7) == gdn.GDN_ERR_INVALID_ARG
    assert call(ws=None) == gdn.GDN_ERR_WORKSPACE
    assert call(wsb=16) == gdn.GDN_ERR_WORKSPACE
    assert call(N=0) == gdn.GDN_OK
