"""The C ABI without a GPU: the library loads, exports every function include/hsa.h declares, sizes
its workspaces, and rejects invalid calls on the host before any launch."""
import ctypes
import os
import re

import pytest

from ultra_long_context_b200 import hsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hsa.h")

# a fake, 256-byte aligned address: only ever passed to calls that fail validation first
FAKE = ctypes.c_void_p(1 << 20)
ODD = ctypes.c_void_p((1 << 20) + 2)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_ ]*?\**\s*\**(hsa_[a-z0-9_]+)\s*\(",
                                 text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"hsa_forward", "hsa_decode", "hsa_backward", "hsa_last_error"} <= set(names)
    lib = ctypes.CDLL(hsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(hsa.SIGNATURES), "binding must declare every C entry point"


def test_workspace_sizes_are_positive_and_monotone():
    a = hsa.hsa_forward_workspace_size(1, 4, 4096, 64, 64, 8)
    b = hsa.hsa_forward_workspace_size(2, 8, 32768, 128, 64, 16)
    assert 0 < a < b
    assert b >= 2 * 8 * 32768 * 128 * 4          # holds the fp32 output accumulator
    assert hsa.hsa_decode_workspace_size(1, 8, 1 << 24, 128, 64, 32) > 0
    assert hsa.hsa_backward_workspace_size(1, 8, 65536, 128, 64, 16) > 0
    assert hsa.hsa_forward_workspace_size(0, 4, 4096, 64, 64, 8) == 0


def _fwd(**kw):
    args = dict(Q=FAKE, K=FAKE, V=FAKE, L=FAKE, B=1, H=1, T=256, D=64, chunk=64, topk=8, scale=0.0, out=FAKE,
                sel_idx=None, sel_w=None, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return hsa.lib().hsa_forward(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), -2), (dict(D=256), -2), (dict(chunk=32), -2), (dict(topk=65), -2),
    (dict(topk=0), -1), (dict(B=0), -1), (dict(T=0), -1), (dict(Q=None), -1), (dict(out=None), -1),
    (dict(L=None), -1), (dict(K=ODD), -1), (dict(sel_w=ODD), -1),
    (dict(ws=None), -3), (dict(ws_bytes=100), -3), (dict(ws=ctypes.c_void_p((1 << 20) + 16)), -3),
])
def test_forward_rejects_invalid_calls_on_host(kw, status):
    assert _fwd(**kw) == status
    assert hsa.hsa_last_error() != ""


def _dec(**kw):
    args = dict(q=FAKE, Kc=FAKE, Vc=FAKE, Lc=FAKE, cache_len=FAKE, Tmax=1 << 20, B=2, H=2, D=128, chunk=64,
                topk=16, scale=0.0, out=FAKE, sel_idx=None, sel_w=None, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return hsa.lib().hsa_decode(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(D=80), -2), (dict(topk=65), -2), (dict(chunk=128), -2), (dict(Tmax=-1), -1), (dict(cache_len=None), -1),
    (dict(Lc=ODD), -1), (dict(ws_bytes=8), -3),
])
def test_decode_rejects_invalid_calls_on_host(kw, status):
    assert _dec(**kw) == status


def _bwd(**kw):
    args = dict(Q=FAKE, K=FAKE, V=FAKE, L=FAKE, out=FAKE, dout=FAKE, sel_idx=FAKE, sel_w=FAKE, B=1, H=1, T=256,
                D=128, chunk=64, topk=16, scale=0.0, dQ=FAKE, dK=FAKE, dV=FAKE, dL=FAKE, ws=FAKE, ws_bytes=1 << 40,
                stream=None)
    args.update(kw)
    return hsa.lib().hsa_backward(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(D=32), -2), (dict(topk=65), -2), (dict(sel_idx=None), -1), (dict(dL=None), -1), (dict(dout=ODD), -1),
    (dict(ws=None), -3),
])
def test_backward_rejects_invalid_calls_on_host(kw, status):
    assert _bwd(**kw) == status


def test_binding_raises_with_message():
    with pytest.raises(hsa.HSAError, match="HSA_ERR_UNSUPPORTED"):
        hsa._check("hsa_forward", _fwd(D=96))


def test_workspace_status_rejects_null_on_host():
    """hsa_workspace_status validates its argument before touching the device."""
    assert hsa.lib().hsa_workspace_status(None, None) == -1
    assert "workspace" in hsa.hsa_last_error()


def _fwd_ex(**kw):
    args = dict(Qs=None, Q=FAKE, K=FAKE, V=FAKE, L=FAKE, B=1, H=4, Hkv=4, T=256, D=64, chunk=64, topk=8, scale=0.0,
                flags=0, out=FAKE, sel_idx=None, sel_w=None, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return hsa.lib().hsa_forward_ex(*args.values())


def _bwd_ex(**kw):
    args = dict(Qs=None, Q=FAKE, K=FAKE, V=FAKE, L=FAKE, out=FAKE, dout=FAKE, sel_idx=FAKE, sel_w=FAKE, B=1, H=4,
                Hkv=4, T=256, D=128, chunk=64, topk=16, scale=0.0, flags=0, dQ=FAKE, dK=FAKE, dV=FAKE, dL=FAKE,
                dQs=None, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return hsa.lib().hsa_backward_ex(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(flags=2), -1), (dict(flags=0x80000000), -1), (dict(Hkv=3), -1), (dict(Hkv=0), -1), (dict(Hkv=8), -1),
    (dict(Qs=ODD), -1), (dict(D=96), -2), (dict(ws_bytes=100, flags=1), -3),
])
def test_forward_ex_rejects_invalid_calls_on_host(kw, status):
    assert _fwd_ex(**kw) == status
    assert hsa.hsa_last_error() != ""


@pytest.mark.parametrize("kw,status", [
    (dict(Qs=FAKE), -1), (dict(dQs=FAKE), -1), (dict(flags=4), -1), (dict(Hkv=5), -1), (dict(ws=None, flags=1), -3),
])
def test_backward_ex_rejects_invalid_calls_on_host(kw, status):
    assert _bwd_ex(**kw) == status


def test_decode_ex_rejects_invalid_calls_on_host():
    args = dict(qs=None, q=FAKE, Kc=FAKE, Vc=FAKE, Lc=FAKE, cache_len=FAKE, Tmax=1 << 20, B=2, H=2, Hkv=2, Tq=1,
                D=128, chunk=64, topk=16, scale=0.0, flags=8, out=FAKE, sel_idx=None, sel_w=None, ws=FAKE,
                ws_bytes=1 << 40, stream=None)
    assert hsa.lib().hsa_decode_ex(*args.values()) == -1
    for kw, status in ((dict(flags=1, Hkv=3), -1), (dict(flags=0, Tq=0), -1), (dict(flags=0, Tq=65), -1),
                       (dict(flags=0, Tq=2, topk=40), -2), (dict(flags=0, Tq=4, ws_bytes=16), -3)):
        a = dict(args, **kw)
        assert hsa.lib().hsa_decode_ex(*a.values()) == status, kw


def test_ex_workspace_sizes_cover_the_options():
    base = hsa.hsa_forward_workspace_size(1, 4, 4096, 128, 64, 16)
    assert hsa.hsa_forward_ex_workspace_size(1, 4, 4, 4096, 128, 64, 16, 0) == base
    # query-key normalisation keeps bf16 copies of Q and K
    assert hsa.hsa_forward_ex_workspace_size(1, 4, 4, 4096, 128, 64, 16, 1) >= base + 2 * 4 * 4096 * 128 * 2
    assert hsa.hsa_backward_ex_workspace_size(1, 4, 4, 4096, 128, 64, 16, 0) >= \
        hsa.hsa_backward_workspace_size(1, 4, 4096, 128, 64, 16) + 4 * 4096 * 16 * 4  # ds per pair
    assert hsa.hsa_decode_ex_workspace_size(1, 8, 8, 1 << 20, 128, 64, 32, 1) == \
        hsa.hsa_decode_workspace_size(1, 8, 1 << 20, 128, 64, 32)


def _fwd_varlen(**kw):
    args = dict(Qs=None, Q=FAKE, K=FAKE, V=FAKE, L=FAKE, cu=FAKE, B=3, max_seqlen=1000, H=4, Hkv=2, D=128, chunk=64,
                topk=8, scale=0.0, flags=0, out=FAKE, sel_idx=FAKE, sel_w=FAKE, ws=FAKE, ws_bytes=1 << 40, stream=None)
    args.update(kw)
    return hsa.lib().hsa_forward_varlen(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(cu=None), -1), (dict(cu=ctypes.c_void_p((1 << 20) + 2)), -1), (dict(max_seqlen=0), -1), (dict(B=0), -1),
    (dict(Hkv=3), -1), (dict(flags=2), -1), (dict(out=None), -1), (dict(sel_w=None), -1), (dict(Q=ODD), -1),
    (dict(D=96), -2), (dict(topk=65), -2), (dict(ws_bytes=64), -3), (dict(ws=None), -3),
])
def test_forward_varlen_rejects_invalid_calls_on_host(kw, status):
    assert _fwd_varlen(**kw) == status
    assert hsa.hsa_last_error() != ""


def test_backward_varlen_rejects_invalid_calls_on_host():
    args = dict(Qs=None, Q=FAKE, K=FAKE, V=FAKE, L=FAKE, out=FAKE, dout=FAKE, sel_idx=FAKE, sel_w=FAKE, cu=FAKE, B=2,
                max_seqlen=500, H=2, Hkv=2, D=64, chunk=64, topk=8, scale=0.0, flags=0, dQ=FAKE, dK=FAKE, dV=FAKE,
                dL=FAKE, dQs=None, ws=FAKE, ws_bytes=1 << 40, stream=None)
    for kw, status in ((dict(dQs=FAKE), -1), (dict(Qs=FAKE), -1), (dict(dL=None), -1), (dict(cu=None), -1),
                       (dict(ws_bytes=16), -3)):
        a = dict(args, **kw)
        assert hsa.lib().hsa_backward_varlen(*a.values()) == status, kw


def test_varlen_workspace_covers_the_padded_batch():
    B, H, Hkv, T, D, K = 3, 4, 2, 1000, 128, 8
    padded = B * H * T * D * 2  # one padded bf16 query batch
    assert hsa.lib().hsa_forward_varlen_workspace_size(B, H, Hkv, T, D, 64, K, 0) >= \
        hsa.hsa_forward_workspace_size(B, H, T, D, 64, K) + 3 * padded
    assert hsa.lib().hsa_backward_varlen_workspace_size(B, H, Hkv, T, D, 64, K, 0) > \
        hsa.lib().hsa_forward_varlen_workspace_size(B, H, Hkv, T, D, 64, K, 0)
    assert hsa.lib().hsa_forward_varlen_workspace_size(B, H, 3, T, D, 64, K, 0) == 0  # H not a multiple of Hkv


def test_selftest_bounded_wait_checks_its_workspace_on_host():
    """The bounded-wait self-test validates its arguments before launching anything."""
    f = hsa.lib().hsa_selftest_bounded_wait
    assert f(None, 1 << 20, 100, None) == -3
    assert f(ctypes.c_void_p((1 << 20) + 16), 1 << 20, 100, None) == -3   # not 256-byte aligned
    assert f(FAKE, 64, 100, None) == -3                                    # too small
    assert f(FAKE, 1 << 20, 0, None) == -1
    assert f(FAKE, 1 << 20, (1 << 20) + 1, None) == -1
