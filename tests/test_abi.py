"""CPU checks of the C-ABI library: it loads, exports every declared entry point, and
rejects bad arguments on the host before any CUDA call (no GPU needed for those)."""

import ctypes
import os
import re

import pytest

from linear_attention_recurrent_selective_b200 import ssu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssu.h")


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def L():
    from linear_attention_recurrent_selective_b200 import build
    build.build()
    return ssu.lib()


def test_header_declares_the_entry_points():
    assert declared_functions() == list(ssu.ENTRY_POINTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


WAIT_TEST_HEADER = os.path.join(ROOT, "include", "ssu_wait_test.h")


def test_product_library_has_no_test_hooks(L):
    assert declared_functions(WAIT_TEST_HEADER) == ["ssu_test_wait_fault"]
    for name in declared_functions(WAIT_TEST_HEADER):
        assert not hasattr(L, name), name


def test_wait_test_library_exports_both_headers():
    """The test library (same sources, SSU_WAIT_TEST) exports every product entry point and
    the test hook of include/ssu_wait_test.h."""
    from linear_attention_recurrent_selective_b200 import build
    T = ssu.load(build.build(waittest=True))
    for name in declared_functions() + declared_functions(WAIT_TEST_HEADER):
        assert hasattr(T, name), name


def test_status_strings(L):
    for code in range(7):
        assert L.ssu_status_string(code).startswith(b"SSU_")


# Pointers below are never dereferenced: each call fails validation on the host first.
P16 = ctypes.c_void_p(256)


def decode_args(**kw):
    a = dict(x=P16, x_dt=2, A=P16, B=P16, C=P16, bc_dt=2, dt=P16, dt_bias=None, D=None,
             z=None, state=P16, state_dt=0, stride=80 * 64 * 128, P=512, out=P16, idx=P16,
             batch=256, active=256, H=80, G=1, Dm=64, N=128, sp=1, err=None, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), 1), (dict(state=None), 1), (dict(out=None), 1),
    (dict(x_dt=7), 3), (dict(state_dt=-1), 3),
    (dict(active=300), 2), (dict(active=-1), 2), (dict(G=3), 2),
    (dict(stride=100), 2), (dict(idx=None, P=16), 2),
    (dict(N=48, stride=80 * 64 * 48), 4),
    (dict(state=ctypes.c_void_p(264)), 6),
    (dict(stride=80 * 64 * 128 + 1), 6),
])
def test_decode_rejects_bad_arguments(L, kw, status):
    assert L.ssu_decode(*decode_args(**kw)) == status


def test_prefill_rejects_partial_stash(L):
    args = [P16, 2, P16, P16, P16, 2, P16, None, None, None, P16, 0, 80 * 64 * 128, 32, P16,
            None, None, P16, None, P16, P16, 16, 16, 512, 80, 1, 64, 128, 1, None, None]
    assert L.ssu_prefill(*args) == 1
    args[16] = None
    args[17:21] = [None] * 4
    args[22] = -1      # T < 0
    assert L.ssu_prefill(*args) == 2


def test_replay_and_pool_reject_bad_arguments(L):
    assert L.ssu_replay(P16, 0, 8192, 8, P16, P16, P16, P16, None, None, 4, 4, 5, 1, 1, 64,
                        128, None, 0, None, None) == 1
    assert L.ssu_replay(P16, 0, 8192, 8, P16, P16, ctypes.c_void_p(260), P16, P16, None, 4,
                        4, 5, 1, 1, 64, 128, None, 0, None, None) == 6
    # accepted node ids with a negative width
    assert L.ssu_replay(P16, 0, 8192, 8, P16, P16, P16, P16, P16, None, 4, 4, 5, 1, 1, 64,
                        128, P16, -1, None, None) == 2
    assert L.ssu_replay_layers(P16, 2, 0, 8192, 8, P16, None, 4, 4, 5, 1, 1, 64, 128, P16,
                               -3, None, None) == 2
    assert L.pool_clear_slot(P16, 1024, 4, 4, None) == 2
    assert L.pool_clear_slot(P16, 1024, 4, -2, None) == 2
    assert L.pool_clear_slot(None, 1024, 4, 0, None) == 1
    assert L.pool_copy_slot(P16, 4, 4, P16, 8, 0, 1024, None) == 2
    assert L.pool_copy_slot(P16, 4, 0, P16, 8, -1, 1024, None) == 2


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ssu, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ssu, "_lib", None)
    with pytest.raises(ssu.SSULibraryMissing):
        ssu.lib()


def ddtree_args(**kw):
    a = dict(x=P16, x_dt=2, A=P16, B=P16, C=P16, bc_dt=2, dt=P16, dt_bias=None, D=None,
             state=P16, state_dt=0, stride=80 * 64 * 128, P=32, out=P16, par=P16, dep=P16,
             idx=P16, sdA=P16, sU=P16, sB=P16, sdt=P16, batch=16, active=16, T=128, H=80,
             G=1, Dm=64, N=128, sp=1, err=None, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize("kw,status", [
    (dict(par=None), 1), (dict(dep=None), 1), (dict(sU=None), 1), (dict(out=None), 1),
    (dict(x_dt=5), 3), (dict(T=129), 2), (dict(T=-1), 2), (dict(G=3), 2),
    (dict(N=24, stride=80 * 64 * 24), 4),
    (dict(B=ctypes.c_void_p(258)), 6), (dict(state=ctypes.c_void_p(264)), 6),
])
def test_ddtree_rejects_bad_arguments(L, kw, status):
    assert L.ssu_ddtree(*ddtree_args(**kw)) == status


def test_ddtree_empty_calls_need_no_pointers(L):
    nulls = dict(x=None, A=None, B=None, C=None, dt=None, state=None, out=None, par=None,
                 dep=None, sdA=None, sU=None, sB=None, sdt=None)
    assert L.ssu_ddtree(*ddtree_args(active=0, **nulls)) == 0
    assert L.ssu_ddtree(*ddtree_args(T=0, **nulls)) == 0


def test_conv_decode_rejects_bad_arguments(L):
    cd = 80 * 64 + 2 * 128
    good = dict(xbc=P16, x_dt=2, w=P16, b=None, cst=P16, cs=cd * 3, cc=3, ck=1, width=4, silu=1,
                A=P16, dt=P16, dtb=None, D=None, z=None, state=P16, sdt=0,
                stride=80 * 64 * 128, P=512, out=P16, idx=P16, batch=256, active=256, H=80,
                G=1, Dm=64, N=128, sp=1, err=None, stream=None)

    def call(**kw):
        a = dict(good)
        a.update(kw)
        return L.ssu_conv_decode(*a.values())
    assert call(xbc=None) == 1 and call(cst=None) == 1 and call(w=None) == 1
    assert call(width=0) == 2 and call(width=17) == 2
    assert call(cs=cd * 3 - 1) == 2                 # taps would leave the slot
    assert call(x_dt=9) == 3 and call(N=24, stride=80 * 64 * 24) == 4
    assert call(active=0, xbc=None, cst=None, w=None, A=None, dt=None, state=None,
                out=None) == 0
    assert call(width=1, cst=None, cs=0, xbc=None) == 1   # width 1 needs no conv pool


def test_gdn_rejects_bad_arguments(L):
    good = dict(q=P16, k=P16, v=P16, x_dt=2, a=P16, b=P16, A_log=P16, dtb=None, scale=0.0,
                l2=1, state=P16, stride=32 * 128 * 128, P=512, out=P16, idx=P16, batch=256,
                active=256, HK=16, HV=32, K=128, V=128, err=None, stream=None)

    def call(**kw):
        a = dict(good)
        a.update(kw)
        return L.gdn_decode(*a.values())
    assert call(q=None) == 1 and call(state=None) == 1 and call(A_log=None) == 1
    assert call(HV=24) == 2 and call(stride=100) == 2 and call(active=300) == 2
    assert call(x_dt=7) == 3 and call(K=96, stride=32 * 128 * 96) == 4
    assert call(state=ctypes.c_void_p(264)) == 6
    assert call(active=0, q=None, k=None, v=None, state=None) == 0


@pytest.mark.parametrize("idx,batch,active,P,err,status", [
    (None, 4, 4, 8, P16, 1), (P16, 4, 4, 8, None, 1), (P16, 4, 5, 8, P16, 2),
    (P16, 4, -1, 8, P16, 2), (P16, 4, 4, -1, P16, 2), (None, 4, 0, 8, None, 0),
])
def test_check_state_indices_host_validation(L, idx, batch, active, P, err, status):
    assert L.ssu_check_state_indices(idx, batch, active, P, err, None) == status
