"""The C-ABI library: it loads, exports every function include/saga.h declares,
and rejects bad arguments on the host (no GPU needed: every call below fails
validation before anything is enqueued)."""
import ctypes
import os
import re

import pytest

import sparse_decode_attention_step_b200 as saga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(saga.LIB_PATH):
        from sparse_decode_attention_step_b200 import build
        build.build()
    return saga.load()


def declared_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \t\*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M):
            if not m.group(0).lstrip().startswith(("typedef", "#", "return")):
                names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"saga_decode_step", "saga_refresh_threshold", "gqa_dense_decode"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_checked_build_exports_the_same_symbols():
    """The bounds-checked variant (build.py --check) is the same library with
    index checks compiled in: it loads and exports every declared function."""
    from sparse_decode_attention_step_b200 import build
    path = build.CHECK_LIB_PATH
    if not os.path.exists(path):
        build.build(check=True)
    checked = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(checked, n), f"{n} not exported by the checked build"


def test_status_strings(lib):
    for code in range(6):
        assert saga.status_string(code) != "unknown status"
    assert saga.status_string(99) == "unknown status"


def test_shape_contiguous_and_workspace_size(lib):
    s = saga.shape(8, 32, 2, 8, 64, saga.SAGA_BF16, 131072)
    assert (s.q_stride_h, s.q_stride_b) == (64, 32 * 64)
    assert (s.k_stride_h, s.k_stride_b) == (131072 * 64, 2 * 131072 * 64)
    assert s.v_stride_b == 8 * 131072 * 64
    n = saga.workspace_size(s, 2048)
    # error word + partials + one fp32 score row per (b, j)
    assert n >= 256 + 8 * 32 * 131072 * 4
    assert n % 256 == 0


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), saga.SAGA_ERR_INVALID_ARG),
    (dict(h_k=4, h_v=2), saga.SAGA_ERR_INVALID_ARG),
    (dict(h_v=64), saga.SAGA_ERR_INVALID_ARG),
    (dict(h_v=3, h_k=1), saga.SAGA_ERR_UNSUPPORTED),
    (dict(d=96), saga.SAGA_ERR_UNSUPPORTED),
    (dict(dtype=7), saga.SAGA_ERR_INVALID_ARG),
    (dict(h_k=1, h_v=1), saga.SAGA_ERR_UNSUPPORTED),     # group of 32 > 16
    (dict(max_l_kv=5000), saga.SAGA_ERR_INVALID_ARG),    # max_l_kv > cap
])
def test_bad_shapes_rejected(lib, kw, code):
    a = dict(B=1, h_q=32, h_k=2, h_v=8, d=64, dtype=saga.SAGA_BF16, cap=4096, max_l_kv=4096)
    a.update(kw)
    s = saga.shape(a["B"], a["h_q"], a["h_k"], a["h_v"], a["d"], a["dtype"], a["cap"],
                   a["max_l_kv"])
    assert saga.workspace_size(s, 8) == 0
    fake = 1 << 40   # never dereferenced: validation fails first
    rc = lib.saga_decode_step(ctypes.byref(s), fake, fake, fake, fake, fake, fake, None, None,
                              fake, 1 << 30, None)
    assert rc == code


def test_bad_pointers_and_workspace(lib):
    s = saga.shape(1, 32, 2, 8, 64, saga.SAGA_BF16, 4096)
    need = saga.workspace_size(s, 8)
    ok = 1 << 40
    call = lambda **o: lib.saga_decode_step(
        ctypes.byref(s), o.get("q", ok), o.get("K", ok), o.get("V", ok), o.get("l", ok),
        o.get("tau", ok), o.get("out", ok), None, None, o.get("ws", ok), o.get("n", need), None)
    assert call(q=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(K=ok + 8) == saga.SAGA_ERR_INVALID_ARG       # K not 16-byte aligned
    assert call(V=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(tau=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(ws=None) == saga.SAGA_ERR_WORKSPACE
    assert call(ws=ok + 128) == saga.SAGA_ERR_WORKSPACE       # not 256-byte aligned
    assert call(n=need - 1) == saga.SAGA_ERR_WORKSPACE
    # refresh: N >= 1, V and out both given or both absent
    r = lib.saga_refresh_threshold(ctypes.byref(s), ok, ok, ok, ok, 0, ok, ok, None, None,
                                   None, ok, need, None)
    assert r == saga.SAGA_ERR_INVALID_ARG
    r = lib.saga_refresh_threshold(ctypes.byref(s), ok, ok, ok, ok, 8, ok, None, None, None,
                                   None, ok, need, None)
    assert r == saga.SAGA_ERR_INVALID_ARG
    # dense needs h_k == h_v
    r = lib.gqa_dense_decode(ctypes.byref(s), ok, ok, ok, ok, ok, ok, need, None)
    assert r == saga.SAGA_ERR_INVALID_ARG
    # misaligned stride: 8 bf16 elements = 16 bytes is the minimum granule
    s2 = saga.shape(1, 32, 2, 8, 64, saga.SAGA_BF16, 4096)
    s2.k_stride_h = 4096 * 64 + 4
    assert saga.workspace_size(s2, 8) == 0


@pytest.mark.parametrize("hq,hk,hv,code", [
    (16, 2, 16, saga.SAGA_ERR_UNSUPPORTED),     # eight value heads per key head
    (20, 2, 4, saga.SAGA_ERR_UNSUPPORTED),      # group of 10 query heads over 2 value heads
    (32, 2, 8, saga.SAGA_ERR_WORKSPACE),        # supported: gets as far as the workspace check
])
def test_saga_dense_shapes(lib, hq, hk, hv, code):
    s = saga.shape(1, hq, hk, hv, 64, saga.SAGA_BF16, 4096)
    fake = 1 << 40   # never dereferenced: validation fails first
    rc = lib.saga_dense_decode(ctypes.byref(s), fake, fake, fake, fake, fake, None, 0, None)
    assert rc == code


def test_append_kv_host_checks(lib):
    s = saga.shape(2, 16, 2, 4, 64, saga.SAGA_BF16, 4096)
    ok = 1 << 40    # never dereferenced: validation fails first
    call = lambda **o: lib.saga_append_kv(ctypes.byref(s), o.get("kn", ok), o.get("vn", ok),
                                          o.get("K", ok), o.get("V", ok), o.get("l", ok),
                                          o.get("ws", ok), o.get("n", 256), None)
    assert call(kn=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(V=ok + 8) == saga.SAGA_ERR_INVALID_ARG        # not 16-byte aligned
    assert call(ws=None) == saga.SAGA_ERR_WORKSPACE
    assert call(n=255) == saga.SAGA_ERR_WORKSPACE             # room for the error word only


def test_merge_workspace_size(lib):
    ok = saga.merge_shape(8192, 2048, 32, 8, 64)
    n = saga.merge_workspace_size(ok)
    # at least the transposed queries and the keys' hi/lo rows
    assert n >= 8192 * 32 * 64 * 2 + 2 * 8192 * 8 * 64 * 2
    assert n % 256 == 0
    for bad in [dict(T=100), dict(T=64), dict(d_model=60), dict(h_k=3), dict(h_q=12),
                dict(d=96), dict(h_k=18, h_q=36)]:
        kw = dict(T=8192, d_model=2048, h_q=32, h_k=8, d=64)
        kw.update(bad)
        assert saga.merge_workspace_size(saga.merge_shape(**kw)) == 0, bad


def test_merge_host_checks(lib):
    s = saga.merge_shape(1024, 512, 8, 4, 64)
    need = saga.merge_workspace_size(s)
    ok = 1 << 40    # never dereferenced: validation fails first
    call = lambda shp=s, **o: lib.saga_merge_keys(
        ctypes.byref(shp), o.get("X", ok), o.get("W", ok), o.get("Q", ok), o.get("rcond", 1e-6),
        o.get("w", ok), o.get("pairs", ok), o.get("total", None), o.get("W_S", ok),
        o.get("ws", ok), o.get("n", need), None)
    assert call(X=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(W=ok + 8) == saga.SAGA_ERR_INVALID_ARG        # not 16-byte aligned
    assert call(pairs=None) == saga.SAGA_ERR_INVALID_ARG
    assert call(rcond=-1.0) == saga.SAGA_ERR_INVALID_ARG
    assert call(rcond=float("nan")) == saga.SAGA_ERR_INVALID_ARG
    assert call(total=ok + 4) == saga.SAGA_ERR_INVALID_ARG    # float64 output misaligned
    assert call(ws=None) == saga.SAGA_ERR_WORKSPACE
    assert call(ws=ok + 128) == saga.SAGA_ERR_WORKSPACE
    assert call(n=need - 1) == saga.SAGA_ERR_WORKSPACE
    assert call(saga.merge_shape(1024, 512, 8, 3, 64)) == saga.SAGA_ERR_INVALID_ARG   # odd h_k
    assert call(saga.merge_shape(1024, 512, 8, 4, 96)) == saga.SAGA_ERR_UNSUPPORTED   # d
    assert call(saga.merge_shape(1024, 512, 36, 18, 64)) == saga.SAGA_ERR_UNSUPPORTED  # h_k > 16
    assert call(saga.merge_shape((1 << 21) + 8, 512, 8, 4, 64)) == saga.SAGA_ERR_UNSUPPORTED
    assert call(saga.merge_shape(120, 512, 8, 4, 64)) == saga.SAGA_ERR_INVALID_ARG     # T < 128
