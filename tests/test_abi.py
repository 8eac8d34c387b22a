"""C ABI checks that need no GPU: the library loads, exports every entry
point that include/abattn.h declares, and rejects bad arguments on the host
(before any CUDA call) with the documented status codes."""
import ctypes
import math
import os
import re

import pytest

from block_sparse_attention_12_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return abi.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "abattn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(abattn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_set():
    assert declared_functions() == sorted(abi.EXPORTED)


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_version_and_messages(L):
    assert "sm_100a" in abi.version()
    for code in range(0, -11, -1):
        assert abi.strerror(code) not in ("", "unknown status")
    assert abi.strerror(-99) == "unknown status"


D = abi.Dims
P = abi.Params
FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: every call below fails validation first
MISALIGNED = ctypes.c_void_p(0x10008)


def params(**kw):
    p = abi.Config(kv_block=4, budget=0.1).params()
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def fwd(L, dims, p, Q=FAKE, O=FAKE, cap=8):
    return L.abattn_forward(Q, FAKE, FAKE, ctypes.byref(dims), ctypes.byref(p), FAKE, FAKE, FAKE, cap, O, None,
                            None)


@pytest.mark.parametrize("dims,code", [
    (D(1, 1, 0, 128), abi.ERR_SHAPE), (D(0, 1, 128, 128), abi.ERR_SHAPE), (D(1, 1, 128, 96), abi.ERR_SHAPE),
    (D(1, 1, 128, 256), abi.ERR_SHAPE), (D(1, 1, 2**31, 64), abi.ERR_SHAPE),
])
def test_forward_rejects_shapes(L, dims, code):
    assert fwd(L, dims, params()) == code


@pytest.mark.parametrize("field,value", [("kv_block", 3), ("kv_block", 256), ("scale", -1.0),
                                         ("scale", math.inf)])
def test_forward_rejects_params(L, field, value):
    assert fwd(L, D(1, 1, 256, 64), params(**{field: value})) == abi.ERR_PARAM


def test_forward_rejects_null_misaligned_and_capacity(L):
    d = D(1, 1, 256, 64)
    assert fwd(L, d, params(), Q=None) == abi.ERR_NULL
    assert fwd(L, d, params(), O=MISALIGNED) == abi.ERR_ALIGN
    assert fwd(L, d, params(), cap=0) == abi.ERR_SHAPE
    assert fwd(L, d, params(), cap=65) == abi.ERR_SHAPE  # > nKVB


@pytest.mark.parametrize("field,value", [("budget", 0.0), ("budget", 1.5), ("budget", math.nan),
                                         ("n_clusters", 0), ("n_clusters", 9), ("kmeans_iters", -1),
                                         ("q_block", 64), ("mode", 2), ("head_offset", -1)])
def test_plan_rejects_params(L, field, value):
    d = D(1, 1, 256, 64)
    rc = L.abattn_plan(FAKE, FAKE, ctypes.byref(d), ctypes.byref(params(**{field: value})), FAKE, FAKE, FAKE, 8,
                       FAKE, 1 << 30, None)
    assert rc == abi.ERR_PARAM


def test_plan_workspace_and_capacity(L):
    shape = (1, 40, 75600, 128)
    cfg = abi.Config(kv_block=4, budget=0.08)
    cap = abi.capacity(shape, cfg)
    assert cap == min(18900, math.ceil(1512 + 8 * math.sqrt(1512) + 32))
    ws = abi.plan_workspace_bytes(shape, cfg)
    nqb, nkvb = 591, 18900
    lower = 4 * (40 * nkvb * 128 + 40 * nqb * 8 * 128 + 40 * nqb * nkvb)
    assert ws >= lower and ws < lower * 1.1
    d = D(*shape)
    rc = L.abattn_plan(FAKE, FAKE, ctypes.byref(d), ctypes.byref(cfg.params()), FAKE, FAKE, FAKE, cap, FAKE,
                       ws - 1, None)
    assert rc == abi.ERR_WORKSPACE
    rc = L.abattn_plan(FAKE, FAKE, ctypes.byref(d), ctypes.byref(cfg.params()), FAKE, FAKE, FAKE, cap, None,
                       ws, None)
    assert rc == abi.ERR_WORKSPACE


def test_plan_rejects_rows_too_long_for_shared_memory(L):
    d = D(1, 1, 4 * 50000, 64)
    p = params()
    rc = L.abattn_plan_from_pi(FAKE, ctypes.byref(d), ctypes.byref(p), FAKE, FAKE, FAKE, 100, None)
    assert rc == abi.ERR_SHAPE


def test_score_workspace_check(L):
    d = D(1, 2, 1024, 64)
    p = params()
    need = abi.score_workspace_bytes((1, 2, 1024, 64), abi.Config(kv_block=4, budget=0.1))
    rc = L.abattn_score(FAKE, FAKE, FAKE, ctypes.byref(d), ctypes.byref(p), FAKE, FAKE, need - 1, None)
    assert rc == abi.ERR_WORKSPACE


def test_params_struct_layout_matches_header():
    assert ctypes.sizeof(abi.Params) == 40
    assert abi.Params.seed.offset == 24 and abi.Params.scale.offset == 32
    assert abi.Params.head_offset.offset == 36
    assert ctypes.sizeof(abi.Dims) == 32


def test_selftest_library_declares_exports_and_rejects_null():
    """The failure-detection self-test library (include/abattn_selftest.h)
    builds, exports exactly what its header declares, and refuses a NULL
    output pointer on the host, before any CUDA call."""
    text = open(os.path.join(ROOT, "include", "abattn_selftest.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    assert sorted(set(re.findall(r"\b(abattn_[a-z_]+)\s*\(", text))) == ["abattn_selftest_stalled_wait"]
    S = ctypes.CDLL(build.build_selftest())
    f = S.abattn_selftest_stalled_wait
    f.restype, f.argtypes = ctypes.c_int, [ctypes.POINTER(ctypes.c_int), ctypes.c_void_p]
    assert f(None, None) == abi.ERR_NULL
