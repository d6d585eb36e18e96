"""Host-side checks of the C ABI: the library loads, exports every function
include/gptq.h declares, and validates arguments before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def g():
    import __graft_entry__
    __graft_entry__.build()
    import post_weight_quantization_13_b200 as m
    return m


def test_header_declares_the_three_calls():
    names = _declared()
    for n in ("gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer",
              "gptq_workspace_bytes", "gptq_last_error", "gptq_validate_config",
              "gptq_abi_version"):
        assert n in names


def test_library_exports_every_declared_symbol(g):
    for name in _declared():
        assert hasattr(g.lib, name), name
        assert getattr(g.lib, name) is not None


def test_abi_version(g):
    src = open(HEADER).read()
    v = int(re.search(r"#define GPTQ_ABI_VERSION (\d+)", src).group(1))
    assert g.gptq_abi_version() == v


def _cfg(g, **kw):
    c = g.GptqConfig(**kw)
    return c


@pytest.mark.parametrize("kw,code", [
    (dict(bits=5), 1), (dict(bits=1), 1), (dict(group_size=0), 1), (dict(group_size=100), 1),
    (dict(block_size=0), 1), (dict(block_size=96, group_size=128), 1),
    (dict(damp_percent=-0.1), 1), (dict(damp_percent=float("nan")), 1),
    (dict(damp_percent=float("inf")), 1), (dict(group_size=96, block_size=96), 7),
])
def test_validate_config_rejects(g, kw, code):
    in_ = 4096 if kw.get("group_size", 128) != 96 else 96 * 40
    with pytest.raises(g.GptqError) as e:
        g.gptq_validate_config(_cfg(g, **kw), 16, in_)
    assert e.value.status == code
    assert g.gptq_last_error()


@pytest.mark.parametrize("kw", [
    dict(), dict(bits=2, group_size=64), dict(bits=8, group_size=32, block_size=128),
    dict(bits=3, group_size=-1, sym=True), dict(group_size=256, block_size=128),
    dict(group_size=128, block_size=1024), dict(group_size=4096, block_size=4096),
    dict(desc_act=True, damp_percent=0.0),
])
def test_validate_config_accepts(g, kw):
    g.gptq_validate_config(_cfg(g, **kw), 16, 4096)
    assert g.gptq_last_error() == ""


def test_validate_sizes(g):
    with pytest.raises(g.GptqError):
        g.gptq_validate_config(_cfg(g), 16, 0)
    with pytest.raises(g.GptqError):
        g.gptq_validate_config(_cfg(g), -1, 128)
    with pytest.raises(g.GptqError) as e:
        g.gptq_validate_config(_cfg(g, group_size=-1), 16, 40000)
    assert e.value.status == 7


def test_workspace_bytes(g):
    c = _cfg(g)
    prep = g.gptq_workspace_bytes(0, 4096, c)
    full = g.gptq_workspace_bytes(4096, 4096, c)
    assert prep >= 2 * 4096 * 4096 * 4   # R (then L) and M = L^-1, fp32
    assert full >= prep
    assert g.gptq_workspace_bytes(4096, 0, c) == 0
    assert g.gptq_workspace_bytes(11008, 4096, c) >= full


def test_calls_reject_bad_arguments_before_any_launch(g):
    lib = g.lib
    i64 = ctypes.c_int64
    n = i64(0)
    # in < 1, negative tokens, NULL S, ldx < tokens, unknown dtype
    assert lib.gptq_hessian_accumulate(None, 0, None, 0, 10, 10, ctypes.byref(n), None) == 1
    assert lib.gptq_hessian_accumulate(None, 8, None, 0, -1, 10, ctypes.byref(n), None) == 1
    assert lib.gptq_hessian_accumulate(None, 8, None, 0, 10, 10, ctypes.byref(n), None) == 1
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), 8, ctypes.c_void_p(256), 0, 10, 5,
                                       ctypes.byref(n), None) == 1
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p(256), 8, ctypes.c_void_p(256), 9, 10, 10,
                                       ctypes.byref(n), None) == 1
    assert n.value == 0
    c = _cfg(g).c()
    # n <= 0, NULL outputs
    assert lib.gptq_prepare_hinv(ctypes.c_void_p(256), 0, 8, ctypes.byref(c), ctypes.c_void_p(256),
                                 ctypes.c_void_p(256), ctypes.c_void_p(256), None, 0, None) == 1
    c8 = _cfg(g, group_size=8).c()
    assert lib.gptq_prepare_hinv(None, 10, 8, ctypes.byref(c8), None, None, None, None, 0, None) == 1
    # quantize: out == 0 is a no-op; ldw < in and qweight with in*bits % 32 are rejected
    assert lib.gptq_quantize_layer(None, 0, 0, 8, 8, None, None, None, ctypes.byref(c8), None, None,
                                   None, None, None, None, None, 0, None) == 0
    assert lib.gptq_quantize_layer(ctypes.c_void_p(256), 0, 4, 8, 4, *([ctypes.c_void_p(256)] * 3),
                                   ctypes.byref(c8), None, None, *([ctypes.c_void_p(256)] * 3), None,
                                   None, 0, None) == 1
    c3 = _cfg(g, bits=3, group_size=8).c()
    assert lib.gptq_quantize_layer(ctypes.c_void_p(256), 0, 4, 8, 8, *([ctypes.c_void_p(256)] * 3),
                                   ctypes.byref(c3), None, ctypes.c_void_p(256),
                                   *([ctypes.c_void_p(256)] * 3), None, None, 0, None) == 1
    assert "multiple of 32" in g.gptq_last_error()


def test_export_checkpoint_rejects_bad_arguments_before_any_launch(g):
    lib = g.lib
    p = ctypes.c_void_p(256)
    # bits, ngroups, zero_offset, missing input, divisibility of in*bits and out*bits
    assert lib.gptq_export_checkpoint(p, p, p, 8, 32, 5, 1, 1, p, p, p, None) == 1
    assert lib.gptq_export_checkpoint(p, p, p, 8, 32, 4, 0, 1, p, p, p, None) == 1
    assert lib.gptq_export_checkpoint(p, p, p, 8, 32, 4, 33, 1, p, p, p, None) == 1
    assert lib.gptq_export_checkpoint(p, p, p, 8, 32, 4, 1, 2, p, p, p, None) == 1
    assert "zero_offset" in g.gptq_last_error()
    assert lib.gptq_export_checkpoint(None, p, p, 8, 32, 4, 1, 1, p, None, None, None) == 1
    assert lib.gptq_export_checkpoint(p, p, p, 8, 36, 3, 1, 1, p, None, None, None) == 7
    assert lib.gptq_export_checkpoint(p, p, p, 12, 32, 3, 1, 1, None, p, None, None) == 7
    assert "out*bits" in g.gptq_last_error()
    # nothing requested, or out == 0: a no-op that needs no GPU
    assert lib.gptq_export_checkpoint(p, p, p, 8, 32, 4, 1, 1, None, None, None, None) == 0
    assert lib.gptq_export_checkpoint(p, p, p, 0, 32, 4, 1, 1, p, p, p, None) == 0
