"""Failure handling without a GPU fault: the bounded waits every kernel of
the library uses give up after their limit and report GPTQ_ERR_TIMEOUT
through a status word; the context stays usable afterwards."""
import ctypes

import numpy as np
import pytest

import gen
import oracle as O
from gpu_util import code_report, dev, host

GPTQ_ERR_INVALID_ARG, GPTQ_ERR_TIMEOUT = 1, 6


@pytest.fixture(scope="module")
def g():
    import __graft_entry__
    __graft_entry__.build()
    import post_weight_quantization_13_b200 as m
    return m


def test_selftest_rejects_bad_limits_on_the_host(g):
    assert g.lib.gptq_selftest_wait_timeout(0, None) == GPTQ_ERR_INVALID_ARG
    assert g.lib.gptq_selftest_wait_timeout(3 * 10**9, None) == GPTQ_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_times_out_and_the_device_stays_usable(lib):
    import time
    import torch
    t0 = time.perf_counter()
    assert lib.gptq_selftest_wait_timeout(5_000_000) == GPTQ_ERR_TIMEOUT   # 5 ms
    assert time.perf_counter() - t0 < 5.0
    assert "gave up" in lib.gptq_last_error()
    # a full solve right after, checked against the oracle
    W, X = gen.small_case(41, 64, 256, 512, w_dtype="float32", x_dtype="float16")
    q = dict(bits=4, group_size=64, sym=False, desc_act=True, damp_percent=0.01, block_size=128)
    r = lib.solve_layer(dev(W), dev(X, torch.float16), q)
    S, n = O.hessian([torch.from_numpy(X).to(torch.float16).float().numpy()])
    ref = O.gptq_layer(W, S, n, **q)
    assert np.array_equal(host(r["perm"]), ref["perm"])
    rate, _ = code_report(host(r["codes"]), ref["codes"])
    assert rate >= 0.999, rate


def test_workspace_status_rejects_bad_workspaces_on_the_host(g):
    GPTQ_ERR_WORKSPACE = 4
    assert g.lib.gptq_workspace_status(None, 1 << 20, None) == GPTQ_ERR_WORKSPACE
    assert g.lib.gptq_workspace_status(ctypes.c_void_p(256 + 16), 1 << 20, None) == GPTQ_ERR_WORKSPACE
    assert g.lib.gptq_workspace_status(ctypes.c_void_p(1 << 20), 128, None) == GPTQ_ERR_WORKSPACE


@pytest.mark.gpu
def test_quantize_status_reaches_the_caller(lib):
    """gptq_quantize_layer returns before its kernels run; a device-side
    failure reaches the caller through the workspace's status word.  A clean
    quantize reads back GPTQ_OK; a status word holding the timeout flag (the
    flag the bounded waits raise, set here by the test) reads back
    GPTQ_ERR_TIMEOUT; the next quantize clears it again."""
    import torch
    W, X = gen.small_case(42, 48, 256, 512, w_dtype="float32", x_dtype="float16")
    cfg = lib.GptqConfig(bits=4, group_size=64, desc_act=True)
    S = torch.zeros((256, 256), dtype=torch.float32, device="cuda")
    n = lib.gptq_hessian_accumulate(S, dev(X, torch.float16), 0)
    ws = torch.empty(lib.gptq_workspace_bytes(48, 256, cfg), dtype=torch.uint8, device="cuda")
    U = torch.empty((256, 256), dtype=torch.float32, device="cuda")
    perm = torch.empty(256, dtype=torch.int32, device="cuda")
    dead = torch.empty(256, dtype=torch.uint8, device="cuda")
    lib.gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws)
    scales = torch.empty((48, 4), dtype=torch.float32, device="cuda")
    zeros = torch.empty((48, 4), dtype=torch.int32, device="cuda")
    g_idx = torch.empty(256, dtype=torch.int32, device="cuda")
    Wd = dev(W)

    def quantize():
        lib.gptq_quantize_layer(Wd, U, perm, dead, cfg, scales, zeros, g_idx, ws)

    quantize()
    lib.gptq_workspace_status(ws)
    ws[:4].view(torch.int32).fill_(4)           # the timeout flag
    with pytest.raises(lib.GptqError) as e:
        lib.gptq_workspace_status(ws)
    assert e.value.status == GPTQ_ERR_TIMEOUT
    quantize()
    lib.gptq_workspace_status(ws)
