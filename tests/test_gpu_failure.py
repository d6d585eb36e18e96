"""Failure handling without a GPU fault: the bounded waits every kernel of
the library uses give up after their limit and report GPTQ_ERR_TIMEOUT
through a status word; the context stays usable afterwards."""
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
