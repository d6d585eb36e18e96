"""gptq_quantize_layer_noalloc: the quantize call on the library's static
device scratch must give what gptq_quantize_layer gives with a caller
workspace, call after call, and must reject layers whose scratch would not
fit.  (File name sorts last so it also runs after every other test.)"""
import ctypes

import numpy as np
import pytest

import gen
from gpu_util import dev, host

GPTQ_ERR_WORKSPACE = 4


@pytest.fixture(scope="module")
def g():
    import __graft_entry__
    __graft_entry__.build()
    import post_weight_quantization_13_b200 as m
    return m


def test_static_scratch_size_matches_header(g):
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "gptq.h")).read()
    m = re.search(r"#define GPTQ_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == g.GPTQ_STATIC_SCRATCH_BYTES


@pytest.mark.parametrize("out,in_", [(2048, 2048), (1024, 4096), (8192, 512)])
def test_rejects_layers_beyond_the_static_scratch(g, out, in_):
    """Checked on the host before any device work: needs no GPU."""
    cfg = g.GptqConfig(bits=4, group_size=128).c()
    s = g.lib.gptq_quantize_layer_noalloc(None, 0, out, in_, in_, None, None, None,
                                          ctypes.byref(cfg), None, None, None, None, None,
                                          None, None)
    assert s == GPTQ_ERR_WORKSPACE
    msg = g.lib.gptq_last_error().decode()
    assert "needs" in msg and str(g.GPTQ_STATIC_SCRATCH_BYTES) in msg


def _outputs(out, in_, cfg):
    import torch
    ng = 1 if cfg.group_size == -1 else in_ // cfg.group_size
    o = dict(scales=torch.full((out, ng), -1.0, dtype=torch.float32, device="cuda"),
             zeros=torch.full((out, ng), -1, dtype=torch.int32, device="cuda"),
             g_idx=torch.full((in_,), -1, dtype=torch.int32, device="cuda"),
             loss=torch.full((out,), -1.0, dtype=torch.float32, device="cuda"),
             codes=torch.full((out, in_), -1, dtype=torch.int32, device="cuda"))
    if (in_ * cfg.bits) % 32 == 0:
        o["qweight"] = torch.zeros((out, in_ * cfg.bits // 32), dtype=torch.int32, device="cuda")
    return o


@pytest.mark.gpu
@pytest.mark.parametrize("out,in_,bits,gs,sym,desc_act,wdt,seed", [
    (512, 768, 4, 128, False, True, "float16", 31),
    (300, 320, 3, 64, True, False, "bfloat16", 32),
    (1024, 1024, 4, 128, False, True, "float16", 33),   # near the scratch limit
])
def test_noalloc_matches_workspace_call_twice(g, out, in_, bits, gs, sym, desc_act, wdt, seed):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    W, X = gen.small_case(seed, out, in_, 2 * in_, w_dtype="float32", x_dtype="float16",
                          sigma=1.5, outlier_frac=0.01)
    cfg = g.GptqConfig(bits=bits, group_size=gs, sym=sym, desc_act=desc_act)
    W_t = dev(W, {"float16": torch.float16, "bfloat16": torch.bfloat16}[wdt])
    X_t = dev(X, torch.float16)
    S = torch.zeros((in_, in_), dtype=torch.float32, device="cuda")
    n = g.gptq_hessian_accumulate(S, X_t, 0)
    ws = torch.empty(g.gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device="cuda")
    U = torch.empty((in_, in_), dtype=torch.float32, device="cuda")
    perm = torch.empty(in_, dtype=torch.int32, device="cuda")
    dead = torch.empty(in_, dtype=torch.uint8, device="cuda")
    g.gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws)

    ref = _outputs(out, in_, cfg)
    g.gptq_quantize_layer(W_t, U, perm, dead, cfg, ref["scales"], ref["zeros"], ref["g_idx"], ws,
                          codes=ref["codes"], qweight=ref.get("qweight"), loss=ref["loss"])
    torch.cuda.synchronize()
    ref = {k: host(v) for k, v in ref.items()}
    maxq = 2 ** bits - 1
    assert ref["codes"].min() >= 0 and ref["codes"].max() <= maxq

    for call in range(2):
        o = _outputs(out, in_, cfg)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        alloc0 = torch.cuda.memory_allocated()
        g.gptq_quantize_layer_noalloc(W_t, U, perm, dead, cfg, o["scales"], o["zeros"], o["g_idx"],
                                      codes=o["codes"], qweight=o.get("qweight"), loss=o["loss"])
        torch.cuda.synchronize()
        if call == 1:
            # after the first call's set-up, a call takes no device memory:
            # neither from the driver nor from torch's caching allocator
            free1, _ = torch.cuda.mem_get_info()
            assert free1 == free0, (free0, free1)
            assert torch.cuda.memory_allocated() == alloc0
        g.gptq_quantize_layer_noalloc_status()        # no device-side failure
        o = {k: host(v) for k, v in o.items()}
        # integer outputs bit-exact; floating point within 1e-6 relative
        for k in ("codes", "zeros", "g_idx", "qweight"):
            if k in ref:
                assert np.array_equal(o[k], ref[k]), (call, k)
        for k in ("scales", "loss"):
            np.testing.assert_allclose(o[k], ref[k], rtol=1e-6, atol=0, err_msg=f"call {call} {k}")
