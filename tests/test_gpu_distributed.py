"""The sharded layer solve with the library's kernels, as a one-rank NCCL
group (one GPU is all a test here gets): the all-reduce, the row slicing and
the gather must leave solve_layer's result unchanged, bit for bit."""
import datetime
import os
import socket

import pytest

import gen
from gpu_util import dev

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_sharded_solve_equals_solve_layer(lib):
    import torch
    import torch.distributed as dist

    from post_weight_quantization_13_b200.distributed import solve_layer_sharded
    W, X = gen.small_case(77, 300, 512, 2048, w_dtype="float16", x_dtype="float16")
    Wd, Xd = dev(W), dev(X)
    cfg = lib.GptqConfig(bits=4, group_size=64, desc_act=True)
    ref = lib.solve_layer(Wd, Xd, cfg)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        res = solve_layer_sharded(Wd, Xd, cfg)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert res["n"] == ref["n"] and res["rows"] == (0, 300)
    assert torch.equal(torch.triu(res["S"]), torch.triu(ref["S"]))
    for k in ("perm", "dead", "g_idx"):
        assert torch.equal(res[k], ref[k]), k
    assert torch.equal(res["U"], ref["U"])
    for k in ("codes", "scales", "zeros", "loss", "qweight"):
        assert torch.equal(res["all_" + k], ref[k]), k
