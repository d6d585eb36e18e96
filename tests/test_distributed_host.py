"""The sharded layer solve's partition and exchange logic, run as gloo
ranks on the host.  Each rank holds a share of the calibration tokens and
solves a share of the rows; the arithmetic steps are the oracle's (LayerOps
built from it), so the gathered layer must equal the oracle's single-process
solve of the whole layer exactly: the tokens are exact small multiples of a
power of two, so every partial Hessian and their sum are exact in fp64."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed, out, in_, tokens):
    rng = np.random.default_rng(seed)
    X = rng.integers(-4, 5, size=(in_, tokens)).astype(np.float64) * 0.125
    X[3] = 0.0                                   # a dead channel
    W = rng.standard_normal((out, in_)) * 0.05
    return W, X


def oracle_ops():
    """LayerOps from the oracle (fp64 on the host)."""
    import torch

    import oracle as O
    from post_weight_quantization_13_b200.distributed import LayerOps

    def hessian(X, in_, device):
        if X is None:
            return torch.zeros((in_, in_), dtype=torch.float64), 0
        Xn = X.numpy()
        return torch.from_numpy(O.hessian_accumulate(np.zeros((in_, in_)), Xn)), Xn.shape[1]

    def prepare(S, n, cfg):
        p = O.prepare(S.numpy(), n, cfg.damp_percent, bool(cfg.desc_act))
        return torch.from_numpy(p["U"]), torch.from_numpy(p["perm"]), torch.from_numpy(p["dead"])

    def quantize(W, U, perm, dead, cfg):
        Wd = W.numpy().copy()
        perm_n = perm.numpy()
        Wd[:, dead.numpy()] = 0.0
        r = O.sweep_blocked(Wd[:, perm_n], U.numpy(), cfg.bits, cfg.group_size, bool(cfg.sym),
                            cfg.block_size)
        invperm = np.empty_like(perm_n)
        invperm[perm_n] = np.arange(perm_n.size)
        codes = r["codes"][:, invperm]
        res = dict(codes=torch.from_numpy(codes), scales=torch.from_numpy(r["scales"]),
                   zeros=torch.from_numpy(r["zeros"]), loss=torch.from_numpy(r["loss"]),
                   g_idx=torch.from_numpy(O.g_index(perm_n, cfg.group_size)), qweight=None)
        if (W.shape[1] * cfg.bits) % 32 == 0:
            res["qweight"] = torch.from_numpy(O.pack_rows(codes, cfg.bits).astype(np.int64))
        return res

    return LayerOps(hessian, prepare, quantize)


def _rank_main(rank, world, port, case, q):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from post_weight_quantization_13_b200 import GptqConfig
    from post_weight_quantization_13_b200.distributed import shard_bounds, solve_layer_sharded
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seed, out, in_, tokens, cfgd = case
        W, X = _layer(seed, out, in_, tokens)
        t0, t1 = shard_bounds(tokens, world, rank)
        res = solve_layer_sharded(torch.from_numpy(W), torch.from_numpy(X[:, t0:t1]),
                                  GptqConfig(**cfgd), ops=oracle_ops())
        keep = {k: (None if res[k] is None else res[k].numpy())
                for k in ("all_codes", "all_scales", "all_zeros", "all_loss", "all_qweight", "g_idx",
                          "perm", "dead", "S")}
        q.put((rank, res["n"], res["rows"], keep))
    finally:
        dist.destroy_process_group()


CASES = [
    (2, (11, 37, 64, 96, dict(bits=4, group_size=32, desc_act=True))),    # rows 19 + 18
    (2, (12, 40, 96, 1, dict(bits=3, group_size=-1, sym=True))),          # rank 1 has no tokens
    (3, (13, 23, 64, 2, dict(bits=2, group_size=16, desc_act=True))),     # rows 8 + 8 + 7; rank 2 no tokens
]


@pytest.mark.parametrize("world,case", CASES)
def test_gloo_ranks_give_the_single_process_solve(world, case):
    import torch.multiprocessing as mp

    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seed, out, in_, tokens, cfgd = case
    W, X = _layer(seed, out, in_, tokens)
    S = O.hessian_accumulate(np.zeros((in_, in_)), X)
    full = dict(bits=4, group_size=128, sym=False, desc_act=False, damp_percent=0.01, block_size=128)
    full.update(cfgd)
    ref = O.gptq_layer(W, S, tokens, **full)
    from post_weight_quantization_13_b200.distributed import shard_bounds
    assert [g[2] for g in got] == [shard_bounds(out, world, r) for r in range(world)]
    for rank, n, rows, k in got:
        assert n == tokens
        assert np.array_equal(k["S"], S)                  # the all-reduced Hessian, exact
        assert np.array_equal(k["perm"], ref["perm"])
        assert np.array_equal(k["dead"], ref["dead"])
        assert np.array_equal(k["g_idx"], ref["g_idx"])
        assert np.array_equal(k["all_codes"], ref["codes"])
        assert np.array_equal(k["all_scales"], ref["scales"])
        assert np.array_equal(k["all_zeros"], ref["zeros"])
        assert np.array_equal(k["all_loss"], ref["loss"])
        if "qweight" in ref:
            assert np.array_equal(k["all_qweight"], ref["qweight"].astype(np.int64))


def test_shard_bounds_partition():
    from post_weight_quantization_13_b200.distributed import shard_bounds
    for total in (0, 1, 7, 37, 4096, 11008):
        for world in (1, 2, 3, 8):
            parts = [shard_bounds(total, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == total
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard_bounds(4, 0, 0)
    with pytest.raises(ValueError):
        shard_bounds(4, 2, 2)
