"""One layer solved by several GPUs ("AutoGPTQ" artifact page, its
distributed-quantization paragraph: the calibration data are split across
devices and the quantization is coordinated over NCCL or Gloo).

The method's data dependencies fix the partition:

* Hessian: S = sum over tokens of x x^T is a sum, so each rank accumulates
  the tokens it holds into a partial S_r (gptq_hessian_accumulate), and one
  all-reduce (sum) of the in x in fp32 matrix and of the token counts gives
  every rank the whole S and n.  This is the one collective of the solve.
* Prepare: every rank runs gptq_prepare_hinv on the same S and n.  The
  factorisation's order of operations is fixed, so the ranks get identical
  U, perm and dead without a broadcast.
* Sweep: rows of W never interact given U, so rank r quantizes its own
  contiguous block of rows (gptq_quantize_layer on a row slice).  g_idx is
  the same on every rank.
* Gather: the row blocks (packed codes, scales, zeros, loss) are all-gathered
  so that every rank holds the whole layer; blocks are padded to the
  largest one because NCCL's all-gather wants equal sizes.

Each rank launches only its own kernels; the collectives run through
torch.distributed on the caller's process group (NCCL on GPUs, Gloo on the
host).  The arithmetic steps are injected as ``ops`` so that the same
partition and exchange logic runs on the host with any implementation of the
three steps (the CUDA library by default).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

__all__ = ["shard_bounds", "LayerOps", "cuda_ops", "solve_layer_sharded"]


def shard_bounds(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous near-equal split of range(total) into ``world`` parts: the
    first total % world parts get one extra element.  Part ``rank`` is
    [lo, hi)."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(total, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


@dataclass
class LayerOps:
    """The three arithmetic steps of a layer solve.

    hessian(X, in_, device) -> (S, n)
                              S = X X^T (in x in; the upper triangle is
                              what later steps read) over X's tokens (X:
                              in x t, or None for no tokens) and n = t.
    prepare(S, n, cfg) -> (U, perm, dead)
    quantize(W, U, perm, dead, cfg) -> dict with qweight (int32, out x
                              in*bits/32, or None), scales (fp32, out x ng),
                              zeros (int32, out x ng), loss (fp32, out),
                              g_idx (int32, in) and codes (int32, out x in,
                              processing order undone).
    """
    hessian: Callable
    prepare: Callable
    quantize: Callable


def cuda_ops(stream=None) -> LayerOps:
    """The library's kernels as LayerOps (tensors on the current device)."""
    import torch

    from . import (GptqConfig, gptq_hessian_accumulate, gptq_prepare_hinv, gptq_quantize_layer,
                   gptq_workspace_bytes, gptq_workspace_status)

    def hessian(X, in_, device):
        S = torch.zeros((in_, in_), dtype=torch.float32, device=device)
        n = 0 if X is None else gptq_hessian_accumulate(S, X, 0, stream)
        return S, n

    def prepare(S, n, cfg):
        in_ = S.shape[0]
        dev = S.device
        ws = torch.empty(gptq_workspace_bytes(0, in_, cfg), dtype=torch.uint8, device=dev)
        U = torch.empty((in_, in_), dtype=torch.float32, device=dev)
        perm = torch.empty(in_, dtype=torch.int32, device=dev)
        dead = torch.empty(in_, dtype=torch.uint8, device=dev)
        gptq_prepare_hinv(S, n, cfg, U, perm, dead, ws, stream)
        return U, perm, dead

    def quantize(W, U, perm, dead, cfg):
        cfg = GptqConfig.of(cfg)
        out, in_ = W.shape
        dev = W.device
        ng = 1 if cfg.group_size == -1 else in_ // cfg.group_size
        r = dict(scales=torch.empty((out, ng), dtype=torch.float32, device=dev),
                 zeros=torch.empty((out, ng), dtype=torch.int32, device=dev),
                 g_idx=torch.empty(in_, dtype=torch.int32, device=dev),
                 loss=torch.empty(out, dtype=torch.float32, device=dev),
                 codes=torch.empty((out, in_), dtype=torch.int32, device=dev),
                 qweight=(torch.empty((out, in_ * cfg.bits // 32), dtype=torch.int32, device=dev)
                          if (in_ * cfg.bits) % 32 == 0 else None))
        ws = torch.empty(gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device=dev)
        gptq_quantize_layer(W, U, perm, dead, cfg, r["scales"], r["zeros"], r["g_idx"], ws,
                            codes=r["codes"], qweight=r["qweight"], loss=r["loss"], stream=stream)
        gptq_workspace_status(ws, stream)
        return r

    return LayerOps(hessian, prepare, quantize)


def _all_gather_rows(t, rows_of, world: int, group):
    """Concatenate every rank's row block of ``t`` (rank r holds rows_of(r)
    rows) in rank order, through one all-gather of equal-sized padded
    blocks."""
    import torch
    import torch.distributed as dist
    most = max(rows_of(r) for r in range(world))
    pad = torch.zeros((most,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[: t.shape[0]] = t
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][: rows_of(r)] for r in range(world)], 0)


def solve_layer_sharded(W, X_local, cfg, group=None, ops: Optional[LayerOps] = None,
                        gather: bool = True):
    """Solve one layer on every rank of ``group`` together.

    W: the whole out x in weight matrix on every rank (each rank reads only its
      row block).  X_local: this rank's calibration tokens (in x t_r).
    Returns a dict with S and n (the reduced Hessian and token count, equal on
    all ranks), U, perm, dead, g_idx, ``rows`` = this rank's [lo, hi) and, for
    those rows, qweight, scales, zeros, loss and codes; with ``gather`` the
    same keys also hold the whole layer (every rank's rows in order) under
    ``all_`` + name.
    """
    import torch
    import torch.distributed as dist

    from . import GptqConfig

    cfg = GptqConfig.of(cfg)
    ops = ops or cuda_ops()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    out, in_ = W.shape
    dev = W.device
    # 1. partial Hessian over this rank's tokens, then the one all-reduce
    S, n_local = ops.hessian(X_local if X_local is not None and X_local.shape[1] > 0 else None, in_, dev)
    n_t = torch.tensor([n_local], dtype=torch.int64, device=dev)
    dist.all_reduce(S, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(n_t, op=dist.ReduceOp.SUM, group=group)
    n = int(n_t.item())
    # 2. the same prepare on every rank
    U, perm, dead = ops.prepare(S, n, cfg)
    # 3. this rank's rows
    lo, hi = shard_bounds(out, world, rank)
    part = ops.quantize(W[lo:hi], U, perm, dead, cfg)
    res = dict(S=S, n=n, U=U, perm=perm, dead=dead, g_idx=part["g_idx"], rows=(lo, hi))
    for k in ("qweight", "scales", "zeros", "loss", "codes"):
        res[k] = part.get(k)
    if gather:
        def rows_of(r):
            a, b = shard_bounds(out, world, r)
            return b - a
        for k in ("qweight", "scales", "zeros", "loss", "codes"):
            v = part.get(k)
            res["all_" + k] = None if v is None else _all_gather_rows(v, rows_of, world, group)
    return res
