"""Seeded synthetic inputs for the GPTQ layer solver: weights W (out x in) and
calibration activations X (in x tokens).

This module only draws random numbers and casts them; it holds none of the
solver's arithmetic.  Both the CPU oracle (through the tests) and the GPU path
(through the tests and ``bench.py``) take their inputs from here, so the two
sides always see the same values.

Shapes and distributions follow the workloads the GPTQ pages calibrate on:
128 calibration sequences of 2048 tokens each ("Using AutoGPTQ in Practice",
the calibration-data step of the workflow; the "gptq" agent-skill page,
"Quantization configurations") and Llama-7B-shaped linear layers.  The pages
calibrate on C4 text, which is not available here; the synthetic activations
below stand in for it and no dataset item is reproduced.

Recipe (all draws use ``numpy.random.default_rng([workload_tag, site_or_layer,
stream])``, cast to the stated dtype with round-to-nearest-even):

* W ~ N(0, 0.02^2), stream 0 of tag ``100 + layer_id``.
* scaled-normal X: X[c, t] = s_c * z, z ~ N(0, 1), s_c = exp(sigma * N(0, 1))
  (stream 1); a fraction of channels (stream 2, without replacement) gets an
  extra factor (x20 outliers).
* SiLU-gated X (down_proj input): X = silu(a) * b with a, b ~ N(0, 1).
* correlated X: x = s * (z + P y), P in x r ~ N(0, 1) (stream 2), y ~ N(0, I_r):
  an identity-plus-low-rank mixing that makes H strongly non-diagonal.
* token chunk c (``chunk`` tokens) is drawn from stream ``3 + c`` so chunks can
  be generated independently and in parallel.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Site", "Layer", "QuantSpec", "Workload", "WORKLOADS",
    "weight", "channel_scales", "x_chunk", "x_full", "small_case",
    "correlated_tiny",
]


@dataclass(frozen=True)
class Site:
    """One calibration-activation stream: the input of one or more layers,
    hence one Hessian."""
    name: str
    tag: int            # site id inside the workload's seed tuple
    in_: int
    kind: str = "scaled_normal"   # scaled_normal | silu_gated | correlated
    sigma: float = 1.5
    outlier_frac: float = 0.0
    outlier_mult: float = 20.0
    rank: int = 16


@dataclass(frozen=True)
class Layer:
    name: str
    out: int
    in_: int
    site: str
    layer_id: int


@dataclass(frozen=True)
class QuantSpec:
    bits: int = 4
    group_size: int = 128
    sym: bool = False
    desc_act: bool = False
    damp_percent: float = 0.01
    block_size: int = 128

    def as_dict(self):
        return dict(bits=self.bits, group_size=self.group_size, sym=self.sym,
                    desc_act=self.desc_act, damp_percent=self.damp_percent,
                    block_size=self.block_size)


@dataclass(frozen=True)
class Workload:
    name: str
    tag: int
    tokens: int
    chunk: int
    w_dtype: str
    x_dtype: str
    sites: tuple
    layers: tuple
    quant: tuple = field(default_factory=lambda: (QuantSpec(),))

    def site(self, name):
        for s in self.sites:
            if s.name == name:
                return s
        raise KeyError(name)

    def layer(self, name):
        for l in self.layers:
            if l.name == name:
                return l
        raise KeyError(name)


_ATTN = Site("attn", 0, 4096, "scaled_normal", 1.5, 0.01, 20.0)
_O = Site("o", 1, 4096, "scaled_normal", 1.5, 0.01, 20.0)
_MLP = Site("mlp", 2, 4096, "scaled_normal", 1.5, 0.01, 20.0)
_DOWN = Site("down", 3, 11008, "silu_gated")

WORKLOADS = {
    # 256x256 fp32 layer, 1024 fp32 tokens, lognormal(0, 1) channel scales.
    "layer256_fp32": Workload(
        "layer256_fp32", 0, 1024, 1024, "float32", "float32",
        (Site("x", 0, 256, "scaled_normal", 1.0, 0.0),),
        (Layer("w", 256, 256, "x", 0),),
        (QuantSpec(4, 128, False, False, 0.01, 128),)),
    # Llama-7B q_proj: 4096x4096 fp16, 128 x 2048 fp16 tokens,
    # lognormal(0, 1.5) channel scales, 1% of channels x20.
    "llama7b_q_proj": Workload(
        "llama7b_q_proj", 1, 262144, 2048, "float16", "float16",
        (_ATTN,), (Layer("q_proj", 4096, 4096, "attn", 0),),
        (QuantSpec(4, 128, False, False, 0.01, 128),)),
    # Same layer and activations, act-order on: b4 g128, b8 g64, b2 g64.
    "llama7b_q_proj_actorder": Workload(
        "llama7b_q_proj_actorder", 1, 262144, 2048, "float16", "float16",
        (_ATTN,), (Layer("q_proj", 4096, 4096, "attn", 0),),
        (QuantSpec(4, 128, False, True), QuantSpec(8, 64, False, True),
         QuantSpec(2, 64, False, True))),
    # Llama-7B MLP pair, 3-bit symmetric, act-order on.
    "llama7b_mlp": Workload(
        "llama7b_mlp", 3, 262144, 2048, "float16", "float16",
        (_MLP, _DOWN),
        (Layer("up_proj", 11008, 4096, "mlp", 5),
         Layer("down_proj", 4096, 11008, "down", 6)),
        (QuantSpec(3, 128, True, True),)),
    # A whole Llama-7B-shaped decoder block: 4 Hessians, 7 solves.
    "llama7b_block": Workload(
        "llama7b_block", 4, 262144, 2048, "float16", "float16",
        (_ATTN, _O, _MLP, _DOWN),
        (Layer("q_proj", 4096, 4096, "attn", 0),
         Layer("k_proj", 4096, 4096, "attn", 1),
         Layer("v_proj", 4096, 4096, "attn", 2),
         Layer("o_proj", 4096, 4096, "o", 3),
         Layer("gate_proj", 11008, 4096, "mlp", 4),
         Layer("up_proj", 11008, 4096, "mlp", 5),
         Layer("down_proj", 4096, 11008, "down", 6)),
        (QuantSpec(4, 128, False, True),)),
    # The q_proj shape with strongly correlated channels (8192 tokens), so
    # that error compensation is exercised hard.
    "q_proj_correlated": Workload(
        "q_proj_correlated", 5, 8192, 2048, "float16", "float16",
        (Site("x", 0, 4096, "correlated", 1.0, 0.0, 20.0, 16),),
        (Layer("q_proj", 4096, 4096, "x", 0),),
        (QuantSpec(4, 128, False, True),)),
}


def _rng(*key):
    return np.random.default_rng([int(k) for k in key])


def weight(wl: Workload, layer: Layer | str) -> np.ndarray:
    """W ~ N(0, 0.02^2), shape (out, in), in the workload's weight dtype."""
    if isinstance(layer, str):
        layer = wl.layer(layer)
    z = _rng(wl.tag, 100 + layer.layer_id, 0).standard_normal(
        (layer.out, layer.in_), dtype=np.float32)
    return (z * np.float32(0.02)).astype(wl.w_dtype)


def channel_scales(wl: Workload, site: Site | str) -> np.ndarray:
    """Per-channel scale s_c (float32), including outlier channels."""
    if isinstance(site, str):
        site = wl.site(site)
    if site.kind == "silu_gated":
        return np.ones(site.in_, np.float32)
    s = np.exp(site.sigma * _rng(wl.tag, site.tag, 1).standard_normal(site.in_))
    n_out = int(round(site.outlier_frac * site.in_))
    if n_out:
        idx = _rng(wl.tag, site.tag, 2).choice(site.in_, n_out, replace=False)
        s[idx] *= site.outlier_mult
    return s.astype(np.float32)


def _mixing(wl: Workload, site: Site) -> np.ndarray:
    return _rng(wl.tag, site.tag, 2).standard_normal(
        (site.in_, site.rank), dtype=np.float32)


def x_chunk(wl: Workload, site: Site | str, c: int, tokens: int | None = None,
            scales: np.ndarray | None = None, mixing: np.ndarray | None = None
            ) -> np.ndarray:
    """Token chunk c of X: shape (in, tokens), the workload's activation dtype."""
    if isinstance(site, str):
        site = wl.site(site)
    t = wl.chunk if tokens is None else tokens
    r = _rng(wl.tag, site.tag, 3 + c)
    if site.kind == "silu_gated":
        a = r.standard_normal((site.in_, t), dtype=np.float32)
        b = r.standard_normal((site.in_, t), dtype=np.float32)
        x = a / (np.float32(1) + np.exp(-a)) * b
    elif site.kind == "correlated":
        if scales is None:
            scales = channel_scales(wl, site)
        if mixing is None:
            mixing = _mixing(wl, site)
        z = r.standard_normal((site.in_, t), dtype=np.float32)
        y = r.standard_normal((site.rank, t), dtype=np.float32)
        x = (z + mixing @ y) * scales[:, None]
    else:
        if scales is None:
            scales = channel_scales(wl, site)
        x = r.standard_normal((site.in_, t), dtype=np.float32) * scales[:, None]
    x = x.astype(wl.x_dtype)
    if not np.all(np.isfinite(x)):
        raise OverflowError("synthetic activations overflowed the target dtype")
    return x


def x_full(wl: Workload, site: Site | str, tokens: int | None = None,
           out: np.ndarray | None = None, threads: int | None = None
           ) -> np.ndarray:
    """The whole of X, shape (in, tokens): chunk c fills columns
    [c*chunk, (c+1)*chunk).  ``out`` may be a caller-provided (e.g. pinned)
    array of that shape and dtype."""
    if isinstance(site, str):
        site = wl.site(site)
    n = wl.tokens if tokens is None else tokens
    if out is None:
        out = np.empty((site.in_, n), dtype=wl.x_dtype)
    assert out.shape == (site.in_, n) and out.dtype == np.dtype(wl.x_dtype)
    scales = channel_scales(wl, site)
    mixing = _mixing(wl, site) if site.kind == "correlated" else None
    nchunks = (n + wl.chunk - 1) // wl.chunk

    def fill(c):
        t0 = c * wl.chunk
        t1 = min(n, t0 + wl.chunk)
        out[:, t0:t1] = x_chunk(wl, site, c, t1 - t0, scales, mixing)

    threads = threads or max(1, min(16, len(os.sched_getaffinity(0))))
    if threads == 1 or nchunks == 1:
        for c in range(nchunks):
            fill(c)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def small_case(seed: int, out: int, in_: int, tokens: int, w_dtype="float32",
               x_dtype="float32", sigma=1.0, outlier_frac=0.0,
               kind="scaled_normal", rank=4):
    """An arbitrary-size layer with the same recipe (for parity tests that need
    odd or ragged shapes).  Returns (W, X)."""
    wl = Workload(f"small{seed}", 1000 + seed, tokens, tokens, w_dtype, x_dtype,
                  (Site("x", 0, in_, kind, sigma, outlier_frac, 20.0, rank),),
                  (Layer("w", out, in_, "x", 0),))
    return weight(wl, "w"), x_full(wl, "x", threads=1)


def correlated_tiny(seed: int, out: int, in_: int, tokens: int = 32):
    """Tiny layer with X = A Z, A ~ N(0, 1) (in x in), Z ~ N(0, 1) (in x tokens):
    strongly correlated channels, for brute-force checks.  float64 arrays."""
    r = _rng(2000, seed, 0)
    w = r.standard_normal((out, in_))
    a = r.standard_normal((in_, in_))
    z = r.standard_normal((in_, tokens))
    return w, a @ z
