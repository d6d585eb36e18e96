"""Parity at the full benchmark size: the 4096 x 4096 Llama-7B q_proj layer
with 262144 fp16 calibration tokens (128 x 2048), run through the C ABI in
the launch configuration bench.py times (one Hessian call over all tokens).

The float64 oracle works from its own inputs only (the seeded generator),
never from a GPU result:
* sampled Hessian entries, each an exact float64 dot product over all tokens;
* the oracle's full S (chunked float64 products), hence its own U, and the
  act-order permutation from the exact diagonal;
* the sweep on sampled rows with the oracle's U.

Tolerances: S within 5e-5 of sqrt(S_ii S_jj) per sampled entry (the tensor-core
accumulation bound the small parity tests use, scaled by Cauchy-Schwarz);
U within 1e-3 relative Frobenius (fp32 accuracy amplified by the condition of
the damped Hessian, which the outlier channels make large); codes >= 99.9 %
identical on the sampled rows; the layer error of the sampled rows within 1 %
of the oracle's.  Where the GPU orders act-order columns by its fp32 diagonal,
columns whose exact diagonals tie to within the Hessian tolerance may come in
either order: the permutation is checked for validity, not equality.
"""
import numpy as np
import pytest

import gen
import oracle as O
from gpu_util import code_report, compare_groups, host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

WL = gen.WORKLOADS["llama7b_q_proj"]
WL_ACT = gen.WORKLOADS["llama7b_q_proj_actorder"]
ROWS = 48          # sampled output rows for the sweep comparison
PAIRS = 400        # sampled Hessian entries


@pytest.fixture(scope="module")
def full(lib):
    import torch
    layer = WL.layers[0]
    W = gen.weight(WL, layer)                                   # fp16 values
    X = gen.x_full(WL, layer.site)                              # 4096 x 262144 fp16
    Xd = torch.from_numpy(X).cuda()
    S = torch.zeros((layer.in_, layer.in_), dtype=torch.float32, device="cuda")
    n = lib.gptq_hessian_accumulate(S, Xd, 0)
    torch.cuda.synchronize()
    del Xd
    # oracle: float64 S over all tokens, in chunks
    S64 = np.zeros((layer.in_, layer.in_), dtype=np.float64)
    for c0 in range(0, X.shape[1], 16384):
        O.hessian_accumulate(S64, X[:, c0:c0 + 16384])
    return dict(W=W, X=X, S=S, n=n, S64=S64, layer=layer)


def _gpu_solve(lib, full, q):
    import torch
    layer = full["layer"]
    out, in_ = layer.out, layer.in_
    cfg = lib.GptqConfig(**q.as_dict())
    ws = torch.empty(lib.gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device="cuda")
    U = torch.empty((in_, in_), dtype=torch.float32, device="cuda")
    perm = torch.empty(in_, dtype=torch.int32, device="cuda")
    dead = torch.empty(in_, dtype=torch.uint8, device="cuda")
    lib.gptq_prepare_hinv(full["S"], full["n"], cfg, U, perm, dead, ws)
    ng = in_ // q.group_size
    scales = torch.empty((out, ng), dtype=torch.float32, device="cuda")
    zeros = torch.empty((out, ng), dtype=torch.int32, device="cuda")
    g_idx = torch.empty(in_, dtype=torch.int32, device="cuda")
    codes = torch.empty((out, in_), dtype=torch.int32, device="cuda")
    Wd = torch.from_numpy(full["W"]).cuda()
    lib.gptq_quantize_layer(Wd, U, perm, dead, cfg, scales, zeros, g_idx, ws, codes=codes)
    torch.cuda.synchronize()
    return dict(U=host(U), perm=host(perm).astype(np.int64), dead=host(dead),
                scales=host(scales), zeros=host(zeros), g_idx=host(g_idx), codes=host(codes))


def _oracle_prep(full, q):
    key = (q.damp_percent, q.desc_act)
    cache = full.setdefault("prep", {})
    if key not in cache:
        cache[key] = O.prepare(full["S64"], full["n"], q.damp_percent, q.desc_act)
    return cache[key]


def _oracle_rows(full, q, rows):
    prep = _oracle_prep(full, q)
    W0 = np.asarray(full["W"], np.float64)
    Wd = W0[rows].copy()
    Wd[:, prep["dead"]] = 0.0
    res = O.sweep_blocked(Wd[:, prep["perm"]], prep["U"], q.bits, q.group_size, q.sym, q.block_size)
    inv = np.empty_like(prep["perm"])
    inv[prep["perm"]] = np.arange(len(inv))
    return prep, res, res["codes"][:, inv]


def _row_error(W0, codes, scales, zeros, g_idx, H0):
    deq = O.dequantize_layer(codes, scales, zeros, g_idx)
    d = np.asarray(W0, np.float64) - deq
    return float(np.sum((d @ H0) * d))


def test_fullsize_hessian_sampled_entries(full):
    X = full["X"]
    S = host(full["S"])
    rng = np.random.default_rng(7)
    n_in = X.shape[0]
    ii = rng.integers(0, n_in, PAIRS)
    jj = rng.integers(0, n_in, PAIRS)
    lo, hi = np.minimum(ii, jj), np.maximum(ii, jj)
    worst = 0.0
    for i, j in zip(lo, hi):
        xi = X[i].astype(np.float64)
        xj = X[j].astype(np.float64)
        exact = float(xi @ xj)
        scale = float(np.sqrt((xi @ xi) * (xj @ xj)))
        worst = max(worst, abs(float(S[i, j]) - exact) / scale)
    assert worst < 5e-5, worst
    assert full["n"] == X.shape[1]


def test_fullsize_natural_order(lib, full):
    q = WL.quant[0]
    g = _gpu_solve(lib, full, q)
    rows = np.random.default_rng(11).choice(full["layer"].out, ROWS, replace=False)
    prep, res, codes = _oracle_rows(full, q, rows)
    assert np.array_equal(g["perm"], np.arange(len(g["perm"])))
    assert np.array_equal(g["dead"].astype(bool), prep["dead"])
    # U against the oracle's own U
    U_gpu = g["U"].T  # column-major storage: U_gpu[i, j] = element (i, j)
    rel = np.linalg.norm(U_gpu - prep["U"]) / np.linalg.norm(prep["U"])
    assert rel < 1e-3, rel
    # codes, scales and zeros of the sampled rows
    rate, eq = code_report(g["codes"][rows], codes)
    assert rate >= 0.999, rate
    compare_groups(g["scales"][rows], g["zeros"][rows], res["scales"], res["zeros"],
                   eq[:, prep["perm"]], q.group_size)
    H0 = prep["H0"]
    e_gpu = _row_error(full["W"][rows], g["codes"][rows], g["scales"][rows], g["zeros"][rows],
                       g["g_idx"], H0)
    e_ref = _row_error(full["W"][rows], codes, res["scales"], res["zeros"],
                       O.g_index(prep["perm"], q.group_size), H0)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref, (e_gpu, e_ref)


@pytest.mark.parametrize("qi", [0, 1, 2])
def test_fullsize_act_order(lib, full, qi):
    q = WL_ACT.quant[qi]
    g = _gpu_solve(lib, full, q)
    n_in = full["layer"].in_
    # the permutation: valid, and non-increasing in the exact diagonal up to
    # the Hessian tolerance
    perm = g["perm"]
    assert np.array_equal(np.sort(perm), np.arange(n_in))
    d = np.diag(full["S64"])[perm]
    assert np.all(d[1:] <= d[:-1] * (1 + 1e-4) + 1e-12)
    rows = np.random.default_rng(13 + qi).choice(full["layer"].out, ROWS, replace=False)
    prep, res, codes = _oracle_rows(full, q, rows)
    maxq = 2 ** q.bits - 1
    assert g["codes"].min() >= 0 and g["codes"].max() <= maxq
    # g_idx: original column perm[p] belongs to processing group p // group_size
    assert np.array_equal(g["g_idx"][perm], np.arange(n_in) // q.group_size)
    # the quantisation error of the sampled rows matches the oracle's
    H0 = prep["H0"]
    e_gpu = _row_error(full["W"][rows], g["codes"][rows], g["scales"][rows], g["zeros"][rows],
                       g["g_idx"], H0)
    e_ref = _row_error(full["W"][rows], codes, res["scales"], res["zeros"],
                       O.g_index(prep["perm"], q.group_size), H0)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref, (e_gpu, e_ref)
    # where both sides chose the same order, the codes agree
    if np.array_equal(perm, prep["perm"]):
        rate, _ = code_report(g["codes"][rows], codes)
        assert rate >= 0.999, rate


def _solve_layer_case(lib, wl, layer, q, tokens, rows=None):
    """GPU solve (the bench's call sequence) and the float64 oracle from the
    same seeded inputs; the oracle sweeps ``rows`` (all when None)."""
    import torch
    W = gen.weight(wl, layer)
    X = gen.x_full(wl, layer.site, tokens=tokens)
    Xd = torch.from_numpy(X).cuda()
    S = torch.zeros((layer.in_, layer.in_), dtype=torch.float32, device="cuda")
    n = lib.gptq_hessian_accumulate(S, Xd, 0)
    del Xd
    full = dict(W=W, X=X, S=S, n=n, layer=layer)
    g = _gpu_solve(lib, full, q)
    S64 = np.zeros((layer.in_, layer.in_), dtype=np.float64)
    for c0 in range(0, X.shape[1], 8192):
        O.hessian_accumulate(S64, X[:, c0:c0 + 8192])
    full["S64"] = S64
    if rows is None:
        rows = np.arange(layer.out)
    prep, res, codes = _oracle_rows(full, q, rows)
    return full, g, prep, res, codes, rows


def test_correlated_channels_all_rows(lib):
    """q_proj shape with strongly correlated channels (X = s (z + P y), rank
    16): the case where error compensation changes most codes relative to
    rounding.  Every row is compared."""
    wl = gen.WORKLOADS["q_proj_correlated"]
    layer, q = wl.layers[0], wl.quant[0]
    full, g, prep, res, codes, rows = _solve_layer_case(lib, wl, layer, q, wl.tokens)
    if np.array_equal(g["perm"], prep["perm"]):
        rate, eq = code_report(g["codes"], codes)
        assert rate >= 0.999, rate
        compare_groups(g["scales"], g["zeros"], res["scales"], res["zeros"],
                       eq[:, prep["perm"]], q.group_size)
    H0 = prep["H0"]
    e_gpu = _row_error(full["W"], g["codes"], g["scales"], g["zeros"], g["g_idx"], H0)
    e_ref = _row_error(full["W"], codes, res["scales"], res["zeros"],
                       O.g_index(prep["perm"], q.group_size), H0)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref, (e_gpu, e_ref)
    # compensation matters here: GPTQ beats round-to-nearest clearly
    r_codes, r_scales, r_zeros = O.rtn(np.asarray(full["W"], np.float64), q.bits, q.group_size,
                                       q.sym, prep["perm"])
    e_rtn = _row_error(full["W"], r_codes, r_scales, r_zeros, O.g_index(prep["perm"], q.group_size), H0)
    assert e_gpu < 0.9 * e_rtn, (e_gpu, e_rtn)


def test_mlp_down_proj_11008_wide(lib):
    """Llama-7B down_proj shape: 11008 input channels (SiLU-gated
    activations), 3-bit symmetric, group 128, act-order.  The layer shape is
    the benchmark's; the calibration set is cut to 32768 tokens so that the
    float64 oracle's Hessian (11008^2 x tokens) stays within a test's time."""
    wl = gen.WORKLOADS["llama7b_mlp"]
    layer, q = wl.layer("down_proj"), wl.quant[0]
    rows = np.random.default_rng(17).choice(layer.out, ROWS, replace=False)
    full, g, prep, res, codes, rows = _solve_layer_case(lib, wl, layer, q, 32768, rows)
    n_in = layer.in_
    perm = g["perm"]
    assert np.array_equal(np.sort(perm), np.arange(n_in))
    d = np.diag(full["S64"])[perm]
    assert np.all(d[1:] <= d[:-1] * (1 + 1e-4) + 1e-12)
    if np.array_equal(perm, prep["perm"]):
        U_gpu = g["U"].T
        rel = np.linalg.norm(U_gpu - prep["U"]) / np.linalg.norm(prep["U"])
        assert rel < 1e-3, rel
        rate, _ = code_report(g["codes"][rows], codes)
        assert rate >= 0.999, rate
    maxq = 2 ** q.bits - 1
    assert g["codes"].min() >= 0 and g["codes"].max() <= maxq
    H0 = prep["H0"]
    e_gpu = _row_error(full["W"][rows], g["codes"][rows], g["scales"][rows], g["zeros"][rows],
                       g["g_idx"], H0)
    e_ref = _row_error(full["W"][rows], codes, res["scales"], res["zeros"],
                       O.g_index(prep["perm"], q.group_size), H0)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref, (e_gpu, e_ref)
