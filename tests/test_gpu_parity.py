"""GPU parity: every ABI call against the CPU oracle on the same seeded inputs.

Tolerances (from the method's specification): Hessian within 1e-3 relative
Frobenius; perm, dead, g_idx and bit packing exact; codes >= 99.9 % identical;
scales within 1e-4 relative and zeros equal on groups not preceded by a code
mismatch in their row; layer reconstruction error within 1 % of the oracle's.
Where the oracle's and the GPU's floating-point inputs to an integer decision
are identical (diagonal Hessian: no compensation), codes must match exactly.
"""
import os

import numpy as np
import pytest

import gen
import oracle as O
from gpu_util import code_report, compare_groups, dev, exact_values, host, rel_fro

pytestmark = pytest.mark.gpu


def _cfg(lib, **kw):
    return lib.GptqConfig(**kw)


def _S_gpu(lib, X_t, in_):
    import torch
    S = torch.full((in_, in_), -7.0, dtype=torch.float32, device="cuda")
    iu = torch.triu_indices(in_, in_, device="cuda")
    S[iu[0], iu[1]] = 0.0
    n = lib.gptq_hessian_accumulate(S, X_t, 0)
    torch.cuda.synchronize()
    return S, n


# ----------------------------------------------------------------- Hessian
@pytest.mark.parametrize("in_,tokens,dtype,seed", [
    (8, 100, "float16", 1), (72, 1, "float16", 2), (136, 1000, "bfloat16", 3),
    (256, 1024, "float32", 4), (300, 4097, "float16", 5), (1000, 2048, "bfloat16", 6),
    (4096, 2048, "float16", 7), (520, 333, "float32", 8),
])
def test_hessian_accumulate(lib, in_, tokens, dtype, seed):
    _, X32 = gen.small_case(seed, 1, in_, tokens, sigma=1.5, outlier_frac=0.01)
    Xt, X64 = exact_values(X32, dtype)
    S, n = _S_gpu(lib, Xt.cuda(), in_)
    assert n == tokens
    Sg = host(S)
    ref = X64 @ X64.T
    iu = np.triu_indices(in_)
    err = rel_fro(Sg[iu], ref[iu])
    assert err < 1e-3, err
    assert err < 5e-5, err          # fp32 accumulation of exact products, <= 8192 per drain
    il = np.tril_indices(in_, -1)
    assert np.all(Sg[il] == -7.0)   # the strictly lower triangle is untouched


def test_hessian_chunked_equals_one_pass(lib):
    import torch
    in_, t = 520, 3 * 2048
    _, X32 = gen.small_case(11, 1, in_, t, sigma=1.5, outlier_frac=0.01)
    Xt, X64 = exact_values(X32, "float16")
    Xd = Xt.cuda()
    S1 = torch.zeros((in_, in_), dtype=torch.float32, device="cuda")
    n = 0
    for c in range(3):
        n = lib.gptq_hessian_accumulate(S1, Xd[:, c * 2048:(c + 1) * 2048], n)
    S2 = torch.zeros_like(S1)
    n2 = lib.gptq_hessian_accumulate(S2, Xd, 0)
    assert n == n2 == t
    iu = np.triu_indices(in_)
    ref = X64 @ X64.T
    assert rel_fro(host(S1)[iu], ref[iu]) < 5e-5
    assert rel_fro(host(S1)[iu], host(S2)[iu]) < 5e-5
    # repeated calls are bitwise reproducible
    S3 = torch.zeros_like(S1)
    lib.gptq_hessian_accumulate(S3, Xd, 0)
    assert torch.equal(S2, S3)


def test_hessian_strided_and_unaligned_views(lib):
    import torch
    in_, t = 200, 777
    _, X32 = gen.small_case(12, 1, in_, t + 5, sigma=1.0)
    Xt, X64 = exact_values(X32, "float16")
    Xd = Xt.cuda()
    for view, ref_x in ((Xd[:, :t], X64[:, :t]), (Xd[:, 3:3 + t], X64[:, 3:3 + t])):
        S = torch.zeros((in_, in_), dtype=torch.float32, device="cuda")
        lib.gptq_hessian_accumulate(S, view, 0)
        iu = np.triu_indices(in_)
        assert rel_fro(host(S)[iu], (ref_x @ ref_x.T)[iu]) < 1e-5


def test_hessian_zero_tokens_is_noop(lib):
    import torch
    S = torch.ones((16, 16), dtype=torch.float32, device="cuda")
    X = torch.zeros((16, 0), dtype=torch.float16, device="cuda")
    assert lib.gptq_hessian_accumulate(S, X, 5) == 5
    assert torch.all(S == 1)


# ----------------------------------------------------------------- prepare
def _prep_inputs(seed, in_, tokens, kind="scaled_normal", dead=()):
    _, X = gen.small_case(seed, 1, in_, tokens, sigma=1.5, outlier_frac=0.02, kind=kind)
    X = X.astype(np.float64)
    for d in dead:
        X[d] = 0.0
    S = (X @ X.T).astype(np.float32)     # the fp32 S both sides receive
    return S, tokens


def _run_prepare(lib, S32, n, cfg):
    import torch
    in_ = S32.shape[0]
    ws = torch.empty(lib.gptq_workspace_bytes(0, in_, cfg), dtype=torch.uint8, device="cuda")
    U = torch.empty((in_, in_), dtype=torch.float32, device="cuda")
    perm = torch.empty(in_, dtype=torch.int32, device="cuda")
    dead = torch.empty(in_, dtype=torch.uint8, device="cuda")
    lib.gptq_prepare_hinv(dev(S32), n, cfg, U, perm, dead, ws)
    return host(U).T, host(perm), host(dead).astype(bool)   # U stored column-major


@pytest.mark.parametrize("in_,tokens,kind,desc_act,damp", [
    (8, 64, "scaled_normal", True, 0.01), (72, 500, "scaled_normal", False, 0.01),
    (136, 1000, "scaled_normal", True, 0.1), (256, 2048, "correlated", True, 0.01),
    (520, 4096, "scaled_normal", True, 0.01), (1000, 3000, "correlated", False, 0.01),
    # wider than one 4096 super-block: two and three cooperative launches
    # joined by tensor-core panel and trailing updates
    (4500, 6000, "scaled_normal", True, 0.01), (9000, 12000, "scaled_normal", False, 0.01),
])
def test_prepare_hinv(lib, in_, tokens, kind, desc_act, damp):
    S32, n = _prep_inputs(in_ + tokens, in_, tokens, kind, dead=(3, 5) if in_ > 8 else ())
    cfg = _cfg(lib, desc_act=desc_act, damp_percent=damp, group_size=-1)
    U, perm, dead = _run_prepare(lib, S32, n, cfg)
    ref = O.prepare(S32.astype(np.float64), n, damp, desc_act)
    assert np.array_equal(dead, ref["dead"])
    assert np.array_equal(perm, ref["perm"])
    assert np.all(np.tril(U, -1) == 0)
    assert np.all(np.diag(U) > 0)
    err = rel_fro(U, ref["U"])
    # measured on B200: at most 1.2e-6 up to 9000 channels with the damped
    # Hessian's condition number up to 1.7e5 (3xTF32 products, fp32 leaves)
    assert err < 1e-4, err


def test_prepare_reports_not_pd_and_nonfinite(lib):
    S = np.array([[1.0, 2.0], [0.0, 1.0]], np.float32)     # upper triangle of an indefinite H
    S = np.pad(S, ((0, 6), (0, 6)))
    S[np.arange(2, 8), np.arange(2, 8)] = 1.0
    cfg = _cfg(lib, group_size=-1, damp_percent=0.0)
    with pytest.raises(lib.GptqError) as e:
        _run_prepare(lib, S, 2, cfg)
    assert e.value.status == 2
    S2 = np.eye(8, dtype=np.float32)
    S2[1, 4] = np.nan
    with pytest.raises(lib.GptqError) as e:
        _run_prepare(lib, S2, 2, cfg)
    assert e.value.status == 3


# ----------------------------------------------------------------- quantize
def _run_quantize(lib, W_t, Ucm, perm, dead, cfg):
    import torch
    out, in_ = W_t.shape
    ws = torch.empty(lib.gptq_workspace_bytes(out, in_, cfg), dtype=torch.uint8, device="cuda")
    ng = 1 if cfg.group_size == -1 else in_ // cfg.group_size
    scales = torch.empty((out, ng), dtype=torch.float32, device="cuda")
    zeros = torch.empty((out, ng), dtype=torch.int32, device="cuda")
    g_idx = torch.empty(in_, dtype=torch.int32, device="cuda")
    loss = torch.empty(out, dtype=torch.float32, device="cuda")
    codes = torch.empty((out, in_), dtype=torch.int32, device="cuda")
    qweight = None
    if (in_ * cfg.bits) % 32 == 0:
        qweight = torch.empty((out, in_ * cfg.bits // 32), dtype=torch.int32, device="cuda")
    lib.gptq_quantize_layer(W_t, dev(Ucm), dev(perm.astype(np.int32)), dev(dead.astype(np.uint8)),
                            cfg, scales, zeros, g_idx, ws, codes=codes, qweight=qweight, loss=loss)
    r = dict(scales=host(scales), zeros=host(zeros), g_idx=host(g_idx), loss=host(loss),
             codes=host(codes))
    if qweight is not None:
        r["qweight"] = host(qweight).view(np.uint32)
    return r


def _check_quantize(lib, W_t, W64, S32, n, cfg, min_match=0.999):
    ref = O.gptq_layer(W64, S32.astype(np.float64), n, bits=cfg.bits, group_size=cfg.group_size,
                       sym=cfg.sym, desc_act=cfg.desc_act, damp_percent=cfg.damp_percent,
                       block_size=cfg.block_size)
    Ucm = np.ascontiguousarray(ref["U"].T).astype(np.float32)
    g = _run_quantize(lib, W_t, Ucm, ref["perm"], ref["dead"], cfg)
    rate, eq = code_report(g["codes"], ref["codes"])
    assert rate >= min_match, rate
    assert np.array_equal(g["g_idx"], ref["g_idx"])
    eq_p = eq[:, ref["perm"]]
    compare_groups(g["scales"], g["zeros"], ref["scales"], ref["zeros"], eq_p, cfg.group_size)
    maxq = 2 ** cfg.bits - 1
    assert g["codes"].min() >= 0 and g["codes"].max() <= maxq
    if "qweight" in g:
        assert np.array_equal(g["qweight"], O.pack_rows(g["codes"], cfg.bits))
    deq = O.dequantize_layer(g["codes"], g["scales"], g["zeros"], g["g_idx"])
    e_gpu, _ = O.layer_error(W64, deq, ref["H0"], n)
    deq_r = O.dequantize_layer(ref["codes"], ref["scales"], ref["zeros"], ref["g_idx"])
    e_ref, _ = O.layer_error(W64, deq_r, ref["H0"], n)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref + 1e-30, (e_gpu, e_ref)
    clean = eq.all(1)                    # rows whose codes all match
    np.testing.assert_allclose(g["loss"][clean], ref["loss"][clean], rtol=1e-3, atol=1e-12)
    return g, ref


@pytest.mark.parametrize("out,in_,bits,gs,sym,desc_act,wdt", [
    (33, 128, 4, 128, False, False, "float16"),
    (3, 72, 3, 8, True, True, "float32"),
    (64, 256, 2, 64, False, True, "bfloat16"),
    (17, 136, 8, -1, False, True, "float16"),
    (100, 512, 4, 32, False, True, "float16"),
    (40, 384, 3, 128, True, False, "float32"),
    (1, 256, 4, 256, False, True, "float16"),
])
def test_quantize_layer(lib, out, in_, bits, gs, sym, desc_act, wdt):
    S32, n = _prep_inputs(out * 7 + in_, in_, 2 * in_ + 64, "correlated")
    W32, _ = gen.small_case(out + in_, out, in_, 8)
    W_t, W64 = exact_values(W32, wdt)
    cfg = _cfg(lib, bits=bits, group_size=gs, sym=sym, desc_act=desc_act)
    _check_quantize(lib, W_t.cuda(), W64, S32, n, cfg)


def test_diagonal_hessian_gives_round_to_nearest_exactly(lib):
    rng = np.random.default_rng(3)
    for bits, gs, sym, da in [(4, 128, False, False), (3, 64, True, True), (2, 32, False, True),
                              (8, -1, False, False)]:
        in_, out = 256, 48
        S32 = np.diag(rng.uniform(0.5, 8.0, in_)).astype(np.float32)
        W32, _ = gen.small_case(bits * 100 + gs, out, in_, 8)
        W_t, W64 = exact_values(W32, "float16")
        cfg = _cfg(lib, bits=bits, group_size=gs, sym=sym, desc_act=da)
        U, perm, dead = _run_prepare(lib, S32, 64, cfg)
        ref = O.prepare(S32.astype(np.float64), 64, 0.01, da)
        assert np.array_equal(perm, ref["perm"])
        g = _run_quantize(lib, W_t.cuda(), np.ascontiguousarray(U.T), perm, dead, cfg)
        codes, s, z = O.rtn(W64, bits, gs, sym, perm=ref["perm"])
        assert np.array_equal(g["codes"], codes)
        assert np.array_equal(g["scales"], s)
        assert np.array_equal(g["zeros"], z)


def test_divide_free_quotient_matches_ieee_division(lib):
    """The sweep's x / scale without a divide (reciprocal and two fma
    corrections) against CUDA's IEEE division, bit for bit, on 2^30 pairs,
    three quarters of them next to a half-integer quotient."""
    n = 1 << 30
    checked, bad = lib.gptq_selftest_quotient(n, seed=20261203)
    assert checked > 0.9 * n, checked
    assert bad == 0, bad


@pytest.mark.parametrize("gs,sym", [(128, False), (32, True), (-1, False)])
def test_tiny_weights_take_the_divide_and_scale_exactly(lib, gs, sym):
    """Weights scaled by 2^-70 put every x / scale outside the divide-free
    quotient's range, so every sub-block is replayed with the divide.  A
    power-of-two scale is exact in fp32 and leaves every quotient as it was:
    codes and zeros must equal the unscaled layer's, scales be 2^-70 times
    theirs, and both match the oracle."""
    import torch
    S32, n = _prep_inputs(95, 384, 900, "correlated")
    W32, _ = gen.small_case(96, 130, 384, 8)
    W_t, W64 = exact_values(W32, "float32")
    cfg = _cfg(lib, bits=4, group_size=gs, sym=sym, desc_act=True)
    g1, ref = _check_quantize(lib, W_t.cuda(), W64, S32, n, cfg)
    tiny = 2.0 ** -70
    Wt2 = (W_t * tiny).contiguous()
    Ucm = np.ascontiguousarray(ref["U"].T).astype(np.float32)
    g2 = _run_quantize(lib, Wt2.cuda(), Ucm, ref["perm"], ref["dead"], cfg)
    g1b = _run_quantize(lib, W_t.cuda(), Ucm, ref["perm"], ref["dead"], cfg)
    assert np.array_equal(g2["codes"], g1b["codes"])
    assert np.array_equal(g2["zeros"], g1b["zeros"])
    assert np.array_equal(g2["scales"], (g1b["scales"].astype(np.float64) * tiny).astype(np.float32))
    assert torch.all(torch.isfinite(torch.from_numpy(g2["loss"])))


def test_block_size_variants_agree(lib):
    S32, n = _prep_inputs(91, 512, 1500, "correlated")
    W32, _ = gen.small_case(92, 64, 512, 8)
    W_t, W64 = exact_values(W32, "float32")
    res = []
    for B in (32, 128, 256, 512):
        cfg = _cfg(lib, bits=4, group_size=32, desc_act=True, block_size=B)
        g, ref = _check_quantize(lib, W_t.cuda(), W64, S32, n, cfg)
        res.append(g["codes"])
    for r in res[1:]:
        assert (r == res[0]).mean() >= 0.999


_SIMT_CHILD = """
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import post_weight_quantization_13_b200 as g
X = torch.from_numpy(np.load(sys.argv[2])).cuda()
S = torch.zeros((X.shape[0], X.shape[0]), dtype=torch.float32, device="cuda")
g.gptq_hessian_accumulate(S, X)
np.save(sys.argv[3], S.cpu().numpy())
"""


def test_tensor_core_and_cuda_core_paths_agree(lib, tmp_path):
    """The Hessian's SYRK on the tensor cores against the same product on the
    CUDA cores.  The library reads GPTQ_FORCE_SIMT once per process, so the
    CUDA-core run happens in a child process started with it set.  Both
    accumulate exact products in fp32 from the same fp16 X: they differ by
    rounding order only, and each stays within the header's 5e-5 bound of
    the exact S."""
    import subprocess
    import sys

    import torch
    rng = np.random.default_rng(93)
    X = (rng.standard_normal((640, 3000)) * 0.5).astype(np.float16)
    S1 = torch.zeros((640, 640), dtype=torch.float32, device="cuda")
    lib.gptq_hessian_accumulate(S1, torch.from_numpy(X).cuda())
    np.save(tmp_path / "X.npy", X)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, GPTQ_FORCE_SIMT="1")
    subprocess.run([sys.executable, "-c", _SIMT_CHILD, root, str(tmp_path / "X.npy"),
                    str(tmp_path / "S.npy")], env=env, check=True, timeout=300)
    S2 = np.load(tmp_path / "S.npy")
    S1 = S1.cpu().numpy()
    assert rel_fro(S1, S2) < 5e-5
    Xd = X.astype(np.float64)
    assert rel_fro(np.triu(S1), np.triu(Xd @ Xd.T)) < 5e-5
    assert rel_fro(np.triu(S2), np.triu(Xd @ Xd.T)) < 5e-5


def test_act_order_exact_on_near_tie_diagonals(lib):
    """Act-order ranks the diagonal the way the oracle does, on the same fp32
    S: channels whose S_ii are one fp32 ulp apart stay in strict order (a
    product with 2/n rounded to fp32 would merge a good share of such pairs
    and fall back to index order), exact ties keep index order, and dead
    channels (S_ii = 0, ranked as H_ii = 1) sit where H_ii = 1 puts them."""
    in_, n = 512, 3
    rng = np.random.default_rng(21)
    base = rng.uniform(0.5, 3.0, in_ // 4).astype(np.float32)
    d = np.empty(in_, np.float32)
    d[0::4] = base
    d[1::4] = np.nextafter(base, np.float32(np.inf))
    d[2::4] = base
    d[3::4] = np.nextafter(base, np.float32(0))
    d[7] = np.float32(1.5)                      # H_ii = 2 * 1.5 / 3: ties with a dead channel's 1
    dead_idx = np.array([3, 100, 257, 400])
    d[dead_idx] = 0.0
    off = np.triu(rng.uniform(-1e-3, 1e-3, (in_, in_)), 1).astype(np.float32)
    S32 = np.diag(d) + off + off.T             # symmetric: the oracle reads both triangles
    S32[dead_idx, :] = 0.0
    S32[:, dead_idx] = 0.0
    for damp in (0.01, 0.0):
        cfg = _cfg(lib, desc_act=True, damp_percent=damp, group_size=-1)
        U, perm, dead = _run_prepare(lib, S32, n, cfg)
        ref = O.prepare(S32.astype(np.float64), n, damp, True)
        assert np.array_equal(dead, ref["dead"])
        assert np.array_equal(perm, ref["perm"])
        assert rel_fro(U, ref["U"]) < 1e-4


def test_group32_damp0005_prepare_and_quantize_at_4096(lib):
    """The agent-skill page's configuration example with group_size 32 and
    damp_percent 0.005, through prepare and quantize on a 4096-wide layer:
    both sides get the same fp32 S, so perm, g_idx and codes compare
    exactly."""
    in_, out, tokens = 4096, 256, 8192
    S32, n = _prep_inputs(77, in_, tokens, "correlated")
    W32, _ = gen.small_case(78, out, in_, 8)
    W_t, W64 = exact_values(W32, "float16")
    cfg = _cfg(lib, bits=4, group_size=32, desc_act=True, damp_percent=0.005)
    U, perm, dead = _run_prepare(lib, S32, n, cfg)
    ref = O.gptq_layer(W64, S32.astype(np.float64), n, bits=4, group_size=32, sym=False,
                       desc_act=True, damp_percent=0.005, block_size=128)
    assert np.array_equal(perm, ref["perm"])
    assert rel_fro(U, ref["U"]) < 1e-3
    g = _run_quantize(lib, W_t.cuda(), np.ascontiguousarray(U.T), perm, dead, cfg)
    rate, eq = code_report(g["codes"], ref["codes"])
    assert rate >= 0.999, rate
    assert np.array_equal(g["g_idx"], ref["g_idx"])
    compare_groups(g["scales"], g["zeros"], ref["scales"], ref["zeros"], eq[:, ref["perm"]], 32)
    assert np.array_equal(g["qweight"], O.pack_rows(g["codes"], 4))
    deq = O.dequantize_layer(g["codes"], g["scales"], g["zeros"], g["g_idx"])
    e_gpu, _ = O.layer_error(W64, deq, ref["H0"], n)
    e_ref, _ = O.layer_error(W64, O.dequantize_layer(ref["codes"], ref["scales"], ref["zeros"],
                                                     ref["g_idx"]), ref["H0"], n)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref, (e_gpu, e_ref)


# ----------------------------------------------------------------- end to end
@pytest.mark.parametrize("name", ["layer256_fp32"])
def test_end_to_end_small_workload(lib, name):
    wl = gen.WORKLOADS[name]
    layer = wl.layers[0]
    W = gen.weight(wl, layer)
    X = gen.x_full(wl, layer.site, threads=1)
    q = wl.quant[0]
    S, n = O.hessian([X])
    ref = O.gptq_layer(W, S, n, **q.as_dict())
    r = lib.solve_layer(dev(W), dev(X), q.as_dict())
    iu = np.triu_indices(layer.in_)
    assert rel_fro(host(r["S"])[iu], S[iu]) < 1e-3
    assert np.array_equal(host(r["perm"]), ref["perm"])
    rate, eq = code_report(host(r["codes"]), ref["codes"])
    assert rate >= 0.999, rate
    compare_groups(host(r["scales"]), host(r["zeros"]), ref["scales"], ref["zeros"],
                   eq[:, ref["perm"]], q.group_size)
    deq = O.dequantize_layer(host(r["codes"]), host(r["scales"]), host(r["zeros"]), host(r["g_idx"]))
    e_gpu, _ = O.layer_error(W, deq, ref["H0"], n)
    e_ref, _ = O.layer_error(W, O.dequantize_layer(ref["codes"], ref["scales"], ref["zeros"],
                                                   ref["g_idx"]), ref["H0"], n)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref
    assert np.array_equal(host(r["qweight"]).view(np.uint32), ref["qweight"]) or rate < 1.0
