"""Pins for the CPU oracle: it is checked against what the pages and the
mathematics fix -- closed forms, brute force on tiny layers, invariances and a
hand-worked example -- never against itself."""
import json
import os

import numpy as np
import pytest

import gen
import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _spd(rng, n, cond_mix=1.0):
    a = rng.standard_normal((n, n))
    return a @ a.T * cond_mix + n * np.eye(n)


# ------------------------------------------------------------- worked example
def test_hand_worked_example():
    g = _load("hand_worked_2bit.json")
    i, e = g["inputs"], g["expected"]
    W = np.array(i["W"])
    S = np.array(i["S"])
    r = O.gptq_layer(W, S, i["n"], bits=i["bits"], group_size=i["group_size"],
                     sym=i["sym"], desc_act=i["desc_act"],
                     damp_percent=i["damp_percent"])
    assert r["codes"].tolist() == e["codes"]
    np.testing.assert_allclose(r["scales"], e["scales"], rtol=1e-7)
    assert r["zeros"].tolist() == e["zeros"]
    np.testing.assert_allclose(r["U"], e["U"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["loss"], e["loss"], rtol=1e-5)
    deq = O.dequantize_layer(r["codes"], r["scales"], r["zeros"], r["g_idx"])
    err, _ = O.layer_error(W, deq, r["H0"], i["n"])
    assert err == pytest.approx(e["layer_error"], rel=1e-5)
    codes, s, z = O.rtn(W, i["bits"], i["group_size"], i["sym"])
    assert codes.tolist() == e["rtn_codes"]
    err_rtn, _ = O.layer_error(W, O.dequantize_layer(codes, s, z, r["g_idx"]),
                               r["H0"], i["n"])
    assert err_rtn == pytest.approx(e["rtn_layer_error"], rel=1e-5)


def test_pages_figures():
    g = _load("pages_figures.json")
    ex = g["group_count_example"]
    out, nin = ex["shape"]
    W = np.zeros((out, nin), np.float32)
    # one scale and one zero per group of group_size weights
    codes, s, z = O.rtn(W[:, :ex["group_size"] * 2], 4, ex["group_size"], False)
    assert s.shape == (out, 2)
    assert out * (nin // ex["group_size"]) == ex["groups"]
    m = g["memory_reduction_4bit"]
    words = O.pack_rows(np.zeros((4, 4096), np.int64), m["bits"])
    assert words.nbytes * m["packed_ratio_vs_fp16"] == 4 * 4096 * m["fp16_bytes_per_weight"]
    for b in g["bit_widths"]["bits"]:
        assert O.maxq_of(b) == 2 ** b - 1
    with pytest.raises(ValueError):
        O.maxq_of(5)


# ------------------------------------------------------------- step 1: Hessian
def test_hessian_explicit_loop_and_chunking():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((6, 40)).astype(np.float32)
    S, n = O.hessian([X[:, :13], X[:, 13:29], X[:, 29:]])
    assert n == 40
    ref = np.zeros((6, 6))
    for t in range(40):
        x = X[:, t].astype(np.float64)
        for a in range(6):
            for b in range(6):
                ref[a, b] += x[a] * x[b]
    np.testing.assert_allclose(S, ref, rtol=1e-13, atol=1e-13)
    S1, _ = O.hessian([X])
    np.testing.assert_allclose(S, S1, rtol=1e-13, atol=1e-12)
    assert np.array_equal(S, S.T)
    assert np.linalg.eigvalsh(S).min() > -1e-10


def test_hessian_resume_equals_one_pass():
    """(S, n) is additive: accumulating chunks 0-1, then 2-3, equals one pass."""
    wl = gen.WORKLOADS["layer256_fp32"]
    x = gen.x_full(wl, "x", threads=1)
    a, na = O.hessian([x[:, :256], x[:, 256:512]])
    b, nb = O.hessian([x[:, 512:768], x[:, 768:]])
    full, nf = O.hessian([x])
    np.testing.assert_allclose(a + b, full, rtol=1e-12, atol=1e-9)
    assert na + nb == nf


def test_normalize_and_layer_error_identity():
    """||(W - Q) X||^2 equals (n/2) delta H0 delta^T with H0 = 2 X X^T / n."""
    rng = np.random.default_rng(1)
    X = rng.standard_normal((7, 30))
    W = rng.standard_normal((3, 7))
    Q = W + 0.01 * rng.standard_normal((3, 7))
    S, n = O.hessian([X])
    H0 = O.normalize_hessian(S, n)
    np.testing.assert_allclose(H0, 2 * X @ X.T / 30, rtol=1e-14)
    e, rel = O.layer_error(W, Q, H0, n)
    direct = np.sum(((W - Q) @ X) ** 2)
    assert e == pytest.approx(direct, rel=1e-12)
    assert rel == pytest.approx(direct / np.sum((W @ X) ** 2), rel=1e-12)


# ------------------------------------------------------------- step 2: damp, dead
def test_dampen_definition():
    H = np.diag([1.0, 3.0, 8.0]) + 0.1
    D = O.dampen(H, 0.05)
    lam = 0.05 * np.mean(np.diag(H))
    np.testing.assert_allclose(np.diag(D) - np.diag(H), lam)
    off = ~np.eye(3, dtype=bool)
    assert np.array_equal(D[off], H[off])
    with pytest.raises(ValueError):
        O.dampen(H, -0.1)


def test_dead_channels():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((8, 64))
    X[[2, 5]] = 0.0
    W = rng.standard_normal((4, 8))
    S, n = O.hessian([X])
    r = O.gptq_layer(W, S, n, bits=4, group_size=4, damp_percent=0.01)
    assert r["dead"].tolist() == [False, False, True, False, False, True, False, False]
    # dead columns: weight zeroed, no compensation into or out of them
    U = r["U"]
    for c in (2, 5):
        assert np.all(U[c, np.arange(8) != c] == 0) and np.all(U[np.arange(8) != c, c] == 0)
        deq = O.dequantize_layer(r["codes"], r["scales"], r["zeros"], r["g_idx"])
        assert np.all(deq[:, c] == 0)


def test_fix_dead_sets_unit_diagonal_before_dampening():
    """A channel with H_ii = 0 gets H_ii = 1 and nothing else changes; with no
    dampening the fixed Hessian still has a Cholesky factor, and the damping
    mean counts the fixed 1."""
    H = np.array([[2.0, 0.0, 0.5],
                  [0.0, 0.0, 0.0],
                  [0.5, 0.0, 3.0]])
    F, dead = O.fix_dead(H)
    assert dead.tolist() == [False, True, False]
    assert F[1, 1] == 1.0
    keep = np.ones_like(H, dtype=bool)
    keep[1, 1] = False
    assert np.array_equal(F[keep], H[keep])
    O.upper_cholesky_of_inverse(O.dampen(F, 0.0))   # positive definite
    # lambda = 0.3 * mean(2, 1, 3) = 0.6 (the fixed diagonal counts)
    np.testing.assert_allclose(np.diag(O.dampen(F, 0.3)), [2.6, 1.6, 3.6])
    S = H * 5.0
    r = O.prepare(S, 10, 0.0, False)     # H0 = 2 S / 10 = H
    assert r["dead"].tolist() == [False, True, False] and r["Hp"][1, 1] == 1.0


# ------------------------------------------------------------- step 3: act order
def test_act_order_is_stable_descending_permutation():
    d = np.array([3.0, 1.0, 3.0, 7.0, 1.0, 0.5, 7.0])
    p = O.act_order(d, True)
    assert sorted(p.tolist()) == list(range(7))
    assert p.tolist() == [3, 6, 0, 2, 1, 4, 5]          # ties keep column order
    assert np.all(np.diff(d[p]) <= 0)
    assert O.act_order(d, False).tolist() == list(range(7))


def test_act_order_on_sorted_diagonal_equals_natural_order():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((16, 64)) * np.linspace(3, 1, 16)[:, None]
    S, n = O.hessian([X])
    order = np.argsort(-np.diag(S), kind="stable")
    S = S[np.ix_(order, order)]                          # diagonal now descending
    W = rng.standard_normal((5, 16))
    a = O.gptq_layer(W, S, n, bits=3, group_size=8, desc_act=True)
    b = O.gptq_layer(W, S, n, bits=3, group_size=8, desc_act=False)
    assert a["perm"].tolist() == list(range(16))
    for k in ("codes", "scales", "zeros", "g_idx"):
        assert np.array_equal(a[k], b[k])


def test_g_idx_maps_columns_to_processing_groups():
    perm = np.array([4, 0, 5, 1, 3, 2, 7, 6])
    g = O.g_index(perm, 2)
    # processing position of column c: invperm[c]
    assert g.tolist() == [0, 1, 2, 2, 0, 1, 3, 3]
    assert O.g_index(perm, -1).tolist() == [0] * 8


# ------------------------------------------------------------- step 4: U
def test_upper_cholesky_of_inverse_closed_form_2x2():
    for a, b, c in [(2.0, 1.0, 2.0), (5.0, -1.5, 0.7), (1.0, 0.9, 1.0)]:
        H = np.array([[a, b], [b, c]])
        det = a * c - b * b
        U = O.upper_cholesky_of_inverse(H)
        ref = np.array([[np.sqrt(c / det), -b / np.sqrt(c * det)],
                        [0.0, 1.0 / np.sqrt(c)]])
        np.testing.assert_allclose(U, ref, rtol=1e-12, atol=1e-14)


def test_upper_cholesky_of_inverse_properties():
    rng = np.random.default_rng(4)
    H = _spd(rng, 12)
    U = O.upper_cholesky_of_inverse(H)
    assert np.all(np.tril(U, -1) == 0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ H, np.eye(12), atol=1e-10)
    # last diagonal entry depends on H's last diagonal entry only
    assert U[-1, -1] == pytest.approx(1 / np.sqrt(H[-1, -1]), rel=1e-12)
    assert U[0, 0] == pytest.approx(np.sqrt(np.linalg.inv(H)[0, 0]), rel=1e-12)


def test_not_positive_definite_is_reported():
    S = np.array([[1.0, 2.0], [2.0, 1.0]])       # indefinite
    with pytest.raises(O.NotPositiveDefinite):
        O.gptq_layer(np.ones((1, 2)), S, 2, bits=4, group_size=-1)


# ------------------------------------------------------------- quantizer
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_quantizer_range_and_grid(bits, sym):
    rng = np.random.default_rng(bits * 10 + sym)
    w = rng.standard_normal((50, 16)) * 0.02
    w[3] = 0.0                                     # an all-zero group
    w[4] = np.abs(w[4])                            # one-signed groups
    w[5] = -np.abs(w[5])
    s, z = O.group_params(w, bits, sym)
    maxq = 2 ** bits - 1
    assert s.dtype == np.float32 and np.all(s > 0)
    assert np.all((z >= 0) & (z <= maxq))
    q = np.stack([O.quantize_codes(w[:, j], s, z, bits) for j in range(16)], 1)
    assert np.all((q >= 0) & (q <= maxq))
    deq = np.stack([O.dequantize_codes(q[:, j], s, z) for j in range(16)], 1)
    # dequantized values sit on each group's grid s * (k - z)
    k = deq / s.astype(np.float64)[:, None] + z[:, None]
    np.testing.assert_allclose(k, np.rint(k), atol=1e-9)
    # within range the rounding error is at most half a step
    inside = (q > 0) & (q < maxq)
    assert np.all(np.abs(w - deq)[inside] <= 0.5 * s.astype(np.float64)[:, None].repeat(16, 1)[inside] * (1 + 1e-6))
    if sym:
        assert np.all(z == (maxq + 1) // 2)
        # the grid spans [-max|w|, max|w|]: scale = 2 max|w| / maxq
        a_ = np.max(np.abs(w.astype(np.float32)), axis=1)
        a_[a_ == 0] = 1
        assert np.array_equal(s, (np.float32(2) * a_) / np.float32(maxq))
    else:
        # zero is exactly representable
        zq = O.quantize_codes(np.zeros(50), s, z, bits)
        assert np.all(O.dequantize_codes(zq, s, z) == 0)
        # asym range covers [min, max] of the group
        assert np.all(deq.min(1) <= w.min(1) + 0.5 * s + 1e-12)


def test_quantizer_hand_values():
    """Worked by hand.  sym, 4 bits, w = (0.3, -0.6, 0.1): max|w| = 0.6,
    scale = 1.2 / 15 = 0.08, zero = 8; w / scale = 3.75, -7.5, 1.25 round
    (half to even) to 4, -8, 1, so the codes are 12, 0, 9.  asym, 2 bits,
    w = (-0.2, 0.1, 0.4): range [-0.2, 0.4], scale = 0.6 / 3 = 0.2, zero =
    rint(0.2 / 0.2) = 1; w / scale = -1, 0.5, 2 round to -1, 0, 2, so the
    codes are 0, 1, 3."""
    w = np.array([[0.3, -0.6, 0.1]])
    s, z = O.group_params(w, 4, True)
    np.testing.assert_allclose(s, [0.08], rtol=1e-6)
    assert z.tolist() == [8]
    q = [O.quantize_codes(w[:, j], s, z, 4)[0] for j in range(3)]
    assert q == [12, 0, 9]
    w = np.array([[-0.2, 0.1, 0.4]])
    s, z = O.group_params(w, 2, False)
    np.testing.assert_allclose(s, [0.2], rtol=1e-6)
    assert z.tolist() == [1]
    assert [O.quantize_codes(w[:, j], s, z, 2)[0] for j in range(3)] == [0, 1, 3]


# ------------------------------------------------------------- step 5: sweep
def test_diagonal_hessian_equals_rtn_exactly():
    rng = np.random.default_rng(5)
    for bits in (2, 3, 4, 8):
        for gs, sym, da in [(4, False, False), (8, True, True), (-1, False, True), (16, True, False)]:
            W = rng.standard_normal((9, 16)) * 0.02
            S = np.diag(rng.uniform(0.5, 5.0, 16))
            r = O.gptq_layer(W, S, 32, bits=bits, group_size=gs, sym=sym,
                             desc_act=da, damp_percent=0.01)
            codes, s, z = O.rtn(W, bits, gs, sym, perm=r["perm"])
            assert np.array_equal(r["codes"], codes)
            assert np.array_equal(r["scales"], s)
            assert np.array_equal(r["zeros"], z)


def test_blocked_equals_unblocked():
    rng = np.random.default_rng(6)
    A = rng.standard_normal((64, 64))
    H = A @ A.T / 64 + 0.1 * np.eye(64)
    U = O.upper_cholesky_of_inverse(H)
    W = rng.standard_normal((12, 64)) * 0.02
    ref = O.sweep_unblocked(W, U, 3, 16, False)
    for B in (1, 5, 16, 32, 48, 64, 128):
        r = O.sweep_blocked(W, U, 3, 16, False, B)
        assert np.array_equal(r["codes"], ref["codes"]), B
        assert np.array_equal(r["zeros"], ref["zeros"])
        np.testing.assert_allclose(r["scales"], ref["scales"], rtol=1e-6)
        np.testing.assert_allclose(r["err"], ref["err"], rtol=1e-9, atol=1e-13)


def test_loss_equals_damped_quadratic_error():
    """sum_j e_j^2 = delta H delta^T (delta = W - deq, damped H, processing
    order): the update rule makes delta = E U, and U H U^T = I."""
    rng = np.random.default_rng(7)
    X = rng.standard_normal((24, 24)) @ rng.standard_normal((24, 100))
    W = rng.standard_normal((6, 24)) * 0.02
    S, n = O.hessian([X])
    r = O.gptq_layer(W, S, n, bits=4, group_size=8, desc_act=True)
    Wp = W[:, r["perm"]]
    s = r["scales"][:, np.arange(24) // 8]
    z = r["zeros"][:, np.arange(24) // 8]
    d = Wp - s.astype(np.float64) * (r["codes_p"] - z)
    quad = np.einsum("ri,ij,rj->r", d, r["Hp"], d)
    np.testing.assert_allclose(r["loss"], quad, rtol=1e-9)
    np.testing.assert_allclose(d, r["err_p"] @ r["U"], rtol=1e-9, atol=1e-14)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("gs", [4, 8, -1])
def test_brute_force_tiny(seed, gs):
    W, X = gen.correlated_tiny(seed, 7, 8)
    W *= 0.02
    S, n = O.hessian([X])
    for bits, sym in ((2, False), (3, True), (4, False)):
        r = O.gptq_layer(W, S, n, bits=bits, group_size=gs, sym=sym,
                         desc_act=(seed % 2 == 1), damp_percent=0.01)
        codes, s, z, deq = O.brute_force_sweep(W[:, r["perm"]], r["Hp"], bits, gs, sym)
        assert np.array_equal(r["codes_p"], codes)
        assert np.array_equal(r["zeros"], z)
        np.testing.assert_allclose(r["scales"], s, rtol=1e-6)
        e_or, _ = O.layer_error(W, O.dequantize_layer(r["codes"], r["scales"], r["zeros"], r["g_idx"]), r["H0"], n)
        e_bf, _ = O.layer_error(W[:, r["perm"]], deq, r["H0"][np.ix_(r["perm"], r["perm"])], n)
        assert e_or == pytest.approx(e_bf, rel=1e-9)


def test_gptq_beats_rtn_on_correlated_tiny_layers():
    for bits in (2, 3, 4):
        for gs in (4, 8, -1):
            wins = 0
            for seed in range(200):
                W, X = gen.correlated_tiny(seed, 16, 8)
                W *= 0.02
                S, n = O.hessian([X])
                r = O.gptq_layer(W, S, n, bits=bits, group_size=gs)
                deq = O.dequantize_layer(r["codes"], r["scales"], r["zeros"], r["g_idx"])
                e_g, _ = O.layer_error(W, deq, r["H0"], n)
                c, s, z = O.rtn(W, bits, gs, False)
                e_r, _ = O.layer_error(W, O.dequantize_layer(c, s, z, r["g_idx"]), r["H0"], n)
                wins += e_g <= e_r * (1 + 1e-12)
            assert wins >= 190, (bits, gs, wins)


# ------------------------------------------------------------- invariances
def _small_layer(seed, out=10, nin=32, tokens=80):
    W, X = gen.small_case(seed, out, nin, tokens, sigma=1.0)
    X = X.astype(np.float64)
    mix = np.random.default_rng(seed).standard_normal((nin, nin)) * 0.3 + np.eye(nin)
    S, n = O.hessian([mix @ X])
    return W.astype(np.float64), S, n


def test_power_of_two_scaling_of_S_is_bitwise_invariant():
    W, S, n = _small_layer(11)
    for da in (False, True):
        a = O.gptq_layer(W, S, n, bits=3, group_size=8, desc_act=da)
        b = O.gptq_layer(W, 4.0 * S, n, bits=3, group_size=8, desc_act=da)
        for k in ("codes", "scales", "zeros", "g_idx", "perm"):
            assert np.array_equal(a[k], b[k]), k


def test_row_permutation_equivariance():
    W, S, n = _small_layer(12)
    p = np.random.default_rng(0).permutation(W.shape[0])
    a = O.gptq_layer(W, S, n, bits=4, group_size=8, desc_act=True)
    b = O.gptq_layer(W[p], S, n, bits=4, group_size=8, desc_act=True)
    assert np.array_equal(a["codes"][p], b["codes"])
    assert np.array_equal(a["scales"][p], b["scales"])
    assert np.array_equal(a["zeros"][p], b["zeros"])


def test_group_size_in_equals_per_row():
    W, S, n = _small_layer(13)
    a = O.gptq_layer(W, S, n, bits=4, group_size=32, desc_act=True)
    b = O.gptq_layer(W, S, n, bits=4, group_size=-1, desc_act=True)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"])
    assert np.all(a["g_idx"] == 0) and np.all(b["g_idx"] == 0)


def test_block_size_near_invariance_on_generated_layer():
    W, S, n = _small_layer(14, out=8, nin=256, tokens=600)
    ref = O.gptq_layer(W, S, n, bits=4, group_size=64, desc_act=True, blocked=False)
    for B in (16, 32, 64, 128, 256):
        r = O.gptq_layer(W, S, n, bits=4, group_size=64, desc_act=True, block_size=B)
        assert np.array_equal(r["codes"], ref["codes"]), B


# ------------------------------------------------------------- packing
def test_pack_known_answers():
    assert O.pack_rows(np.array([list(range(8))]), 4).tolist() == [[0x76543210]]
    assert O.pack_rows(np.array([[1, 2, 3, 4]]), 8).tolist() == [[0x04030201]]
    assert O.pack_rows(np.array([[3] + [0] * 15]), 2).tolist() == [[0x3]]
    assert O.pack_rows(np.array([[7] * 32]), 3).tolist() == [[0xFFFFFFFF] * 3]
    # 3-bit field 10 sits at bits 30..32 and straddles words 0 and 1:
    # 5 = 0b101 -> bit 30 set in word 0, bit 0 set in word 1
    c = np.zeros((1, 32), np.int64)
    c[0, 10] = 5
    assert O.pack_rows(c, 3).tolist() == [[0x40000000, 0x00000001, 0]]
    c = np.zeros((1, 32), np.int64)
    c[0, 21] = 6                      # bits 63..65: 0b110 -> bit 63 clear, bits 64,65 set
    assert O.pack_rows(c, 3).tolist() == [[0, 0, 0x3]]
    c[0, 21] = 1                      # bit 63 = word 1 bit 31
    assert O.pack_rows(c, 3).tolist() == [[0, 0x80000000, 0]]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip(bits):
    rng = np.random.default_rng(bits)
    c = rng.integers(0, 2 ** bits, (5, 96))
    assert np.array_equal(O.unpack_rows(O.pack_rows(c, bits), bits, 96), c)
    with pytest.raises(ValueError):
        O.pack_rows(c + 2 ** bits, bits)
