"""Property checks of the oracle's integer and packing steps over many random
shapes and values (hypothesis), beyond the fixed cases of the pins."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

BITS = st.sampled_from([2, 3, 4, 8])


@settings(max_examples=60, deadline=None)
@given(bits=BITS, rows=st.integers(1, 6), words=st.integers(1, 4), seed=st.integers(0, 2**31 - 1))
def test_pack_unpack_roundtrip_any_shape(bits, rows, words, seed):
    # n codes fill whole words: 32 * words / bits when bits divides it,
    # otherwise (3 bits) 32 * words codes fill 3 * words words
    n = 32 * words // bits if (32 * words) % bits == 0 else 32 * words
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** bits, (rows, n))
    words_ = O.pack_rows(codes, bits)
    assert words_.shape == (rows, n * bits // 32)
    assert np.array_equal(O.unpack_rows(words_, bits, n), codes)


@settings(max_examples=60, deadline=None)
@given(bits=BITS, out_w=st.integers(1, 3), in_w=st.integers(1, 3), ng=st.integers(1, 4),
       off=st.sampled_from([0, 1]), seed=st.integers(0, 2**31 - 1))
def test_checkpoint_layout_is_the_transposed_packing(bits, out_w, in_w, ng, off, seed):
    out, in_ = 32 * out_w, 32 * in_w          # any bits: out * bits and in * bits are word multiples
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** bits, (out, in_))
    zeros = rng.integers(0, 2 ** bits, (out, ng))
    scales = rng.random((out, ng)).astype(np.float32)
    r = O.checkpoint_layout(codes, scales, zeros, np.zeros(in_), bits, off)
    assert np.array_equal(r["qweight"].T, O.pack_rows(codes, bits))
    assert np.array_equal(O.unpack_rows(r["qzeros"], bits, out), (zeros.T - off) % 2 ** bits)
    assert np.array_equal(r["scales"], scales.T.astype(np.float16))


@settings(max_examples=80, deadline=None)
@given(bits=BITS, sym=st.booleans(), seed=st.integers(0, 2**31 - 1), width=st.integers(1, 64),
       scale=st.sampled_from([1e-4, 0.02, 1.0, 300.0]))
def test_codes_in_range_and_on_the_grid(bits, sym, seed, width, scale):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((5, width)) * scale
    s, z = O.group_params(w, bits, sym)
    maxq = 2 ** bits - 1
    assert np.all(s > 0) and np.all((z >= 0) & (z <= maxq))
    q = np.stack([O.quantize_codes(w[:, j], s, z, bits) for j in range(width)], 1)
    assert np.all((q >= 0) & (q <= maxq))
    deq = np.stack([O.dequantize_codes(q[:, j], s, z) for j in range(width)], 1)
    k = deq / s.astype(np.float64)[:, None] + z[:, None]
    np.testing.assert_allclose(k, np.rint(k), atol=1e-6)
    if not sym:
        # the asymmetric grid s (k - z), k = 0..maxq, spans the group's range
        # [min(0, min w), max(0, max w)] to within half a step at each end
        lo = np.minimum(w.min(1), 0)
        hi = np.maximum(w.max(1), 0)
        step = s.astype(np.float64)
        g_lo = step * (0 - z)
        g_hi = step * (maxq - z)
        assert np.all(g_lo <= lo + 0.5 * step * (1 + 1e-5))
        assert np.all(g_hi >= hi - 0.5 * step * (1 + 1e-5))


@settings(max_examples=40, deadline=None)
@given(n=st.integers(1, 40), gs=st.sampled_from([1, 2, 4, 8, -1]), seed=st.integers(0, 2**31 - 1))
def test_g_index_counts_group_members(n, gs, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n)
    g = O.g_index(perm, gs)
    if gs == -1:
        assert np.all(g == 0)
        return
    # the column processed at position p belongs to group p // gs
    assert np.array_equal(g[perm], np.arange(n) // gs)
    counts = np.bincount(g)
    assert np.all(counts[:-1] == gs) and 1 <= counts[-1] <= gs
