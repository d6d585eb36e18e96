"""Pins of the oracle's checkpoint layout (the loaders' transposed packing):
hand-worked words, agreement with the independently written row packer and
unpacker, the zero offset, float16 rounding of the scales, and the layer the
layout describes dequantizing to the same weights."""
import json
import os

import numpy as np
import pytest

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "checkpoint_layout_hand.json")


def _hex(words):
    return [int(w, 16) for w in words]


def _case(c):
    bits = c["bits"]
    if bits == 4:
        out, in_ = 8, 8
        codes = np.array([[(o + j) % 16 for j in range(in_)] for o in range(out)])
        zeros = np.array([[o, 8] for o in range(out)])
    elif bits == 3:
        out, in_ = 32, 32
        codes = np.array([[(o + j) % 8 for j in range(in_)] for o in range(out)])
        zeros = np.array([[o % 8 + 1] for o in range(out)])
    else:
        out, in_ = 16, 16
        codes = 3 * np.eye(out, in_, dtype=np.int64)
        zeros = np.full((out, 1), 2)
    scales = np.ones(zeros.shape, np.float32)
    return O.checkpoint_layout(codes, scales, zeros, np.zeros(in_), bits, c["zero_offset"])


def test_hand_worked_words():
    g = json.load(open(GOLD))
    c4, c3, c2 = g["cases"]
    r = _case(c4)
    assert r["qweight"].shape == (1, 8) and r["qzeros"].shape == (2, 1)
    assert list(r["qweight"][0]) == _hex(c4["qweight_row0"])
    assert [list(x) for x in r["qzeros"]] == [_hex(x) for x in c4["qzeros"]]
    r = _case(c3)
    assert r["qweight"].shape == (3, 32) and r["qzeros"].shape == (1, 3)
    assert list(r["qweight"][:, 0]) == _hex(c3["qweight_col0"])
    assert list(r["qzeros"][0]) == _hex(c3["qzeros_row0"])
    r = _case(c2)
    for o, w in c2["qweight_row0"].items():
        assert r["qweight"][0, int(o)] == int(w, 16)
    assert [list(x) for x in r["qzeros"]] == [_hex(x) for x in c2["qzeros"]]


def test_scales_round_to_nearest_even_float16():
    g = json.load(open(GOLD))["scales_to_float16"]
    n = len(g["values"])
    s = np.ones((8, 1), np.float32)  # out 8 so that the zeros fill one word
    s[:n, 0] = g["values"]
    with np.errstate(over="ignore"):
        r = O.checkpoint_layout(np.zeros((8, 32), np.int64), s, np.zeros((8, 1)), np.zeros(32), 4, 0)
    assert list(r["scales"][0, :n].view(np.uint16)) == _hex(g["bits"])


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_transpose_of_the_row_packing(bits):
    rng = np.random.default_rng(bits)
    out, in_, ng = 64, 96, 3
    codes = rng.integers(0, 2 ** bits, (out, in_))
    zeros = rng.integers(0, 2 ** bits, (out, ng))
    r = O.checkpoint_layout(codes, rng.random((out, ng)), zeros, np.arange(in_) // 32, bits, 1)
    assert r["qweight"].dtype == np.uint32 and r["qweight"].shape == (in_ * bits // 32, out)
    # column o of qweight is row o of the row-major packing
    assert np.array_equal(r["qweight"].T, O.pack_rows(codes, bits))
    assert np.array_equal(O.unpack_rows(r["qweight"].T, bits, in_), codes)
    # qzeros rows unpack to the zeros less one, wrapped into [0, maxq]
    assert r["qzeros"].shape == (ng, out * bits // 32)
    back = O.unpack_rows(r["qzeros"], bits, out)
    assert np.array_equal(back, (zeros.T - 1) % (2 ** bits))
    assert np.array_equal(r["g_idx"], np.arange(in_) // 32) and r["g_idx"].dtype == np.int32


def test_zero_offset_zero_keeps_zeros():
    rng = np.random.default_rng(7)
    zeros = rng.integers(0, 16, (32, 2))
    r = O.checkpoint_layout(np.zeros((32, 8), np.int64), np.ones((32, 2)), zeros, np.zeros(8), 4, 0)
    assert np.array_equal(O.unpack_rows(r["qzeros"], 4, 32), zeros.T)
    with pytest.raises(ValueError):
        O.checkpoint_layout(np.zeros((32, 8), np.int64), np.ones((32, 2)), zeros, np.zeros(8), 4, 2)
    with pytest.raises(ValueError):
        O.checkpoint_layout(np.full((32, 8), 16), np.ones((32, 2)), zeros, np.zeros(8), 4, 0)


def test_layout_dequantizes_to_the_layer():
    """A reader of the layout (unpack along the input dimension, add the
    offset back, float16 scales) recovers the oracle's dequantized layer up
    to the float16 rounding of the scales."""
    rng = np.random.default_rng(11)
    W = rng.standard_normal((32, 128)) * 0.02
    codes, s, z = O.rtn(W, 4, 32, False)
    g_idx = O.g_index(np.arange(128), 32)
    r = O.checkpoint_layout(codes, s, z, g_idx, 4, 1)
    q = O.unpack_rows(r["qweight"].T, 4, 128)
    zr = O.unpack_rows(r["qzeros"], 4, 32).T + 1
    sr = r["scales"].T.astype(np.float64)
    deq = sr[:, g_idx] * (q - zr[:, g_idx])
    ref = O.dequantize_layer(codes, s, z, g_idx)
    assert np.array_equal(q, codes)
    np.testing.assert_allclose(deq, ref, rtol=2 ** -11, atol=0)
