"""gptq_export_checkpoint against the oracle's checkpoint layout, bit for bit.

Inputs are seeded random codes, scales and zeros; the solver-layout qweight
the call reads is the oracle's row packing of those codes.  Words are
integers and the float16 scales are one round-to-nearest-even conversion of
the same float32 values on both sides, so every output must match exactly.
The last test runs a whole solve and checks that the exported layer reads
back to the solver's own codes and dequantizes like it.
"""
import numpy as np
import pytest

import gen
import oracle as O
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


def _case(seed, out, in_, bits, ng):
    rng = np.random.default_rng([13, seed])
    maxq = 2 ** bits - 1
    codes = rng.integers(0, maxq + 1, (out, in_))
    zeros = rng.integers(0, maxq + 1, (out, ng)).astype(np.int32)
    zeros[0, 0] = 0  # wraps to maxq under the offset of 1
    scales = (np.abs(rng.standard_normal((out, ng))) * 0.01 + 1e-4).astype(np.float32)
    # float16 edge values: a tie to even, the overflow tie, a subnormal
    special = np.array([1.00048828125, 1.00146484375, 65520.0, 6e-08, 3e-09], np.float32)
    flat = scales.reshape(-1)
    flat[:min(len(special), flat.size)] = special[:flat.size]
    return codes, scales, zeros


def _run(lib, codes, scales, zeros, bits, zero_offset, want=(True, True, True)):
    import torch
    out, in_ = codes.shape
    ng = scales.shape[1]
    qweight = O.pack_rows(codes, bits).view(np.int32)
    sentinel = -0x5A5A5A5B  # 0xA5A5A5A5
    qt = torch.full((in_ * bits // 32, out), sentinel, dtype=torch.int32, device="cuda")
    qz = torch.full((ng, out * bits // 32), sentinel, dtype=torch.int32, device="cuda") \
        if (out * bits) % 32 == 0 else None
    sh = torch.full((ng, out), -1.0, dtype=torch.float16, device="cuda")
    lib.gptq_export_checkpoint(dev(qweight), dev(scales), dev(zeros), out, in_, bits, ng, zero_offset,
                               qt if want[0] else None, qz if want[1] else None,
                               sh if want[2] else None)
    torch.cuda.synchronize()
    return host(qt).view(np.uint32), None if qz is None else host(qz).view(np.uint32), \
        host(sh).view(np.uint16)


@pytest.mark.parametrize("out,in_,bits,ng,off", [
    (64, 256, 4, 2, 1),
    (32, 96, 3, 3, 1),      # 3-bit fields straddle words along both dimensions
    (48, 64, 2, 1, 0),
    (40, 512, 8, 8, 1),
    (96, 4128, 3, 129, 1),  # ragged 32 x 32 tiles in both dimensions
    (4096, 512, 4, 4, 1),
])
def test_export_bit_exact(lib, out, in_, bits, ng, off):
    codes, scales, zeros = _case(out + in_ + bits, out, in_, bits, ng)
    qt, qz, sh = _run(lib, codes, scales, zeros, bits, off)
    with np.errstate(over="ignore"):
        ref = O.checkpoint_layout(codes, scales, zeros, np.zeros(in_), bits, off)
    assert np.array_equal(qt, ref["qweight"])
    assert np.array_equal(qz, ref["qzeros"])
    assert np.array_equal(sh, ref["scales"].view(np.uint16))


def test_export_transpose_only_when_out_is_not_a_word_multiple(lib):
    """out * bits not a multiple of 32: qweight_t and scales_h are still
    written; qzeros cannot be and is not requested."""
    codes, scales, zeros = _case(5, 33, 128, 4, 4)
    qt, _, sh = _run(lib, codes, scales, zeros, 4, 1, want=(True, False, True))
    assert np.array_equal(qt, O.pack_rows(codes, 4).T)
    with np.errstate(over="ignore"):
        assert np.array_equal(sh, scales.T.astype(np.float16).view(np.uint16))


def test_export_skips_null_outputs(lib):
    codes, scales, zeros = _case(6, 32, 64, 4, 2)
    qt, qz, sh = _run(lib, codes, scales, zeros, 4, 1, want=(False, True, False))
    assert np.all(qt == 0xA5A5A5A5)
    assert np.all(sh == np.float16(-1.0).view(np.uint16))
    with np.errstate(over="ignore"):
        ref = O.checkpoint_layout(codes, scales, zeros, np.zeros(64), 4, 1)
    assert np.array_equal(qz, ref["qzeros"])


def test_export_of_a_solved_layer_reads_back(lib):
    """A reader of the exported layout (unpack along the input dimension,
    zeros plus the offset, float16 scales, g_idx) gets the solver's codes and
    the solver's dequantized layer up to the float16 rounding of the
    scales."""
    import torch
    W, X = gen.small_case(71, 64, 256, 1024, x_dtype="float16")
    Wt = dev(W, torch.float16)
    res = lib.solve_layer(Wt, dev(X, torch.float16), dict(bits=4, group_size=32, desc_act=True))
    ck = lib.export_checkpoint(res, 4, zero_offset=1)
    torch.cuda.synchronize()
    codes = host(res["codes"])
    q = O.unpack_rows(host(ck["qweight"]).view(np.uint32).T, 4, 256)
    assert np.array_equal(q, codes)
    # zeros plus the offset, modulo 2^bits (a zero of 0 is stored wrapped)
    z = (O.unpack_rows(host(ck["qzeros"]).view(np.uint32), 4, 64).T + 1) % 16
    assert np.array_equal(z, host(res["zeros"]))
    g_idx = host(ck["g_idx"])
    s16 = host(ck["scales"]).T.astype(np.float64)
    deq_ck = s16[:, g_idx] * (q - z[:, g_idx])
    deq = torch.empty((64, 256), dtype=torch.float32, device="cuda")
    lib.gptq_dequantize_layer(res["qweight"], res["scales"], res["zeros"], res["g_idx"], 4, deq)
    torch.cuda.synchronize()
    np.testing.assert_allclose(deq_ck, host(deq), rtol=1.01 * 2 ** -11, atol=1e-30)
