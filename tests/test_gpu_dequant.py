"""gptq_dequantize_layer against the oracle's dequantisation, bit for bit.

Inputs are seeded random codes, scales, zeros and group maps (natural and
act-order style), packed by the oracle's packer.  The oracle's value
scale * (code - zero) is exact in float64; rounding it to fp32 and then to the
output type is the same two roundings the kernel makes (fp32 product, one
conversion), so the outputs must match exactly.
"""
import numpy as np
import pytest

import oracle as O
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


def _case(seed, out, in_, bits, gs, act_order):
    rng = np.random.default_rng([9, seed])
    maxq = 2 ** bits - 1
    ng = 1 if gs == -1 else in_ // gs
    codes = rng.integers(0, maxq + 1, (out, in_))
    scales = (np.abs(rng.standard_normal((out, ng))) * 0.01 + 1e-4).astype(np.float32)
    zeros = rng.integers(0, maxq + 1, (out, ng)).astype(np.int32)
    if act_order:
        perm = rng.permutation(in_)
        g_idx = O.g_index(perm, gs)
    else:
        g_idx = O.g_index(np.arange(in_), gs)
    return codes, scales, zeros, np.asarray(g_idx, np.int32), ng


def _expected(codes, scales, zeros, g_idx, torch_dtype):
    import torch
    deq32 = O.dequantize_layer(codes, scales, zeros, g_idx).astype(np.float32)
    return torch.from_numpy(deq32).to(torch_dtype)


@pytest.mark.parametrize("out,in_,bits,gs,act,dt,pad", [
    (64, 256, 4, 128, False, "float16", 0),
    (33, 96, 3, 32, True, "bfloat16", 0),
    (17, 64, 2, -1, False, "float32", 0),
    (40, 512, 8, 64, True, "float16", 8),
    (9, 128, 4, 8, True, "float16", 3),      # unaligned row stride: scalar stores
    (5, 64, 3, 64, False, "bfloat16", 1),
    (4096, 4096, 4, 128, True, "float16", 0),
])
def test_dequantize_bit_exact(lib, out, in_, bits, gs, act, dt, pad):
    import torch
    tdt = {"float16": torch.float16, "bfloat16": torch.bfloat16, "float32": torch.float32}[dt]
    codes, scales, zeros, g_idx, ng = _case(out + in_ + bits, out, in_, bits, gs, act)
    qweight = O.pack_rows(codes, bits).astype(np.uint32)
    Wbuf = torch.full((out, in_ + pad), 7.0, dtype=tdt, device="cuda")
    Wq = Wbuf[:, :in_]
    lib.gptq_dequantize_layer(dev(qweight.view(np.int32)), dev(scales), dev(zeros), dev(g_idx), bits, Wq)
    torch.cuda.synchronize()
    exp = _expected(codes, scales, zeros, g_idx, tdt)
    got = Wq.cpu()
    assert torch.equal(got.view(torch.int16 if tdt != torch.float32 else torch.int32),
                       exp.view(torch.int16 if tdt != torch.float32 else torch.int32))
    if pad:  # the padding columns are untouched
        assert torch.all(Wbuf[:, in_:].cpu() == 7.0)


def test_dequantize_rejects_unsupported_shapes(lib):
    import torch
    Wq = torch.empty((4, 12), dtype=torch.float16, device="cuda")
    q = torch.zeros((4, 3), dtype=torch.int32, device="cuda")
    s = torch.ones((4, 1), dtype=torch.float32, device="cuda")
    z = torch.zeros((4, 1), dtype=torch.int32, device="cuda")
    g = torch.zeros(12, dtype=torch.int32, device="cuda")
    with pytest.raises(lib.GptqError) as e:
        lib.gptq_dequantize_layer(q, s, z, g, 8, Wq)    # in % 8 != 0
    assert e.value.status == 7
