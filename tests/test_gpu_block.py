"""solve_block: the layers of a decoder block, with one Hessian and one
prepare per activation site shared by the layers that read it, and the
layers of a site quantized concurrently on separate streams.  Every layer is
compared with the oracle's independent solve of that layer."""
import numpy as np
import pytest

import gen
import oracle as O
from gpu_util import code_report, compare_groups, dev, host

pytestmark = pytest.mark.gpu


def test_block_layers_match_independent_oracle_solves(lib):
    import torch
    q = dict(bits=4, group_size=64, sym=False, desc_act=True, damp_percent=0.01, block_size=128)
    # two sites: "attn" (in 256) read by q/k/v, "o" (in 384) read by o
    _, Xa = gen.small_case(51, 1, 256, 2048, x_dtype="float16", sigma=1.5, outlier_frac=0.01)
    _, Xo = gen.small_case(52, 1, 384, 1536, x_dtype="float16", sigma=1.5, outlier_frac=0.01)
    shapes = {"q_proj": (128, "attn"), "k_proj": (192, "attn"), "v_proj": (64, "attn"), "o_proj": (96, "o")}
    Ws = {}
    for i, (name, (out, site)) in enumerate(shapes.items()):
        in_ = 256 if site == "attn" else 384
        Ws[name], _ = gen.small_case(60 + i, out, in_, 8, w_dtype="float16")
    acts = {"attn": dev(Xa, torch.float16), "o": dev(Xo, torch.float16)}
    layers = [(name, dev(Ws[name], torch.float16), site) for name, (_, site) in shapes.items()]
    res = lib.solve_block(layers, acts, q)
    # layers of one site share the prepared factor
    assert res["q_proj"]["U"] is res["k_proj"]["U"] is res["v_proj"]["U"]
    for name, (out, site) in shapes.items():
        X = torch.from_numpy(Xa if site == "attn" else Xo).to(torch.float16).float().numpy()
        S, n = O.hessian([X])
        ref = O.gptq_layer(np.asarray(Ws[name], np.float64), S, n, **q)
        r = res[name]
        assert np.array_equal(host(r["perm"]), ref["perm"]), name
        rate, eq = code_report(host(r["codes"]), ref["codes"])
        assert rate >= 0.999, (name, rate)
        compare_groups(host(r["scales"]), host(r["zeros"]), ref["scales"], ref["zeros"],
                       eq[:, ref["perm"]], q["group_size"])
        assert np.array_equal(host(r["qweight"]).view(np.uint32), O.pack_rows(host(r["codes"]), 4))
