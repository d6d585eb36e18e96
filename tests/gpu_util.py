"""Helpers shared by the GPU parity tests: moving seeded inputs to the device
and comparing the library's outputs with the oracle's."""
import numpy as np


def dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()


def torch_dtype(name):
    import torch
    return {"float16": torch.float16, "bfloat16": torch.bfloat16,
            "float32": torch.float32}[name]


def exact_values(x32, dtype_name):
    """The exact values a float32 array takes in ``dtype_name``, as float64,
    cast on the CPU (so the oracle sees precisely what the GPU gets)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch_dtype(dtype_name))
    return t, t.float().numpy().astype(np.float64)


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def code_report(gpu_codes, ref_codes):
    """Match rate of integer codes and, per row, the first mismatching
    processing column (rows with an earlier mismatch are excluded from the
    scale comparison, since their later groups legitimately diverge)."""
    g = np.asarray(gpu_codes)
    r = np.asarray(ref_codes)
    eq = g == r
    return float(eq.mean()), eq


def compare_groups(gpu_s, gpu_z, ref_s, ref_z, codes_p_eq, group_size, rtol=1e-4, max_flips=1e-3):
    """Compare scales (relative) and zeros on every group whose row had no
    code mismatch before the group's first column (processing order).

    A zero is an integer decided in fp32 from the group's current weights,
    like the codes: where the two sides' weights differ in the last bits and
    -lo / scale sits at a half-integer, the zero can come out one apart, and
    then every code of the group differs by one as well.  So zeros must be
    equal on every compared group whose codes all agree; groups whose zero
    differs are decision flips, bounded like codes (at most ``max_flips`` of
    the compared groups).  Returns (n_compared, n_excluded, n_zero_flips)."""
    out, ng = ref_s.shape
    n = codes_p_eq.shape[1]
    gs = n if group_size == -1 else group_size
    first_bad = np.where(codes_p_eq.all(1), n, np.argmin(codes_p_eq, axis=1))
    ok = np.zeros((out, ng), bool)
    grp_eq = np.zeros((out, ng), bool)
    for g in range(ng):
        ok[:, g] = first_bad >= g * gs   # no mismatch strictly before the group start
        grp_eq[:, g] = codes_p_eq[:, g * gs:(g + 1) * gs].all(1)
    gs_ = np.asarray(gpu_s, np.float64)[ok]
    rs_ = np.asarray(ref_s, np.float64)[ok]
    np.testing.assert_allclose(gs_, rs_, rtol=rtol)
    zeq = np.asarray(gpu_z) == np.asarray(ref_z)
    assert np.all(zeq[ok & grp_eq]), "zero differs on a group whose codes all agree"
    flips = int((ok & ~zeq).sum())
    assert flips <= max_flips * max(int(ok.sum()), 1), (flips, int(ok.sum()))
    return int(ok.sum()), int((~ok).sum()), flips
