"""GPTQ layer solver -- plain float64 CPU oracle.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may use this
module.  The GPU library never imports it and shares no code with it.

It restates, step by step and without blocking or fusion beyond what the
method itself states, what the GPTQ pages say the solver computes:

1. Hessian from calibration data ("gptq" glossary page, "Algorithm" (1):
   H = d2L/dW2 approximated from calibration data).  For the layer loss
   L = ||W X - W^ X||^2 averaged over n tokens this is H = 2 X X^T / n.
2. Dampening: a fraction ``damp_percent`` of the mean of diag(H) is added to
   the diagonal ("Using AutoGPTQ in Practice", "Key Parameters",
   damp_percent).
3. desc_act / ActOrder: columns are processed by decreasing Hessian diagonal
   (same section, desc_act).
4. Cholesky factorisation ("Using AutoGPTQ in Practice", opening paragraph):
   the sweep uses U, the upper Cholesky factor of H^-1 (U^T U = H^-1).
5. For each weight in order: quantize it, compute its error and adjust the
   remaining weights with H^-1 ("gptq" glossary page, "Algorithm" (2), and
   "Key innovation"), with one scale/zero per group of ``group_size`` weights
   ("gptq" agent-skill page, "Group-wise quantization"; "gptq" glossary page,
   "Group quantization"), symmetric or asymmetric ("AutoGPTQ" artifact page,
   quantization-scheme paragraph), at 2/3/4/8 bits.

Where the pages are silent the plainest reading is taken; each reading is
named at the function that makes it:

* quantizer grid: asymmetric range [min(0, min w), max(0, max w)] (an all-zero
  group uses [-1, 1]), scale = (hi - lo) / maxq, zero = rint(-lo / scale);
  symmetric: scale = 2 max|w| / maxq (max|w| = 0 -> 1), zero = (maxq + 1) / 2;
  code = clamp(rint(w / scale) + zero, 0, maxq); rint rounds half to even.
* the code decision (scale, zero, code) is taken in IEEE float32 -- the GPU
  kernel's precision -- so both sides decide integers the same way; all other
  arithmetic is float64.
* group parameters come from the current, fully updated weights at the
  group's first column (in processing order); groups are consecutive runs of
  ``group_size`` columns in processing order; group_size = -1 means one group
  per output row.
* dead channels (H_ii == 0) get H_ii = 1 and their weights set to zero,
  before dampening; the act-order sort key is diag(H) after that fix, ties
  broken by ascending column index.
* codes are packed LSB-first into little-endian uint32 words, row by row, in
  original column order.
* the loaders' checkpoint layout (``checkpoint_layout``) is the transpose:
  codes packed along the input dimension, zeros along the output dimension
  less an offset of 1, scales in float16.

Every function here is pinned by ``tests/test_oracle_*.py`` against closed
forms, brute force on tiny layers, invariances and hand-worked examples.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "NotPositiveDefinite", "hessian_accumulate", "hessian", "normalize_hessian",
    "fix_dead", "dampen", "act_order", "upper_cholesky_of_inverse",
    "group_params", "quantize_codes", "dequantize_codes", "sweep_unblocked",
    "sweep_blocked", "prepare", "gptq_layer", "rtn", "pack_rows", "unpack_rows",
    "g_index", "dequantize_layer", "layer_error", "brute_force_sweep",
    "maxq_of", "checkpoint_layout",
]


class NotPositiveDefinite(ValueError):
    """The damped Hessian (or its inverse) has no Cholesky factor."""


def maxq_of(bits: int) -> int:
    if bits not in (2, 3, 4, 8):
        raise ValueError("bits must be 2, 3, 4 or 8")
    return (1 << bits) - 1


# ---------------------------------------------------------------- step 1
def hessian_accumulate(S: np.ndarray, X: np.ndarray) -> np.ndarray:
    """S += X X^T in float64 (X: in x tokens, values taken exactly)."""
    X64 = np.asarray(X, dtype=np.float64)
    S += X64 @ X64.T
    return S


def hessian(chunks) -> tuple[np.ndarray, int]:
    """(S, n): S = sum_c X_c X_c^T over calibration chunks, n = total tokens."""
    S = None
    n = 0
    for X in chunks:
        if S is None:
            S = np.zeros((X.shape[0], X.shape[0]), dtype=np.float64)
        hessian_accumulate(S, X)
        n += X.shape[1]
    return S, n


def normalize_hessian(S: np.ndarray, n: int) -> np.ndarray:
    """H = 2 S / n: the Hessian of the mean squared layer-output error."""
    if n <= 0:
        raise ValueError("no calibration tokens")
    return (2.0 / n) * np.asarray(S, dtype=np.float64)


# ---------------------------------------------------------------- step 2
def fix_dead(H: np.ndarray):
    """Reading: a channel with H_ii == 0 never fires; set H_ii = 1 so H stays
    positive definite (its weights are zeroed by the caller).  Returns
    (H fixed copy, dead mask)."""
    H = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(H) == 0.0
    idx = np.nonzero(dead)[0]
    H[idx, idx] = 1.0
    return H, dead


def dampen(H: np.ndarray, damp_percent: float) -> np.ndarray:
    """H + lambda I with lambda = damp_percent * mean(diag H)
    ("Using AutoGPTQ in Practice", "Key Parameters", damp_percent)."""
    if not (damp_percent >= 0 and np.isfinite(damp_percent)):
        raise ValueError("damp_percent must be finite and >= 0")
    lam = damp_percent * float(np.mean(np.diag(H)))
    H = np.array(H, dtype=np.float64, copy=True)
    H[np.diag_indices_from(H)] += lam
    return H


# ---------------------------------------------------------------- step 3
def act_order(diag_h: np.ndarray, desc_act: bool) -> np.ndarray:
    """perm[p] = original column processed at position p.  desc_act: decreasing
    Hessian diagonal ("Using AutoGPTQ in Practice", "Key Parameters",
    desc_act); ties keep ascending column index.  Otherwise identity."""
    n = len(diag_h)
    if not desc_act:
        return np.arange(n, dtype=np.int64)
    # stable sort on the negated key == stable descending sort
    return np.argsort(-np.asarray(diag_h, dtype=np.float64), kind="stable")


# ---------------------------------------------------------------- step 4
def _chol_lower(A: np.ndarray) -> np.ndarray:
    try:
        return np.linalg.cholesky(A)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from None


def upper_cholesky_of_inverse(H: np.ndarray) -> np.ndarray:
    """U upper triangular with positive diagonal and U^T U = H^-1, by the plain
    definition: H^-1 from the Cholesky factor of H, then the Cholesky factor
    of H^-1 ("Using AutoGPTQ in Practice": Hessian computation, Cholesky
    factorization)."""
    n = H.shape[0]
    L = _chol_lower(H)                       # H = L L^T
    Linv = np.linalg.solve(L, np.eye(n))     # L^-1
    Hinv = Linv.T @ Linv                     # H^-1 = L^-T L^-1
    Hinv = 0.5 * (Hinv + Hinv.T)
    C = _chol_lower(Hinv)                    # H^-1 = C C^T
    return C.T                               # U = C^T: U^T U = H^-1


# ---------------------------------------------------------------- step 5
def group_params(wg: np.ndarray, bits: int, sym: bool):
    """Scale (float32) and integer zero for each row of the group ``wg``
    (rows x group columns, current values).  Computed in IEEE float32: the
    precision the GPU kernel decides codes in."""
    maxq = maxq_of(bits)
    w32 = np.asarray(wg, dtype=np.float64).astype(np.float32)
    fmaxq = np.float32(maxq)
    if sym:
        a = np.max(np.abs(w32), axis=1)
        a = np.where(a == 0, np.float32(1), a).astype(np.float32)
        scale = (np.float32(2) * a) / fmaxq
        zero = np.full(w32.shape[0], (maxq + 1) // 2, dtype=np.int64)
    else:
        lo = np.minimum(np.min(w32, axis=1), np.float32(0))
        hi = np.maximum(np.max(w32, axis=1), np.float32(0))
        both = (lo == 0) & (hi == 0)
        lo = np.where(both, np.float32(-1), lo).astype(np.float32)
        hi = np.where(both, np.float32(1), hi).astype(np.float32)
        scale = (hi - lo) / fmaxq
        zero = np.rint(-lo / scale).astype(np.int64)
    return scale.astype(np.float32), zero


def quantize_codes(w: np.ndarray, scale: np.ndarray, zero: np.ndarray,
                   bits: int) -> np.ndarray:
    """code = clamp(rint(w / scale) + zero, 0, maxq); w rounded to float32 and
    divided in float32 (round half to even)."""
    maxq = maxq_of(bits)
    w32 = np.asarray(w, dtype=np.float64).astype(np.float32)
    q = np.rint(w32 / scale.astype(np.float32)).astype(np.int64) + zero
    return np.clip(q, 0, maxq)


def dequantize_codes(q, scale, zero) -> np.ndarray:
    """scale * (code - zero), exact in float64."""
    return scale.astype(np.float64) * (np.asarray(q, np.int64) - zero)


def _ngroups(n: int, group_size: int) -> int:
    return 1 if group_size == -1 else (n + group_size - 1) // group_size


def _group_of(j: int, group_size: int) -> int:
    return 0 if group_size == -1 else j // group_size


def _group_start(j: int, group_size: int) -> bool:
    return j == 0 if group_size == -1 else j % group_size == 0


def _group_end(j: int, n: int, group_size: int) -> int:
    return n if group_size == -1 else min(n, j + group_size)


def sweep_unblocked(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int,
                    sym: bool):
    """The column-sequential sweep, one column at a time ("gptq" glossary
    page, "Algorithm" (2)): for column j, quantize, e = (w - deq) / U_jj,
    W[:, j+1:] -= e U[j, j+1:].  Wp and U are in processing order.

    Returns dict(codes, scales, zeros, err, loss) with scales/zeros indexed
    [row, group] by processing-order group, err the e values (out x n) and
    loss[r] = sum_j e_rj^2."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    out, n = W.shape
    ng = _ngroups(n, group_size)
    codes = np.zeros((out, n), np.int64)
    scales = np.zeros((out, ng), np.float32)
    zeros = np.zeros((out, ng), np.int64)
    err = np.zeros((out, n), np.float64)
    s = z = None
    for j in range(n):
        if _group_start(j, group_size):
            g = _group_of(j, group_size)
            s, z = group_params(W[:, j:_group_end(j, n, group_size)], bits, sym)
            scales[:, g], zeros[:, g] = s, z
        q = quantize_codes(W[:, j], s, z, bits)
        e = (W[:, j] - dequantize_codes(q, s, z)) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        codes[:, j] = q
        err[:, j] = e
    return dict(codes=codes, scales=scales, zeros=zeros, err=err,
                loss=np.sum(err * err, axis=1))


def sweep_blocked(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int,
                  sym: bool, block_size: int = 128):
    """The same sweep with lazy batching: inside a block of ``block_size``
    columns the updates are applied eagerly to the block; the block's errors
    then update all later columns at once, W[:, b1:] -= E_blk U[blk, b1:].
    This is an exact reorganisation of ``sweep_unblocked``.  Group parameters
    need the current values of the group's columns; where a group reaches past
    the block, the pending in-block updates are applied to those columns
    first."""
    if block_size <= 0:
        raise ValueError("block_size must be positive")
    W = np.array(Wp, dtype=np.float64, copy=True)
    out, n = W.shape
    ng = _ngroups(n, group_size)
    codes = np.zeros((out, n), np.int64)
    scales = np.zeros((out, ng), np.float32)
    zeros = np.zeros((out, ng), np.int64)
    err = np.zeros((out, n), np.float64)
    s = z = None
    for b0 in range(0, n, block_size):
        b1 = min(n, b0 + block_size)
        for j in range(b0, b1):
            if _group_start(j, group_size):
                g = _group_of(j, group_size)
                ge = _group_end(j, n, group_size)
                cur = W[:, j:ge].copy()
                if ge > b1:   # columns past the block still miss E[:, b0:j]
                    cur[:, b1 - j:] -= err[:, b0:j] @ U[b0:j, b1:ge]
                s, z = group_params(cur, bits, sym)
                scales[:, g], zeros[:, g] = s, z
            q = quantize_codes(W[:, j], s, z, bits)
            e = (W[:, j] - dequantize_codes(q, s, z)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            codes[:, j] = q
            err[:, j] = e
        W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return dict(codes=codes, scales=scales, zeros=zeros, err=err,
                loss=np.sum(err * err, axis=1))


# ---------------------------------------------------------------- packing
def pack_rows(codes: np.ndarray, bits: int) -> np.ndarray:
    """Reading (the pages name a packed format but give no layout): each row's
    codes, in original column order, form an LSB-first bit stream of
    ``bits``-wide fields in little-endian uint32 words."""
    codes = np.asarray(codes, dtype=np.uint64)
    out, n = codes.shape
    if (n * bits) % 32:
        raise ValueError("in * bits must be a multiple of 32")
    if np.any(codes >> np.uint64(bits)):
        raise ValueError("code out of range")
    words = np.zeros((out, n * bits // 32), dtype=np.uint64)
    for c in range(n):
        bit = c * bits
        w, off = divmod(bit, 32)
        words[:, w] |= (codes[:, c] << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[:, w + 1] |= codes[:, c] >> np.uint64(32 - off)
    return words.astype(np.uint32)


def unpack_rows(words: np.ndarray, bits: int, n: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint64)
    out = words.shape[0]
    mask = np.uint64((1 << bits) - 1)
    codes = np.zeros((out, n), np.int64)
    for c in range(n):
        bit = c * bits
        w, off = divmod(bit, 32)
        v = words[:, w] >> np.uint64(off)
        if off + bits > 32:
            v |= words[:, w + 1] << np.uint64(32 - off)
        codes[:, c] = (v & mask).astype(np.int64)
    return codes



# ------------------------------------------------------- checkpoint layout
def _stream_words(fields: np.ndarray, bits: int) -> np.ndarray:
    """Words of the LSB-first stream of ``bits``-wide fields taken along the
    last axis: field i fills stream bits [i bits, (i + 1) bits) from its least
    significant bit up, and stream bit t is bit t % 32 of word t // 32.  Built
    bit by bit, independently of ``pack_rows``."""
    f = np.asarray(fields, np.uint64)
    n = f.shape[-1]
    if (n * bits) % 32:
        raise ValueError("the packed axis times bits must be a multiple of 32")
    one = np.uint64(1)
    stream = (f[..., None] >> np.arange(bits, dtype=np.uint64)) & one
    stream = stream.reshape(*f.shape[:-1], n * bits // 32, 32)
    return (stream << np.arange(32, dtype=np.uint64)).sum(axis=-1).astype(np.uint32)


def checkpoint_layout(codes, scales, zeros, g_idx, bits: int, zero_offset: int = 1):
    """The quantized layer in the checkpoint layout of the GPTQ loaders.

    Reading (the "AutoGPTQ" artifact page, "Why AutoGPTQ Matters", names the
    GPTQ format that ExLlamaV2 and vLLM load, and the "gptq" agent-skill page,
    "Marlin", loads it from disk; neither prints the layout): tensors are
    stored input-dimension-major, the transpose of this solver's row-major
    outputs --

    * qweight uint32 [in bits/32][out]: column o is the LSB-first stream of
      row o's codes along the input dimension, in original column order;
    * qzeros uint32 [ngroups][out bits/32]: row g is the LSB-first stream,
      along the output dimension, of (zeros[:, g] - zero_offset) mod 2^bits
      (zero_offset 1 is the convention of the format's first version, whose
      readers add the 1 back; a zero of 0 then wraps to maxq);
    * scales float16 [ngroups][out]: scales^T rounded to nearest, ties to
      even;
    * g_idx int32 [in], unchanged.
    """
    codes = np.asarray(codes, np.int64)
    zeros = np.asarray(zeros, np.int64)
    if zero_offset not in (0, 1):
        raise ValueError("zero_offset must be 0 or 1")
    if np.any(codes < 0) or np.any(codes >= (1 << bits)):
        raise ValueError("code out of range")
    qweight = _stream_words(codes, bits).T.copy()
    qzeros = _stream_words(np.mod(zeros.T - zero_offset, 1 << bits), bits)
    return dict(qweight=qweight, qzeros=qzeros,
                scales=np.asarray(scales, np.float32).T.astype(np.float16),
                g_idx=np.asarray(g_idx).astype(np.int32))


def g_index(perm: np.ndarray, group_size: int) -> np.ndarray:
    """g_idx[c] = group of original column c = (its processing position) //
    group_size; 0 for group_size = -1."""
    n = len(perm)
    if group_size == -1:
        return np.zeros(n, np.int64)
    invperm = np.empty(n, np.int64)
    invperm[np.asarray(perm)] = np.arange(n)
    return invperm // group_size


# ---------------------------------------------------------------- pipeline
def prepare(S: np.ndarray, n: int, damp_percent: float, desc_act: bool):
    """Steps 1-4 from the accumulated S: returns dict(H0, dead, perm, Hp, U),
    Hp and U in processing order, H0 = 2 S / n undamped."""
    H0 = normalize_hessian(S, n)
    if not np.all(np.isfinite(H0)):
        raise FloatingPointError("non-finite Hessian")
    H, dead = fix_dead(H0)
    perm = act_order(np.diag(H), desc_act)
    H = dampen(H, damp_percent)
    Hp = H[np.ix_(perm, perm)]
    U = upper_cholesky_of_inverse(Hp)
    return dict(H0=H0, dead=dead, perm=perm, Hp=Hp, U=U)


def gptq_layer(W: np.ndarray, S: np.ndarray, n: int, bits=4, group_size=128,
               sym=False, desc_act=False, damp_percent=0.01, block_size=128,
               blocked=True):
    """The whole layer solve.  W: out x in (any float dtype, taken exactly);
    S: accumulated sum of X X^T; n: tokens.  Outputs are in original column
    order except scales/zeros, which are indexed by processing-order group
    (g_idx maps original column -> group)."""
    W0 = np.asarray(W, dtype=np.float64)
    nin = W0.shape[1]
    if group_size != -1 and (group_size <= 0 or nin % group_size):
        raise ValueError("group_size must be -1 or a positive divisor of in")
    prep = prepare(S, n, damp_percent, desc_act)
    perm = prep["perm"]
    Wd = W0.copy()
    Wd[:, prep["dead"]] = 0.0
    Wp = Wd[:, perm]
    if blocked:
        res = sweep_blocked(Wp, prep["U"], bits, group_size, sym, block_size)
    else:
        res = sweep_unblocked(Wp, prep["U"], bits, group_size, sym)
    invperm = np.empty(nin, np.int64)
    invperm[perm] = np.arange(nin)
    codes = res["codes"][:, invperm]
    g_idx = g_index(perm, group_size)
    out = dict(prep)
    out.update(codes=codes, scales=res["scales"], zeros=res["zeros"],
               g_idx=g_idx, err_p=res["err"], loss=res["loss"],
               codes_p=res["codes"], invperm=invperm)
    if (nin * bits) % 32 == 0:
        out["qweight"] = pack_rows(codes, bits)
    return out


def rtn(W: np.ndarray, bits: int, group_size: int, sym: bool,
        perm: np.ndarray | None = None):
    """Round-to-nearest with the same quantizer and no compensation (the
    "blind quantization" GPTQ improves on).  Groups are formed in processing
    order ``perm`` (identity by default).  Returns (codes in original order,
    scales, zeros) with scales/zeros indexed by processing-order group."""
    W0 = np.asarray(W, dtype=np.float64)
    nin = W0.shape[1]
    perm = np.arange(nin) if perm is None else np.asarray(perm)
    Wp = W0[:, perm]
    ng = _ngroups(nin, group_size)
    codes_p = np.zeros(Wp.shape, np.int64)
    scales = np.zeros((W0.shape[0], ng), np.float32)
    zeros = np.zeros((W0.shape[0], ng), np.int64)
    for g in range(ng):
        j0 = 0 if group_size == -1 else g * group_size
        j1 = nin if group_size == -1 else min(nin, j0 + group_size)
        s, z = group_params(Wp[:, j0:j1], bits, sym)
        scales[:, g], zeros[:, g] = s, z
        for j in range(j0, j1):
            codes_p[:, j] = quantize_codes(Wp[:, j], s, z, bits)
    invperm = np.empty(nin, np.int64)
    invperm[perm] = np.arange(nin)
    return codes_p[:, invperm], scales, zeros


def dequantize_layer(codes, scales, zeros, g_idx) -> np.ndarray:
    """deq[r, c] = scales[r, g_idx[c]] * (codes[r, c] - zeros[r, g_idx[c]])."""
    g_idx = np.asarray(g_idx, np.int64)
    s = np.asarray(scales, np.float32).astype(np.float64)[:, g_idx]
    z = np.asarray(zeros, np.int64)[:, g_idx]
    return s * (np.asarray(codes, np.int64) - z)


def layer_error(W0: np.ndarray, deq: np.ndarray, H0: np.ndarray, n: int):
    """(||(W0 - Deq) X||_F^2, same / ||W0 X||_F^2) using X X^T = (n/2) H0."""
    W0 = np.asarray(W0, np.float64)
    d = W0 - deq
    e = 0.5 * n * float(np.einsum("ri,ij,rj->", d, H0, d, optimize=True))
    ref = 0.5 * n * float(np.einsum("ri,ij,rj->", W0, H0, W0, optimize=True))
    return e, (e / ref if ref > 0 else float("nan"))


# ---------------------------------------------------------------- brute force
def brute_force_sweep(Wp: np.ndarray, Hp: np.ndarray, bits: int,
                      group_size: int, sym: bool):
    """The column-sequential procedure restated without any Cholesky factor
    (for tiny layers): before column j, the already quantized columns F are
    fixed at their dequantized values and the rest R take their optimal
    continuous values W_R = W0_R + (W0_F - Deq_F) H_FR H_RR^-1 (the minimiser
    of (w - w^) H (w - w^)^T over w^_R).  Column j is quantized from those
    values.  Hp: damped Hessian in processing order.  Returns (codes, scales,
    zeros, deq) in processing order."""
    W0 = np.asarray(Wp, np.float64)
    out, n = W0.shape
    ng = _ngroups(n, group_size)
    codes = np.zeros((out, n), np.int64)
    deq = np.zeros((out, n))
    scales = np.zeros((out, ng), np.float32)
    zeros = np.zeros((out, ng), np.int64)
    s = z = None
    for j in range(n):
        F = np.arange(j)
        R = np.arange(j, n)
        if j:
            shift = (W0[:, F] - deq[:, F]) @ Hp[np.ix_(F, R)] @ \
                np.linalg.inv(Hp[np.ix_(R, R)])
            cur = W0[:, R] + shift
        else:
            cur = W0.copy()
        if _group_start(j, group_size):
            g = _group_of(j, group_size)
            ge = _group_end(j, n, group_size)
            s, z = group_params(cur[:, :ge - j], bits, sym)
            scales[:, g], zeros[:, g] = s, z
        codes[:, j] = quantize_codes(cur[:, 0], s, z, bits)
        deq[:, j] = dequantize_codes(codes[:, j], s, z)
    return codes, scales, zeros, deq
