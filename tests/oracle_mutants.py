"""Plausible mistakes planted in the CPU oracle, one at a time, to show that
its pins catch each of them (test infrastructure; used by
``test_oracle_mutants.py``).

A mutant rewrites the source of one or more oracle functions by plain text
substitution (a dropped term, a flipped sign, a transposed operand, a wrong
index, a wrong rounding) and rebinds the result in the oracle module and the
``oracle`` package, so that every caller -- the pins and the oracle's own
pipeline -- sees the mistake.  Nothing here touches the GPU library.
"""
import inspect
import textwrap

# name -> [(function, text in its source, replacement), ...]
MUTANTS = {
    # step 1: Hessian
    "hessian_drops_factor_2": [("normalize_hessian", "(2.0 / n)", "(1.0 / n)")],
    "hessian_transposed_operand": [("hessian_accumulate", "X64 @ X64.T", "X64.T @ X64")],
    # step 2: dead channels and dampening
    "dead_diagonal_left_zero": [("fix_dead", "H[idx, idx] = 1.0", "H[idx, idx] = 0.0")],
    "damp_uses_max_of_diagonal": [("dampen", "np.mean(np.diag(H))", "np.max(np.diag(H))")],
    "damp_added_to_every_entry": [("dampen", "H[np.diag_indices_from(H)] += lam", "H += lam")],
    "damp_before_dead_fix": [("prepare", "    H, dead = fix_dead(H0)\n",
                              "    H, dead = fix_dead(dampen(H0, damp_percent))\n"),
                             ("prepare", "    H = dampen(H, damp_percent)\n", "")],
    # step 3: act-order
    "act_order_ascending": [("act_order", "np.argsort(-np.asarray(diag_h, dtype=np.float64), kind=\"stable\")",
                             "np.argsort(np.asarray(diag_h, dtype=np.float64), kind=\"stable\")")],
    "act_order_ties_by_descending_index": [
        ("act_order", "np.argsort(-np.asarray(diag_h, dtype=np.float64), kind=\"stable\")",
         "np.lexsort((-np.arange(n), -np.asarray(diag_h, dtype=np.float64)))")],
    "permuted_rows_only": [("prepare", "Hp = H[np.ix_(perm, perm)]", "Hp = H[perm]")],
    # step 4: U
    "U_is_inverse_transposed_cholesky": [("upper_cholesky_of_inverse", "return C.T", "return Linv.T")],
    "U_lower_triangular": [("upper_cholesky_of_inverse", "return C.T", "return C")],
    "U_from_H_not_its_inverse": [("upper_cholesky_of_inverse", "C = _chol_lower(Hinv)", "C = _chol_lower(H)")],
    # step 5: quantizer
    "zero_sign_flipped": [("group_params", "np.rint(-lo / scale)", "np.rint(lo / scale)")],
    "scale_over_maxq_plus_1": [("group_params", "scale = (hi - lo) / fmaxq", "scale = (hi - lo) / (fmaxq + 1)")],
    "sym_zero_maxq_half": [("group_params", "(maxq + 1) // 2", "maxq // 2")],
    "sym_scale_drops_factor_2": [("group_params", "(np.float32(2) * a) / fmaxq", "a / fmaxq")],
    "codes_floor": [("quantize_codes", "np.rint(w32 / scale.astype(np.float32))",
                     "np.floor(w32 / scale.astype(np.float32))")],
    "codes_round_half_away_from_zero": [("quantize_codes", "np.rint(w32 / scale.astype(np.float32))",
                                         "np.trunc(w32 / scale.astype(np.float32) + np.copysign(np.float32(0.5), w32))")],
    "codes_not_clamped": [("quantize_codes", "np.clip(q, 0, maxq)", "q")],
    "codes_without_zero": [("quantize_codes", ".astype(np.int64) + zero", ".astype(np.int64)")],
    # step 5: the sweep (both forms, so that blocked == unblocked still holds)
    "error_not_divided_by_U_jj": [
        ("sweep_unblocked", "e = (W[:, j] - dequantize_codes(q, s, z)) / U[j, j]",
         "e = (W[:, j] - dequantize_codes(q, s, z))"),
        ("sweep_blocked", "e = (W[:, j] - dequantize_codes(q, s, z)) / U[j, j]",
         "e = (W[:, j] - dequantize_codes(q, s, z))")],
    "compensation_sign_flipped": [
        ("sweep_unblocked", "W[:, j + 1:] -= np.outer(e, U[j, j + 1:])", "W[:, j + 1:] += np.outer(e, U[j, j + 1:])"),
        ("sweep_blocked", "W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])",
         "W[:, j + 1:b1] += np.outer(e, U[j, j + 1:b1])"),
        ("sweep_blocked", "W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]", "W[:, b1:] += err[:, b0:b1] @ U[b0:b1, b1:]"),
        ("sweep_blocked", "cur[:, b1 - j:] -= err", "cur[:, b1 - j:] += err")],
    "compensation_uses_U_column": [
        ("sweep_unblocked", "np.outer(e, U[j, j + 1:])", "np.outer(e, U[j + 1:, j])"),
        ("sweep_blocked", "np.outer(e, U[j, j + 1:b1])", "np.outer(e, U[j + 1:b1, j])"),
        ("sweep_blocked", "err[:, b0:b1] @ U[b0:b1, b1:]", "err[:, b0:b1] @ U[b1:, b0:b1].T"),
        ("sweep_blocked", "err[:, b0:j] @ U[b0:j, b1:ge]", "err[:, b0:j] @ U[b1:ge, b0:j].T")],
    "blocked_lazy_update_dropped": [("sweep_blocked", "W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]", "pass")],
    "blocked_group_params_miss_pending_updates": [("sweep_blocked", "if ge > b1:", "if False:")],
    "group_params_from_the_original_weights": [
        ("sweep_unblocked", "group_params(W[:, j:_group_end(j, n, group_size)]",
         "group_params(np.asarray(Wp, np.float64)[:, j:_group_end(j, n, group_size)]"),
        ("sweep_blocked", "cur = W[:, j:ge].copy()", "cur = np.array(Wp, np.float64)[:, j:ge]"),
        ("sweep_blocked", "if ge > b1:", "if False:")],
    "loss_of_unscaled_error": [
        ("sweep_unblocked", "loss=np.sum(err * err, axis=1)", "loss=np.sum(np.abs(err), axis=1)"),
        ("sweep_blocked", "loss=np.sum(err * err, axis=1)", "loss=np.sum(np.abs(err), axis=1)")],
    # layer pipeline
    "dead_weights_kept": [("gptq_layer", "Wd[:, prep[\"dead\"]] = 0.0", "pass")],
    "codes_unpermuted_with_perm": [("gptq_layer", "codes = res[\"codes\"][:, invperm]",
                                    "codes = res[\"codes\"][:, perm]")],
    "g_idx_from_perm_not_inverse": [("g_index", "return invperm // group_size",
                                     "return np.asarray(perm) // group_size")],
    "dequantize_ignores_g_idx": [("dequantize_layer", "[:, g_idx]", "[:, np.arange(len(g_idx)) * "
                                  "len(np.unique(g_idx)) // len(g_idx)]")],
    "layer_error_drops_half_n": [("layer_error", "e = 0.5 * n * float(", "e = float(")],
    # packing and the checkpoint layout
    "pack_msb_first": [("pack_rows", "(codes[:, c] << np.uint64(off))",
                        "(codes[:, c] << np.uint64(32 - bits - off if off + bits <= 32 else off))")],
    "pack_drops_straddling_bits": [("pack_rows", "if off + bits > 32:", "if False:")],
    "checkpoint_ignores_zero_offset": [("checkpoint_layout", "zeros.T - zero_offset", "zeros.T")],
    "checkpoint_offset_added": [("checkpoint_layout", "zeros.T - zero_offset", "zeros.T + zero_offset")],
    "checkpoint_scales_truncated": [
        ("checkpoint_layout", "scales=np.asarray(scales, np.float32).T.astype(np.float16)",
         "scales=(np.asarray(scales, np.float32).T.view(np.uint32) & np.uint32(0xFFFFE000))"
         ".view(np.float32).astype(np.float16)")],
    "checkpoint_stream_msb_first": [("_stream_words", "np.arange(bits, dtype=np.uint64)",
                                     "np.arange(bits - 1, -1, -1, dtype=np.uint64)")],
    "checkpoint_qweight_not_transposed": [("checkpoint_layout", "_stream_words(codes, bits).T.copy()",
                                           "_stream_words(codes, bits)")],
}


def _rewrite(module, fname, edits):
    src = textwrap.dedent(inspect.getsource(getattr(module, fname)))
    for old, new in edits:
        if old not in src:
            raise ValueError(f"mutant text not found in {fname}: {old!r}")
        src = src.replace(old, new)
    ns = {}
    exec(compile(src, f"<mutant of {fname}>", "exec"), module.__dict__, ns)
    return ns[fname]


def apply(name):
    """Plant mutant ``name`` in the oracle (module and package)."""
    import oracle
    from oracle import gptq_oracle as M
    by_fn = {}
    for fname, old, new in MUTANTS[name]:
        by_fn.setdefault(fname, []).append((old, new))
    for fname, edits in by_fn.items():
        fn = _rewrite(M, fname, edits)
        setattr(M, fname, fn)
        if hasattr(oracle, fname):
            setattr(oracle, fname, fn)
