"""Planted mistakes in the oracle, run by tests/test_oracle_mutants.py.

Each mutant swaps one snippet of the oracle's source (oracle/isa_oracle.py)
for a plausible mistake: a transposed operand, a dropped term, a wrong
index region, sign, divisor, tie rule or rounding.  Loaded as a pytest
plugin (``-p oracle_mutants``) with ``ORACLE_MUTANT=<name>``, it executes the
changed source as the oracle module before any test imports it, so the
oracle's pin tests run against the mistake and at least one must fail.
``ORACLE_MUTANT=none`` loads the unchanged source the same way (the
control).  Only the tests use this module.
"""
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCE = os.path.join(ROOT, "oracle", "isa_oracle.py")

# name -> (snippet of the oracle source, replacement); each snippet occurs
# exactly once in the source.
MUTANTS = {
    # step (1): pooling and coarse scores
    "pool_divides_by_block_size": (
        "sum(axis=0) / float(n)", "sum(axis=0) / float(counts.max())"),
    "scores_transposed": (
        "return (Qc @ Kc.T) * s", "return (Kc @ Qc.T) * s"),
    "scores_scale_squared": (
        "return (Qc @ Kc.T) * s", "return (Qc @ Kc.T) * (s * s)"),
    # step (2): context importance and TopK
    "importance_from_context_rows": (
        "return S[:T_src, T_src:].sum(axis=0)", "return S[T_src:, T_src:].sum(axis=0)"),
    "importance_region_transposed": (
        "return S[:T_src, T_src:].sum(axis=0)", "return S[T_src:, :T_src].sum(axis=1)"),
    "topk_ties_to_higher_index": (
        "np.lexsort((np.arange(len(scores)), -np.asarray(scores, np.float64)))",
        "np.lexsort((-np.arange(len(scores)), -np.asarray(scores, np.float64)))"),
    "context_count_rounded_down": (
        "math.ceil(_f32(alpha_s) * T_ctx)", "math.floor(_f32(alpha_s) * T_ctx)"),
    "kept_drops_source_blocks": (
        "kept = np.concatenate([np.arange(T_src), T_src + ctx_sel])", "kept = (T_src + ctx_sel)"),
    "kept_context_ids_not_offset": (
        "kept = np.concatenate([np.arange(T_src), T_src + ctx_sel])",
        "kept = np.concatenate([np.arange(T_src), ctx_sel])"),
    "context_last_block_full": (
        "counts.append(min(b, L_ctx - c * b))", "counts.append(b)"),
    # step (3): sharpness and the split
    "sharpness_without_softmax": (
        "P = softmax_rows(X) if use_softmax else X", "P = X"),
    "sharpness_over_source_columns": (
        'if cols == "all":\n        X = S\n', 'if cols == "all":\n        X = S[:, :T_src]\n'),
    "split_flat_takes_sharpest": (
        "sharp = np.sort(order[:T - n_flat])\n    flat = np.sort(order[T - n_flat:])",
        "flat = np.sort(order[:n_flat])\n    sharp = np.sort(order[n_flat:])"),
    "split_ties_to_higher_index": (
        "np.lexsort((np.arange(T), -np.asarray(M, np.float64)))",
        "np.lexsort((-np.arange(T), -np.asarray(M, np.float64)))"),
    "flat_count_rounded_up": (
        "math.floor(_f32(alpha_f) * T)", "math.ceil(_f32(alpha_f) * T)"),
    # step (5) lists
    "exact_count_over_all_blocks": (
        'base = len(kept) if p.ns_base == "kept" else T', "base = T"),
    "exact_lists_from_score_column": (
        "topk_lower_index(S[i, kept], n_ex)", "topk_lower_index(S[kept, i], n_ex)"),
    # steps (4)-(5): attention
    "sharp_attends_every_token": (
        "    cols = _kept_tokens(plan, plan.kept)\n    logits = ",
        "    cols = np.arange(k.shape[0])\n    logits = "),
    "taylor_drops_count_weight": (
        "logw = np.concatenate([np.zeros(len(tok)), np.log(plan.counts[pooled_blocks].astype(np.float64))])",
        "logw = np.zeros(len(tok) + len(pooled_blocks))"),
    "taylor_uses_pooled_query": (
        "logits_p = (q[rows] @ plan.Kc[pooled_blocks].T) * s",
        "logits_p = np.repeat((plan.Qc[i] @ plan.Kc[pooled_blocks].T)[None, :] * s, len(rows), axis=0)"),
    "taylor_value_is_first_token": (
        "values = np.concatenate([v[tok].astype(np.float64), plan.Vc[pooled_blocks]], axis=0)",
        "values = np.concatenate([v[tok].astype(np.float64), v[plan.starts[pooled_blocks]]], axis=0)"),
    "weights_left_out_of_softmax": (
        "    z = logits + log_weights[None, :]\n    m = z.max",
        "    z = logits\n    m = z.max"),
    "lse_without_row_maximum": (
        "return (e @ values) / den, (m + np.log(den))[:, 0]", "return (e @ values) / den, np.log(den)[:, 0]"),
    # backward
    "backward_dq_drops_pooled_keys": (
        "dq[rows] += s * (dz[:, :nt] @ k[tok] + dz[:, nt:] @ plan.Kc[pooled])",
        "dq[rows] += s * (dz[:, :nt] @ k[tok])"),
    "backward_drops_delta": (
        "return P * (dP - delta), P.T @ dout", "return P * dP, P.T @ dout"),
    "backward_pooled_gradient_not_averaged": (
        "        dk[t] += dKc[j] / plan.counts[j]\n        dv[t] += dVc[j] / plan.counts[j]\n    return dq, dk, dv\n",
        "        dk[t] += dKc[j]\n        dv[t] += dVc[j]\n    return dq, dk, dv\n"),
    "backward_dk_without_scale": (
        "dk[tok] += s * (dz[:, :nt].T @ q[rows])", "dk[tok] += dz[:, :nt].T @ q[rows]"),
    # gamma * O_coarse
    "coarse_softmax_over_columns": (
        "return softmax_rows(plan.S) @ plan.Vc", "return softmax_rows(plan.S.T).T @ plan.Vc"),
    "coarse_without_gamma": (
        "= gamma * oc[i]", "= oc[i]"),
    "coarse_backward_not_averaged": (
        "dq[t] += dQc[j] / plan.counts[j]", "dq[t] += dQc[j]"),
    "coarse_dgamma_scaled_by_gamma": (
        "dgamma = float((dO * oc).sum())", "dgamma = gamma * float((dO * oc).sum())"),
    # decoupled RoPE
    "rope_positions_continue_into_context": (
        "np.concatenate([np.arange(L_src), np.arange(L_ctx)]).astype(np.float64)",
        "np.arange(L_src + L_ctx).astype(np.float64)"),
    "rope_rotation_sign": (
        "y[..., 0::2] = xe * c - xo * s", "y[..., 0::2] = xe * c + xo * s"),
    "rope_frequency_exponent": (
        "theta = base ** (-2.0 * np.arange(D // 2) / D)", "theta = base ** (-1.0 * np.arange(D // 2) / D)"),
    "rope_pairs_halves": (
        "xe, xo = x[..., 0::2], x[..., 1::2]", "xe, xo = x[..., :D // 2], x[..., D // 2:]"),
}


def mutated_source(name: str) -> str:
    src = open(SOURCE).read()
    if name == "none":
        return src
    old, new = MUTANTS[name]
    n = src.count(old)
    if n != 1:
        raise RuntimeError(f"mutant {name}: snippet found {n} times in the oracle source")
    return src.replace(old, new)


def install(name: str) -> None:
    """Execute the (changed) oracle source as ``oracle.isa_oracle`` and
    re-export its names from the ``oracle`` package."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import oracle
    mod = types.ModuleType("oracle.isa_oracle")
    mod.__file__ = SOURCE
    mod.__package__ = "oracle"
    sys.modules["oracle.isa_oracle"] = mod
    exec(compile(mutated_source(name), SOURCE, "exec"), mod.__dict__)
    oracle.isa_oracle = mod
    for key, val in vars(mod).items():
        if not key.startswith("__"):
            setattr(oracle, key, val)


def pytest_configure(config):
    name = os.environ.get("ORACLE_MUTANT")
    if name:
        install(name)
