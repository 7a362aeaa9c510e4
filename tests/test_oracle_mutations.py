"""The oracle's pins catch plausible mistakes: each case plants one mistake in
a temporary copy of the oracle (a dropped square root, a transposed operand, a
floor for the ceiling, the wrong tie rule, an unscaled INT8 weight, one
selection for every batch item, ...) and
runs the pin suite against that copy, which must fail. The oracle itself is
never modified."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle", "rmm_oracle.py")

# name: (text in the oracle, planted replacement)
MUTATIONS = {
    "keep_count_floor": ("return int(math.ceil(rho * K))", "return int(math.floor(rho * K))"),
    "keep_count_round": ("return int(math.ceil(rho * K))", "return int(round(rho * K))"),
    "column_norm_without_sqrt": ("return np.sqrt(np.sum(A * A, axis=0))", "return np.sum(A * A, axis=0)"),
    "column_norm_l1": ("return np.sqrt(np.sum(A * A, axis=0))", "return np.sum(np.abs(A), axis=0)"),
    "row_norm_without_sqrt": ("return np.sqrt(np.sum(B * B, axis=1))", "return np.sum(B * B, axis=1)"),
    "row_norm_over_columns": ("return np.sqrt(np.sum(B * B, axis=1))",
                              "return np.resize(np.sqrt(np.sum(B * B, axis=0)), B.shape[0])"),
    "score_sum_not_product": ("return a * row_norms(B)", "return a + row_norms(B)"),
    "a_only_mode_ignored": ("    if mode == SCORE_A_ONLY:\n        return a\n", ""),
    "ties_to_higher_index": ('order = np.argsort(-s, kind="stable")',
                             'order = (len(s) - 1 - np.argsort(-s[::-1], kind="stable"))'),
    "kept_indices_unsorted": ("return np.sort(order[:k_keep]).astype(np.int64)",
                              "return order[:k_keep].astype(np.int64)"),
    "keeps_smallest_scores": ('order = np.argsort(-s, kind="stable")', 'order = np.argsort(s, kind="stable")'),
    "keeps_one_too_few": ("return np.sort(order[:k_keep]).astype(np.int64)",
                          "return np.sort(order[:max(1, k_keep - 1)]).astype(np.int64)"),
    "pack_misaligns_B_rows": ("return A[:, idx], B[idx, :]", "return A[:, idx], B[np.sort(idx)[::-1], :]"),
    "int8_scale_per_row": ("return Wq.astype(np.float64) * np.asarray(scale, dtype=np.float64)[None, :]",
                           "return Wq.astype(np.float64) * np.resize(np.asarray(scale, dtype=np.float64), "
                           "Wq.shape[0])[:, None]"),
    "int8_scale_dropped": ("return Wq.astype(np.float64) * np.asarray(scale, dtype=np.float64)[None, :]",
                           "return Wq.astype(np.float64)"),
    "pv_contracts_over_queries": ("return matmul_reduced_batched(P, V, rho, mode)",
                                  "return matmul_reduced_batched(np.swapaxes(P, 1, 2), V, rho, mode)"),
    "near_tie_window_absolute": ("ok = all(abs(s[k] - t) <= rel_window * t for k in diff)",
                                 "ok = all(abs(s[k] - t) <= rel_window for k in diff)"),
    "relative_error_unnormalised": ("return float(num / den)", "return float(num)"),
    "keeps_one_too_many": ("return np.sort(order[:k_keep]).astype(np.int64)",
                           "return np.sort(order[:min(len(order), k_keep + 1)]).astype(np.int64)"),
    "batch_items_share_one_selection": ("        C, idx, s = matmul_reduced(A[b], B[b], rho, mode)\n",
                                        "        C, idx, s = matmul_reduced(A[b], B[b], rho, mode)\n"
                                        "        if b > 0:\n"
                                        "            idx = idxs[0]\n"
                                        "            C = reduced_product(A[b], B[b], idx)\n"),
    "product_over_dropped_slices": ("    return A_S @ B_S\n",
                                    "    keep = np.setdiff1d(np.arange(np.asarray(A).shape[1]), idx)\n"
                                    "    return np.asarray(A, dtype=np.float64)[:, keep] @ "
                                    "np.asarray(B, dtype=np.float64)[keep, :]\n"),
    "selection_range_unchecked": ("    if any(i < 0 or i >= s.shape[0] for i in g_list) or len(set(g_list)) != len(g_list):\n"
                                  "        return False, 0\n", ""),
    "pack_range_unchecked": ("        raise IndexError(f\"kept index outside [0, {K})\")\n", "        pass\n"),
    "bf16_rounding_truncates": ("    out[nz] = np.rint(q) * np.exp2(e - 7)  # np.rint rounds halves to even\n",
                                "    out[nz] = np.trunc(q) * np.exp2(e - 7)\n"),
    "causal_mask_off_by_one": ("        visible = k <= q + (S_k - S_q)\n", "        visible = k < q + (S_k - S_q)\n"),
    "causal_mask_aligned_to_the_first_query": ("        visible = k <= q + (S_k - S_q)\n", "        visible = k <= q\n"),
    "softmax_over_queries": ("    m = np.max(L, axis=-1, keepdims=True)\n    E = np.exp(L - m)\n"
                             "    return E / np.sum(E, axis=-1, keepdims=True)\n",
                             "    m = np.max(L, axis=-2, keepdims=True)\n    E = np.exp(L - m)\n"
                             "    return E / np.sum(E, axis=-2, keepdims=True)\n"),
    "softmax_scale_ignored": ("    L = np.asarray(L, dtype=np.float64) * scale\n", "    L = np.asarray(L, dtype=np.float64)\n"),
    "near_tie_threshold_is_the_largest_kept": ("t = float(np.min(s[list(o)]))", "t = float(np.max(s[list(o)]))"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(ORACLE).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, f"mutation {name} no longer matches the oracle"
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    (tmp_path / "oracle").mkdir()
    (tmp_path / "oracle" / "__init__.py").write_text("")
    (tmp_path / "oracle" / "rmm_oracle.py").write_text(src.replace(old, new))
    os.symlink(os.path.join(ROOT, "input_adaptive_reduced_02_b200"), tmp_path / "input_adaptive_reduced_02_b200")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=tmp_path, capture_output=True, text=True,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)}, timeout=300)
    assert r.returncode == 1, f"pins did not catch {name}:\n{r.stdout[-400:]}"
