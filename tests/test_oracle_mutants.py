"""Plant plausible mistakes in a copy of the oracle and check that the pins in
test_oracle.py (quantizer, packing, GEMM), test_oracle_gptq.py (GPTQ),
test_oracle_search.py (the alpha search) and test_oracle_w4a8.py (W4A8) catch
every one of them.  CPU only;
the real oracle is untouched."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "step_denominator_2^N": ("delta = ((mx - mn) / F64(qmax)).astype(F16)",
                             "delta = ((mx - mn) / F64(qmax + 1)).astype(F16)"),
    "zero_point_sign": ("z = np.clip(np.rint(-mn / delta.astype(F64)), 0, qmax) + 0.0",
                        "z = np.clip(np.rint(mn / delta.astype(F64)), 0, qmax) + 0.0"),
    "round_half_up": ("u = np.clip(np.rint(g / d) + zz, 0, 2 ** bits - 1)",
                      "u = np.clip(np.floor(g / d + 0.5) + zz, 0, 2 ** bits - 1)"),
    "joint_rounding": ("u = np.clip(np.rint(g / d) + zz, 0, 2 ** bits - 1)",
                       "u = np.clip(np.rint(g / d + zz), 0, 2 ** bits - 1)"),
    "act_scale_max": ("sx = np.abs(X.astype(F64)).mean(axis=0)",
                      "sx = np.abs(X.astype(F64)).max(axis=0)"),
    "act_scale_no_abs": ("sx = np.abs(X.astype(F64)).mean(axis=0)",
                         "sx = (X.astype(F64)).mean(axis=0)"),
    "scale_rows_not_channels": ("(W.astype(F64) * s.astype(F64)[None, :])",
                                "(W.astype(F64) * s.astype(F64)[:W.shape[0], None])"),
    "sym_step_2^(N-1)-1": ("delta = (amax / F64(half)).astype(F16)",
                           "delta = (amax / F64(half - 1)).astype(F16)"),
    "slot_order_linear": ("SLOT_TO_ELEM = (0, 2, 4, 6, 1, 3, 5, 7)",
                          "SLOT_TO_ELEM = (0, 1, 2, 3, 4, 5, 6, 7)"),
    "dequant_drops_zero": ("return (u - z) * d", "return u * d"),
    "zero_range_rule": ("delta[delta == 0] = F16(1.0 / qmax)", "delta[delta == 0] = F16(1.0)"),
    "bound_not_absolute": ("bound = np.abs(x64) @ np.abs(w_hat).T", "bound = np.abs(x64 @ w_hat.T)"),
    # GPTQ: caught by tests/test_oracle_gptq.py
    "gptq_lower_factor": ("return np.linalg.cholesky(np.linalg.inv(np.asarray(H, dtype=F64))).T",
                          "return np.linalg.cholesky(np.linalg.inv(np.asarray(H, dtype=F64)))", "gptq"),
    "gptq_no_diagonal_division": ("e = (w - (ui - z) * d) / G[i, i]", "e = (w - (ui - z) * d)", "gptq"),
    "gptq_error_sign": ("Wc[:, i + 1:b1] = Wc[:, i + 1:b1] - e[:, None] * G[i, i + 1:b1][None, :]",
                        "Wc[:, i + 1:b1] = Wc[:, i + 1:b1] + e[:, None] * G[i, i + 1:b1][None, :]", "gptq"),
    "gptq_no_trailing_update": ("Wc[:, b1:] = Wc[:, b1:] - acc", "Wc[:, b1:] = Wc[:, b1:]", "gptq"),
    "gptq_trailing_row_shift": ("acc = acc + errs[:, i - b0][:, None] * G[i, b1:][None, :]",
                                "acc = acc + errs[:, i - b0][:, None] * G[max(i - 1, 0), b1:][None, :]", "gptq"),
    "gptq_no_damping": ("return H + lam * np.eye(H.shape[0])", "return H", "gptq"),
    "gptq_hessian_without_2": ("H = 2.0 * (Xf.T @ Xf)", "H = Xf.T @ Xf", "gptq"),
    "gptq_stats_from_original": ("d16, z16 = group_params(Wc[:, b0:b1], bits, mode, group)",
                                 "d16, z16 = group_params(np.asarray(W, dtype=F16)[:, b0:b1], bits, mode, group)",
                                 "gptq"),
    "gptq_code_from_original": ("w = Wc[:, i].copy()", "w = np.asarray(W, dtype=F16)[:, i].astype(F64)", "gptq"),
    # alpha search: caught by tests/test_oracle_search.py
    "search_multiplies_activation": ("return (X / np.asarray(s, dtype=F16).astype(F64)[None, :]).astype(F16)",
                                     "return (X * np.asarray(s, dtype=F16).astype(F64)[None, :]).astype(F16)",
                                     "search"),
    "search_output_not_rounded": ("y_q = (divide_activation(X, s).astype(F64) @ w_hat.T).astype(F16).astype(F64)",
                                  "y_q = divide_activation(X, s).astype(F64) @ w_hat.T", "search"),
    "search_target_divided": ("y = np.asarray(X, dtype=F16).astype(F64) @ np.asarray(W, dtype=F16).astype(F64).T",
                              "y = divide_activation(X, s).astype(F64) @ np.asarray(W, dtype=F16).astype(F64).T",
                              "search"),
    "search_argmax": ("return losses, int(np.argmin(losses))", "return losses, int(np.argmax(losses))", "search"),
    "search_sum_not_mean": ("return float(np.mean((y_q - y) ** 2))", "return float(np.sum((y_q - y) ** 2))",
                            "search"),
    "search_alpha_ignored": ("s = act_scale(X, alpha)", "s = act_scale(X, 0.5)", "search"),
    # W4A8: caught by tests/test_oracle_w4a8.py
    "w4a8_level1_range_127": ("W4A8_L1 = 119", "W4A8_L1 = 127", "w4a8"),
    "w4a8_floor_step": ("s2 = np.maximum(1, -((mn - mx) // 15))", "s2 = np.maximum(1, (mx - mn) // 15)", "w4a8"),
    "w4a8_unscaled_zero": ("(z2 * s2).astype(np.uint8)", "z2.astype(np.uint8)", "w4a8"),
    "w4a8_range_without_zero": ("mx, mn = np.maximum(g.max(axis=-1), 0), np.minimum(g.min(axis=-1), 0)",
                                "mx, mn = g.max(axis=-1), g.min(axis=-1)", "w4a8"),
    "w4a8_activation_range_128": ("W4A8_ACT = 127", "W4A8_ACT = 128", "w4a8"),
    "w4a8_output_without_s1": ("* np.asarray(s1, dtype=F16).astype(F64)[None, :]).astype(F16)",
                               ").astype(F16)", "w4a8"),
}

PIN_FILES = {None: "tests/test_oracle.py", "gptq": "tests/test_oracle_gptq.py", "search": "tests/test_oracle_search.py",
             "w4a8": "tests/test_oracle_w4a8.py"}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    before, after, *which = MUTANTS[name]
    pins = PIN_FILES[which[0] if which else None]
    src = open(os.path.join(ROOT, "oracle", "w4a16_oracle.py")).read()
    assert before in src, "mutation site moved; update the mutant"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle")
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "w4a16_oracle.py").write_text(src.replace(before, after))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        pins], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0, f"mutant {name} survived:\n{r.stdout[-2000:]}"
