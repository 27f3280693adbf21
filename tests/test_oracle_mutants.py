"""Plant plausible mistakes in a copy of the oracle and check that the pins in
test_oracle.py catch every one of them.  CPU only; the real oracle is untouched."""
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
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(os.path.join(ROOT, "oracle", "w4a16_oracle.py")).read()
    assert before in src, "mutation site moved; update the mutant"
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle")
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    (tmp_path / "oracle" / "w4a16_oracle.py").write_text(src.replace(before, after))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle.py"], cwd=tmp_path, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0, f"mutant {name} survived:\n{r.stdout[-2000:]}"
