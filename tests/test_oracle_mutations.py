"""Plants plausible mistakes in a scratch copy of the oracle (CPU only) and checks
that the pins in test_oracle_pins.py catch every one of them."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "drop_D_skip": ("if (Dskip) yt += Dskip[d] * ut;\n        if (z) yt *= ora_silu(z[row + t]);\n        y[row + t] = yt;",
                    "if (z) yt *= ora_silu(z[row + t]);\n        y[row + t] = yt;"),
    "conv_index_reversed": ("const long s = t + k - pad_left;", "const long s = t - k + pad_left;"),
    "aux_mean_over_L": ("const double m = s / (double)T;", "const double m = s / (double)(T + 2);"),
    "reset_at_last_token": ("const int reset = (p % L) == 0;", "const int reset = (p % L) == L - 1;"),
    "A_sign_flipped": ("const double abar = exp(delta * A[d * N + n]);\n          const double bbar",
                       "const double abar = exp(-delta * A[d * N + n]);\n          const double bbar"),
    "no_gate": ("if (z) yt *= ora_silu(z[row + t]);\n        y[row + t] = yt;", "y[row + t] = yt;"),
    "bwd_adjoint_no_carry": ("const double carry = (t + 1 < L) ? abar[(t + 1) * N + n] * g[n] : 0.0;",
                             "const double carry = 0.0;"),
    "bwd_dA_missing_delta": ("dA[d * N + n] += da * abar[t * N + n] * delta[t];", "dA[d * N + n] += da * abar[t * N + n];"),
    "softplus_threshold": ("return v > 20.0 ? v : log1p(exp(v));", "return v > 2.0 ? v : log1p(exp(v));"),
    "swap_keeps_head": ("yr[0] = yr[L - 1];", "yr[0] = yr[0];"),
    "conv_bwd_index": ("const long t = s - k + pad_left;", "const long t = s + k - pad_left;"),
    "aux_bwd_no_mean_share": ("const double share = (g[0] + g[L - 1]) / (double)T;", "const double share = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    src = open(os.path.join(ROOT, "oracle", "sfm_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, "mutation site moved: " + name
    work = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (work / "oracle" / "sfm_oracle.c").write_text(src.replace(old, new, 1))
    shutil.copytree(os.path.join(ROOT, "tests"), work / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    os.symlink(os.path.join(ROOT, "selective_scan_sfm_b200"), work / "selective_scan_sfm_b200")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=work, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "planted mistake %s was not caught:\n%s" % (name, r.stdout[-2000:])
