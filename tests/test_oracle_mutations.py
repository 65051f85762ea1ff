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


# mistakes in the ragged composition (oracle/__init__.py), caught by test_oracle_ragged_pins.py
RAGGED_MUTATIONS = {
    "ragged_x_offset": ("return (a - 2 * s, e - 2 * s - 2) if aux else (a, e)",
                        "return (a - s, e - s - 2) if aux else (a, e)"),
    "ragged_swap_dropped": ("aux_init_in=aux_init_in, swap_out=swap_out, pad_left=pad_left, dt_softplus=dt_softplus,\n"
                            "                          want_state=want_state)",
                            "aux_init_in=aux_init_in, swap_out=False, pad_left=pad_left, dt_softplus=dt_softplus,\n"
                            "                          want_state=want_state)"),
    "literal_no_reset": ("carried = np.zeros_like(h) if p in starts else np.exp(delta[:, p:p + 1] * Af) * h",
                         "carried = np.exp(delta[:, p:p + 1] * Af) * h"),
    "literal_conv_crosses_offsets": ("if 0 <= q < Lt and owner[q] == owner[p] and owner[p] >= 0:",
                                     "if 0 <= q < Lt and owner[p] >= 0:"),
    "literal_reset_multiplies": ("carried = np.zeros_like(h) if p in starts else np.exp(delta[:, p:p + 1] * Af) * h",
                                 "carried = (0.0 if p in starts else np.exp(delta[:, p:p + 1] * Af)) * h"),
}


def _run_mutated(tmp_path, fname, old, new, pins, name):
    src = open(os.path.join(ROOT, "oracle", fname)).read()
    assert src.count(old) >= 1, "mutation site moved: " + name
    work = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (work / "oracle" / fname).write_text(src.replace(old, new, 1))
    shutil.copytree(os.path.join(ROOT, "tests"), work / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    os.symlink(os.path.join(ROOT, "selective_scan_sfm_b200"), work / "selective_scan_sfm_b200")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", pins], cwd=work,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "planted mistake %s was not caught:\n%s" % (name, r.stdout[-2000:])


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTATIONS[name]
    _run_mutated(tmp_path, "sfm_oracle.c", old, new, "tests/test_oracle_pins.py", name)


@pytest.mark.parametrize("name", sorted(RAGGED_MUTATIONS))
def test_ragged_pins_catch_planted_mistake(tmp_path, name):
    old, new = RAGGED_MUTATIONS[name]
    _run_mutated(tmp_path, "__init__.py", old, new, "tests/test_oracle_ragged_pins.py", name)
