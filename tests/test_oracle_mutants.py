"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C++ source (on the CPU,
never in the product), builds it, and runs the pin suite against it through
GDN_ORACLE_LIB.  The suite must fail for every mutant.
"""
import os
import pathlib
import subprocess
import sys

import pytest

ROOT = pathlib.Path(__file__).resolve().parent.parent
SRC = (ROOT / "oracle" / "gdn_oracle.cpp").read_text()

MUTANTS = {
    "sign_of_projection": ("(r == c ? 1.0 : 0.0) - be * kv[r] * kv[c]", "(r == c ? 1.0 : 0.0) + be * kv[r] * kv[c]"),
    "beta_dropped_from_write": ("a * SP[j * dk + i] + be * vv[j] * kv[i]", "a * SP[j * dk + i] + vv[j] * kv[i]"),
    "alpha_on_write_term": ("a * SP[j * dk + i] + be * vv[j] * kv[i]", "a * (SP[j * dk + i] + be * vv[j] * kv[i])"),
    "state_transposed": ("S[j * dk + i] = static_cast<double>(M[i * dv + j]);", "S[j * dk + i] = static_cast<double>(M[j * dk + i]);"),
    "key_head_modulo": ("const int64_t hk = h / G;", "const int64_t hk = h % p.Hk;"),
    "readout_with_k": ("acc += static_cast<double>(Sf[j * dk + i]) * qv[i];", "acc += static_cast<double>(Sf[j * dk + i]) * kv[i];"),
    "carry_unrounded": ("S[j * dk + i] = static_cast<double>(Sf[j * dk + i]);", "S[j * dk + i] = s_new;"),
    "commit_first_token": ("cur[b * T + (a - 1)]", "cur[b * T]"),
    "skip_check_dropped": ("if (d < 0 || d >= p.num_slots) return false;", "(void)d;"),
    "fused_beta_sign": ("double beta_of(double y) { return 1.0 / (1.0 + std::exp(-y)); }",
                        "double beta_of(double y) { return 1.0 / (1.0 + std::exp(y)); }"),
    "fused_alpha_softplus_sign": ("double alpha_of(double x) { return std::exp(-softplus(x)); }",
                                  "double alpha_of(double x) { return std::exp(-softplus(-x)); }"),
    "fused_norm_without_sqrt": ("const double n = std::sqrt(ss + 1e-6);", "const double n = ss + 1e-6;"),
    "check_in_place_for_all_T": ("if (w != b || T > 1) return 5;", "if (w != b) return 5;"),
    "check_ignores_padding_flag": ("auto live = [&](int64_t b) { return src_idx[b] != -1; };",
                                   "auto live = [&](int64_t b) { return b >= 0; };"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    src = tmp_path / "mutant.cpp"
    src.write_text(SRC.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    "-o", str(lib), str(src)], check=True)
    env = dict(os.environ, GDN_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        str(ROOT / "tests" / "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pin suite:\n{r.stdout[-2000:]}"
