"""Plant plausible mistakes in a copy of the oracle source and check that the
pins in test_oracle_pins.py catch each one (CPU only).

Each mutant is compiled into a temporary library and the pin tests are run
against it in a child process through ``ORACLE_LIB``; a mutant survives if all
pins still pass."""

import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "engram_oracle.cpp")

MUTANTS = {
    "remap_identity": ("canon[i] = P[x];", "canon[i] = x;"),
    "hash_no_plus_one": ("x ^= (s[j] + 1u) * mult", "x ^= (s[j]) * mult"),
    "hash_sum_not_xor": ("x ^= (s[j] + 1u)", "x += (s[j] + 1u)"),
    "hash_reversed_multipliers": ("mult[jt * 4 + j]", "mult[jt * 4 + (n - 1 - j)]"),
    "hash_pad_zero": ("s[j] = (uint64_t)Vc;  // PAD", "s[j] = 0;"),
    "hash_first_table_prime": ("x % (uint64_t)M[jt]", "x % (uint64_t)M[0]"),
    "gather_no_table_offset": ("off += M[j];", "off += 0;"),
    "project_drops_last_term": ("q < d_mem; ++q) acc", "q < d_mem - 1; ++q) acc"),
    "gate_drops_key_gain": ("(gk[c] * ki[c] / rk)", "(ki[c] / rk)"),
    "gate_no_sqrt_d": ("-dot / std::sqrt((double)d)", "-dot"),
    "gate_sign": ("std::exp(-dot", "std::exp(dot"),
    "gate_sum_not_mean": ("std::sqrt(sh / d + eps)", "std::sqrt(sh + eps)"),
    "gate_eps_outside": ("std::sqrt(sk / d + eps)", "(std::sqrt(sk / d) + eps)"),
    "conv_reversed_taps": ("cw[(int64_t)c * w + j]", "cw[(int64_t)c * w + (w - 1 - j)]"),
    "conv_history_reversed": ("hist[(int64_t)(w - 1 + tt) * d + c]", "hist[(int64_t)(-tt - 1) * d + c]"),
    "silu_is_sigmoid": ("return x / (1.0 + std::exp(-x));", "return 1.0 / (1.0 + std::exp(-x));"),
    "residual_dropped": ("if (add_residual) r += h[i];", "(void)add_residual;"),
    "bf16_truncates": ("std::nearbyint(std::ldexp(m, 8))", "std::trunc(std::ldexp(m, 8))"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_kill_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle source"
    mutant_src = tmp_path / "mutant.cpp"
    mutant_src.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-shared", "-fPIC",
                           "-o", str(lib), str(mutant_src)])
    env = dict(os.environ, ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
