"""Plant plausible mistakes in a copy of the oracle source and check that the
pins in test_oracle_pins.py catch each one (CPU only).

A mutant of the C++ steps is compiled into a temporary library and the pin
tests run against it in a child process through ``ORACLE_LIB``.  A mutant of
the Python composition (``oracle/__init__.py``: the per-sequence split of the
conv, the zero rows of the row gather, the sequence of a sampled row) goes
into a copy of the package that ``ORACLE_PKG`` puts first on the child's
import path.  A mutant survives if all pins still pass."""

import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "engram_oracle.cpp")
PY = os.path.join(ROOT, "oracle", "__init__.py")

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
}

PY_MUTANTS = {
    # one conv over the flat [B*L][d] rows: history leaks from sequence b-1 into b
    "conv_no_sequence_split": ("    for b in range(wl.B):\n        seg = slice(b * L, (b + 1) * L)\n",
                               "    for b in range(wl.B):\n        seg = slice(0, wl.B * L)\n"),
    "multibranch_no_sequence_split": ("        for b in range(wl.B):\n            seg = slice(b * L, (b + 1) * L)\n",
                                      "        for b in range(wl.B):\n            seg = slice(0, wl.B * L)\n"),
    # every sequence takes the first sequence's conv history
    "conv_history_wrong_sequence": ("u[seg] = conv(vt[seg], inp.conv_w, None if hist is None else hist[b])",
                                    "u[seg] = conv(vt[seg], inp.conv_w, None if hist is None else hist[0])"),
    "rows_history_wrong_sequence": ("u = conv(seg, inp.conv_w, hist[b])[-1:]",
                                    "u = conv(seg, inp.conv_w, hist[0])[-1:]"),
    # an index >= M_j gathers row 0 instead of a zero row
    "gather_rows_no_zeroing": ("        vals = np.where(ok[:, None], vals, 0)\n", ""),
    # every branch gated with branch 0's key projection
    "multibranch_shared_key": ("        k = project(e, br.Wk)\n", "        k = project(e, branches[0].Wk)\n"),
    # every branch convolved with branch 0's history
    "multibranch_history_of_branch0": ("None if hist is None else hist[m][b])", "None if hist is None else hist[0][b])"),
    # the table gradient counts invalid lookups as row 0's
    "table_grad_keeps_invalid": ("    valid = r < np.asarray(rows, dtype=np.int64)[None, :]\n",
                                 "    valid = r < np.iinfo(np.int64).max\n"),
    # the table gradient without the table offsets (tables' rows collide)
    "table_grad_no_offset": ("    keys = (r + off[None, :])[valid]\n", "    keys = r[valid]\n"),
    # E4M3 exponent bias 8 instead of 7
    "e4m3_bias": ("np.exp2((e - 7).astype(np.float64))", "np.exp2((e - 8).astype(np.float64))"),
    # subnormals without the 2^-6 scale
    "e4m3_subnormal": ("m / 8.0 * 2.0 ** -6", "m / 8.0 * 2.0 ** -7"),
    # a sampled row's window taken from the wrong sequence
    "rows_sequence_index": ("    for p in positions:\n        b, t = divmod(int(p), L)\n",
                            "    for p in positions:\n        b, t = divmod(int(p), L + 1)\n"),
}


def _run_pins(env):
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


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
    r = _run_pins(env)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_kill_python_mutant(name, tmp_path):
    import oracle
    old, new = PY_MUTANTS[name]
    src = open(PY).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique in the oracle package"
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(src.replace(old, new))
    env = dict(os.environ, ORACLE_PKG=str(tmp_path), ORACLE_LIB=oracle.build())
    r = _run_pins(env)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """The copy mechanism itself: the unchanged package passes the pins."""
    import oracle
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(PY).read())
    env = dict(os.environ, ORACLE_PKG=str(tmp_path), ORACLE_LIB=oracle.build())
    r = _run_pins(env)
    assert r.returncode == 0, r.stdout[-2000:]
