"""The benchmark's DRAM-traffic bookkeeping: a captured figure is reported
only while the kernel's code is the code that was captured.  Editing a
comment leaves the digest alone; editing code changes it."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


SRC = """// leading comment
__global__ void k(int* x) {
    /* block
       comment */
    x[0] = 1;   // trailing comment

}
"""


def _digest(m, text):
    return m.source_digest(["a.cu"], read=lambda name: text)


def test_comment_edits_keep_the_digest():
    m = _bench()
    base = _digest(m, SRC)
    assert _digest(m, SRC.replace("leading comment", "another note")) == base
    assert _digest(m, SRC.replace("trailing comment", "")) == base
    assert _digest(m, SRC.replace("/* block\n       comment */", "")) == base
    assert _digest(m, SRC + "\n\n// appended note\n") == base


def test_code_edits_change_the_digest():
    m = _bench()
    base = _digest(m, SRC)
    assert _digest(m, SRC.replace("x[0] = 1;", "x[0] = 2;")) != base
    assert _digest(m, SRC.replace("int* x", "long* x")) != base


def test_captured_traffic_matches_current_sources_or_is_none():
    m = _bench()
    for (workload, kernel), (digest, nbytes) in m.CAPTURED_TRAFFIC.items():
        got = m.captured_traffic(workload, kernel)
        current = m.source_digest(m.KERNEL_SOURCES[kernel])
        assert got == (nbytes if current == digest else None)
    assert m.captured_traffic("c2", "no_such_kernel") is None
    assert m.captured_traffic("no_such_workload", "vconv_tc") is None


def test_table_grad_bytes_by_hand():
    """Two tokens, two tables of 4-wide bf16 rows, three distinct rows: the
    reduce reads 2*2 slices of 8 bytes and writes 3 sums of 16 bytes; the
    update reads the 3 sums and 3 row ids and reads and writes 3 rows of 8
    bytes; the step adds the 4 indices read and the 3 row ids written."""
    m = _bench()
    b = m.table_grad_bytes(n=2, J=2, D=4, es=2, U=3)
    assert b["grad_reduce"] == 4 * 8 + 3 * 16
    assert b["table_sgd"] == 3 * 16 + 3 * 8 + 2 * 3 * 8
    assert b["step"] == b["grad_reduce"] + b["table_sgd"] + 4 * 4 + 3 * 8
