"""Host side of the host-memory tier, on the CPU: the row packing that the
tier's threads run (engram_pack_rows is the same routine behind a C call)
and the rule that sizes the host-memory workload to the machine."""

import numpy as np
import pytest

import synth


@pytest.fixture(scope="module")
def eb():
    import hashed_gram_embedding_02_b200 as eb
    return eb


@pytest.mark.parametrize("n_threads", [1, 3, 16])
def test_pack_rows_equals_fancy_indexing(eb, n_threads):
    rng = np.random.default_rng(7)
    total, row_bytes = 5003, 256
    tables = rng.integers(0, 256, size=(total, row_bytes), dtype=np.uint8)
    rows = rng.integers(0, total, size=12345).astype(np.uint64)      # repeats included
    dst = np.zeros((len(rows), row_bytes), dtype=np.uint8)
    eb.engram_pack_rows(tables, total, row_bytes, rows, len(rows), dst, n_threads)
    assert np.array_equal(dst, tables[rows.astype(np.int64)])


def test_pack_rows_rejects_rows_outside_the_tables(eb):
    tables = np.zeros((10, 16), dtype=np.uint8)
    dst = np.full((2, 16), 7, dtype=np.uint8)
    with pytest.raises(eb.EngramError):
        eb.engram_pack_rows(tables, 10, 16, np.array([3, 10], dtype=np.uint64), 2, dst, 2)
    assert (dst == 7).all()                       # checked before any copy
    eb.engram_pack_rows(tables, 10, 16, np.zeros(1, dtype=np.uint64), 0, dst, 1)   # n = 0 is a no-op


def test_host_scaled_picks_the_largest_fitting_prime():
    wl = synth.WORKLOADS["c5"]
    per_row = wl.J * wl.D * 2
    for gib in (1, 7, 90):
        m = synth.host_scaled(wl, gib << 30).M
        assert synth._is_prime(m) and m * per_row <= gib << 30
        nxt = m + 1
        while not synth._is_prime(nxt):
            nxt += 1
        assert nxt * per_row > gib << 30 or nxt > wl.M
    assert synth.host_scaled(wl, 1 << 50).M == wl.M == 48828139
