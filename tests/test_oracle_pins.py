"""Pins of the oracle against what the pages and mathematics fix (CPU only).

Each oracle step is checked against something other than itself: hand-derived
golden cases (tests/golden/), closed forms, library routines (numpy matmul,
numpy convolve, torch's bf16 conversion) and invariants the pages state.
"""

import math
import os

import numpy as np
import pytest

import oracle
import synth


def _load_rows(path):
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append(line.split())
    return rows


# ------------------------------------------------------------------ remap

def test_remap_golden(golden_dir):
    rows = {r[0]: [int(x) for x in r[1:]] for r in _load_rows(os.path.join(golden_dir, "remap_case.txt"))}
    canon, bad = oracle.remap(np.array(rows["tok"]), np.array(rows["P"]))
    assert bad == 0
    assert canon.tolist() == rows["canon"]


def test_remap_out_of_range_marks_invalid():
    P = np.array([1, 0, 2, 1])
    canon, bad = oracle.remap(np.array([0, 4, -1, 3]), P)
    assert bad == 2
    assert canon.tolist() == [1, -1, -1, 1]


# ------------------------------------------------------------------ hash

def test_hash_single_head_golden(golden_dir):
    for r in _load_rows(os.path.join(golden_dir, "hash_cases.txt")):
        n, M, a0, a1, a2, s0, s1, s2, want = (int(x) for x in r)
        s = [s0, s1, s2][:n]
        canon = np.array([list(reversed(s))], dtype=np.int32)  # s_0 is the last position
        mult = np.array([[a0, a1, a2, 0]], dtype=np.uint64)
        idx, bad = oracle.hash_ids(canon, 1 << 30, [n], 1, mult, np.array([M]), t_begin=n - 1)
        assert bad == 0
        assert idx.shape == (1, 1)
        assert int(idx[0, 0]) == want, r


def test_hash_sequence_golden_with_padding(golden_dir):
    rows = _load_rows(os.path.join(golden_dir, "hash_sequence.txt"))
    canon = np.array([[4, 7, 2]], dtype=np.int32)
    mult = np.array([[1, 2, 0, 0], [1, 2, 4, 0]], dtype=np.uint64)
    idx, bad = oracle.hash_ids(canon, 10, [2, 3], 1, mult, np.array([97, 97]))
    assert bad == 0
    for t, i2, i3, _ in ((int(x) for x in r) for r in rows):
        assert idx[t].tolist() == [i2, i3]
    idx13, _ = oracle.hash_ids(canon, 10, [2, 3], 1, mult, np.array([97, 13]))
    for t, i2, _, i3 in ((int(x) for x in r) for r in rows):
        assert idx13[t].tolist() == [i2, i3]
    # decode form: only the last position, n-gram windows reach back into context
    idx_last, _ = oracle.hash_ids(canon, 10, [2, 3], 1, mult, np.array([97, 97]), t_begin=2)
    assert idx_last.tolist() == [idx[2].tolist()]


def test_hash_invalid_canonical_id():
    canon = np.array([[1, -1, 2, 3]], dtype=np.int32)
    mult = np.array([[3, 5, 0, 0]], dtype=np.uint64)
    idx, bad = oracle.hash_ids(canon, 10, [2], 1, mult, np.array([7]))
    # n-grams containing position 1 (t = 1 and t = 2) are invalid
    assert bad == 2
    assert idx[:, 0].tolist()[1:3] == [0xFFFFFFFF, 0xFFFFFFFF]
    assert idx[0, 0] < 7 and idx[3, 0] < 7


@pytest.fixture(scope="module")
def c1():
    inp = synth.Inputs(synth.WORKLOADS["c1"])
    canon, bad = oracle.remap(inp.tok, inp.P)
    assert bad == 0
    idx, badh = oracle.hash_ids(canon, inp.wl.Vc, inp.wl.orders, inp.wl.K, inp.mult, inp.rows)
    assert badh == 0
    return inp, canon, idx


def _ngrams_bruteforce(seq, n, pad):
    """Naive listing of suffix n-grams (most recent first), padded at the start."""
    out = []
    for t in range(len(seq)):
        out.append(tuple(seq[t - j] if t - j >= 0 else pad for j in range(n)))
    return out


def test_hash_indices_in_range_and_deterministic(c1):
    inp, canon, idx = c1
    wl = inp.wl
    assert idx.shape == (wl.n_tok, wl.J)
    assert np.all(idx < wl.M)
    for o, n in enumerate(wl.orders):
        grams = _ngrams_bruteforce(canon[0].tolist(), n, wl.Vc)
        seen = {}
        for t, g in enumerate(grams):
            tup = tuple(idx[t, o * wl.K:(o + 1) * wl.K].tolist())
            if g in seen:
                # equal n-grams at different positions give equal indices
                assert seen[g] == tup
            else:
                seen[g] = tup
        # distinct n-grams never collide on all K heads at this size
        assert len(set(seen.values())) == len(seen)


def test_hash_collisions_within_birthday_bound():
    # many distinct n-grams into a small prime table: per-head collision count
    # near the birthday expectation n_d^2 / (2M)
    wl = synth.WORKLOADS["c1"].replace(T=4096, B=4)
    inp = synth.Inputs(wl)
    canon, _ = oracle.remap(inp.tok, inp.P)
    M = 10007
    idx, _ = oracle.hash_ids(canon, wl.Vc, wl.orders, wl.K, inp.mult, np.full(wl.J, M))
    for o, n in enumerate(wl.orders):
        distinct = {}
        for b in range(wl.B):
            grams = _ngrams_bruteforce(canon[b].tolist(), n, wl.Vc)
            for t, g in enumerate(grams):
                distinct.setdefault(g, b * wl.T + t)
        nd = len(distinct)
        rows = np.array(list(distinct.values()))
        expect = nd * (nd - 1) / (2.0 * M)
        for k in range(wl.K):
            col = idx[rows, o * wl.K + k]
            _, counts = np.unique(col, return_counts=True)
            pairs = float(np.sum(counts * (counts - 1) / 2))
            assert 0.7 * expect < pairs < 1.3 * expect, (n, k, nd, pairs, expect)


def test_hash_depends_only_on_ids(c1):
    inp, canon, idx = c1
    # the same ids placed in another sequence slot give the same indices
    wl = inp.wl
    two = np.concatenate([canon, canon], axis=0)
    idx2, _ = oracle.hash_ids(two, wl.Vc, wl.orders, wl.K, inp.mult, inp.rows)
    assert np.array_equal(idx2[: wl.T], idx) and np.array_equal(idx2[wl.T:], idx)


# ------------------------------------------------------------------ gather

def test_gather_matches_numpy_take():
    rng = np.random.default_rng(3)
    J, M, D, n = 5, 11, 7, 40
    tables = rng.standard_normal((J, M, D)).astype(np.float32)
    idx = rng.integers(0, M, size=(n, J)).astype(np.uint32)
    idx[3, 2] = M        # out of range -> zero row
    idx[7, 0] = 0xFFFFFFFF
    e = oracle.gather(idx, np.full(J, M), tables)
    want = np.concatenate([np.where((idx[:, j] < M)[:, None], tables[j][np.minimum(idx[:, j], M - 1)], 0)
                           for j in range(J)], axis=1)
    assert np.array_equal(e, want)
    # bit patterns (bf16 stored as uint16) are copied exactly
    bits = rng.integers(0, 65535, size=(J, M, D)).astype(np.uint16)
    eb = oracle.gather(idx, np.full(J, M), bits)
    assert eb.dtype == np.uint16
    assert np.array_equal(eb[5].reshape(J, D), np.stack([bits[j, idx[5, j]] for j in range(J)]))


def test_gather_rows_matches_full_gather(c1):
    inp, canon, idx = c1
    tables = inp.all_tables()
    e_full = oracle.gather(idx, inp.rows, tables)
    e_rows = oracle.gather_rows(idx, inp.rows, inp.table_rows)
    assert np.array_equal(e_full, e_rows.astype(np.float32))


# ------------------------------------------------------------------ projections

def test_gather_rows_zero_rows_for_invalid_indices():
    """An index >= M_j, and the invalid-n-gram marker 0xFFFFFFFF, gather a zero
    row; every other index gathers its table row (numpy indexing)."""
    M, D, J = 11, 4, 3
    tables = (np.arange(J * M * D, dtype=np.float64).reshape(J, M, D) + 1.0)
    idx = np.array([[0, 10, 11], [0xFFFFFFFF, 5, 12], [3, 0xFFFFFFFF, 0], [11, 11, 10]], dtype=np.uint32)
    got = oracle.gather_rows(idx, np.full(J, M, dtype=np.uint32), lambda j, r: tables[j][r])
    want = np.zeros((idx.shape[0], J * D))
    for i in range(idx.shape[0]):
        for j in range(J):
            if idx[i, j] < M:
                want[i, j * D:(j + 1) * D] = tables[j, idx[i, j]]
    assert np.array_equal(got, want)
    assert np.count_nonzero(np.all(got.reshape(-1, J, D) == 0, axis=2)) == 6


def test_project_matches_numpy_matmul():
    rng = np.random.default_rng(5)
    e = rng.standard_normal((9, 13))
    W = rng.standard_normal((6, 13))
    np.testing.assert_allclose(oracle.project(e, W), e @ W.T, rtol=1e-12, atol=1e-12)


def test_project_identity_returns_e():
    rng = np.random.default_rng(6)
    e = rng.standard_normal((4, 8))
    W = np.vstack([np.eye(8), np.zeros((3, 8))])  # d_mem <= d, W = [I; 0]
    k = oracle.project(e, W)
    assert np.array_equal(k[:, :8], e) and np.all(k[:, 8:] == 0)


# ------------------------------------------------------------------ gate

def test_gate_orthogonal_is_half():
    h = np.array([[1.0, 1.0, 0.0, 0.0]])
    k = np.array([[0.0, 0.0, 1.0, -1.0]])
    a = oracle.gate(h, k, np.ones(4), np.ones(4), 1e-6)
    assert a[0] == 0.5


@pytest.mark.parametrize("c", [0.3, 1.0, 4.0])
def test_gate_parallel_closed_form(c):
    rng = np.random.default_rng(7)
    d = 64
    h = rng.standard_normal((1, d))
    eps = 1e-6
    m = np.mean(h * h)
    dot = d * c * m / (math.sqrt(m + eps) * math.sqrt(c * c * m + eps))
    want = 1.0 / (1.0 + math.exp(-dot / math.sqrt(d)))
    got = oracle.gate(h, c * h, np.ones(d), np.ones(d), eps)[0]
    assert abs(got - want) < 1e-14
    got_neg = oracle.gate(h, -c * h, np.ones(d), np.ones(d), eps)[0]
    assert abs(got_neg - (1.0 - want)) < 1e-14
    # with d = 64 the aligned key gives sigma(~8) -> near 1, the opposed one near 0
    assert got > 0.999 and got_neg < 0.001


def test_gate_gains_scale_the_logit():
    rng = np.random.default_rng(8)
    d = 32
    h = rng.standard_normal((3, d))
    k = rng.standard_normal((3, d))
    a1 = oracle.gate(h, k, np.ones(d), np.ones(d), 1e-6)
    a6 = oracle.gate(h, k, np.full(d, 2.0), np.full(d, 3.0), 1e-6)
    logit = lambda a: np.log(a / (1 - a))
    np.testing.assert_allclose(logit(a6), 6.0 * logit(a1), rtol=1e-10)


def test_gate_in_open_unit_interval():
    rng = np.random.default_rng(9)
    a = oracle.gate(rng.standard_normal((200, 48)) * 5, rng.standard_normal((200, 48)),
                    np.ones(48), np.ones(48), 1e-6)
    assert np.all(a > 0) and np.all(a < 1)


# ------------------------------------------------------------------ conv

def test_conv_matches_numpy_convolve():
    rng = np.random.default_rng(10)
    L, d, w = 20, 5, 4
    vt = rng.standard_normal((L, d))
    cw = rng.standard_normal((d, w))
    u = oracle.conv(vt, cw)
    for c in range(d):
        np.testing.assert_allclose(u[:, c], np.convolve(vt[:, c], cw[c])[:L], rtol=1e-12, atol=1e-12)


def test_conv_impulse_response_and_causality():
    rng = np.random.default_rng(11)
    L, d, w = 12, 3, 4
    cw = rng.standard_normal((d, w))
    vt = np.zeros((L, d))
    vt[5] = 1.0
    u = oracle.conv(vt, cw)
    for j in range(w):
        assert np.array_equal(u[5 + j], cw[:, j])
    assert np.all(u[:5] == 0) and np.all(u[5 + w:] == 0)
    base = rng.standard_normal((L, d))
    pert = base.copy()
    pert[7] += 3.0
    ub, up = oracle.conv(base, cw), oracle.conv(pert, cw)
    assert np.array_equal(ub[:7], up[:7])
    assert not np.allclose(ub[7], up[7])


def test_conv_history_equals_concatenation():
    rng = np.random.default_rng(12)
    L, d, w = 6, 4, 4
    cw = rng.standard_normal((d, w))
    hist = rng.standard_normal((w - 1, d))
    vt = rng.standard_normal((L, d))
    u = oracle.conv(vt, cw, hist)
    u_cat = oracle.conv(np.vstack([hist, vt]), cw)[w - 1:]
    np.testing.assert_allclose(u, u_cat, rtol=0, atol=1e-15)


def test_output_special_cases():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 0.7310585786300049) < 1e-15
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    rng = np.random.default_rng(13)
    vt = rng.standard_normal((8, 3))
    h = rng.standard_normal((8, 3))
    zero_u = oracle.conv(vt, np.zeros((3, 4)))
    assert np.array_equal(oracle.output(vt, zero_u, h, False), vt)        # conv_w = 0 -> Y = v~
    assert np.array_equal(oracle.output(vt, zero_u, h, True), vt + h)     # plus the residual
    cw = np.zeros((3, 4))
    cw[:, 1] = [0.5, -2.0, 1.5]                                            # one-hot tap j = 1
    y = oracle.output(vt, oracle.conv(vt, cw), h, False)
    for t in range(1, 8):
        for c in range(3):
            x = cw[c, 1] * vt[t - 1, c]
            assert abs(y[t, c] - (vt[t, c] + x / (1 + math.exp(-x)))) < 1e-14


# ------------------------------------------------------------------ whole path

def test_forward_full_c1_properties(c1):
    inp, canon, idx = c1
    r = oracle.forward_full(inp)
    assert np.array_equal(r.idx, idx)
    assert np.all(r.alpha > 0) and np.all(r.alpha < 1)
    # the gate is not saturated on these inputs
    assert 0.05 < np.std(r.alpha) < 0.45
    assert np.all(np.isfinite(r.y))
    assert np.max(np.abs(r.y)) < 4.0


def test_forward_rows_equals_forward_full(c1):
    inp, _, _ = c1
    full = oracle.forward_full(inp, add_residual=True)
    pos = synth.sample_positions(inp.wl, 24, seed=1)
    rows = oracle.forward_rows(inp, pos, add_residual=True)
    np.testing.assert_allclose(rows.y, full.y[pos], rtol=0, atol=1e-12)
    np.testing.assert_allclose(rows.alpha, full.alpha[pos], rtol=0, atol=1e-15)


def test_decode_step_equals_last_prefill_row(c1):
    inp, _, _ = c1
    wl = inp.wl
    full = oracle.forward_full(inp)
    dec_wl = wl.replace(t_begin=wl.T - 1)
    dec = synth.Inputs(dec_wl)
    hist = full.vt[None, wl.T - wl.w:wl.T - 1]        # the last w-1 gated rows before t = T-1
    dec.hidden_rows = lambda rows: inp.hidden_rows(np.asarray(rows) + (wl.T - 1))
    r = oracle.forward_rows(dec, np.array([0]), hist=hist)
    np.testing.assert_allclose(r.y[0], full.y[wl.T - 1], rtol=0, atol=1e-12)


# ------------------------------------------------------------------ batches of sequences

def _one_sequence(inp, b, tables, h_all):
    """The inputs of sequence b alone, as a workload with B = 1."""
    import types
    wl = inp.wl
    L = wl.T - wl.t_begin
    one = types.SimpleNamespace(**{k: getattr(inp, k) for k in ("P", "mult", "rows", "Wk", "Wv", "gq", "gk",
                                                                    "conv_w")})
    one.wl = wl.replace(B=1)
    one.tok = inp.tok[b:b + 1]
    return one, h_all[b * L:(b + 1) * L]


@pytest.fixture(scope="module")
def c1_batch():
    inp = synth.Inputs(synth.WORKLOADS["c1"].replace(name="c1b3", B=3, T=96, seed=21), gamma="random")
    return inp, inp.all_tables(), inp.all_hidden()


@pytest.mark.parametrize("with_hist", [False, True])
def test_batch_equals_independent_sequences(c1_batch, with_hist):
    """The conv is causal within each sequence ("DeepSeek AI II" digest,
    section "DeepSeek Engram": per-channel causal convolution over a
    sequence): a batch of three sequences gives, row for row, what three
    single-sequence runs give, each with its own history (zero or its own
    conv_state row)."""
    inp, tables, h_all = c1_batch
    wl = inp.wl
    L = wl.T
    hist = inp.state_rows(np.arange(wl.B)) if with_hist else None
    batch = oracle.forward_full(inp, add_residual=True, tables=tables, h=h_all, hist=hist)
    for b in range(wl.B):
        one, h_b = _one_sequence(inp, b, tables, h_all)
        r = oracle.forward_full(one, add_residual=True, tables=tables, h=h_b,
                                hist=None if hist is None else hist[b:b + 1])
        np.testing.assert_array_equal(batch.y[b * L:(b + 1) * L], r.y)
        np.testing.assert_array_equal(batch.alpha[b * L:(b + 1) * L], r.alpha)
    # the sequences differ, so a history leaking across them would show
    assert not np.allclose(batch.y[:4], batch.y[L:L + 4])


@pytest.mark.parametrize("with_hist", [False, True])
def test_forward_rows_equals_forward_full_batch(c1_batch, with_hist):
    """forward_rows (one position at a time, its window rebuilt per sequence)
    against forward_full on B = 3: every sequence's first four and last rows."""
    inp, tables, h_all = c1_batch
    wl = inp.wl
    L = wl.T
    hist = inp.state_rows(np.arange(wl.B)) if with_hist else None
    full = oracle.forward_full(inp, add_residual=True, tables=tables, h=h_all, hist=hist)
    pos = np.array([b * L + t for b in range(wl.B) for t in (0, 1, 2, 3, L - 1)], dtype=np.int64)
    rows = oracle.forward_rows(inp, pos, add_residual=True, hist=hist)
    np.testing.assert_allclose(rows.y, full.y[pos], rtol=0, atol=1e-12)
    np.testing.assert_allclose(rows.alpha, full.alpha[pos], rtol=0, atol=1e-15)
    np.testing.assert_allclose(rows.vt_win, oracle.vt_windows(full.vt, wl.B, L, wl.w, hist)[pos], rtol=0, atol=1e-15)


# ------------------------------------------------------------------ multi-branch

@pytest.fixture(scope="module")
def mb():
    inp = synth.Inputs(synth.WORKLOADS["c1"].replace(name="mb", B=2, T=80, seed=23), gamma="random")
    branches = [synth.branch_inputs(inp, m) for m in range(3)]
    return inp, branches, inp.all_tables()


def _hybrid(inp, br):
    """branch br's key, gains and hidden rows on inp's tokens, tables, W_V and taps."""
    import types
    one = types.SimpleNamespace(**{k: getattr(inp, k) for k in ("wl", "tok", "P", "mult", "rows", "Wv", "conv_w")})
    one.Wk, one.gq, one.gk = br.Wk, br.gq, br.gk
    one.hidden_rows = br.hidden_rows
    one.table_rows = inp.table_rows
    return one


def test_multibranch_one_branch_is_the_single_branch_forward(mb):
    inp, branches, tables = mb
    r = oracle.forward_multibranch(branches[:1], add_residual=True, tables=tables)
    f = oracle.forward_full(inp, add_residual=True, tables=tables)
    np.testing.assert_array_equal(r.y[0], f.y)
    np.testing.assert_array_equal(r.alpha[0], f.alpha)


@pytest.mark.parametrize("with_hist", [False, True])
def test_multibranch_branch_m_uses_its_own_key_and_hidden(mb, with_hist):
    """Branch m equals the single-branch module run with W_K^(m), its gains and
    h^(m) on the shared tables, W_V and taps (the pages: one W_V, M W_K, a gate
    per branch applied to the shared value)."""
    inp, branches, tables = mb
    M = len(branches)
    hist = np.stack([b.state_rows(np.arange(inp.wl.B)) for b in branches]) if with_hist else None
    r = oracle.forward_multibranch(branches, add_residual=True, tables=tables, hist=hist)
    assert r.y.shape == (M, inp.wl.n_tok, inp.wl.d)
    for m in range(M):
        f = oracle.forward_full(_hybrid(inp, branches[m]), add_residual=True, tables=tables,
                                h=branches[m].all_hidden(), hist=None if hist is None else hist[m])
        np.testing.assert_array_equal(r.y[m], f.y)
        np.testing.assert_array_equal(r.alpha[m], f.alpha)
    # the branches differ, and they share v: v~^(m) / alpha^(m) is the same vector
    assert not np.allclose(r.alpha[0], r.alpha[1])
    np.testing.assert_allclose(r.vt[1] / r.alpha[1][:, None], r.vt[2] / r.alpha[2][:, None], rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------------ table backward

def test_table_grad_brute_force():
    """Against a plain loop over the lookups, on a case small enough to read:
    three tables of 5 rows, rows touched several times, one invalid index."""
    D = 2
    rows = np.array([5, 5, 5], dtype=np.uint32)
    idx = np.array([[0, 4, 2], [0, 1, 2], [3, 0xFFFFFFFF, 2], [0, 4, 7]], dtype=np.uint32)
    de = np.arange(idx.shape[0] * 3 * D, dtype=np.float64).reshape(idx.shape[0], 3 * D) + 1.0
    want = {}
    for t in range(idx.shape[0]):
        for j in range(3):
            if idx[t, j] < 5:
                key = j * 5 + int(idx[t, j])
                want[key] = want.get(key, 0) + de[t, j * D:(j + 1) * D]
    keys, grad = oracle.table_grad(idx, rows, de, D)
    assert keys.tolist() == sorted(want)
    for k, g in zip(keys, grad):
        np.testing.assert_array_equal(g, want[int(k)])
    # table 0 row 0 three times: 1+2, 7+8, 19+20 -> [1+7+19, 2+8+20]
    np.testing.assert_array_equal(grad[list(keys).index(0)], [27.0, 30.0])


def test_table_grad_conserves_the_total(c1):
    """The gradients of all rows add up to the sum of every valid slice of
    dL/de (nothing lost, nothing counted twice)."""
    inp, _, idx = c1
    wl = inp.wl
    rng = np.random.default_rng(3)
    de = rng.standard_normal((wl.n_tok, wl.d_mem))
    keys, grad = oracle.table_grad(idx, inp.rows, de, wl.D)
    assert len(np.unique(keys)) == len(keys)
    valid = (idx.astype(np.int64) < inp.rows[None, :].astype(np.int64))
    total = de.reshape(wl.n_tok, wl.J, wl.D)[valid].sum(axis=0)
    np.testing.assert_allclose(grad.sum(axis=0), total, rtol=0, atol=1e-9)
    assert len(keys) == len(np.unique((idx.astype(np.int64) + (np.arange(wl.J) * wl.M)[None, :])[valid]))


def test_table_grad_of_a_union_is_the_sum_of_the_parts():
    """The sharded backward rests on linearity: the gradient of the union of
    the ranks' batches is, row by row, the sum of each rank's own gradient
    (a row missing from a rank contributes nothing).  Three batches with
    integer-valued slices, so every sum is exact."""
    D, J, M = 3, 2, 7
    rows = np.full(J, M, dtype=np.uint32)
    rng = np.random.default_rng(11)
    parts = []
    for r in range(3):
        n = 5 + 4 * r
        idx = rng.integers(0, M, size=(n, J)).astype(np.uint32)
        idx[0, 1] = 0xFFFFFFFF                                   # an invalid lookup in every batch
        de = rng.integers(-5, 6, size=(n, J * D)).astype(np.float64)
        parts.append((idx, de))
    keys_u, grad_u = oracle.table_grad(np.concatenate([p[0] for p in parts]), rows,
                                       np.concatenate([p[1] for p in parts]), D)
    total = {}
    for idx, de in parts:
        keys, grad = oracle.table_grad(idx, rows, de, D)
        for k, g in zip(keys.tolist(), grad):
            total[k] = total.get(k, 0) + g
    assert keys_u.tolist() == sorted(total)
    for k, g in zip(keys_u.tolist(), grad_u):
        np.testing.assert_array_equal(g, total[k])


# ------------------------------------------------------------------ FP8 E4M3 codes

def test_decode_e4m3_hand_values_and_all_codes():
    assert oracle.decode_e4m3(np.array([0x38]))[0] == 1.0          # exponent 7 = bias, mantissa 0
    assert oracle.decode_e4m3(np.array([0xB8]))[0] == -1.0
    assert oracle.decode_e4m3(np.array([0x7E]))[0] == 448.0        # 1.75 * 2^8, the largest finite value
    assert oracle.decode_e4m3(np.array([0x01]))[0] == 2.0 ** -9    # smallest subnormal, 1/8 * 2^-6
    assert oracle.decode_e4m3(np.array([0x08]))[0] == 2.0 ** -6    # smallest normal
    assert oracle.decode_e4m3(np.array([0x3C]))[0] == 1.5
    assert np.isnan(oracle.decode_e4m3(np.array([0x7F, 0xFF]))).all()
    assert oracle.decode_e4m3(np.array([0x80]))[0] == 0.0
    # every code against torch's float8_e4m3fn conversion (a library routine)
    import torch
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
