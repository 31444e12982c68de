"""The seeded input generators (CPU only)."""

import numpy as np

import synth


def test_splitmix64_published_outputs():
    # first outputs of SplitMix64 seeded with 0 (reference implementation by
    # Sebastiano Vigna, splitmix64.c)
    assert synth.splitmix64_stream(0, 3) == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_surjection_is_onto_and_23_percent_smaller():
    for name in ("c1", "c2"):
        wl = synth.WORKLOADS[name]
        P = synth.surjection(wl)
        assert P.shape == (wl.V,)
        assert P.min() >= 0 and P.max() < wl.Vc
        assert len(np.unique(P)) == wl.Vc
        assert abs(1 - wl.Vc / wl.V - 0.23) < 0.005


def test_zipf_tokens_rank_frequency():
    wl = synth.WORKLOADS["c2"]
    tok = synth.zipf_tokens(wl, B=1, T=200000)
    cnt = np.bincount(tok.ravel(), minlength=wl.V)
    assert tok.min() >= 0 and tok.max() < wl.V
    # frequency of rank r ~ r^-s: ratio between ranks 1 and 10 near 10^1.1
    ratio = cnt[0] / cnt[9]
    assert 8.0 < ratio < 17.0


def test_multipliers_odd_and_layout():
    wl = synth.WORKLOADS["c2"]
    a = synth.hash_multipliers(wl)
    assert a.shape == (wl.J, 4)
    for o, n in enumerate(wl.orders):
        for k in range(wl.K):
            row = a[o * wl.K + k]
            assert all(int(x) & 1 for x in row[:n])
            assert all(int(x) == 0 for x in row[n:])
    assert len({int(x) for x in a[a != 0]}) == int(np.count_nonzero(a))


def test_normal_values_statistics_and_torch_agreement():
    import torch
    v = synth.normal_np(1, synth.TAG_TABLES, np.arange(1 << 18), 1.0)
    assert abs(float(v.mean())) < 0.01 and abs(float(v.std()) - 1.0) < 0.01
    assert float(np.abs(v).max()) <= 2.0 * np.sqrt(3.0) + 1e-6
    t = synth.normal_torch(1, synth.TAG_TABLES, 1000, 5000, 0.02, "cpu").numpy()
    assert np.array_equal(t, synth.normal_np(1, synth.TAG_TABLES, np.arange(1000, 6000), 0.02))


def test_bf16_helpers():
    x = synth.to_bf16_values(np.array([1.0 + 2 ** -8, 3.0, -0.5], dtype=np.float32))
    assert x.tolist() == [1.0, 3.0, -0.5]
    assert synth.bf16_bits(x).tolist() == [0x3F80, 0x4040, 0xBF00]


def test_sample_positions_cover_sequence_edges():
    wl = synth.WORKLOADS["c2"]
    pos = synth.sample_positions(wl, 64)
    L = wl.T
    for b in range(wl.B):
        for t in (0, 1, 2, 3, L - 1):
            assert b * L + t in pos
    assert pos.max() < wl.n_tok
