"""Seeded input generators: determinism and the workload structure they
promise (shapes, id mix, segment lengths).  No GPU needed."""

import numpy as np

import synth
from synth.workloads import config, zipf_lengths


def test_same_seed_same_bytes():
    a = synth.config(2, seed=77)
    b = synth.workloads._CONFIGS[2](77)
    assert np.array_equal(a.ids, b.ids)
    assert np.array_equal(a.x(0), b.x(0))
    A1, B1 = a.adapter(3, 0)
    A2, B2 = b.adapter(3, 0)
    assert np.array_equal(A1, A2) and np.array_equal(B1, B2)
    assert not np.array_equal(a.adapter(4, 0)[0], A1)


def test_prefetch_matches_single_draws():
    w = synth.workloads._CONFIGS[1](5)
    w2 = synth.workloads._CONFIGS[1](5)
    w.prefetch(range(4), [0], threads=3)
    for s in range(4):
        assert np.array_equal(w.adapter(s, 0)[0], w2.adapter(s, 0)[0])


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 65504.0], dtype=np.float32)
    assert [hex(v) for v in synth.f32_to_bf16_bits(vals)] == ['0x3f80', '0x3f80', '0x3f82', '0xc020', '0x4780']
    assert np.array_equal(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(vals[:2])), [1.0, 1.0])


def test_zipf_lengths():
    assert zipf_lengths(4096, 8, 1.2) == [1753, 764, 470, 333, 255, 205, 171, 145]
    for total, n, s in [(10, 10, 1.0), (1000, 7, 0.8), (33, 2, 3.0)]:
        L = zipf_lengths(total, n, s)
        assert sum(L) == total and min(L) >= 1 and L == sorted(L, reverse=True)


def test_workload_structure():
    w1 = config(1)
    assert w1.T == 16 and set(w1.ids.tolist()) <= {0, 1, 2, 3}
    w3 = config(3)
    assert np.diff(w3.seg_offsets).tolist() == zipf_lengths(4096, 8, 1.2)
    assert sorted(w3.seg_slot.tolist()) == list(range(8))
    w4 = config(4)
    assert (w4.ids == -1).sum() == 26 and set(np.unique(w4.rank)) <= {8, 16, 32, 64}
    assert w4.targets == [(4096, 11008), (11008, 4096)] and w4.r_max == 64
    w5 = config(5)
    assert w5.T == 512 and len(w5.targets) == 128 and w5.active_slots.size == 64
    assert w5.page_bytes == 1 << 20 and w5.n_slots == 1000


def test_value_distributions():
    w = config(2)
    x = synth.bf16_bits_to_f32(w.x(0)).astype(np.float64)
    A, B = w.adapter(0, 0)
    A = synth.bf16_bits_to_f32(A).astype(np.float64)
    B = synth.bf16_bits_to_f32(B).astype(np.float64)
    assert abs(x.std() - 1.0) < 0.02
    assert abs(A.std() * 64 - 1.0) < 0.03               # std 1/sqrt(4096)
    assert abs(B.var() / 0.02 - 1.0) < 0.05
