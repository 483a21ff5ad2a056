"""The seeded synthetic workloads against the statistics they stand in for (the VBQ paper's section 5.1 width
allocation, as read in the design notes): mean bits and width shares of each mix, the LM head's 1.09 mean bits
with 92.5% of rows pure 1-bit, the edge sweep's exactly-half 8-bit rows, value ranges, and seeding."""
import numpy as np

import vbq_synth as S

BITS = np.array([1, 2, 4, 8])


def shares(widths):
    return np.array([(widths == k).mean() for k in BITS])


def test_width_mixes_have_their_stated_means_and_shares():
    g = np.random.default_rng(0)
    for p, mean in ((S.P_BASE, 1.85), (S.P_FIRST_MLP, 2.50), (S.P_HEAD_TOP, 2.20)):
        w = S.widths_iid(4096, 256, p, g)
        assert abs(w.mean() - mean) < 0.01
        assert np.all(np.abs(shares(w) - np.asarray(p)) < 0.003)
        assert abs(float(np.dot(p, BITS)) - mean) < 1e-9


def test_decode_step_layers_use_the_base_mix_and_a_first_block_mlp():
    l0 = {m.name: m for m in S.cfg5_layer(0)}
    l1 = {m.name: m for m in S.cfg5_layer(1)}
    for n in ("q", "o", "gate", "down"):
        assert abs(l1[n].widths.mean() - 1.85) < 0.01
    for n in ("gate", "up", "down"):
        assert abs(l0[n].widths.mean() - 2.50) < 0.01
        assert abs((l0[n].widths == 8).mean() - 0.10) < 0.005
    assert abs(l0["q"].widths.mean() - 1.85) < 0.01
    assert (l0["gate"].N, l0["gate"].K, l0["down"].N, l0["down"].K) == (14336, 4096, 4096, 14336)


def test_lm_head_mean_bits_and_pure_one_bit_rows():
    h = S.cfg5_head()
    assert (h.N, h.K) == (32000, 4096)
    assert abs(h.widths.mean() - 1.09) < 0.005
    pure = np.all(h.widths == 1, axis=1)
    assert pure.mean() == 0.925                              # rows 2400.. are pure 1-bit, rows 0..2399 are not
    assert not pure[:2400].any() and pure[2400:].all()
    extra8 = (h.widths[:1000] == 8).any(axis=1).mean()
    assert 0.04 <= extra8 <= 0.20                           # 4.8% forced, plus the top mix has no 8-bit groups


def test_edge_sweep_rows_are_exactly_half_eight_bit():
    mix = [m for m in S.cfg3() if m.name == "mix1_8"][0]
    per_row = (mix.widths == 8).sum(axis=1)
    assert np.all(per_row == mix.G // 2) and np.all((mix.widths == 1).sum(axis=1) == mix.G // 2)
    starts = np.array([np.flatnonzero(r == 8)[0] for r in mix.widths[:64]])
    assert len(set(starts.tolist())) > 8                    # positions shuffled per row


def test_value_ranges_and_seeding():
    m = S.make_matrix(4, "q", 512, 1024)
    s = m.scales.view(np.float16).astype(np.float64)
    assert s.min() >= 0.0099 and s.max() <= 0.1001
    kk = np.repeat(m.widths.astype(np.int64), 64, axis=1)
    assert np.all(m.codes < (1 << kk))
    for k in (1, 2, 4, 8):                                   # codes uniform over their range
        c = m.codes[kk == k].astype(np.int64)
        assert abs(c.mean() - ((1 << k) - 1) / 2) < 0.05 * (1 << k)
    x = S.make_x(4, "q", 16, 4096).view(np.int16).astype(np.int32) << 16
    xf = x.astype(np.uint32).view(np.float32).astype(np.float64)
    assert abs(xf.mean()) < 0.02 and abs(xf.std() - 1.0) < 0.02
    again = S.make_matrix(4, "q", 512, 1024)
    assert np.array_equal(m.widths, again.widths) and np.array_equal(m.codes, again.codes)
    other = S.make_matrix(4, "k", 512, 1024)
    assert not np.array_equal(m.codes, other.codes)
