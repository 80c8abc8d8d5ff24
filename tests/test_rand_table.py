"""Pins for the oracle's random block table generator."""

import os

import numpy as np
import pytest
from scipy import stats

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "splitmix64_seed0.txt")


def _golden_values():
    with open(GOLDEN) as f:
        return [int(line, 16) for line in f
                if line.strip() and not line.startswith("#")]


def test_splitmix64_matches_published_outputs():
    rng = oracle.SplitMix64(0)
    assert [rng.next() for _ in range(3)] == _golden_values()


@pytest.mark.parametrize("nb,r", [(1, 3), (2, 3), (3, 2), (4, 3), (5, 1),
                                  (5, 3), (8, 6), (16, 3), (64, 3), (65, 0),
                                  (256, 3), (33, 9)])
def test_table_properties(nb, r):
    H = 4
    t = oracle.rand_table(1234, H, nb, r)
    assert t.shape == (H, nb, r) and t.dtype == np.int32
    for h in range(H):
        for i in range(nb):
            row = t[h, i]
            if i == 0 or i == nb - 1:
                assert (row == -1).all()
                continue
            cand = [j for j in range(1, nb - 1) if abs(j - i) > 1]
            r_eff = min(r, len(cand))
            chosen = row[:r_eff]
            assert (row[r_eff:] == -1).all()
            assert len(set(chosen.tolist())) == r_eff          # distinct
            assert all(c in cand for c in chosen.tolist())      # off-window
            assert (np.diff(chosen) > 0).all()                  # sorted


def test_table_deterministic_and_varies():
    a = oracle.rand_table(5, 3, 32, 3)
    b = oracle.rand_table(5, 3, 32, 3)
    assert np.array_equal(a, b)
    assert not np.array_equal(a[0], a[1])          # heads differ
    c = oracle.rand_table(6, 3, 32, 3)
    assert not np.array_equal(a, c)                # seeds differ


def test_table_uniform_chi_square():
    """Over many seeds each candidate of a row is chosen equally often, and
    the chosen count per row is r."""
    nb, i, r = 12, 5, 3
    cand = [j for j in range(1, nb - 1) if abs(j - i) > 1]
    counts = {j: 0 for j in cand}
    for s in range(6000):
        row = oracle.rand_table(s, 1, nb, r)[0, i]
        for j in row.tolist():
            counts[j] += 1
    obs = np.array([counts[j] for j in cand], dtype=float)
    assert obs.sum() == 6000 * r
    p = stats.chisquare(obs).pvalue
    assert p > 1e-3, p


# ---- the layer's table options: drawn for the maximum length, capped ----

def test_layer_options_off_is_the_base_table():
    for nb, r in ((16, 3), (33, 9), (5, 2)):
        assert np.array_equal(oracle.rand_table(9, 3, nb, r, 0, 0),
                              oracle.rand_table(9, 3, nb, r))
        assert np.array_equal(oracle.rand_table(9, 3, nb, r, nb, 0),
                              oracle.rand_table(9, 3, nb, r))


@pytest.mark.parametrize("nb,nbb,r", [(16, 64, 3), (32, 64, 3), (3, 64, 2),
                                      (40, 41, 6), (64, 64, 3)])
def test_truncation_keeps_the_prefix_of_the_full_build(nb, nbb, r):
    """Rows of a table drawn for nbb blocks and kept for nb are the rows of
    the full nbb-block table restricted to this table's middle blocks."""
    full = oracle.rand_table(3, 4, nbb, r)
    part = oracle.rand_table(3, 4, nb, r, max_blocks=nbb)
    for h in range(4):
        assert (part[h, 0] == -1).all() and (part[h, nb - 1] == -1).all()
        for i in range(1, nb - 1):
            want = sorted(j for j in full[h, i].tolist()
                          if 0 <= j <= nb - 2)
            got = part[h, i]
            assert got[:len(want)].tolist() == want
            assert (got[len(want):] == -1).all()


@pytest.mark.parametrize("nb,last,r", [(64, 16, 3), (64, 16, 6), (32, 4, 3),
                                       (64, 1, 3), (20, 30, 2)])
def test_cap_keeps_random_blocks_below_last_block(nb, last, r):
    t = oracle.rand_table(11, 3, nb, r, last_block=last)
    for h in range(3):
        for i in range(1, nb - 1):
            cand = [j for j in range(1, nb - 1) if abs(j - i) > 1 and j < last]
            r_eff = min(r, len(cand))
            row = t[h, i]
            chosen = row[:r_eff].tolist()
            assert (row[r_eff:] == -1).all()
            assert len(set(chosen)) == r_eff and all(c in cand for c in chosen)
            assert chosen == sorted(chosen)


def test_pages_configuration_stays_inside_short_sequences():
    """The pages' layer: block 64, table for 4096 tokens, random blocks
    before token 1024, seed = layer index; every kept id is a middle block
    of the running sequence, below 16, off the row's window."""
    for layer in range(12):
        for L in (1024, 2048, 4096):
            nb = L // 64
            t = oracle.rand_table(layer, 12, nb, 3, max_blocks=64,
                                  last_block=16)
            ids = t[t >= 0]
            assert ids.min() >= 1 and ids.max() <= min(15, nb - 2)
            for i in range(1, nb - 1):
                for j in t[:, i][t[:, i] >= 0].tolist():
                    assert abs(j - i) > 1


def test_capped_choice_uniform_chi_square():
    """Over many seeds a capped row chooses each allowed candidate equally
    often."""
    nb, i, r, last = 64, 30, 3, 16
    cand = [j for j in range(1, nb - 1) if abs(j - i) > 1 and j < last]
    counts = dict.fromkeys(cand, 0)
    n = 3000
    for s in range(n):
        for j in oracle.rand_table(s, 1, nb, r, last_block=last)[0, i]:
            counts[int(j)] += 1
    assert sum(counts.values()) == n * r
    assert stats.chisquare(list(counts.values())).pvalue > 1e-4


def test_layer_options_reject_bad_arguments():
    with pytest.raises(ValueError):
        oracle.rand_table(0, 1, 32, 3, max_blocks=16)
    with pytest.raises(ValueError):
        oracle.rand_table(0, 1, 32, 3, last_block=-1)
