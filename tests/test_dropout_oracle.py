"""Pins for the oracle's seeded attention dropout.

The generator is checked against the published Philox4x32-10 known-answer
vectors; the keep rule against a byte-level restatement of its layout; the
dropped forward and backward against a dense torch fp64 formulation with the
same keep mask (autograd for the gradients) and against central finite
differences; the rate handling against its closed forms.
"""

import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
from test_oracle import _case, _dense, _token_bias

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "philox4x32_10_kat.txt")


def _kat():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                w = [int(x, 16) for x in line.split()]
                rows.append((tuple(w[:4]), tuple(w[4:6]), tuple(w[6:])))
    return rows


def test_philox_matches_published_kat():
    kat = _kat()
    assert len(kat) == 3
    for ctr, key, want in kat:
        got = tuple(int(x) for x in oracle.philox4x32_10(ctr, key))
        assert got == want


def test_philox_vectorised_equals_scalar_calls():
    rng = np.random.default_rng(3)
    ctr = [rng.integers(0, 2**32, size=17, dtype=np.uint64) for _ in range(4)]
    key = (0x01234567, 0x89ABCDEF)
    vec = oracle.philox4x32_10(ctr, key)
    for n in range(17):
        one = oracle.philox4x32_10([c[n] for c in ctr], key)
        assert [int(w[n]) for w in vec] == [int(w) for w in one]


@pytest.mark.parametrize("rate,thr", [(0.0, 0), (0.1, 26), (0.5, 128),
                                      (1.0 / 512, 1), (0.9, 230),
                                      (254.4 / 256, 254), (255.49 / 256, 255)])
def test_threshold_rounds_to_nearest_256th(rate, thr):
    assert oracle.dropout_threshold(rate) == thr
    assert oracle.dropout_scale(rate) == 256.0 / (256 - thr)


@pytest.mark.parametrize("rate", [-0.01, 1.0, 1.5, 255.5 / 256, 0.9999])
def test_threshold_rejects_rates_outside_range(rate):
    with pytest.raises(ValueError):
        oracle.dropout_threshold(rate)


def test_keep_uses_little_endian_bytes_of_one_call_per_16_keys():
    """Restates the keep rule with struct packing: the 16 bytes of the call
    with counter (g, t, h, b) are the key tokens 16 g .. 16 g + 15."""
    seed = 0x1122334455667788
    b, h, rate = 3, 5, 0.3
    thr = oracle.dropout_threshold(rate)
    rows = np.array([0, 1, 63, 64, 1000, 4095])
    cols = np.arange(0, 96)
    keep = oracle.dropout_keep(seed, b, h, rows, cols, rate)
    for a, t in enumerate(rows):
        for g in range(6):
            words = oracle.philox4x32_10((g, int(t), h, b),
                                         (seed & 0xFFFFFFFF, seed >> 32))
            raw = struct.pack("<4I", *(int(w) for w in words))
            for j in range(16):
                assert keep[a, 16 * g + j] == (raw[j] >= thr)


@pytest.mark.parametrize("rate", [0.1, 0.5, 0.9])
def test_keep_fraction_is_binomial(rate):
    thr = oracle.dropout_threshold(rate)
    keep = oracle.dropout_keep(7, 1, 2, np.arange(512), np.arange(1024), rate)
    n = keep.size
    pk = (256 - thr) / 256
    sigma = math.sqrt(n * pk * (1 - pk))
    assert abs(keep.sum() - n * pk) < 5 * sigma
    # the mean factor is 1: dropped probabilities are unbiased
    f = oracle.Dropout(rate, 7).factors(1, 2, np.arange(512), np.arange(1024))
    assert abs(f.mean() - 1.0) < 5 * sigma / n * oracle.dropout_scale(rate)


def test_keep_bytes_uniform_chi_square():
    """Byte values behind the decisions are uniform: bucket counts of the
    keep rule at every threshold 16 k follow the uniform distribution."""
    from scipy import stats
    rows, cols = np.arange(256), np.arange(512)
    counts = []
    prev = np.ones((256, 512), dtype=bool)
    for k in range(1, 17):
        rate = 16 * k / 256 if k < 16 else None
        cur = (oracle.dropout_keep(11, 0, 0, rows, cols, rate)
               if rate is not None else np.zeros_like(prev))
        counts.append(int((prev & ~cur).sum()))
        prev = cur
    assert sum(counts) == 256 * 512
    assert stats.chisquare(counts).pvalue > 1e-4


def test_keep_depends_on_every_coordinate_and_seed():
    base = oracle.dropout_keep(5, 1, 1, np.arange(64), np.arange(64), 0.5)
    for seed, b, h in ((6, 1, 1), (5 + (1 << 32), 1, 1), (5, 0, 1), (5, 1, 0)):
        other = oracle.dropout_keep(seed, b, h, np.arange(64), np.arange(64),
                                    0.5)
        assert (other != base).mean() > 0.3
    # shifting the query rows or the key columns by one changes the draw
    sh_t = oracle.dropout_keep(5, 1, 1, np.arange(1, 65), np.arange(64), 0.5)
    sh_u = oracle.dropout_keep(5, 1, 1, np.arange(64), np.arange(1, 65), 0.5)
    assert (sh_t != base).mean() > 0.3 and (sh_u != base).mean() > 0.3


def _dense_dropout(q, k, v, key_mask, table, bs, scale, mask_value, drop):
    """Dense masked softmax attention with the keep factors applied to the
    probabilities (torch fp64, differentiable); lse of the undropped
    softmax."""
    B, H, L, d = q.shape
    nb = L // bs
    outs, lses = [], []
    for b in range(B):
        ob, lb = [], []
        for h in range(H):
            bias = _token_bias(table, h, nb, bs,
                               None if key_mask is None else key_mask[b],
                               mask_value)
            s = scale * (q[b, h] @ k[b, h].T) + bias
            f = torch.from_numpy(drop.factors(b, h, np.arange(L), np.arange(L)))
            ob.append((torch.softmax(s, dim=-1) * f) @ v[b, h])
            lb.append(torch.logsumexp(s, dim=-1))
        outs.append(torch.stack(ob))
        lses.append(torch.stack(lb))
    return torch.stack(outs), torch.stack(lses)


DROP_CASES = [
    # seed, B, H, nb, bs, d, r, masked, own_table, rate
    (40, 1, 1, 1, 4, 4, 0, False, False, 0.1),
    (41, 2, 2, 5, 4, 8, 1, True, False, 0.5),
    (42, 1, 2, 9, 8, 8, 2, True, True, 0.1),
    (43, 2, 1, 12, 4, 4, 3, False, False, 0.9),
    (44, 1, 2, 6, 32, 8, 1, True, False, 0.25),
]


@pytest.mark.parametrize("case", DROP_CASES)
def test_dropout_forward_equals_dense(case):
    seed, B, H, nb, bs, d, r, masked, own, rate = case
    q, k, v, dout, km, table = _case(seed, B, H, nb, bs, d, r, masked, own)
    drop = oracle.Dropout(rate, 1000 + seed)
    o, lse = oracle.forward(q, k, v, km, table, bs, dropout=drop)
    t = lambda x: torch.from_numpy(np.asarray(x, dtype=np.float64))
    od, lsed = _dense_dropout(t(q), t(k), t(v), km, table, bs,
                              1.0 / math.sqrt(d), -10000.0, drop)
    np.testing.assert_allclose(o, od.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lsed.numpy(), atol=1e-10, rtol=0)
    # the lse is that of the undropped softmax
    _, lse0 = oracle.forward(q, k, v, km, table, bs)
    np.testing.assert_array_equal(lse, lse0)


@pytest.mark.parametrize("case", DROP_CASES)
def test_dropout_backward_equals_autograd(case):
    seed, B, H, nb, bs, d, r, masked, own, rate = case
    q, k, v, dout, km, table = _case(seed, B, H, nb, bs, d, r, masked, own)
    drop = oracle.Dropout(rate, 1000 + seed)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, bs, dropout=drop)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, _ = _dense_dropout(tq, tk, tv, km, table, bs, 1.0 / math.sqrt(d),
                           -10000.0, drop)
    (od * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10, rtol=0)


def test_dropout_backward_finite_differences():
    q, k, v, dout, km, table = _case(45, 1, 1, 7, 4, 4, 2, True, False)
    drop = oracle.Dropout(0.3, 99)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, 4, dropout=drop)

    def loss(q_, k_, v_):
        o, _ = oracle.forward(q_, k_, v_, km, table, 4, dropout=drop)
        return float((o * dout).sum())

    h = 1e-6
    rng = np.random.default_rng(8)
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in q.shape)
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += h
            up = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * h
            dn = loss(args["q"], args["k"], args["v"])
            fd = (up - dn) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_dropout_rate_zero_is_the_plain_operation():
    q, k, v, dout, km, table = _case(46, 2, 2, 6, 4, 8, 2, True, False)
    drop = oracle.Dropout(0.0, 12345)
    o0, l0 = oracle.forward(q, k, v, km, table, 4)
    o1, l1 = oracle.forward(q, k, v, km, table, 4, dropout=drop)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)
    g0 = oracle.backward(q, k, v, dout, km, table, 4)
    g1 = oracle.backward(q, k, v, dout, km, table, 4, dropout=drop)
    for a, b in zip(g0, g1):
        np.testing.assert_array_equal(a, b)


def test_dropout_output_is_unbiased_over_seeds():
    """Averaged over seeds, the dropped output approaches the undropped one
    (each factor has mean 1 and the draws of different seeds are
    independent)."""
    q, k, v, dout, km, table = _case(47, 1, 1, 5, 4, 4, 1, False, False)
    o0, _ = oracle.forward(q, k, v, km, table, 4)
    n = 400
    acc = np.zeros_like(o0)
    sq = np.zeros_like(o0)
    for s in range(n):
        o, _ = oracle.forward(q, k, v, km, table, 4,
                              dropout=oracle.Dropout(0.5, s))
        acc += o
        sq += o * o
    mean = acc / n
    se = np.sqrt(np.maximum(sq / n - mean * mean, 0) / n) + 1e-12
    assert np.max(np.abs(mean - o0) / se) < 6.0


def test_slice_offsets_reproduce_the_whole_call():
    """A (b, h) slice run as its own problem with offsets (b, h) draws the
    decisions of the whole call's batch b, head h."""
    q, k, v, dout, km, table = _case(48, 2, 3, 6, 4, 8, 2, True, False)
    whole = oracle.Dropout(0.3, 77)
    o, _ = oracle.forward(q, k, v, km, table, 4, dropout=whole)
    g = oracle.backward(q, k, v, dout, km, table, 4, dropout=whole)
    for b in range(2):
        for h in range(3):
            sl = lambda x: x[b:b + 1, h:h + 1]
            part = oracle.Dropout(0.3, 77, b0=b, h0=h)
            kmb = km[b:b + 1]
            os_, _ = oracle.forward(sl(q), sl(k), sl(v), kmb, table[h:h + 1],
                                    4, dropout=part)
            np.testing.assert_array_equal(os_[0, 0], o[b, h])
            gs = oracle.backward(sl(q), sl(k), sl(v), sl(dout), kmb,
                                 table[h:h + 1], 4, dropout=part)
            for a, c in zip(gs, g):
                np.testing.assert_array_equal(a[0, 0], c[b, h])
