"""Pins for the oracle's query-side (from) mask: rows of padding tokens
output zero and pass no gradient.  Checked against a dense torch fp64
formulation with autograd, finite differences, and the reductions the rule
fixes (all-real mask = the plain operation; real rows unchanged)."""

import math

import numpy as np
import pytest
import torch

import oracle
from test_oracle import _case, _dense

CASES = [
    # seed, B, H, nb, bs, d, r, masked, own_table
    (60, 1, 1, 1, 4, 4, 0, True, False),
    (61, 2, 2, 5, 4, 8, 1, True, False),
    (62, 1, 2, 9, 8, 8, 2, True, True),
    (63, 2, 1, 12, 4, 4, 3, False, False),
]


def _qmask(seed, B, L):
    rng = np.random.default_rng(seed + 100)
    m = (rng.random((B, L)) > 0.35).astype(np.uint8)
    m[:, 0] = 1
    return m


def _dense_q(q, k, v, km, table, bs, scale, qm):
    o, lse = _dense(q, k, v, km, table, bs, scale, -10000.0)
    return o * torch.from_numpy(qm.astype(np.float64))[:, None, :, None], lse


@pytest.mark.parametrize("case", CASES)
def test_query_mask_forward_and_backward_equal_dense_autograd(case):
    seed, B, H, nb, bs, d, r, masked, own = case
    q, k, v, dout, km, table = _case(seed, B, H, nb, bs, d, r, masked, own)
    qm = _qmask(seed, B, nb * bs)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.forward(q, k, v, km, table, bs, query_mask=qm)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, bs, query_mask=qm)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, lsed = _dense_q(tq, tk, tv, km, table, bs, scale, qm)
    np.testing.assert_allclose(o, od.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lsed.detach().numpy(), atol=1e-10, rtol=0)
    (od * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10, rtol=0)


def test_query_mask_rows_zero_and_real_rows_unchanged():
    q, k, v, dout, km, table = _case(64, 2, 2, 6, 4, 8, 2, True, False)
    qm = _qmask(64, 2, 24)
    o0, l0 = oracle.forward(q, k, v, km, table, 4)
    o1, l1 = oracle.forward(q, k, v, km, table, 4, query_mask=qm)
    pad = qm == 0
    assert pad.any() and (~pad).any()
    for b in range(2):
        assert (o1[b][:, pad[b]] == 0).all()
        np.testing.assert_array_equal(o1[b][:, ~pad[b]], o0[b][:, ~pad[b]])
    np.testing.assert_array_equal(l0, l1)
    dq1, _, _ = oracle.backward(q, k, v, dout, km, table, 4, query_mask=qm)
    for b in range(2):
        assert (dq1[b][:, pad[b]] == 0).all()


def test_query_mask_all_real_is_the_plain_operation():
    q, k, v, dout, km, table = _case(65, 1, 2, 7, 4, 8, 2, True, False)
    ones = np.ones((1, 28), dtype=np.uint8)
    for a, b in zip(oracle.forward(q, k, v, km, table, 4),
                    oracle.forward(q, k, v, km, table, 4, query_mask=ones)):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(oracle.backward(q, k, v, dout, km, table, 4),
                    oracle.backward(q, k, v, dout, km, table, 4,
                                    query_mask=ones)):
        np.testing.assert_array_equal(a, b)


def test_query_mask_finite_differences():
    q, k, v, dout, km, table = _case(66, 1, 1, 7, 4, 4, 2, True, False)
    qm = _qmask(66, 1, 28)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, 4, query_mask=qm)

    def loss(q_, k_, v_):
        o, _ = oracle.forward(q_, k_, v_, km, table, 4, query_mask=qm)
        return float((o * dout).sum())

    h = 1e-6
    rng = np.random.default_rng(9)
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


def test_query_mask_with_dropout_matches_dense():
    q, k, v, dout, km, table = _case(67, 1, 2, 6, 4, 8, 1, True, False)
    qm = _qmask(67, 1, 24)
    drop = oracle.Dropout(0.2, 5)
    o, _ = oracle.forward(q, k, v, km, table, 4, dropout=drop, query_mask=qm)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, 4, dropout=drop,
                                 query_mask=qm)
    from test_dropout_oracle import _dense_dropout
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, _ = _dense_dropout(tq, tk, tv, km, table, 4, 1.0 / math.sqrt(8),
                           -10000.0, drop)
    od = od * torch.from_numpy(qm.astype(np.float64))[:, None, :, None]
    np.testing.assert_allclose(o, od.detach().numpy(), atol=1e-12, rtol=0)
    (od * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10, rtol=0)
