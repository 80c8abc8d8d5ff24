"""Property-based checks on the CPU (hypothesis, derandomised so every run
draws the same cases): random small shapes of the oracle against the dense
formulation and autograd, and random arguments of the C table builder
against the oracle's table, bit for bit."""

import math

import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from block_sparse_long_bwd_b200 import binding as bb
from test_oracle import _dense, _random_table

SETTINGS = dict(max_examples=30, deadline=None, derandomize=True)


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    H = draw(st.integers(1, 2))
    nb = draw(st.integers(1, 12))
    bs = draw(st.sampled_from([2, 4, 8]))
    d = draw(st.sampled_from([4, 8]))
    r = draw(st.integers(0, 6))
    masked = draw(st.booleans())
    seed = draw(st.integers(0, 2**32 - 1))
    own = draw(st.booleans())
    return B, H, nb, bs, d, r, masked, seed, own


def _inputs(B, H, nb, bs, d, r, masked, seed, own):
    rng = np.random.default_rng(seed)
    L = nb * bs
    q, k, v, dout = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    km = (rng.random((B, L)) > 0.3).astype(np.uint8) if masked else None
    table = (_random_table(rng, H, nb, r) if own
             else oracle.rand_table(seed, H, nb, r))
    return q, k, v, dout, km, table


@settings(**SETTINGS)
@given(problems())
def test_oracle_equals_dense_autograd_on_random_shapes(prob):
    B, H, nb, bs, d, r, masked, seed, own = prob
    q, k, v, dout, km, table = _inputs(*prob)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.forward(q, k, v, km, table, bs)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, bs)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, lsed = _dense(tq, tk, tv, km, table, bs, scale, -10000.0)
    np.testing.assert_allclose(o, od.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lsed.detach().numpy(), atol=1e-10, rtol=0)
    (od * torch.from_numpy(dout)).sum().backward()
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, want.grad.numpy(), atol=1e-10, rtol=0)


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**64 - 1), H=st.integers(0, 4),
       nb=st.integers(0, 70), r=st.integers(0, 9),
       extra=st.integers(0, 40), last=st.integers(0, 80))
def test_c_table_equals_oracle_on_random_arguments(seed, H, nb, r, extra,
                                                   last):
    mx = nb + extra if extra else 0
    got = bb.bb_rand_attn_build_ex(seed, H, nb, r, mx, last).numpy()
    want = oracle.rand_table(seed, H, nb, r, max_blocks=mx, last_block=last)
    assert np.array_equal(got, want)


@settings(**SETTINGS)
@given(problems(), st.sampled_from([0.0, 0.1, 0.5]), st.booleans(),
       st.integers(0, 2**64 - 1))
def test_oracle_options_equal_dense_autograd_on_random_shapes(prob, rate,
                                                              qmask, dseed):
    """Dropout and the query mask on random shapes: the oracle against dense
    softmax attention with the same keep factors and masked output rows."""
    from test_dropout_oracle import _dense_dropout
    B, H, nb, bs, d, r, masked, seed, own = prob
    q, k, v, dout, km, table = _inputs(*prob)
    L = nb * bs
    qm = None
    if qmask:
        qm = (np.random.default_rng(seed + 7).random((B, L)) > 0.3).astype(
            np.uint8)
    drop = oracle.Dropout(rate, dseed)
    o, _ = oracle.forward(q, k, v, km, table, bs, dropout=drop, query_mask=qm)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, bs, dropout=drop,
                                 query_mask=qm)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, _ = _dense_dropout(tq, tk, tv, km, table, bs, 1.0 / math.sqrt(d),
                           -10000.0, drop)
    if qm is not None:
        od = od * torch.from_numpy(qm.astype(np.float64))[:, None, :, None]
    np.testing.assert_allclose(o, od.detach().numpy(), atol=1e-12, rtol=0)
    (od * torch.from_numpy(dout)).sum().backward()
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, want.grad.numpy(), atol=1e-10, rtol=0)
