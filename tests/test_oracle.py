"""Pins for the fp64 oracle, independent of the oracle's own code paths.

Each check compares the oracle with something it does not share code with:
a dense token-level formulation written here (attention mask built from the
pattern's definition, torch softmax / logsumexp), torch fp64 autograd, central
finite differences, torch's scaled_dot_product_attention where the pattern is
dense, a closed-form read-out of the adjacency, and invariants of softmax.
"""

import math

import numpy as np
import pytest
import torch

import oracle

ATOL = 1e-12


def _random_table(rng, H, nb, r):
    """A valid table drawn independently of the oracle's generator: for each
    middle row, r_eff distinct non-window middle blocks, sorted, -1 padded."""
    t = np.full((H, nb, r), -1, dtype=np.int32)
    for h in range(H):
        for i in range(1, nb - 1):
            cand = [j for j in range(1, nb - 1) if j < i - 1 or j > i + 1]
            n = min(r, len(cand))
            if n:
                t[h, i, :n] = np.sort(rng.choice(cand, size=n, replace=False))
    return t


def _token_bias(table, h, nb, bs, key_mask_b, mask_value):
    """[L, L] additive bias: -inf outside the ITC pattern, mask_value on masked
    keys inside it, 0 elsewhere.  Written from the pattern's definition with
    dense boolean algebra on block ids."""
    L = nb * bs
    blk = torch.arange(L) // bs
    qb = blk[:, None]
    kb = blk[None, :]
    allowed = ((qb == 0) | (qb == nb - 1) | (kb == 0) | (kb == nb - 1)
               | ((qb - kb).abs() <= 1))
    rnd = torch.zeros(nb, nb, dtype=torch.bool)
    for i in range(nb):
        for j in table[h, i]:
            if j >= 0:
                rnd[i, int(j)] = True
    allowed = allowed | rnd[qb, kb]
    keyoff = torch.zeros(L, dtype=torch.float64)
    if key_mask_b is not None:
        keyoff = torch.where(torch.as_tensor(key_mask_b).bool(),
                             torch.tensor(0.0, dtype=torch.float64),
                             torch.tensor(float(mask_value),
                                          dtype=torch.float64))
    return torch.where(allowed, keyoff[None, :].expand(L, L),
                       torch.tensor(-math.inf, dtype=torch.float64))


def _dense(q, k, v, key_mask, table, bs, scale, mask_value):
    """Dense masked softmax attention in torch fp64 (differentiable)."""
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
            ob.append(torch.softmax(s, dim=-1) @ v[b, h])
            lb.append(torch.logsumexp(s, dim=-1))
        outs.append(torch.stack(ob))
        lses.append(torch.stack(lb))
    return torch.stack(outs), torch.stack(lses)


def _case(seed, B, H, nb, bs, d, r, masked, own_table):
    rng = np.random.default_rng(seed)
    L = nb * bs
    q = rng.standard_normal((B, H, L, d))
    k = rng.standard_normal((B, H, L, d))
    v = rng.standard_normal((B, H, L, d))
    dout = rng.standard_normal((B, H, L, d))
    key_mask = None
    if masked:
        key_mask = (rng.random((B, L)) > 0.3).astype(np.uint8)
    if own_table:
        table = _random_table(rng, H, nb, r)
    else:
        table = oracle.rand_table(seed, H, nb, r)
    return q, k, v, dout, key_mask, table


CASES = [
    # seed, B, H, nb, bs, d, r, masked, own_table
    (0, 1, 1, 1, 4, 4, 0, False, False),
    (1, 1, 2, 2, 4, 8, 2, True, False),
    (2, 2, 1, 3, 4, 4, 1, True, True),
    (3, 1, 2, 4, 8, 8, 3, False, False),
    (4, 1, 1, 5, 4, 8, 0, True, False),
    (5, 2, 2, 5, 4, 4, 1, False, True),
    (6, 1, 2, 6, 4, 8, 2, True, True),
    (7, 1, 1, 8, 8, 16, 3, True, False),
    (8, 2, 2, 9, 4, 4, 2, False, True),
    (9, 1, 2, 12, 4, 8, 3, True, True),
    (10, 1, 1, 16, 4, 4, 6, True, False),
    (11, 1, 2, 11, 4, 8, 4, False, False),
]


@pytest.mark.parametrize("case", CASES)
def test_forward_equals_dense_bruteforce(case):
    seed, B, H, nb, bs, d, r, masked, own = case
    q, k, v, dout, km, table = _case(seed, B, H, nb, bs, d, r, masked, own)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.forward(q, k, v, km, table, bs)
    t = lambda x: torch.from_numpy(np.asarray(x, dtype=np.float64))
    od, lsed = _dense(t(q), t(k), t(v), km, table, bs, scale, -10000.0)
    np.testing.assert_allclose(o, od.numpy(), atol=ATOL, rtol=0)
    np.testing.assert_allclose(lse, lsed.numpy(), atol=1e-10, rtol=0)


def test_forward_custom_scale_and_mask_value():
    q, k, v, dout, km, table = _case(21, 1, 2, 7, 4, 8, 2, True, False)
    o, lse = oracle.forward(q, k, v, km, table, 4, scale=0.3,
                            mask_value=-7.5)
    t = lambda x: torch.from_numpy(np.asarray(x, dtype=np.float64))
    od, lsed = _dense(t(q), t(k), t(v), km, table, 4, 0.3, -7.5)
    np.testing.assert_allclose(o, od.numpy(), atol=ATOL, rtol=0)
    np.testing.assert_allclose(lse, lsed.numpy(), atol=1e-10, rtol=0)


@pytest.mark.parametrize("case", CASES)
def test_backward_equals_autograd(case):
    seed, B, H, nb, bs, d, r, masked, own = case
    q, k, v, dout, km, table = _case(seed, B, H, nb, bs, d, r, masked, own)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, bs)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True)
                  for x in (q, k, v))
    od, _ = _dense(tq, tk, tv, km, table, bs, scale, -10000.0)
    (od * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-10, rtol=0)


def test_backward_finite_differences():
    q, k, v, dout, km, table = _case(31, 1, 1, 7, 4, 4, 2, True, False)
    dq, dk, dv = oracle.backward(q, k, v, dout, km, table, 4)

    def loss(q_, k_, v_):
        o, _ = oracle.forward(q_, k_, v_, km, table, 4)
        return float((o * dout).sum())

    h = 1e-6
    rng = np.random.default_rng(5)
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


@pytest.mark.parametrize("nb,r", [(1, 0), (2, 3), (3, 1), (4, 0), (4, 5),
                                  (5, 1), (5, 3)])
def test_reduces_to_library_sdpa_when_dense(nb, r):
    """With nb <= 4 (any r), or nb = 5 with r >= 1, every query block attends
    every key block, so the result is plain masked softmax attention."""
    bs, d = 8, 16
    q, k, v, dout, km, table = _case(40 + nb + r, 2, 2, nb, bs, d, r, True,
                                     False)
    o, lse = oracle.forward(q, k, v, km, table, bs)
    bias = torch.where(torch.from_numpy(km).bool(), 0.0, -10000.0)
    bias = bias.to(torch.float64)[:, None, None, :]
    t = lambda x: torch.from_numpy(np.asarray(x, dtype=np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=bias)
    np.testing.assert_allclose(o, ref.numpy(), atol=ATOL, rtol=0)


def test_nb5_r0_is_not_dense():
    """nb = 5, r = 0: rows 1 and 3 each miss one block (pair counts
    [5, 4, 5, 4, 5]); the result must differ from dense attention."""
    table = oracle.rand_table(0, 1, 5, 0)
    counts = [len(oracle.attended_blocks(i, 5, table[0, i])) for i in range(5)]
    assert counts == [5, 4, 5, 4, 5]
    q, k, v, dout, km, table = _case(50, 1, 1, 5, 4, 4, 0, False, False)
    o, _ = oracle.forward(q, k, v, None, table, 4)
    t = lambda x: torch.from_numpy(np.asarray(x, dtype=np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))
    assert np.abs(o - ref.numpy()).max() > 1e-3


@pytest.mark.parametrize("nb,r", [(6, 0), (9, 2), (13, 3), (20, 6)])
def test_pattern_identity_closed_form(nb, r):
    """K = 0 and no mask make every attended key equally likely, so with
    V[u] = onehot(block(u)) the output row of query block i is 1/|A(i)| on the
    attended blocks and 0 elsewhere.  The count |A(i)| has a closed form:
    nb for rows 0 and nb-1; 4 + r_eff for rows 1 and nb-2 (the window holds a
    global block); 5 + r_eff otherwise, with r_eff = min(r, |cand(i)|) and
    |cand(i)| = nb - 4 for rows 1 and nb-2 and nb - 5 for the rest."""
    bs = 2
    H = 2
    L = nb * bs
    table = oracle.rand_table(7, H, nb, r)
    q = np.random.default_rng(1).standard_normal((1, H, L, nb))
    k = np.zeros((1, H, L, nb))
    v = np.zeros((1, H, L, nb))
    for u in range(L):
        v[0, :, u, u // bs] = 1.0
    o, _ = oracle.forward(q, k, v, None, table, bs)
    for h in range(H):
        for i in range(nb):
            row = o[0, h, i * bs]
            hit = np.nonzero(row > 1e-9)[0]
            if i in (0, nb - 1):
                n = nb
            elif i in (1, nb - 2):
                n = 4 + min(r, nb - 4)
            else:
                n = 5 + min(r, nb - 5)
            assert len(hit) == n
            np.testing.assert_allclose(row[hit], 1.0 / n, atol=1e-14)
            if i not in (0, nb - 1):
                want = {0, nb - 1, i - 1, i, i + 1}
                want |= {int(j) for j in table[h, i] if j >= 0}
                assert set(hit.tolist()) == want


def test_softmax_rows_sum_to_one_and_constant_v():
    q, k, v, dout, km, table = _case(60, 1, 2, 10, 4, 8, 3, True, False)
    for i in range(10):
        _, p, _ = oracle.block_probs(q, k, km, table, 4, 0, 1, i)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
    vc = np.broadcast_to(np.arange(8, dtype=np.float64), v.shape).copy()
    o, _ = oracle.forward(q, k, vc, km, table, 4)
    np.testing.assert_allclose(o, vc, atol=1e-12)


def test_masked_keys_get_vanishing_probability():
    q, k, v, dout, km, table = _case(61, 1, 1, 8, 4, 8, 2, True, False)
    km[0, :4] = 1  # block 0 has valid keys, so every row has one
    for i in range(8):
        cols, p, _ = oracle.block_probs(q, k, km, table, 4, 0, 0, i)
        masked = km[0, cols] == 0
        assert p[:, masked].max(initial=0.0) < 1e-300 or not masked.any()


def test_global_key_and_query_rows():
    """Rows 0 and nb-1 attend all blocks; every row attends blocks 0, nb-1."""
    table = oracle.rand_table(3, 2, 12, 3)
    for h in range(2):
        for i in range(12):
            a = oracle.attended_blocks(i, 12, table[h, i])
            assert 0 in a and 11 in a
            if i in (0, 11):
                assert a == list(range(12))


def test_pair_count_formula():
    """Pairs per head = 7 nb - 12 + sum r_eff (nb >= 5)."""
    for nb, r in [(5, 1), (8, 3), (16, 3), (64, 3), (9, 6)]:
        table = oracle.rand_table(0, 1, nb, r)
        r_eff = int((table[0] >= 0).sum())
        assert oracle.pair_count(nb, table[0]) == 7 * nb - 12 + r_eff
