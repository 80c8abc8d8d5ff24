"""Pins of the oracle's projections (the dense layers either side of the
attention, [GC] section "两条构建路径：EncoderScaffold 与 BigBirdEncoder"):
element-by-element sums written as explicit loops on tiny shapes, and
identity weights that read the input back out in the head layout."""

import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("B,L,hidden,H,d", [(1, 3, 4, 2, 2), (2, 2, 5, 1, 3), (1, 1, 6, 3, 1)])
def test_qkv_projection_matches_explicit_sums(B, L, hidden, H, d):
    r = _rng(B * 100 + L)
    x = r.standard_normal((B, L, hidden))
    w = r.standard_normal((3 * H * d, hidden))
    bias = r.standard_normal(3 * H * d)
    q, k, v = oracle.qkv_projection(x, w, bias, H, d)
    D = H * d
    for part, t in enumerate((q, k, v)):
        assert t.shape == (B, H, L, d)
        for b in range(B):
            for h in range(H):
                for l in range(L):
                    for j in range(d):
                        f = part * D + h * d + j
                        want = bias[f]
                        for c in range(hidden):
                            want += x[b, l, c] * w[f, c]
                        assert abs(t[b, h, l, j] - want) < 1e-12


@pytest.mark.parametrize("B,L,H,d,hidden", [(1, 3, 2, 2, 5), (2, 2, 3, 1, 4)])
def test_output_projection_matches_explicit_sums(B, L, H, d, hidden):
    r = _rng(B * 10 + H)
    o = r.standard_normal((B, H, L, d))
    w = r.standard_normal((hidden, H * d))
    bias = r.standard_normal(hidden)
    out = oracle.output_projection(o, w, bias)
    assert out.shape == (B, L, hidden)
    for b in range(B):
        for l in range(L):
            for n in range(hidden):
                want = bias[n]
                for h in range(H):
                    for j in range(d):
                        want += o[b, h, l, j] * w[n, h * d + j]
                assert abs(out[b, l, n] - want) < 1e-12


def test_identity_weights_read_the_heads_back():
    """hidden = H d and W_q = W_k = W_v = I: q = k = v = x split into heads;
    w_o = I then puts the heads back in token order."""
    B, L, H, d = 2, 5, 3, 4
    x = _rng(7).standard_normal((B, L, H * d))
    eye = np.eye(H * d)
    q, k, v = oracle.qkv_projection(x, np.concatenate([eye, eye, eye]), None, H, d)
    for t in (q, k, v):
        for h in range(H):
            assert np.array_equal(t[:, h], x[:, :, h * d:(h + 1) * d])
    back = oracle.output_projection(q, eye, None)
    assert np.array_equal(back, x)


def test_bias_only():
    """Zero weights: every row of q, k, v is its part of the bias."""
    B, L, hidden, H, d = 1, 4, 8, 2, 4
    bias = np.arange(3 * H * d, dtype=np.float64)
    q, k, v = oracle.qkv_projection(np.ones((B, L, hidden)), np.zeros((3 * H * d, hidden)),
                                    bias, H, d)
    for part, t in enumerate((q, k, v)):
        for h in range(H):
            for l in range(L):
                assert np.array_equal(t[0, h, l], bias[part * H * d + h * d:part * H * d + (h + 1) * d])
