"""GPU parity of the seeded attention dropout: the CUDA path through the C ABI
against the fp64 oracle drawing the same keep decisions (Philox4x32-10 on
(seed, b, h, t, u)), on the tensor-core path (bf16) and the CUDA-core path
(fp32), plus the properties the rule fixes: the lse is that of the undropped
softmax, a rate that rounds to 0 is the plain operation, and the result is a
deterministic function of the seed.  The tensor-core runs store the
forward's decisions for the backward (the binding's default); the stored
bits are checked against the keep rule, and against runs that draw them in
every pass."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice, run_gpu

pytestmark = pytest.mark.gpu

ALL = ("out", "lse", "dq", "dk", "dv")
SEED = 0x5EED0123456789AB


def _cfg(B, H, L, bs, r, dtype, mask=None, seed=21):
    return dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype=dtype,
                seed=seed, mask=mask, passes="fwd+bwd")


def _check(cfg, res, inp, rate, slices=None):
    tol = ATOL[cfg["dtype"]]
    if slices is None:
        slices = [(b, h) for b in range(cfg["B"]) for h in range(cfg["H"])]
    for b, h in slices:
        ora = oracle_slice(cfg, inp, res["table"], b, h, dropout=rate,
                           dropout_seed=SEED)
        assert_close(res, ora, b, h, tol, ALL)


DROP_SMALL = [
    # B, H, L, bs, r, dtype, mask, rate
    (2, 2, 1088, 64, 3, "bf16", "tail", 0.1),      # nb = 17: global chunks
    (1, 2, 256, 64, 3, "bf16", None, 0.1),         # nb = 4: dense
    (1, 2, 1024, 32, 3, "bf16", "random5", 0.1),   # bs = 32
    (1, 2, 2048, 128, 3, "bf16", None, 0.1),       # bs = 128
    (1, 2, 448, 64, 1, "f32", "tail", 0.1),        # CUDA-core path
    (2, 1, 1024, 32, 6, "f32", None, 0.5),
]


@pytest.mark.parametrize("case", DROP_SMALL)
def test_dropout_small_shapes_full_compare(case):
    *shape, rate = case
    cfg = _cfg(*shape)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=rate, dropout_seed=SEED)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check(cfg, res, inp, rate)


def test_dropout_long_split_path_sampled():
    """L = 16384: the global key blocks take the hi/lo split dK/dV launch."""
    cfg = _cfg(1, 2, 16384, 64, 3, "bf16", None)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check(cfg, res, inp, 0.1, slices=[(0, 1)])


def test_dropout_large_train_sampled():
    cfg = synth.WORKLOADS["large_train_l4096"]
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check(cfg, res, inp, 0.1, slices=[(0, 0), (3, 15)])


def test_dropout_determinism_seed_and_lse():
    cfg = _cfg(2, 2, 2048, 64, 3, "bf16", "tail", seed=22)
    inp = synth.make_inputs(cfg)
    plain = run_gpu(cfg, inp)
    a = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED)
    b = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED)
    c = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED + 1)
    for n in ALL:
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["out"], c["out"])
    # the lse is that of the undropped softmax
    torch.testing.assert_close(a["lse"], plain["lse"], rtol=0, atol=1e-6)
    # a rate that rounds to 0 (below 1/512) is the plain operation
    z = run_gpu(cfg, inp, dropout=0.001, dropout_seed=SEED)
    for n in ALL:
        assert torch.equal(z[n], plain[n]), n


# ---- the forward's keep decisions stored for the backward -----------------

STORED = [
    # B, H, L, bs, r, dtype, mask, mask_queries
    (2, 2, 1088, 64, 3, "bf16", "tail", 0),     # nb = 17, masked tiles skipped
    (2, 2, 1088, 64, 3, "bf16", "tail", 1),     # with the query-side mask
    (1, 2, 256, 64, 3, "bf16", None, 0),        # nb = 4: dense
    (1, 2, 1024, 32, 3, "bf16", "random5", 0),  # bs = 32: two blocks per tile
    (1, 2, 2048, 128, 6, "bf16", None, 0),      # bs = 128: two tiles per block
    (1, 2, 16384, 64, 3, "bf16", None, 0),      # global key blocks split
]


@pytest.mark.parametrize("case", STORED)
def test_stored_keep_bits_give_the_redrawn_results_bitwise(case):
    """Loading the forward's decisions instead of drawing them again changes
    no bit of any output."""
    *shape, mq = case
    cfg = _cfg(*shape)
    inp = synth.make_inputs(cfg)
    kw = dict(dropout=0.1, dropout_seed=SEED, mask_queries=mq)
    a = run_gpu(cfg, inp, keep_dropout_bits=True, **kw)
    b = run_gpu(cfg, inp, keep_dropout_bits=False, **kw)
    assert "dropout_bits" in a and "dropout_bits" not in b
    for r in (a, b):
        assert r["status_fwd"] == 0 and r["status_bwd"] == 0
    for n in ALL:
        assert torch.equal(a[n], b[n]), n


def _slot(nb, r, row, i, u):
    """Slot of the attended pair (i, u) in a (b, h)'s keep bits, as the
    header states the layout."""
    if i == 0:
        return u
    if i == nb - 1:
        return nb + u
    c = (int(u > 0) + int(i >= 2 and i - 1 < u) + int(i < u)
         + int(i + 1 <= nb - 2 and i + 1 < u)
         + sum(1 for j in row if 0 <= j < u))
    return 2 * nb + (i - 1) * (5 + r) + c


@pytest.mark.parametrize("L,bs,r", [(1024, 64, 3), (1024, 32, 3), (2048, 128, 3),
                                    (256, 64, 2)])
def test_stored_keep_bits_follow_the_keep_rule(L, bs, r):
    """Every attended element's stored bit is the oracle's keep decision, at
    the place the header's layout gives it."""
    cfg = _cfg(2, 2, L, bs, r, "bf16", None)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED, backward=False)
    assert res["status_fwd"] == 0
    words = res["dropout_bits"].numpy().view(np.uint32)
    nb, table = L // bs, np.asarray(res["table"])
    S = 1 if nb == 1 else 2 * nb + (nb - 2) * (5 + r)
    per_slot = bs * bs // 32
    assert words.size == cfg["B"] * cfg["H"] * S * per_slot
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            base = (b * cfg["H"] + h) * S
            for i in range(nb):
                rows = np.arange(i * bs, (i + 1) * bs)
                for u in oracle.attended_blocks(i, nb, table[h, i]):
                    keep = oracle.dropout_keep(SEED, b, h, rows,
                                               np.arange(u * bs, (u + 1) * bs), 0.1)
                    want = (keep.reshape(bs, bs // 32, 32).astype(np.uint64)
                            * weights).sum(axis=2).astype(np.uint32).ravel()
                    s = base + _slot(nb, r, table[h, i], i, int(u))
                    got = words[s * per_slot:(s + 1) * per_slot]
                    assert np.array_equal(got, want), (b, h, i, int(u))


def test_cuda_core_path_leaves_the_keep_bits_alone():
    """fp32 runs on the CUDA-core kernels, which draw in every pass: the
    buffer is neither written nor read, and the results match the oracle."""
    cfg = _cfg(1, 2, 448, 64, 1, "f32", "tail")
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=0.1, dropout_seed=SEED, bits_fill=0xA5)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    assert bool((res["dropout_bits"] == 0xA5).all())
    _check(cfg, res, inp, 0.1)
