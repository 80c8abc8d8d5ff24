"""GPU parity of the seeded attention dropout: the CUDA path through the C ABI
against the fp64 oracle drawing the same keep decisions (Philox4x32-10 on
(seed, b, h, t, u)), on the tensor-core path (bf16) and the CUDA-core path
(fp32), plus the properties the rule fixes: the lse is that of the undropped
softmax, a rate that rounds to 0 is the plain operation, and the result is a
deterministic function of the seed."""

import pytest
import torch

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
