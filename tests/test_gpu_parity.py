"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes are compared element by element over every (b, h).  The
full-size workloads run in the launch configuration the benchmark times:
the BigBird-base, BigBird-large and 16K workloads on every (b, h) slice, the
54 sweep points on two slices each (rows of one (b, h) depend on nothing
else, so a slice is an exact check of its rows)."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_bwd_b200 import synth
from gpu_util import (ATOL, assert_bf16_is_rounded_fp32, assert_close,
                      oracle_slice, run_gpu)

pytestmark = pytest.mark.gpu

FWD = ("out", "lse")
ALL = ("out", "lse", "dq", "dk", "dv")


def _small(B, H, L, bs, r, dtype, mask=None, seed=11):
    return dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype=dtype,
                seed=seed, mask=mask, passes="fwd+bwd")


def _check_all(cfg, res, inp, names=ALL, **kw):
    tol = ATOL[cfg["dtype"]]
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ora = oracle_slice(cfg, inp, res["table"], b, h,
                               backward="dq" in names, **kw)
            assert_close(res, ora, b, h, tol, names)


def test_tiny_fp32_workload_full_compare():
    cfg = synth.WORKLOADS["tiny_fp32_l1024"]
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check_all(cfg, res, inp)


SMALL = [
    # B, H, L, bs, r, dtype, mask
    (1, 1, 64, 64, 3, "bf16", None),        # nb = 1
    (2, 1, 128, 64, 3, "bf16", "tail"),     # nb = 2
    (1, 2, 192, 64, 2, "f32", None),        # nb = 3
    (1, 2, 256, 64, 3, "bf16", "random5"),  # nb = 4: dense
    (2, 1, 320, 64, 0, "bf16", None),       # nb = 5, r = 0: not dense
    (1, 3, 448, 64, 1, "f32", "tail"),      # nb = 7
    (3, 2, 1088, 64, 3, "bf16", "tail"),    # nb = 17
    (1, 2, 1024, 32, 3, "bf16", "random5"),  # bs = 32
    (2, 1, 1024, 32, 6, "f32", None),
    (1, 2, 1024, 128, 6, "bf16", None),     # clamped: fully dense
    (2, 1, 2048, 128, 3, "bf16", "random5"),
    (1, 1, 1152, 128, 2, "f32", "tail"),
    (1, 5, 2112, 64, 6, "bf16", None),
]


@pytest.mark.parametrize("case", SMALL)
def test_small_shapes_full_compare(case):
    cfg = _small(*case)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check_all(cfg, res, inp)


def test_custom_scale_and_mask_value():
    cfg = _small(1, 2, 640, 64, 2, "f32", "random5", seed=12)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, scale=0.2, mask_value=-5.0)
    _check_all(cfg, res, inp, scale=0.2, mask_value=-5.0)


def test_corrupt_table_is_flagged_and_ignored():
    cfg = _small(1, 2, 768, 64, 3, "bf16", None, seed=13)
    inp = synth.make_inputs(cfg)
    nb = cfg["L"] // cfg["block_size"]
    table = oracle.rand_table(0, 2, nb, 3)
    table[1, 4, 1] = nb + 7      # out of range: ignored, flagged
    table[0, 5, 0] = -9          # out of range: ignored, flagged
    table[0, 6, 2] = 6           # own window: redundant under set union
    res = run_gpu(cfg, inp, table=table)
    assert res["status_fwd"] == -6 and res["status_bwd"] == -6
    clean = table.copy()
    clean[1, 4, 1] = -1
    clean[0, 5, 0] = -1
    res["table"] = clean
    _check_all(cfg, res, inp)


def test_deterministic_bitwise():
    cfg = _small(2, 3, 2048, 64, 3, "bf16", "tail", seed=14)
    inp = synth.make_inputs(cfg)
    a = run_gpu(cfg, inp)
    b = run_gpu(cfg, inp)
    for n in ALL:
        assert torch.equal(a[n], b[n]), n


def test_deterministic_bitwise_many_items_per_cta():
    """BigBird-large step: 2560 items over 296 CTAs taken from a dynamic
    counter, so which CTA computes which item differs between runs; every
    output row is still written by exactly one item (or summed in a fixed
    order), so the results are bitwise equal."""
    cfg = synth.WORKLOADS["large_train_l4096"]
    inp = synth.make_inputs(cfg)
    a = run_gpu(cfg, inp)
    b = run_gpu(cfg, inp)
    for n in ALL:
        assert torch.equal(a[n], b[n]), n


def _all_slices(cfg):
    return [(b, h) for b in range(cfg["B"]) for h in range(cfg["H"])]


def _full(cfg, samples, backward, direct_grads=True):
    """Full-size workload in the benchmark's launch configuration.

    The forward outputs (bf16 O, fp32 lse) are compared with the oracle at
    the bf16 tolerance on the sampled (b, h) slices.  The backward runs
    twice: with fp32 gradient outputs, compared with the oracle at the same
    tolerance, and with bf16 gradients, which must equal the fp32 ones
    rounded to nearest even bit for bit.  direct_grads: also compare the
    bf16 gradients themselves with the oracle (where every exact gradient is
    small enough that its bf16 rounding stays within the tolerance)."""
    inp = synth.make_inputs(cfg, with_grad=backward)
    res = run_gpu(cfg, inp, backward=backward)
    assert res["status_fwd"] == 0
    tol = ATOL[cfg["dtype"]]
    if backward:
        assert res["status_bwd"] == 0
        r32 = run_gpu(cfg, inp, backward=True, grad_fp32=1)
        assert r32["status_bwd"] == 0
        assert_bf16_is_rounded_fp32(res, r32)
        for n in ("out", "lse"):
            assert torch.equal(res[n], r32[n]), n
    for n in (ALL if backward else FWD):
        assert torch.isfinite(res[n]).all(), n
    for b, h in samples:
        ora = oracle_slice(cfg, inp, res["table"], b, h, backward=backward)
        assert_close(res, ora, b, h, tol, FWD)
        if backward:
            assert_close(r32, ora, b, h, tol, ("dq", "dk", "dv"))
            if direct_grads:
                assert_close(res, ora, b, h, tol, ("dq", "dk", "dv"))


def test_full_base_fwd_l4096():
    """BigBird-base forward with its padded batch: every (b, h) slice."""
    cfg = synth.WORKLOADS["base_fwd_l4096"]
    _full(cfg, _all_slices(cfg), False)


def test_full_large_train_l4096():
    """BigBird-large training step: every (b, h) slice, forward and
    backward."""
    cfg = synth.WORKLOADS["large_train_l4096"]
    _full(cfg, _all_slices(cfg), True)


def test_full_long_l16384():
    """16K-token pattern with 5 % masked keys: every (b, h) slice."""
    cfg = synth.WORKLOADS["long_l16384"]
    _full(cfg, _all_slices(cfg), True)


SWEEP = [(L, bs, r) for L in synth.SWEEP_L for bs in synth.SWEEP_BS
         for r in synth.SWEEP_R]


@pytest.mark.parametrize("L,bs,r", SWEEP)
def test_full_sweep_point(L, bs, r):
    """Every point of the length / block / random-count sweep, two (b, h)
    slices each.  The gradients are checked at the bf16 tolerance through
    the fp32 outputs: at long lengths and small blocks the two global key
    blocks' exact gradients exceed 4 in magnitude (7.6 at L = 32768, block
    32, r = 0), where bf16's own spacing (1/32) alone exceeds 1e-2."""
    cfg = synth.sweep_point(L, bs, r)
    _full(cfg, [(0, 0), (cfg["B"] - 1, cfg["H"] - 1)], True,
          direct_grads=False)


def test_full_planning_fallback_l131072():
    """A length whose per-head transposed adjacency does not fit in shared
    memory (block 32: 4096 blocks), so the backward plans through the CSR
    builder in global memory; also the two-launch dK/dV path and a key mask.
    Every row meets 1e-2 max-abs: the forward directly, the gradients through
    their fp32 outputs (the global key blocks' exact dK reaches 10 here, where
    a bf16 value is only good to 1/32), and the bf16 gradients are those
    fp32 values rounded to nearest even."""
    cfg = dict(B=1, H=2, L=131072, block_size=32, d=64, r=3, dtype="bf16",
               seed=7, mask="random5", passes="fwd+bwd")
    _full(cfg, [(0, 1)], True, direct_grads=False)
