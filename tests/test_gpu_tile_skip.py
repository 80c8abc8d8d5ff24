"""GPU parity of the forward's skipping of fully masked key tiles.

A 64-key tile whose keys are all masked is dropped from an item's tile list
when every row of the batch has a valid attended key (a valid key among the
first 32, which lie in global block 0); a masked key's probability is then
exp(-10000 + ...), zero in fp32 and below 1e-4000 in the fp64 oracle, so the
result is the oracle's.  Global chunks can lose all their tiles (empty
partials).  Cases: the BigBird-base workload with the query-side mask on
every (b, h) slice; a batch whose first 32 keys are masked (skipping must
stay off there) beside one that skips; short valid lengths that empty
whole chunks; block sizes 32 and 128.  The backward uses the same bitmap:
dQ drops the key tiles, dK/dV writes zeros for key items whose keys are all
masked, and with the query-side mask dQ skips items of padding rows and
dK/dV's walks leave out query tiles of padding rows (their P is 0)."""

import numpy as np
import pytest
import torch

from block_sparse_long_bwd_b200 import synth
from gpu_util import (ATOL, assert_bf16_is_rounded_fp32, assert_close, oracle_slice,
                      run_gpu)

pytestmark = pytest.mark.gpu

FWD = ("out", "lse")


def _compare(cfg, inp, res, mask_queries=0):
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ora = oracle_slice(cfg, inp, res["table"], b, h, backward=False,
                               mask_queries=mask_queries)
            assert_close(res, ora, b, h, ATOL[cfg["dtype"]], FWD)


def test_base_fwd_with_query_mask_every_slice():
    cfg = synth.WORKLOADS["base_fwd_l4096"]
    inp = synth.make_inputs(cfg, with_grad=False)
    res = run_gpu(cfg, inp, backward=False, mask_queries=1)
    assert res["status_fwd"] == 0
    km = inp["key_mask"]
    for b in range(cfg["B"]):
        assert (res["out"][b][:, km[b] == 0] == 0).all()
    _compare(cfg, inp, res, mask_queries=1)


@pytest.mark.parametrize("bs", [32, 64, 128])
def test_skip_rule_per_batch(bs):
    """Batch 0: keys 0..31 masked and a masked run of whole tiles: no tile
    is skipped there, rows see the -10000 offset as defined (every row still
    has a valid key in the last block).  Batch 1: only 1024 valid keys
    of 4096, so most tiles, and whole global chunks, are skipped.  Batch 2:
    keys 0..31 valid, a masked run of whole tiles in the middle."""
    L = 4096
    cfg = dict(B=3, H=2, L=L, block_size=bs, d=64, r=3, dtype="bf16",
               seed=71, mask=None, passes="fwd")
    inp = synth.make_inputs(cfg, with_grad=False)
    km = np.ones((3, L), np.uint8)
    km[0, :32] = 0
    km[0, 1024:2048] = 0
    km[1, 1024:] = 0
    km[2, 1280:2560] = 0
    inp["key_mask"] = torch.from_numpy(km)
    res = run_gpu(cfg, inp, backward=False)
    assert res["status_fwd"] == 0
    _compare(cfg, inp, res)


# ---- the backward: the same bitmap, in dQ's tile lists and dK/dV's items --


def _compare_backward(cfg, inp, mask_queries):
    """Forward outputs at the bf16 tolerance; gradients through their fp32
    form (with few valid keys the global key blocks' exact gradients exceed
    4, where bf16's own spacing is above 1e-2), the bf16 gradients of the
    same kernels being those values rounded to nearest even."""
    res = run_gpu(cfg, inp, mask_queries=mask_queries)
    r32 = run_gpu(cfg, inp, mask_queries=mask_queries, grad_fp32=1)
    for r in (res, r32):
        assert r["status_fwd"] == 0 and r["status_bwd"] == 0
    assert_bf16_is_rounded_fp32(res, r32)
    tol = ATOL[cfg["dtype"]]
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ora = oracle_slice(cfg, inp, res["table"], b, h,
                               mask_queries=mask_queries)
            assert_close(res, ora, b, h, tol, FWD)
            assert_close(r32, ora, b, h, tol, ("dq", "dk", "dv"))
    return res


@pytest.mark.parametrize("bs", [32, 64, 128])
@pytest.mark.parametrize("mq", [0, 1])
def test_backward_skip_rule_per_batch(bs, mq):
    """dQ drops key tiles whose keys are all masked (and, with the
    query-side mask, whole items of padding rows); dK/dV writes zeros for
    key items whose keys are all masked.  Same batches as the forward case:
    batch 0 keeps every tile (keys 0..31 masked), batch 1 has 1024 valid
    keys of 4096 (most items and whole global chunks empty), batch 2 a
    masked run in the middle."""
    L = 4096
    cfg = dict(B=3, H=2, L=L, block_size=bs, d=64, r=3, dtype="bf16",
               seed=72, mask=None, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    km = np.ones((3, L), np.uint8)
    km[0, :32] = 0
    km[0, 1024:2048] = 0
    km[1, 1024:] = 0
    km[2, 1280:2560] = 0
    inp["key_mask"] = torch.from_numpy(km)
    res = _compare_backward(cfg, inp, mq)
    # fully masked keys get exactly zero dK and dV (batch 1's tail)
    assert bool((res["dk"][1, :, 1024:] == 0).all())
    assert bool((res["dv"][1, :, 1024:] == 0).all())
    if mq:  # and padding rows exactly zero dQ
        assert bool((res["dq"][1, :, 1024:] == 0).all())


def test_backward_skip_base_layer_shape():
    """The BigBird-base shape (B 8, H 12, its tail mask) through fwd + bwd
    with the query-side mask: whole global rows, skipped tiles on both
    sides; every (b, h) slice against the oracle."""
    cfg = dict(synth.WORKLOADS["base_fwd_l4096"])
    cfg["passes"] = "fwd+bwd"
    inp = synth.make_inputs(cfg)
    _compare_backward(cfg, inp, 1)


@pytest.mark.parametrize("L,bs", [(8192, 64), (1024, 32)])
def test_backward_heavy_padding_without_query_mask(L, bs):
    """Three quarters of the keys masked and the padding rows computed (no
    query-side mask): their probability concentrates on the global blocks'
    valid keys, whose gradients then grow like a long sequence's.  Block 64
    at 8192 tokens takes the split dK/dV variant (the bf16 low part), block
    32 at 1024 does not need it; both within the tolerance."""
    cfg = dict(B=1, H=2, L=L, block_size=bs, d=64, r=3, dtype="bf16",
               seed=73, mask=None, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    km = np.zeros((1, L), np.uint8)
    km[0, :L // 4] = 1
    inp["key_mask"] = torch.from_numpy(km)
    _compare_backward(cfg, inp, 0)


def test_backward_query_skip_long_chunked():
    """16384 tokens with the query-side mask and a tail of padding: the
    global key blocks run in their own split launch on 8-tile chunks of
    query tiles, and the chunks that lie wholly in the padding lose every
    query tile (zero partials merged by the finish launch); the middle key
    items drop their padded query tiles.  Every slice against the oracle."""
    L = 16384
    cfg = dict(B=2, H=1, L=L, block_size=64, d=64, r=3, dtype="bf16",
               seed=74, mask=None, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    km = np.ones((2, L), np.uint8)
    km[0, 5000:] = 0          # 11384 padding tokens (tiles 79..255 dead)
    km[1, 9000:12288] = 0     # a padded run inside the sequence
    inp["key_mask"] = torch.from_numpy(km)
    res = _compare_backward(cfg, inp, 1)
    assert bool((res["dq"][0, :, 5000:] == 0).all())


def test_backward_query_skip_with_stored_dropout():
    """Dropout with the forward's decisions stored, together with the
    query-side mask: the dK/dV softmax warps load each visited tile's keep
    words (one tile ahead when its entry is already published), over walks
    with padded query tiles left out."""
    L = 4096
    cfg = dict(B=2, H=2, L=L, block_size=64, d=64, r=3, dtype="bf16",
               seed=75, mask=None, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    km = np.ones((2, L), np.uint8)
    km[0, 2600:] = 0
    km[1, 700:1900] = 0
    inp["key_mask"] = torch.from_numpy(km)
    seed = 0x1234ABCD5678EF01
    res = run_gpu(cfg, inp, mask_queries=1, dropout=0.1, dropout_seed=seed)
    redrawn = run_gpu(cfg, inp, mask_queries=1, dropout=0.1,
                      dropout_seed=seed, keep_dropout_bits=False)
    for r in (res, redrawn):
        assert r["status_fwd"] == 0 and r["status_bwd"] == 0
    for n in ("out", "lse", "dq", "dk", "dv"):
        assert torch.equal(res[n], redrawn[n]), n
    tol = ATOL[cfg["dtype"]]
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ora = oracle_slice(cfg, inp, res["table"], b, h, dropout=0.1,
                               dropout_seed=seed, mask_queries=1)
            assert_close(res, ora, b, h, tol, ("out", "lse", "dq", "dk", "dv"))
