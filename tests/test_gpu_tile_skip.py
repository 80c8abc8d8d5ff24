"""GPU parity of the forward's skipping of fully masked key tiles.

A 64-key tile whose keys are all masked is dropped from an item's tile list
when every row of the batch has a valid attended key (a valid key among the
first 32, which lie in global block 0); a masked key's probability is then
exp(-10000 + ...), zero in fp32 and below 1e-4000 in the fp64 oracle, so the
result is the oracle's.  Global chunks can lose all their tiles (empty
partials).  Cases: the BigBird-base workload with the query-side mask on
every (b, h) slice; a batch whose first 32 keys are masked (skipping must
stay off there) beside one that skips; short valid lengths that empty
whole chunks; block sizes 32 and 128."""

import numpy as np
import pytest
import torch

from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice, run_gpu

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
