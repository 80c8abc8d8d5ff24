"""GPU parity at the edges of the dispatch: the degenerate and maximum-size
shapes of the tensor-core path (one block of 128 tokens, a single global
block over two tiles; two blocks of 32 tokens, both global blocks inside
one tile; r at the planner's bound with enough blocks for every middle row
to draw it, a full candidate sort and a full tile list per item), bf16
shapes just outside it (run by the CUDA-core kernels), and a random table
built with the pages' layer options."""

import numpy as np
import pytest

import oracle
from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice, run_gpu

pytestmark = pytest.mark.gpu

ALL = ("out", "lse", "dq", "dk", "dv")

EDGES = [
    # B, H, L, bs, r, mask
    (2, 1, 128, 128, 3, None),         # nb = 1 at block 128
    (2, 2, 64, 32, 2, "tail"),         # nb = 2 at block 32
    (1, 1, 4096, 64, 27, "random5"),   # r at the bound, block 64
    (1, 1, 4096, 32, 11, None),        # r at the bound, block 32
    (1, 1, 4096, 128, 11, None),       # r at the bound, block 128
]


@pytest.mark.parametrize("case", EDGES)
def test_edge_shapes_full_compare(case):
    B, H, L, bs, r, mask = case
    import torch
    desc = bb.make_desc(B, H, L, 64, bs, r, torch.bfloat16)
    assert bb.bb_attn_launch_name(desc, 0, 1) == "tc_fwd"  # tensor-core path
    cfg = dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype="bf16",
               seed=61, mask=mask, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    for b in range(B):
        for h in range(H):
            ora = oracle_slice(cfg, inp, res["table"], b, h)
            assert_close(res, ora, b, h, ATOL["bf16"], ALL)


def _cfg(B, H, L, bs, r, mask, seed):
    return dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype="bf16",
                seed=seed, mask=mask, passes="fwd+bwd")


def _check_all(cfg, res, inp):
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ora = oracle_slice(cfg, inp, res["table"], b, h)
            assert_close(res, ora, b, h, ATOL["bf16"], ALL)


FALLBACK = [
    # B, H, L, bs, r, mask: bf16 outside the tensor-core bounds
    (1, 2, 96, 32, 2, "tail"),        # L not a multiple of 64
    (1, 1, 1024, 64, 28, None),       # r past the planner bound
    (1, 1, 1024, 32, 12, "random5"),
]


@pytest.mark.parametrize("case", FALLBACK)
def test_bf16_outside_tensor_core_bounds_full_compare(case):
    import torch
    B, H, L, bs, r, mask = case
    desc = bb.make_desc(B, H, L, 64, bs, r, torch.bfloat16)
    assert bb.bb_attn_launch_name(desc, 0, 0) == "simt_fwd"
    cfg = _cfg(B, H, L, bs, r, mask, 11)
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check_all(cfg, res, inp)


def test_layer_table_options_full_compare():
    """The pages' layer table: drawn for 4096 tokens with random blocks
    before token 1024 and the layer index (5) as seed, used at L = 2048
    (rows truncated, fewer random ids in some rows)."""
    cfg = _cfg(2, 3, 2048, 64, 3, "tail", 15)
    inp = synth.make_inputs(cfg)
    table = bb.bb_rand_attn_build_ex(5, 3, 2048 // 64, 3, 4096 // 64,
                                     1024 // 64)
    assert np.array_equal(table.numpy(),
                          oracle.rand_table(5, 3, 32, 3, 64, 16))
    res = run_gpu(cfg, inp, table=table)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    _check_all(cfg, res, inp)
