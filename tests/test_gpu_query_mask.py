"""GPU parity of the query-side mask (mask_queries = 1): the key mask also
zeroes the output rows of padding tokens, which then pass no gradient; the
CUDA path through the C ABI against the fp64 oracle with query_mask set to
the same mask, on the tensor-core path (middle and global rows, which are
zeroed when their chunks are combined) and the CUDA-core path."""

import pytest
import torch

from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice, run_gpu

pytestmark = pytest.mark.gpu

ALL = ("out", "lse", "dq", "dk", "dv")

CASES = [
    # B, H, L, bs, r, dtype, mask, dropout
    (2, 2, 1088, 64, 3, "bf16", "tail", 0.0),     # padding in the last block
    (1, 2, 1024, 32, 3, "bf16", "random5", 0.0),
    (2, 1, 2048, 128, 3, "bf16", "tail", 0.0),
    (2, 2, 1088, 64, 3, "bf16", "tail", 0.1),     # with dropout
    (1, 2, 448, 64, 1, "f32", "tail", 0.0),       # CUDA-core path
    (1, 2, 96, 32, 2, "bf16", "tail", 0.0),       # bf16 on the CUDA cores
]


@pytest.mark.parametrize("case", CASES)
def test_query_mask_full_compare(case):
    B, H, L, bs, r, dtype, mask, rate = case
    cfg = dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype=dtype,
               seed=51, mask=mask, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp, dropout=rate, dropout_seed=9, mask_queries=1)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    km = inp["key_mask"]
    assert (km == 0).any()  # some padding in the batch
    for b in range(B):
        pad = km[b] == 0
        assert (res["out"][b][:, pad] == 0).all()
        assert (res["dq"][b][:, pad] == 0).all()
        for h in range(H):
            ora = oracle_slice(cfg, inp, res["table"], b, h, dropout=rate,
                               dropout_seed=9, mask_queries=1)
            assert_close(res, ora, b, h, ATOL[dtype], ALL)


def test_query_mask_without_key_mask_is_the_plain_operation():
    cfg = dict(B=1, H=2, L=1024, block_size=64, d=64, r=3, dtype="bf16",
               seed=52, mask=None, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    a = run_gpu(cfg, inp)
    b = run_gpu(cfg, inp, mask_queries=1)
    for n in ALL:
        assert torch.equal(a[n], b[n]), n
