"""Failure detection without a GPU fault: a device wait on a barrier that
nothing completes runs out after its limit, the kernel reports
BB_ERR_TIMEOUT through the status word and exits, and the context stays
usable (a normal call afterwards matches the oracle)."""

import time

import pytest
import torch

from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    bb.bb_debug_wait_probe(ws, armed=0)
    assert bb.bb_attn_check_status(ws) == bb.BB_OK
    t0 = time.perf_counter()
    bb.bb_debug_wait_probe(ws, armed=1)
    status = bb.bb_attn_check_status(ws)
    waited = time.perf_counter() - t0
    assert status == bb.BB_ERR_TIMEOUT
    assert 1.5 < waited < 60.0  # the 2 s limit, not an endless wait
    # the context is still usable
    cfg = dict(B=1, H=2, L=1024, block_size=64, d=64, r=3, dtype="bf16",
               seed=41, mask="tail", passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    res = run_gpu(cfg, inp)
    assert res["status_fwd"] == 0 and res["status_bwd"] == 0
    ora = oracle_slice(cfg, inp, res["table"], 0, 1)
    assert_close(res, ora, 0, 1, ATOL["bf16"],
                 ("out", "lse", "dq", "dk", "dv"))
