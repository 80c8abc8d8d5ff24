"""The forward entry point that allocates nothing (bb_attn_fwd_noalloc).

It serves callers that cannot allocate device memory (an engine that
reserves its memory budget at start-up, a plugin that must not bypass its
host framework's allocator): it runs the ordinary forward with the library's
built-in scratch array in place of a caller workspace.  Both paths run the
same deterministic kernels, so the outputs must be bitwise equal; every call
reuses the same scratch, so the test alternates shapes (and masks) between
calls, which would expose a call that read what an earlier one left behind.
The file sorts last so that a run that stops at the first failure has run
every other test before it."""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, oracle_slice

pytestmark = pytest.mark.gpu

_SEQUENCE = ["large_train_l4096", "base_fwd_l4096", "large_train_l4096",
             "tiny_fp32_l1024", "base_fwd_l4096"]


def _setup(name):
    cfg = synth.WORKLOADS[name]
    inp = synth.make_inputs(cfg, with_grad=False)
    dev = torch.device("cuda")
    att = bb.Attention(cfg["B"], cfg["H"], cfg["L"], cfg["block_size"],
                       cfg["r"], synth.torch_dtype(cfg["dtype"]))
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    return cfg, inp, att, q, k, v, km


def test_no_alloc_forward_bitwise_equal_across_shapes():
    """Calls in a row on different shapes: large, base (tail mask), large
    again, the fp32 CUDA-core case, base again.  Each no-alloc result equals
    the workspace forward's bit for bit, its status word reads OK, and two
    (b, h) slices per shape match the oracle."""
    seen = set()
    for name in _SEQUENCE:
        cfg, inp, att, q, k, v, km = _setup(name)
        out_ref, lse_ref = att.forward(q, k, v, km)
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32,
                         device=q.device)
        bb.bb_attn_fwd_noalloc(att.desc, q, k, v, km, att.table, out, lse)
        assert bb.bb_attn_noalloc_status() == 0, name
        torch.cuda.synchronize()
        assert torch.equal(out, out_ref), name
        assert torch.equal(lse, lse_ref), name
        if name in seen:
            continue
        seen.add(name)
        tol = ATOL[cfg["dtype"]]
        res = {"out": out.float().cpu(), "lse": lse.cpu()}
        for b, h in ((0, 0), (cfg["B"] - 1, cfg["H"] - 1)):
            ora = oracle_slice(cfg, inp, att.table_host, b, h, backward=False)
            for n in ("out", "lse"):
                err = np.abs(res[n][b, h].double().numpy() - ora[n]).max()
                assert err <= tol, (name, n, b, h, err)


def test_no_alloc_status_reports_a_corrupt_table():
    """A table entry outside [-1, nb) is ignored and flagged: the no-alloc
    call's status word must say so, and the next clean call clears it."""
    cfg, inp, att, q, k, v, km = _setup("large_train_l4096")
    nb = cfg["L"] // cfg["block_size"]
    bad = att.table.clone()
    bad[1, 5, 0] = nb + 3
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    bb.bb_attn_fwd_noalloc(att.desc, q, k, v, km, bad, out, lse)
    assert bb.bb_attn_noalloc_status() == bb.BB_ERR_BAD_TABLE
    bb.bb_attn_fwd_noalloc(att.desc, q, k, v, km, att.table, out, lse)
    assert bb.bb_attn_noalloc_status() == 0


def test_no_alloc_rejects_problems_beyond_its_scratch():
    # 1024 (b, h) slices at L = 4096 need far more than the 32 MiB scratch;
    # the call must refuse before touching any pointer.
    desc = bb.make_desc(64, 16, 4096, 64, 64, 3, torch.bfloat16)
    fake = 1 << 20
    rc = bb.lib().bb_attn_fwd_noalloc(ctypes.byref(desc), fake, fake, fake,
                                      None, fake, fake, fake, None)
    assert rc == bb.BB_ERR_WORKSPACE
