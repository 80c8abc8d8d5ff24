"""The forward entry point that allocates nothing (bb_attn_fwd_noalloc).

It exists for callers that cannot allocate device memory (an engine that
reserves its memory budget at start-up, a plugin that must not bypass its
host framework's allocator): it runs the ordinary forward with the library's
built-in scratch array in place of a caller workspace.  Here it is called
through the C ABI and compared with bb_attn_fwd on the same inputs, twice in
a row, since every call reuses the same scratch."""

import ctypes

import pytest
import torch

from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["large_train_l4096", "base_fwd_l4096"])
def test_no_alloc_forward_matches_workspace_forward(name):
    cfg = synth.WORKLOADS[name]
    inp = synth.make_inputs(cfg, with_grad=False)
    dev = torch.device("cuda")
    att = bb.Attention(cfg["B"], cfg["H"], cfg["L"], cfg["block_size"],
                       cfg["r"], torch.bfloat16)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    out_ref, lse_ref = att.forward(q, k, v, km)
    tol = ATOL["bf16"]
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32,
                         device=dev)
        bb.bb_attn_fwd_noalloc(att.desc, q, k, v, km, att.table, out, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
        assert (out.float() - out_ref.float()).abs().max().item() <= tol
        assert (lse - lse_ref).abs().max().item() <= tol


def test_no_alloc_rejects_problems_beyond_its_scratch():
    # 1024 (b, h) slices at L = 4096 need far more than the 32 MiB scratch;
    # the call must refuse before touching any pointer.
    desc = bb.make_desc(64, 16, 4096, 64, 64, 3, torch.bfloat16)
    fake = 1 << 20
    rc = bb.lib().bb_attn_fwd_noalloc(ctypes.byref(desc), fake, fake, fake,
                                      None, fake, fake, fake, None)
    assert rc == -4  # BB_ERR_WORKSPACE
