"""Out-of-bounds write check: every output buffer and the workspace sit
between canary-filled guard regions, and the library gets exactly the
interior.  After a forward and a backward the guards must be untouched, and
no output element may still hold the canary pattern (every element written).
Covers the tensor-core path (with global chunks, and the split dK/dV launch
at L = 16384) and the CUDA-core path."""

import pytest
import torch

from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth
from gpu_util import ATOL, assert_close, oracle_slice

pytestmark = pytest.mark.gpu

CANARY = 0xA5
GUARD = 4096  # bytes on each side (keeps the interior 16-byte aligned)


def _guarded(shape, dtype, dev):
    es = torch.empty((), dtype=dtype).element_size()
    n = 1
    for s in shape:
        n *= s
    pad = GUARD // es
    buf = torch.empty(n + 2 * pad, dtype=dtype, device=dev)
    buf.view(torch.uint8).fill_(CANARY)
    return buf, buf[pad:pad + n].view(shape)


def _guards_intact(buf, dtype):
    raw = buf.view(torch.uint8)
    return bool((raw[:GUARD] == CANARY).all() and (raw[-GUARD:] == CANARY).all())


def _all_written(t):
    """No element still carries the canary byte pattern."""
    raw = t.contiguous().view(torch.uint8).view(-1, t.element_size())
    return not bool((raw == CANARY).all(dim=1).any())


@pytest.mark.parametrize("B,H,L,bs,r,dtype,mask", [
    (2, 3, 2048, 64, 3, "bf16", "tail"),   # tensor cores, global chunks
    (1, 2, 16384, 64, 3, "bf16", None),    # split dK/dV launch
    (1, 2, 1024, 32, 3, "bf16", "random5"),
    (1, 2, 448, 64, 1, "f32", "tail"),     # CUDA-core path
])
def test_outputs_and_workspace_stay_in_bounds(B, H, L, bs, r, dtype, mask):
    dev = torch.device("cuda")
    cfg = dict(B=B, H=H, L=L, block_size=bs, d=64, r=r, dtype=dtype, seed=31,
               mask=mask, passes="fwd+bwd")
    inp = synth.make_inputs(cfg)
    tdt = synth.torch_dtype(dtype)
    desc = bb.make_desc(B, H, L, 64, bs, r, tdt)
    table_host = bb.bb_rand_attn_build(synth.TABLE_SEED, H, L // bs, r)
    table = table_host.to(dev)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    shape = (B, H, L, 64)
    bufs = {}
    for name in ("out", "dq", "dk", "dv"):
        bufs[name] = _guarded(shape, tdt, dev)
    bufs["lse"] = _guarded((B, H, L), torch.float32, dev)
    bufs["ws_f"] = _guarded((bb.bb_attn_workspace_size(desc, 0),),
                            torch.uint8, dev)
    bufs["ws_b"] = _guarded((bb.bb_attn_workspace_size(desc, 1),),
                            torch.uint8, dev)
    out, lse = bufs["out"][1], bufs["lse"][1]
    bb.bb_attn_fwd(desc, q, k, v, km, table, out, lse, bufs["ws_f"][1])
    bb.bb_attn_bwd(desc, q, k, v, out, lse, g, km, table, bufs["dq"][1],
                   bufs["dk"][1], bufs["dv"][1], bufs["ws_b"][1])
    torch.cuda.synchronize()
    assert bb.bb_attn_check_status(bufs["ws_f"][1]) == 0
    assert bb.bb_attn_check_status(bufs["ws_b"][1]) == 0
    for name, (buf, view) in bufs.items():
        assert _guards_intact(buf, view.dtype), name
        if not name.startswith("ws"):
            assert _all_written(view), name
    # the guarded run computes the same as the oracle on one slice
    res = {n: bufs[n][1].float().cpu() for n in ("out", "lse", "dq", "dk", "dv")}
    ora = oracle_slice(cfg, inp, table_host, B - 1, H - 1)
    assert_close(res, ora, B - 1, H - 1, ATOL[dtype],
                 ("out", "lse", "dq", "dk", "dv"))
