"""Helpers for the GPU parity tests: run the library through the C ABI and
the oracle on the same seeded inputs."""

import numpy as np
import torch

import oracle
from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth

# Tolerances the problem statement fixes: max-abs error against the fp64
# oracle, per I/O precision (applied to O, lse, dQ, dK and dV alike).
ATOL = {"f32": 2e-5, "bf16": 1e-2}


def run_gpu(cfg, inp, table_seed=synth.TABLE_SEED, backward=True,
            scale=0.0, mask_value=0.0, table=None, dropout=0.0,
            dropout_seed=0, mask_queries=0, grad_fp32=0,
            keep_dropout_bits=True, bits_fill=None):
    """Forward (and backward) through the C ABI; returns CPU tensors.
    grad_fp32: the backward writes dq, dk, dv as fp32 (returned as such;
    bf16 gradients come back widened to fp32 exactly).
    keep_dropout_bits: with dropout, the forward stores its keep decisions
    for the backward (returned as "dropout_bits", uint8); bits_fill: byte
    written over that buffer before the forward."""
    dev = torch.device("cuda")
    B, H, L = cfg["B"], cfg["H"], cfg["L"]
    att = bb.Attention(B, H, L, cfg["block_size"], cfg["r"],
                       synth.torch_dtype(cfg["dtype"]), d=cfg["d"],
                       seed=table_seed, scale=scale, mask_value=mask_value,
                       dropout=dropout, dropout_seed=dropout_seed,
                       mask_queries=mask_queries, grad_fp32=grad_fp32,
                       keep_dropout_bits=keep_dropout_bits)
    if att.dropout_bits is not None and bits_fill is not None:
        att.dropout_bits.fill_(bits_fill)
    if table is not None:
        att.table_host = torch.as_tensor(table, dtype=torch.int32)
        att.table = att.table_host.to(dev)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    km = None if inp["key_mask"] is None else inp["key_mask"].to(dev)
    out, lse = att.forward(q, k, v, km)
    res = {"out": out, "lse": lse, "table": att.table_host,
           "status_fwd": bb.bb_attn_check_status(att.ws_fwd)}
    if backward:
        dout = inp["dout"].to(dev)
        dq, dk, dv = att.backward(q, k, v, out, lse, dout, km)
        res.update(dq=dq, dk=dk, dv=dv,
                   status_bwd=bb.bb_attn_check_status(att.ws_bwd))
    torch.cuda.synchronize()
    out = {k_: (v_.float().cpu() if torch.is_tensor(v_) and v_.is_cuda
                else v_) for k_, v_ in res.items()}
    if att.dropout_bits is not None:
        out["dropout_bits"] = att.dropout_bits.cpu()
    return out


def oracle_slice(cfg, inp, table, b, h, backward=True, scale=None,
                 mask_value=oracle.DEFAULT_MASK_VALUE, dropout=0.0,
                 dropout_seed=0, mask_queries=0):
    """Oracle on the (b, h) slice: rows of one (b, h) depend on nothing else
    (the dropout decisions are drawn at the slice's own b and h)."""
    sl = lambda x: x[b:b + 1, h:h + 1].double().numpy()
    km = inp["key_mask"]
    km = None if km is None else km[b:b + 1].numpy()
    tab = np.asarray(table)[h:h + 1]
    drop = (oracle.Dropout(dropout, dropout_seed, b0=b, h0=h)
            if dropout else None)
    qm = km if (mask_queries and km is not None) else None
    o, lse = oracle.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), km, tab,
                            cfg["block_size"], scale, mask_value, drop, qm)
    res = {"out": o[0, 0], "lse": lse[0, 0]}
    if backward:
        dq, dk, dv = oracle.backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                     sl(inp["dout"]), km, tab,
                                     cfg["block_size"], scale, mask_value,
                                     drop, qm)
        res.update(dq=dq[0, 0], dk=dk[0, 0], dv=dv[0, 0])
    return res


def assert_close(gpu, ora, b, h, atol, names):
    for n in names:
        g = gpu[n][b, h].double().numpy()
        err = np.abs(g - ora[n]).max()
        assert np.isfinite(g).all(), (n, b, h)
        assert err <= atol, f"{n}[{b},{h}] max-abs err {err:.3e} > {atol}"


def assert_bf16_is_rounded_fp32(g16, g32, names=("dq", "dk", "dv")):
    """bf16 gradients equal the fp32 gradients of the same kernels rounded
    to nearest even, bit for bit (the kernels accumulate in fp32 and round
    only when storing)."""
    for n in names:
        want = g32[n].to(torch.bfloat16).float()
        assert torch.equal(g16[n], want), n
