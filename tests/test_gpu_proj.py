"""GPU parity of the projections either side of the attention (the fused
Q/K/V projection into the [B, H, L, 64] layout and the output projection
from it) against the fp64 oracle, and of the whole layer step
(projection -> block-sparse attention -> output projection).

Tolerance, from the arithmetic: the kernel accumulates bf16 products in
fp32 (error below 2e-3 for these sizes, K <= 1024 terms of unit scale) and
rounds once to bf16, so an element may differ from the exact value by half
a bf16 unit in the last place of that value plus 2e-3."""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_bwd_b200 import binding as bb
from block_sparse_long_bwd_b200 import synth

pytestmark = pytest.mark.gpu


def _tol(ref):
    a = np.abs(ref)
    half_ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.maximum(a, 1e-30))) - 8), 0.0)
    return half_ulp + 2e-3


def _check(got, ref, what):
    g = got.double().cpu().numpy()
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    bad = err > _tol(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max err {err.max():.3e}"


def _ws():
    return torch.zeros(256, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("B,L,hidden,H,bias", [
    (2, 256, 768, 12, True),    # BigBird-base layer widths
    (1, 384, 1024, 16, True),   # BigBird-large layer widths
    (1, 128, 768, 12, False),   # no bias
    (3, 128, 256, 4, True),     # one column tile per Q / K / V
])
def test_qkv_and_out_projection_full_compare(B, L, hidden, H, bias):
    inp = synth.make_proj_inputs(B, L, hidden, H, seed=31, bias=bias)
    dev = torch.device("cuda")
    t = {k_: (None if v_ is None else v_.to(dev)) for k_, v_ in inp.items()}
    ws = _ws()
    q, k, v = bb.bb_qkv_proj(t["x"], t["w_qkv"], t["b_qkv"], H, ws)
    torch.cuda.synchronize()
    assert bb.bb_attn_check_status(ws) == 0
    f = lambda x: None if x is None else x.double().numpy()
    rq, rk, rv = oracle.qkv_projection(f(inp["x"]), f(inp["w_qkv"]), f(inp["b_qkv"]), H)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        _check(got, ref, name)
    if hidden % 256 == 0:
        out = bb.bb_out_proj(q, t["w_o"], t["b_o"], ws)
        torch.cuda.synchronize()
        ro = oracle.output_projection(f(q.cpu()), f(inp["w_o"]), f(inp["b_o"]))
        _check(out, ro, "out")


def test_qkv_projection_full_size_sampled_tokens():
    """The BigBird-base layer at L = 4096, B = 8 (32768 tokens), in the
    launch configuration the benchmark times; 512 sampled tokens compared
    (a token's q, k, v depend on its own row of x only)."""
    B, L, hidden, H = 8, 4096, 768, 12
    inp = synth.make_proj_inputs(B, L, hidden, H, seed=32)
    dev = torch.device("cuda")
    ws = _ws()
    q, k, v = bb.bb_qkv_proj(inp["x"].to(dev), inp["w_qkv"].to(dev), inp["b_qkv"].to(dev), H, ws)
    out = bb.bb_out_proj(q, inp["w_o"].to(dev), inp["b_o"].to(dev), ws)
    torch.cuda.synchronize()
    assert bb.bb_attn_check_status(ws) == 0
    rows = np.random.default_rng(5).choice(B * L, size=512, replace=False)
    bi, li = rows // L, rows % L
    x = inp["x"].double().numpy()[bi, li][None]           # [1, 512, hidden]
    rq, rk, rv = oracle.qkv_projection(x, inp["w_qkv"].double().numpy(),
                                       inp["b_qkv"].double().numpy(), H)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        g = got[bi, :, li].permute(1, 0, 2).unsqueeze(0)  # [1, H, 512, 64]
        _check(g, ref, name)
    o_rows = q[bi, :, li].double().cpu().numpy()[None].transpose(0, 2, 1, 3)  # [1, H, 512, 64]
    ro = oracle.output_projection(o_rows, inp["w_o"].double().numpy(), inp["b_o"].double().numpy())
    _check(out[bi, li].unsqueeze(0), ro, "out")


def test_layer_step_projection_attention_projection():
    """x -> Q, K, V (fused projection) -> block-sparse attention -> output
    projection, against the oracle's composition of the same steps on the
    GPU's own intermediate bf16 tensors (each step compared on its inputs)."""
    B, L, hidden, H, bs, r = 1, 1024, 768, 12, 64, 3
    inp = synth.make_proj_inputs(B, L, hidden, H, seed=33)
    dev = torch.device("cuda")
    ws = _ws()
    q, k, v = bb.bb_qkv_proj(inp["x"].to(dev), inp["w_qkv"].to(dev), inp["b_qkv"].to(dev), H, ws)
    att = bb.Attention(B, H, L, bs, r, torch.bfloat16)
    o, lse = att.forward(q, k, v)
    out = bb.bb_out_proj(o, inp["w_o"].to(dev), inp["b_o"].to(dev), ws)
    torch.cuda.synchronize()
    f = lambda x: x.double().cpu().numpy()
    ro, _ = oracle.forward(f(q), f(k), f(v), None, att.table_host.numpy(), bs)
    assert np.abs(f(o) - ro).max() <= 1e-2
    _check(out, oracle.output_projection(f(o), f(inp["w_o"]), f(inp["b_o"])), "out")


def test_projection_shape_checks():
    dev = torch.device("cuda")
    ws = _ws()
    x = torch.zeros((1, 100, 768), dtype=torch.bfloat16, device=dev)   # L % 128 != 0
    w = torch.zeros((3 * 768, 768), dtype=torch.bfloat16, device=dev)
    with pytest.raises(bb.BBError) as e:
        bb.bb_qkv_proj(x, w, None, 12, ws)
    assert e.value.code == -2
    x = torch.zeros((1, 128, 768), dtype=torch.bfloat16, device=dev)
    with pytest.raises(bb.BBError) as e:
        bb.bb_qkv_proj(x, w, None, 6, ws, q=torch.empty((1, 6, 128, 64), dtype=torch.bfloat16, device=dev))
    assert e.value.code == -2  # H % 4 != 0
