"""The seeded input generators shared by the tests and the bench: the
recipe they state (draw order, dtype cast, mask kinds), determinism, and
that a batch slice equals the corresponding rows of the full inputs."""

import numpy as np
import pytest
import torch

from block_sparse_long_bwd_b200 import synth


def _cfg(**kw):
    base = dict(B=3, H=2, L=512, block_size=64, d=64, r=3, dtype="bf16",
                seed=9, mask="tail", passes="fwd+bwd")
    base.update(kw)
    return base


def test_draw_order_and_cast():
    cfg = _cfg()
    inp = synth.make_inputs(cfg)
    g = torch.Generator().manual_seed(cfg["seed"])
    for name in ("q", "k", "v", "dout"):
        ref = torch.randn((3, 2, 512, 64), generator=g, dtype=torch.float32)
        assert inp[name].dtype == torch.bfloat16
        assert torch.equal(inp[name], ref.to(torch.bfloat16)), name
    f32 = synth.make_inputs(_cfg(dtype="f32"))
    assert f32["q"].dtype == torch.float32
    assert torch.equal(f32["q"].to(torch.bfloat16), inp["q"])


def test_deterministic_and_seed_dependent():
    a = synth.make_inputs(_cfg())
    b = synth.make_inputs(_cfg())
    c = synth.make_inputs(_cfg(seed=10))
    for n in ("q", "k", "v", "dout", "key_mask"):
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["q"], c["q"])
    assert "dout" not in synth.make_inputs(_cfg(), with_grad=False)


@pytest.mark.parametrize("L", [128, 1088, 4096])
def test_tail_mask_lengths(L):
    m = synth.make_key_mask("tail", 64, L, 5).numpy()
    assert m.dtype == np.uint8 and m.shape == (64, L)
    for row in m:
        n = int(row.sum())
        assert (row[:n] == 1).all() and (row[n:] == 0).all()  # a prefix
        assert (n - L // 2) % 64 == 0 and L // 2 <= n <= L
        if (L // 2) % 64 == 0:
            assert n % 64 == 0


def test_random5_mask_count():
    L = 4096
    m = synth.make_key_mask("random5", 8, L, 6).numpy()
    assert ((m == 0).sum(axis=1) == round(0.05 * L)).all()
    assert synth.make_key_mask(None, 8, L, 6) is None
    with pytest.raises(ValueError):
        synth.make_key_mask("bogus", 1, 64, 0)


def test_batch_slice_matches_full_inputs():
    cfg = _cfg(mask="random5")
    full = synth.make_inputs(cfg)
    part = synth.make_inputs(cfg, batch_slice=slice(1, 3))
    for n in ("q", "k", "v", "dout", "key_mask"):
        assert torch.equal(part[n], full[n][1:3]), n


def test_workloads_and_sweep_points():
    for name, cfg in synth.WORKLOADS.items():
        assert cfg["L"] % cfg["block_size"] == 0, name
        assert cfg["d"] == 64
    pts = [synth.sweep_point(L, bs, r) for L in synth.SWEEP_L
           for bs in synth.SWEEP_BS for r in synth.SWEEP_R]
    assert len(pts) == 54
    for p in pts:
        assert p["B"] * p["L"] == synth.SWEEP_TOKENS and p["H"] == 12
