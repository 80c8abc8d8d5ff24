"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws numbers: it holds none of the attention arithmetic.
Recipe (identical for the CUDA path and the oracle):

* q, k, v, dout: drawn in that order from ``torch.Generator().manual_seed(S)``
  as fp32 N(0, 1) of shape [B, H, L, d], then cast to the workload dtype
  (bf16 by round-to-nearest-even).  The oracle reads the same cast values.
* key mask (uint8 [B, L], 1 = attend) from ``numpy.random.default_rng(S+1)``:
  - "tail": per sequence a valid length drawn uniformly from
    L/2, L/2 + 64, ... (<= L) -- the multiples of 64 in [L/2, L] when L/2
    is one, as at L = 4096; keys at t >= length are masked;
  - "random5": exactly round(0.05 L) key positions per sequence, drawn
    uniformly without replacement, are masked;
  - None: no mask (all keys attended).
* The random block table uses seed 0 in every workload.

The named workloads mirror BigBird's published settings: BigBird-base
(12 heads, hidden 768, head dim 64) and BigBird-large (16 heads) at 4096
tokens with block size 64 and 3 random blocks, plus a 16K-token pattern and
a length / block-size / random-count sweep at a fixed token budget.
"""

import numpy as np
import torch

TABLE_SEED = 0

WORKLOADS = {
    # Small fp32 case the oracle finishes instantly.
    "tiny_fp32_l1024": dict(B=1, H=2, L=1024, block_size=64, d=64, r=3,
                            dtype="f32", seed=1, mask=None, passes="fwd+bwd"),
    # BigBird-base attention layer, padded batch, forward only.
    "base_fwd_l4096": dict(B=8, H=12, L=4096, block_size=64, d=64, r=3,
                           dtype="bf16", seed=2, mask="tail", passes="fwd"),
    # BigBird-large attention layer, training step.
    "large_train_l4096": dict(B=4, H=16, L=4096, block_size=64, d=64, r=3,
                              dtype="bf16", seed=3, mask=None,
                              passes="fwd+bwd"),
    # Long-sequence pattern, 5 % random key padding.
    "long_l16384": dict(B=1, H=12, L=16384, block_size=64, d=64, r=3,
                        dtype="bf16", seed=4, mask="random5",
                        passes="fwd+bwd"),
}

SWEEP_L = (1024, 2048, 4096, 8192, 16384, 32768)
SWEEP_BS = (32, 64, 128)
SWEEP_R = (0, 3, 6)
SWEEP_TOKENS = 32768


def sweep_point(L, block_size, r):
    """One point of the sweep: B*L fixed at 32768 tokens, 12 heads, d=64."""
    return dict(B=SWEEP_TOKENS // L, H=12, L=L, block_size=block_size, d=64,
                r=r, dtype="bf16", seed=5, mask=None, passes="fwd+bwd")


def torch_dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_key_mask(kind, B, L, seed):
    """uint8 [B, L] key mask (1 = attend) or None; see module doc."""
    if kind is None:
        return None
    rng = np.random.default_rng(seed + 1)
    mask = np.ones((B, L), dtype=np.uint8)
    if kind == "tail":
        choices = np.arange(L // 2, L + 1, 64)
        lengths = rng.choice(choices, size=B)
        for b in range(B):
            mask[b, int(lengths[b]):] = 0
    elif kind == "random5":
        n = int(round(0.05 * L))
        for b in range(B):
            mask[b, rng.choice(L, size=n, replace=False)] = 0
    else:
        raise ValueError(f"unknown mask kind {kind!r}")
    return torch.from_numpy(mask)


def make_inputs(cfg, with_grad=True, batch_slice=None):
    """CPU tensors q, k, v (and dout) in the workload dtype, plus key_mask.

    batch_slice (optional ``slice``) keeps only those sequences, drawn from
    the same stream as the full batch, so a sample equals the full inputs'
    corresponding rows."""
    B, H, L, d = cfg["B"], cfg["H"], cfg["L"], cfg["d"]
    g = torch.Generator().manual_seed(cfg["seed"])
    dt = torch_dtype(cfg["dtype"])
    names = ["q", "k", "v"] + (["dout"] if with_grad else [])
    out = {}
    for name in names:
        x = torch.randn((B, H, L, d), generator=g, dtype=torch.float32)
        if batch_slice is not None:
            x = x[batch_slice].contiguous()
        out[name] = x.to(dt)
    km = make_key_mask(cfg["mask"], B, L, cfg["seed"])
    if km is not None and batch_slice is not None:
        km = km[batch_slice].contiguous()
    if km is not None:
        # Every query row attends key block 0; keep it non-empty so no row
        # is entirely masked (fp32 parity would otherwise be ill-conditioned).
        bs = cfg["block_size"]
        assert bool((km[:, :bs].sum(dim=1) > 0).all())
    out["key_mask"] = km
    return out


def make_proj_inputs(B, L, hidden, H, seed, d=64, bias=True):
    """Seeded inputs of the projections either side of the attention:
    drawn in the order x, w_qkv, b_qkv, w_o, b_o from
    ``torch.Generator().manual_seed(seed)``; x ~ N(0, 1) [B, L, hidden],
    weights ~ N(0, 1/in_features) (so outputs have unit scale) in the
    linear-layer layout [out, in], biases ~ N(0, 0.01) fp32 (None when
    bias=False).  x and the weights are cast to bf16 (round to nearest
    even); the oracle reads the same values."""
    g = torch.Generator().manual_seed(seed)
    D = H * d
    x = torch.randn((B, L, hidden), generator=g).to(torch.bfloat16)
    w_qkv = (torch.randn((3 * D, hidden), generator=g) / hidden ** 0.5).to(torch.bfloat16)
    b_qkv = torch.randn((3 * D,), generator=g) * 0.1
    w_o = (torch.randn((hidden, D), generator=g) / D ** 0.5).to(torch.bfloat16)
    b_o = torch.randn((hidden,), generator=g) * 0.1
    if not bias:
        b_qkv = b_o = None
    return {"x": x, "w_qkv": w_qkv, "b_qkv": b_qkv, "w_o": w_o, "b_o": b_o}
