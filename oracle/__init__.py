"""fp64 CPU oracle (test infrastructure only; see bigbird_oracle)."""

from .bigbird_oracle import (  # noqa: F401
    DEFAULT_MASK_VALUE,
    Dropout,
    SplitMix64,
    attended_blocks,
    backward,
    block_probs,
    dropout_keep,
    dropout_scale,
    dropout_threshold,
    forward,
    output_projection,
    pair_count,
    philox4x32_10,
    qkv_projection,
    rand_table,
    random_candidates,
)
