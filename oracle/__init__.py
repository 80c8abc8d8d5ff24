"""fp64 CPU oracle (test infrastructure only; see bigbird_oracle)."""

from .bigbird_oracle import (  # noqa: F401
    DEFAULT_MASK_VALUE,
    SplitMix64,
    attended_blocks,
    backward,
    block_probs,
    forward,
    pair_count,
    rand_table,
    random_candidates,
)
