"""CPU oracle (fp64 NumPy) for the block-sparse attention path.

Test infrastructure only: imported by tests, the smoke check and the benchmark's
CPU baseline, never by the product path."""
from .sparse_attn_oracle import (  # noqa: F401
    BLOCK, as_f64, n_blocks, block_mean_pool, pooled_logits, pooled_softmax,
    cumulative_energy_select, plan, attention_masked, attention_tiled, fwd,
)
