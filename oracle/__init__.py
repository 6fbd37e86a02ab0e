"""CPU oracle for the ISPA warmup path. TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
package. The product path (the C-ABI library and its Python binding) never calls it and
shares no code with it.
"""
from .ispa_oracle import (  # noqa: F401
    bf16_round,
    partition_masks,
    masked_attention,
    split_attention,
    lse_merge,
    local_attention,
    stats_init,
    stats_update,
    absorb_solve,
    reconstruction_error,
    select_layers,
    project,
    run_episode,
    live_error,
    rewarm_trigger,
    quantize_int8,
    project_w8a8,
    kv_blocks,
    quantize_i8_q,
    quantize_i8_k,
    split_attention_i8,
)
