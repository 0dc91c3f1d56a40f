"""CPU oracle (test infrastructure only; see ``tp_oracle``)."""

from .tp_oracle import (  # noqa: F401
    ACTIVATIONS,
    apply_activation,
    attention_sharded,
    attention_unsharded,
    column_parallel_linear,
    gelu_tanh,
    heads_per_shard,
    layer_norm,
    mlp_sharded,
    mlp_unsharded,
    reduce_partials_fixed_order,
    rel_err,
    relu,
    round_to_bf16,
    sdpa_head,
    row_parallel_partials,
    shard_width,
    silu,
    transformer_block_sharded,
    transformer_block_unsharded,
)
