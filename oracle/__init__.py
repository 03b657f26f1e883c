"""CPU fp64 oracle (test infrastructure only; see mla_oracle's header)."""
from .mla_oracle import (  # noqa: F401
    DEFAULT_ROPE_BASE,
    attend_sequence,
    build_slot_index,
    cache_rows_rotated,
    decode,
    default_softmax_scale,
    gather_rows,
    latent_append,
    rope,
    rope_angles,
)
