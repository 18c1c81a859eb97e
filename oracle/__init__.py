"""CPU oracle for ReLU-kernel linear attention (fp64). Test infrastructure only: imported by the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``; never by the product
path."""

from .linattn import (  # noqa: F401
    apply_states,
    block_causal_attn,
    block_state_update,
    block_states,
    bruteforce_masked,
    cache_step,
    causal_recurrence,
    linattn_fwd,
    max_rel_err,
    num_blocks,
    phi,
    prefix_states,
    rows_from_states,
)
from .projection import out_projection, qkv_projection  # noqa: F401,E402
from .temporal_conv import centred_conv, temporal_conv_block_causal, temporal_conv_step  # noqa: F401,E402
from .rope import (  # noqa: F401,E402
    block_causal_attn_rope,
    bruteforce_rope,
    default_pairs,
    rope3d_angles,
    rotate_pairs,
    token_positions,
)
