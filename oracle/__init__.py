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
