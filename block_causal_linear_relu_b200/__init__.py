"""ReLU-kernel linear attention (bidirectional and block-causal with a constant-memory cache)
for NVIDIA B200 (sm_100a).

The compute lives in ``libsvlinattn.so`` (hand-written CUDA, C ABI declared in
``include/svlinattn.h``); this package is its thin ctypes binding plus a seeded input generator.
"""

from ._native import (  # noqa: F401
    EXPORTS,
    SV_BF16,
    SV_F32,
    SV_OP_BLOCK_CAUSAL_ATTN,
    SV_OP_BLOCK_STATE_UPDATE,
    SV_OP_CACHE_STEP,
    SV_OP_LINATTN_FWD,
    Rope3dTable,
    SvError,
    SvRope3d,
    Workspace,
    lib_path,
    load,
    make_workspace,
    rope_pairs,
    sv_block_causal_attn,
    sv_block_causal_attn_rope,
    sv_block_state_update,
    sv_cache_step,
    sv_cache_step_noalloc,
    sv_cache_step_noalloc_status,
    sv_linattn_fwd,
    sv_out_projection,
    sv_qkv_projection,
    sv_profile_events,
    sv_rope3d_table,
    sv_rope3d_table_bytes,
    sv_selftest_wait_timeout,
    sv_temporal_conv,
    sv_temporal_conv_step,
    workspace_bytes,
)
