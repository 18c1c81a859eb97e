"""sv_cache_step_noalloc: the streaming step for callers that cannot allocate device memory
(framework operators whose memory belongs to the host, real-time block loops that must not call
cudaMalloc, code recorded into CUDA graphs). It must give what sv_cache_step gives with a
caller-owned workspace, call after call, and refuse blocks that do not fit its 16 MiB scratch.

Kept in a file of its own that pytest collects last; it passes alone in a fresh process and after
the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_causal_linear_relu_b200.inputs import draw_qkv

pytestmark = pytest.mark.gpu

TOL_O = 2e-2      # bf16 output tolerance used by the parity tests
TOL_CACHE = 1e-4  # fp32 cache tolerance used by the parity tests


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()


def test_noalloc_step_matches_workspace_step_two_calls():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as sv
    lib = sv.load()
    vp = ctypes.c_void_p
    B, H, N, D = 1, 20, 2760, 128   # one 720p streaming block (3 latent frames of 23 x 40 tokens)
    blocks = [tuple(_dev(x) for x in draw_qkv((B, H, N, D), seed, "bf16")) for seed in (0, 1)]
    # reference: the existing entry point with a caller-owned workspace
    S_ref = torch.zeros(B, H, D, D, device="cuda")
    z_ref = torch.zeros(B, H, D, device="cuda")
    ws = sv.make_workspace(sv.SV_OP_CACHE_STEP, blocks[0][0])
    assert ws.nbytes <= 16 << 20
    # the no-allocation entry point, called through the C ABI, on the same two blocks in a row
    S = torch.zeros(B, H, D, D, device="cuda")
    z = torch.zeros(B, H, D, device="cuda")
    stream = vp(torch.cuda.current_stream().cuda_stream)
    for q, k, v in blocks:
        o_ref = sv.sv_cache_step(q, k, v, S_ref, z_ref, commit=True, eps=1e-6, ws=ws)
        o = torch.empty_like(q)
        st = lib.sv_cache_step_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(o.data_ptr()),
                                       B, H, N, D, sv.SV_BF16, 1e-6, vp(S.data_ptr()), vp(z.data_ptr()), 1, stream)
        assert st == 0, lib.sv_last_error()
        torch.cuda.synchronize()
        assert _rel(o, o_ref) < TOL_O
        assert _rel(S, S_ref) < TOL_CACHE and _rel(z, z_ref) < TOL_CACHE
    assert ws.status() == 0


def test_noalloc_step_refuses_blocks_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    import block_causal_linear_relu_b200 as sv
    lib = sv.load()
    vp = ctypes.c_void_p
    # the scratch need grows with B*H (one fp32 D x (D+1) partial per (batch, head) and per CTA):
    # eight 720p streams of 20 heads in one call need about 20 MB
    B, H, N, D = 8, 20, 2760, 128
    need = lib.sv_workspace_bytes(sv.SV_OP_CACHE_STEP, B, H, N, D, N, sv.SV_BF16)
    assert need > 16 << 20
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")  # never read: the call is refused first
    S = torch.zeros(16, device="cuda")
    p = vp(x.data_ptr())
    st = lib.sv_cache_step_noalloc(p, p, p, p, B, H, N, D, sv.SV_BF16, 1e-6, vp(S.data_ptr()), vp(S.data_ptr()), 1,
                                   None)
    assert st == sv._native.SV_ERR_INVALID_ARG
    assert b"static scratch" in lib.sv_last_error()
