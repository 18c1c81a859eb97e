"""sv_cache_step_noalloc: the streaming step for callers that cannot allocate device memory
(framework operators whose memory belongs to the host, real-time block loops that must not call
cudaMalloc, code recorded into CUDA graphs). It must give what sv_cache_step gives with a
caller-owned workspace, call after call, agree with the fp64 oracle whichever kernel the block
shape selects, survive shape changes between calls on its one shared static array, and refuse blocks
that do not fit its 16 MiB scratch.

Kept in a file of its own that pytest collects last; it passes alone in a fresh process and after
the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_causal_linear_relu_b200.inputs import draw_qkv, to_f64

pytestmark = pytest.mark.gpu

TOL_O = {"bf16": 2e-2, "f32": 1e-4}  # output tolerances of the parity tests
TOL_CACHE = 1e-4                     # fp32 cache tolerance of the parity tests
EPS = 1e-6


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


def _dev(x, dtype="bf16"):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def _sv():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as sv
    sv.load()
    return sv


def _noalloc(lib, q, k, v, o, S, z, commit, dt):
    vp = ctypes.c_void_p
    B, H, N, D = q.shape
    stream = vp(torch.cuda.current_stream().cuda_stream)
    return lib.sv_cache_step_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(o.data_ptr()), B, H,
                                     N, D, dt, EPS, vp(S.data_ptr()), vp(z.data_ptr()), 1 if commit else 0, stream)


def test_noalloc_step_matches_workspace_step_two_calls():
    sv = _sv()
    lib = sv.load()
    B, H, N, D = 1, 20, 2760, 128   # one 720p streaming block (3 latent frames of 23 x 40 tokens)
    stored = [draw_qkv((B, H, N, D), seed, "bf16") for seed in (0, 1)]
    blocks = [tuple(_dev(x) for x in st) for st in stored]
    # reference: the existing entry point with a caller-owned workspace
    S_ref = torch.zeros(B, H, D, D, device="cuda")
    z_ref = torch.zeros(B, H, D, device="cuda")
    ws = sv.make_workspace(sv.SV_OP_CACHE_STEP, blocks[0][0])
    assert ws.nbytes <= 16 << 20
    S64, z64 = np.zeros((B, H, D, D)), np.zeros((B, H, D))
    # the no-allocation entry point, called through the C ABI, on the same two blocks in a row
    S = torch.zeros(B, H, D, D, device="cuda")
    z = torch.zeros(B, H, D, device="cuda")
    for (q, k, v), st in zip(blocks, stored):
        o_ref = sv.sv_cache_step(q, k, v, S_ref, z_ref, commit=True, eps=EPS, ws=ws)
        o = torch.empty_like(q)
        rc = _noalloc(lib, q, k, v, o, S, z, True, sv.SV_BF16)
        assert rc == 0, lib.sv_last_error()
        torch.cuda.synchronize()
        assert _rel(o, o_ref) < TOL_O["bf16"]
        assert _rel(S, S_ref) < TOL_CACHE and _rel(z, z_ref) < TOL_CACHE
        o64, S64, z64 = oracle.cache_step(*(to_f64(x, "bf16") for x in st), S64, z64, EPS)
        assert oracle.max_rel_err(_host(o), o64) < TOL_O["bf16"]
        assert oracle.max_rel_err(_host(S), S64) < TOL_CACHE and oracle.max_rel_err(_host(z), z64) < TOL_CACHE
    assert ws.status() == 0
    assert sv.sv_cache_step_noalloc_status() == 0


def test_noalloc_interleaved_shapes_against_oracle():
    # Several independent streams of blocks share the one static array, call after call, each shape
    # reaching a different kernel: 20 heads of D=128 (one thread-block cluster per head), 2 x 20
    # heads of D=112 (the flag-synchronised one-launch kernel, whose launch sequence number and
    # flags persist in the array), 4 heads of D=64 (the same kernel on 24 CTAs) and fp32 I/O (the
    # three-kernel path). Each call is checked against the oracle's cache step on the same inputs.
    sv = _sv()
    lib = sv.load()
    streams = {
        "cluster": ((1, 20, 2760, 128), "bf16"),
        "flags40": ((2, 20, 1000, 112), "bf16"),
        "flags4": ((1, 4, 700, 64), "bf16"),
        "fp32": ((1, 3, 300, 32), "f32"),
    }
    order = [("cluster", 1), ("flags40", 1), ("fp32", 0), ("flags40", 0), ("cluster", 1), ("flags4", 1),
             ("flags40", 1), ("fp32", 1), ("flags4", 0), ("cluster", 0), ("flags40", 1)]
    state = {}
    for name, (shape, dtype) in streams.items():
        B, H, N, D = shape
        state[name] = dict(S=torch.zeros(B, H, D, D, device="cuda"), z=torch.zeros(B, H, D, device="cuda"),
                           S64=np.zeros((B, H, D, D)), z64=np.zeros((B, H, D)))
    for i, (name, commit) in enumerate(order):
        shape, dtype = streams[name]
        st = draw_qkv(shape, 50 + i, dtype)
        q, k, v = (_dev(x, dtype) for x in st)
        o = torch.empty_like(q)
        s = state[name]
        rc = _noalloc(lib, q, k, v, o, s["S"], s["z"], commit, sv.SV_BF16 if dtype == "bf16" else sv.SV_F32)
        assert rc == 0, lib.sv_last_error()
        torch.cuda.synchronize()
        o64, S64, z64 = oracle.cache_step(*(to_f64(x, dtype) for x in st), s["S64"], s["z64"], EPS,
                                          commit=bool(commit))
        s["S64"], s["z64"] = S64, z64
        err = oracle.max_rel_err(_host(o), o64)
        assert err < TOL_O[dtype], (i, name, err)
        assert oracle.max_rel_err(_host(s["S"]), S64) < TOL_CACHE, (i, name)
        assert oracle.max_rel_err(_host(s["z"]), z64) < TOL_CACHE, (i, name)
    assert sv.sv_cache_step_noalloc_status() == 0


def test_noalloc_step_refuses_blocks_beyond_its_scratch():
    sv = _sv()
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
    # a bad argument is refused before anything touches the array: a misaligned q
    st = lib.sv_cache_step_noalloc(vp(x.data_ptr() + 2), p, p, p, 1, 1, 128, 128, sv.SV_BF16, 1e-6,
                                   vp(S.data_ptr()), vp(S.data_ptr()), 1, None)
    assert st == sv._native.SV_ERR_INVALID_ARG and b"aligned" in lib.sv_last_error()
    assert sv.sv_cache_step_noalloc_status() == 0
