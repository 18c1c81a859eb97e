"""GPU parity of the block-causal temporal convolution (sv_temporal_conv, sv_temporal_conv_step)
against the fp64 oracle (oracle/temporal_conv.py, the talk's padding-token / carried-token
construction), through the C ABI.

Tolerances (normwise max relative error): bf16 I/O 2e-2 (the path's bf16 bar; the output is rounded
to bf16 once after an fp32 sum of three products and a bias, so the error is about 2^-9 of the
largest output and the tests also require < 5e-3); fp32 I/O 1e-4 (fp32 fused multiply-adds only).
Streaming block by block with the carried frame must equal the one-shot call bit for bit (same
arithmetic in the same order).
"""

import numpy as np
import pytest
import torch

import oracle
from block_causal_linear_relu_b200.inputs import draw_conv, to_f64

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as m
    m.load()
    return m


def dev(x, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,T,S,C,L", [(1, 12, 5, 16, 3), (2, 10, 7, 24, 4), (1, 1, 3, 8, 1), (1, 7, 9, 32, 10),
                                       (2, 9, 33, 64, 2), (1, 13, 4, 8, 13)])
def test_conv_matches_oracle(sv, dtype, B, T, S, C, L):
    x, w, b = draw_conv((B, T, S, C), 3, dtype)
    xd = dev(x, dtype)
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    y = sv.sv_temporal_conv(xd, wd, L, bias=bd)
    y0 = sv.sv_temporal_conv(xd, wd, L)  # no bias
    torch.cuda.synchronize()
    xf = to_f64(x, dtype)
    ref = oracle.temporal_conv_block_causal(xf, w.astype(np.float64), b.astype(np.float64), L)
    err = oracle.max_rel_err(host(y), ref)
    assert err < TOL[dtype], err
    if dtype == "bf16":
        assert err < 5e-3, err
    ref0 = oracle.temporal_conv_block_causal(xf, w.astype(np.float64), None, L)
    assert oracle.max_rel_err(host(y0), ref0) < TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_streaming_with_carry_equals_one_shot_and_oracle(sv, dtype):
    B, T, S, C, L = 2, 11, 6, 40, 3   # blocks of 3 frames, the last one 2 frames
    x, w, b = draw_conv((B, T, S, C), 4, dtype)
    xd = dev(x, dtype)
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    one = sv.sv_temporal_conv(xd, wd, L, bias=bd)
    carry = torch.zeros(B, S, C, dtype=xd.dtype, device="cuda")
    outs = []
    for a in range(0, T, L):
        blk = xd[:, a:a + L].contiguous()
        before = carry.clone()
        y_nc = sv.sv_temporal_conv_step(blk, wd, carry, commit=False, bias=bd)
        torch.cuda.synchronize()
        assert torch.equal(carry, before)                      # commit=0 leaves the carry
        y = sv.sv_temporal_conv_step(blk, wd, carry, commit=True, bias=bd)
        torch.cuda.synchronize()
        assert torch.equal(y, y_nc)
        assert torch.equal(carry, blk[:, -1])                  # the block's last frame is carried
        outs.append(y)
    streamed = torch.cat(outs, dim=1)
    assert torch.equal(streamed, one)                          # bit for bit
    ref = oracle.temporal_conv_block_causal(to_f64(x, dtype), w.astype(np.float64), b.astype(np.float64), L)
    assert oracle.max_rel_err(host(streamed), ref) < TOL[dtype]


def test_in_place_and_validation(sv):
    import ctypes
    x, w, b = draw_conv((1, 8, 5, 16), 5, "bf16")
    xd = dev(x, "bf16")
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    want = sv.sv_temporal_conv(xd, wd, 4, bias=bd)
    xi = xd.clone()
    sv.sv_temporal_conv(xi, wd, 4, bias=bd, y=xi)              # y may equal x
    torch.cuda.synchronize()
    assert torch.equal(xi, want)
    lib = sv.load()
    p = ctypes.c_void_p
    # C not a multiple of 8 for bf16, a misaligned x, a NULL carry: refused before any launch
    assert lib.sv_temporal_conv(p(xd.data_ptr()), p(xd.data_ptr()), 1, 8, 5, 12, 4, p(wd.data_ptr()), None, 0,
                                None) == 2
    assert lib.sv_temporal_conv(p(xd.data_ptr() + 2), p(xd.data_ptr()), 1, 8, 5, 16, 4, p(wd.data_ptr()), None, 0,
                                None) == 1
    assert lib.sv_temporal_conv_step(p(xd.data_ptr()), p(xd.data_ptr()), 1, 8, 5, 16, p(wd.data_ptr()), None, None,
                                     1, 0, None) == 1


def test_conv_720p_full_size(sv):
    # the 720p latent video of the block-causal prefill: 60 frames of 23 x 40 tokens, hidden 2560,
    # blocks of 3 frames; every element against the oracle, 256 channels at a time on the host
    B, T, S, C, L = 1, 60, 920, 2560, 3
    x, w, b = draw_conv((B, T, S, C), 0, "bf16")
    xd = dev(x, "bf16")
    wd, bd = torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda()
    y = sv.sv_temporal_conv(xd, wd, L, bias=bd)
    carry = torch.zeros(B, S, C, dtype=torch.bfloat16, device="cuda")
    ys = [sv.sv_temporal_conv_step(xd[:, a:a + L].contiguous(), wd, carry, bias=bd) for a in range(0, T, L)]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(ys, dim=1), y)
    yh = y.float().cpu().numpy()
    for c0 in range(0, C, 256):
        xs = to_f64(x[..., c0:c0 + 256], "bf16")
        ref = oracle.temporal_conv_block_causal(xs, w[c0:c0 + 256].astype(np.float64), b[c0:c0 + 256].astype(np.float64), L)
        err = oracle.max_rel_err(yh[..., c0:c0 + 256].astype(np.float64), ref)
        assert err < 5e-3, (c0, err)
