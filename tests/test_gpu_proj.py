"""GPU parity of the Q/K/V projection (ReLU on Q and K in the epilogue, [B, H, N, D] outputs) and of
the output projection (reading [B, H, N, D] in place) against the fp64 oracle
(oracle/projection.py), through the C ABI.

Tolerance: normwise max relative error 2e-2 (the bf16 bar of the path); the products of bf16 inputs
are exact in the fp32 accumulator, so the error is the single bf16 rounding of each output (about
2^-9 of the largest output) and the tests also require < 5e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from block_causal_linear_relu_b200.inputs import draw_proj, draw_qkv, to_f64

pytestmark = pytest.mark.gpu

TOL = 2e-2
TIGHT = 5e-3


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from block_causal_linear_relu_b200 import build
    build.build()
    import block_causal_linear_relu_b200 as m
    m.load()
    return m


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("B,N,C,H,D", [(2, 300, 256, 2, 128), (1, 129, 128, 4, 64), (1, 77, 192, 3, 64),
                                       (3, 1, 64, 1, 128), (1, 513, 320, 5, 64)])
def test_qkv_projection_matches_oracle(sv, B, N, C, H, D):
    xb, wb = draw_proj((B, N, C), 3 * H * D, 11)
    q, k, v = sv.sv_qkv_projection(dev(xb), dev(wb), H, D)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_projection(to_f64(xb, "bf16"), to_f64(wb, "bf16"), H, D)
    for got, ref in ((q, rq), (k, rk), (v, rv)):
        err = oracle.max_rel_err(host(got), ref)
        assert err < TIGHT, err
    assert bool((q >= 0).all()) and bool((k >= 0).all()) and bool((v < 0).any())


@pytest.mark.parametrize("B,N,H,D,Co", [(2, 300, 2, 128, 256), (1, 77, 3, 64, 128), (1, 1, 1, 128, 64)])
def test_out_projection_matches_oracle(sv, B, N, H, D, Co):
    ob, wb = draw_proj((B, H, N, D), Co, 12)
    wb = draw_proj((1, H * D), Co, 13)[1]
    y = sv.sv_out_projection(dev(ob), dev(wb))
    torch.cuda.synchronize()
    ref = oracle.out_projection(to_f64(ob, "bf16"), to_f64(wb, "bf16"))
    assert oracle.max_rel_err(host(y), ref) < TIGHT


def test_layer_projection_attention_projection(sv):
    # x -> [q|k|v] -> bidirectional linear attention -> output projection, against the oracle's
    # composition on the same inputs (each GPU stage's bf16 output feeds the next stage, so the
    # oracle is fed the GPU's intermediate tensors stage by stage)
    B, N, C, H, D = 1, 700, 256, 2, 128
    xb, wb = draw_proj((B, N, C), 3 * H * D, 14)
    wob = draw_proj((1, H * D), C, 15)[1]
    q, k, v = sv.sv_qkv_projection(dev(xb), dev(wb), H, D)
    o = sv.sv_linattn_fwd(q, k, v, eps=1e-6)
    y = sv.sv_out_projection(o, dev(wob))
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_projection(to_f64(xb, "bf16"), to_f64(wb, "bf16"), H, D)
    assert oracle.max_rel_err(host(q), rq) < TIGHT
    ro = oracle.linattn_fwd(host(q), host(k), host(v), 1e-6)
    assert oracle.max_rel_err(host(o), ro) < TOL
    ry = oracle.out_projection(host(o), to_f64(wob, "bf16"))
    assert oracle.max_rel_err(host(y), ry) < TIGHT


def test_projections_full_size_2p0_layer(sv):
    # SANA-Video 2.0 layer shape: B=2 (CFG pair), 11 latent frames x 920 = 10,120 tokens, hidden 2560
    # = 20 heads x 128; every element of q, k, v and y against the oracle, one batch at a time
    B, N, C, H, D = 2, 10120, 2560, 20, 128
    xb, wb = draw_proj((B, N, C), 3 * H * D, 0)
    wob = draw_proj((1, H * D), C, 1)[1]
    q, k, v = sv.sv_qkv_projection(dev(xb), dev(wb), H, D)
    y = sv.sv_out_projection(v, dev(wob))   # v as the attention output stand-in: a [B, H, N, D] input
    torch.cuda.synchronize()
    w64, wo64 = to_f64(wb, "bf16"), to_f64(wob, "bf16")
    for b in range(B):
        rq, rk, rv = oracle.qkv_projection(to_f64(xb[b:b + 1], "bf16"), w64, H, D)
        for got, ref in ((q, rq), (k, rk), (v, rv)):
            err = oracle.max_rel_err(host(got[b:b + 1]), ref)
            assert err < TIGHT, (b, err)
        ry = oracle.out_projection(host(v[b:b + 1]), wo64)
        assert oracle.max_rel_err(host(y[b:b + 1]), ry) < TIGHT


def test_projection_validation(sv):
    import ctypes
    lib = sv.load()
    p = ctypes.c_void_p
    x = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    ws = sv.Workspace(256, torch.device("cuda:0"))
    a = p(x.data_ptr())
    assert lib.sv_qkv_projection(a, a, a, a, a, 1, 4, 64, 1, 96, ws.ptr, ws.nbytes, None) == 2    # D = 96
    assert lib.sv_qkv_projection(a, a, a, a, a, 1, 4, 100, 1, 64, ws.ptr, ws.nbytes, None) == 2   # C % 64
    assert lib.sv_qkv_projection(p(x.data_ptr() + 2), a, a, a, a, 1, 4, 64, 1, 64, ws.ptr, ws.nbytes, None) == 1
    assert lib.sv_out_projection(a, a, a, 1, 4, 1, 64, 64, None, 0, None) == 1                     # no workspace
    assert ws.status() == 0
