"""GPU parity of the 3D rotary form (sv_rope3d_table, sv_block_causal_attn_rope) against the fp64
oracle (oracle/rope.py) on the same seeded inputs, every element compared.

Tolerances (normwise max relative error, as in test_gpu_parity.py):
  o : 2e-2 (bf16 I/O), 1e-4 (fp32 I/O).
  z (unturned key sum): 1e-4 for both dtypes, as without the rotation (exact products, fp32 sums).
  S (turned-key state): 1e-4 for fp32 I/O; for bf16 I/O the turned features are rounded to bf16
  (relative error <= 2^-8 each) before the tensor-core products, so S carries that rounding:
  2e-2, the bar of the bf16 outputs (observed ~2e-3).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import rope as R
from block_causal_linear_relu_b200.inputs import draw_qkv, to_f64

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}
TOL_S = {"bf16": 2e-2, "f32": 1e-4}
TOL_Z = 1e-4
EPS = 1e-6


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


def cache_in(B, H, D, seed):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((B, H, D, D)).astype(np.float32)
    z = np.abs(rng.standard_normal((B, H, D))).astype(np.float32) * np.float32(8.0)
    return S, z


@pytest.mark.parametrize("D,frames,height,width", [(128, 60, 23, 40), (112, 21, 15, 26), (24, 3, 2, 5)])
def test_table_matches_the_oracle_angles(sv, D, frames, height, width):
    pairs = R.default_pairs(D)
    tab = sv.sv_rope3d_table(frames, height, width, D, pairs)
    torch.cuda.synchronize()
    got = host(tab.table).reshape(frames + height + width, D // 2, 2)
    # row f is the token at (f, 0, 0), row height + y the token at (0, y, 0), and so on: the other
    # groups' angles are 0 there, i.e. (cos, sin) = (1, 0), as the table holds them
    pos = np.concatenate([np.stack([np.arange(frames), np.zeros(frames), np.zeros(frames)], 1),
                          np.stack([np.zeros(height), np.arange(height), np.zeros(height)], 1),
                          np.stack([np.zeros(width), np.zeros(width), np.arange(width)], 1)]).astype(np.int64)
    ang = R.rope3d_angles(pos, pairs)
    assert np.max(np.abs(got[..., 0] - np.cos(ang))) < 1e-6
    assert np.max(np.abs(got[..., 1] - np.sin(ang))) < 1e-6


def run_rope(sv, dtype, shape, L, height, width, frame0=0, with_cache=True, seed=0, pairs=None):
    B, H, N, D = shape
    st = draw_qkv(shape, seed, dtype)
    q, k, v = (to_f64(x, dtype) for x in st)
    hw = height * width
    frames = frame0 + (N - 1) // hw + 1
    pairs = R.default_pairs(D) if pairs is None else pairs
    tab = sv.sv_rope3d_table(frames, height, width, D, pairs)
    S_in, z_in = cache_in(B, H, D, seed + 1) if with_cache else (None, None)
    S_out = torch.zeros(B, H, D, D, device="cuda")
    z_out = torch.zeros(B, H, D, device="cuda")
    qd, kd, vd = (dev(x, dtype) for x in st)
    o = sv.sv_block_causal_attn_rope(qd, kd, vd, L, tab, frame0=frame0, eps=EPS,
                                     S_in=None if S_in is None else torch.from_numpy(S_in).cuda(),
                                     z_in=None if z_in is None else torch.from_numpy(z_in).cuda(),
                                     S_out=S_out, z_out=z_out)
    torch.cuda.synchronize()
    ang = R.rope3d_angles(R.token_positions(N, height, width, frame0), pairs)
    ref = R.block_causal_attn_rope(q, k, v, L, EPS, ang, S_in, z_in)
    return (host(o), host(S_out), host(z_out)), ref


def check(got, ref, dtype):
    assert oracle.max_rel_err(got[0], ref[0]) < TOL[dtype]
    assert oracle.max_rel_err(got[1], ref[1]) < TOL_S[dtype]
    assert oracle.max_rel_err(got[2], ref[2]) < TOL_Z


@pytest.mark.parametrize("B,H,N,D,L,height,width", [
    (1, 3, 700, 64, 175, 5, 7),      # 4 blocks of 5 frames, ragged tiles
    (2, 2, 1300, 112, 390, 13, 10),  # two atoms, features 112..127 padding, a short last block
    (1, 2, 1000, 128, 1000, 10, 10),  # one block per head (bidirectional), three-kernel path
    (1, 1, 333, 40, 111, 3, 37),     # pairs (8, 6, 6): the row/column boundary inside a 4-pair chunk
    (1, 2, 200, 24, 64, 2, 5),       # pairs (4, 4, 4)
    (1, 2, 97, 8, 40, 1, 97),        # D = 8, blocks not aligned to frames
    (3, 5, 260, 128, 130, 2, 13),    # many heads, one tile + 2 rows per block
])
def test_bf16_matches_oracle(sv, B, H, N, D, L, height, width):
    got, ref = run_rope(sv, "bf16", (B, H, N, D), L, height, width, frame0=2, seed=B * 100 + N)
    check(got, ref, "bf16")


@pytest.mark.parametrize("B,H,N,D,L,height,width", [
    (1, 2, 300, 32, 64, 4, 5),
    (1, 1, 129, 30, 43, 3, 43),
    (2, 1, 256, 128, 256, 16, 16),
])
def test_f32_matches_oracle(sv, B, H, N, D, L, height, width):
    got, ref = run_rope(sv, "f32", (B, H, N, D), L, height, width, frame0=1, seed=N)
    check(got, ref, "f32")


def test_bf16_table_beyond_shared_memory(sv):
    # 4 x 4 tokens per frame: the call touches 188 frames, so the compact (cos, sin) table would
    # need 188 * 22 + 4 * 21 + 4 * 21 = 4304 entries, more than the kernels stage in shared memory
    # (3072): they read the table in global memory instead
    got, ref = run_rope(sv, "bf16", (1, 2, 3000, 128), 800, 4, 4, seed=31)
    check(got, ref, "bf16")


@pytest.mark.parametrize("dtype,D,pairs", [("bf16", 128, (32, 0, 32)), ("bf16", 64, (0, 16, 16)),
                                           ("bf16", 112, (56, 0, 0)), ("f32", 32, (0, 0, 16))])
def test_caller_given_pair_splits(sv, dtype, D, pairs):
    # empty groups, and all pairs on one axis
    got, ref = run_rope(sv, dtype, (1, 2, 600, D), 200, 5, 6, frame0=3, seed=D, pairs=pairs)
    check(got, ref, dtype)


def test_bf16_without_incoming_cache(sv):
    got, ref = run_rope(sv, "bf16", (1, 4, 640, 128), 320, 8, 10, with_cache=False, seed=5)
    check(got, ref, "bf16")


def test_streaming_three_720p_blocks_equals_oracle_prefill(sv):
    # the 720p streaming block [1, 20, 2760, 128] (3 frames of 23 x 40), three blocks through the
    # cache with frame0 = 0, 3, 6, against the oracle's one-shot prefill of the 8280 tokens
    B, H, D, Lb, height, width = 1, 20, 128, 2760, 23, 40
    st = draw_qkv((B, H, 3 * Lb, D), 77, "bf16")
    q, k, v = (to_f64(x, "bf16") for x in st)
    pairs = R.default_pairs(D)
    ang = R.rope3d_angles(R.token_positions(3 * Lb, height, width), pairs)
    ref_o, ref_S, ref_z = R.block_causal_attn_rope(q, k, v, Lb, EPS, ang)
    tab = sv.sv_rope3d_table(9, height, width, D, pairs)
    S = torch.zeros(B, H, D, D, device="cuda")
    z = torch.zeros(B, H, D, device="cuda")
    Sc, zc = np.zeros((B, H, D, D)), np.zeros((B, H, D))
    for c in range(3):
        sl = slice(c * Lb, (c + 1) * Lb)
        qd, kd, vd = (dev(np.ascontiguousarray(x[:, :, sl]), "bf16") for x in st)
        o = sv.sv_block_causal_attn_rope(qd, kd, vd, Lb, tab, frame0=3 * c, eps=EPS, S_in=S, z_in=z, S_out=S, z_out=z)
        torch.cuda.synchronize()
        assert oracle.max_rel_err(host(o), ref_o[:, :, sl]) < TOL["bf16"]
        _, Sc, zc = R.block_causal_attn_rope(q[:, :, sl], k[:, :, sl], v[:, :, sl], Lb, EPS,
                                             ang[sl], Sc, zc)
        assert oracle.max_rel_err(host(S), Sc) < TOL_S["bf16"]
        assert oracle.max_rel_err(host(z), zc) < TOL_Z
    assert oracle.max_rel_err(Sc, ref_S) < 1e-12 and oracle.max_rel_err(zc, ref_z) < 1e-12


def test_720p_prefill_full_size(sv):
    # the 720p block-causal prefill [1, 20, 55200, 128], blocks of 2760 tokens (3 frames of 23 x 40),
    # every output, the turned-key state and the key sum compared
    got, ref = run_rope(sv, "bf16", (1, 20, 55200, 128), 2760, 23, 40, with_cache=False, seed=2)
    check(got, ref, "bf16")
