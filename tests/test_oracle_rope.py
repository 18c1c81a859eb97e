"""Pins of the 3D-RoPE oracle (oracle/rope.py) against things other than itself: the plain pinned
oracle at zero angles, an independent brute force with dense rotation matrices, relative-position
invariance, closed forms worked by hand, streaming == prefill, and planted mistakes."""

import math

import numpy as np
import pytest

import oracle
from oracle import rope as R
from block_causal_linear_relu_b200.inputs import draw_qkv

EPS = 1e-6


def _qkv(shape, seed):
    return tuple(x.astype(np.float64) for x in draw_qkv(shape, seed, "f32"))


def test_token_positions_enumerate_the_grid_frame_major():
    F, Hh, W = 3, 4, 5
    pos = R.token_positions(F * Hh * W, Hh, W, frame0=7)
    n = 0
    for f in range(F):
        for y in range(Hh):
            for x in range(W):
                assert tuple(pos[n]) == (7 + f, y, x)
                n += 1


def test_default_pairs_and_frequencies():
    assert R.default_pairs(128) == (22, 21, 21)
    assert R.default_pairs(112) == (20, 18, 18)
    assert sum(R.default_pairs(64)) == 32
    # one token at frame 1, row 2, column 3: the first pair of each group turns by the position
    # itself (theta = base^0), and inside a group consecutive pairs slow down by base^(-1/P)
    pairs = (4, 2, 2)
    ang = R.rope3d_angles(np.array([[1, 2, 3]]), pairs, base=10000.0)[0]
    assert ang[0] == 1.0 and ang[4] == 2.0 and ang[6] == 3.0
    assert math.isclose(ang[1] / ang[0], 10000.0 ** (-1 / 4), rel_tol=1e-14)
    assert math.isclose(ang[5] / ang[4], 10000.0 ** (-1 / 2), rel_tol=1e-14)
    assert math.isclose(ang[3], 10000.0 ** (-3 / 4), rel_tol=1e-14)


def test_rotation_keeps_pair_lengths():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 8))
    ang = rng.uniform(-50, 50, size=(5, 4))
    y = R.rotate_pairs(x, ang)
    np.testing.assert_allclose(y[:, 0::2] ** 2 + y[:, 1::2] ** 2, x[:, 0::2] ** 2 + x[:, 1::2] ** 2, rtol=1e-12)


@pytest.mark.parametrize("blen", [16, 40, 1000])
def test_zero_angles_reduce_to_the_plain_oracle(blen):
    q, k, v = _qkv((2, 2, 70, 8), 5)
    S_in = np.random.default_rng(1).standard_normal((2, 2, 8, 8))
    z_in = np.abs(np.random.default_rng(2).standard_normal((2, 2, 8)))
    o, S, z = R.block_causal_attn_rope(q, k, v, blen, EPS, np.zeros((70, 4)), S_in, z_in)
    ref = oracle.block_causal_attn(q, k, v, blen, EPS, S_in, z_in)
    assert oracle.max_rel_err(o, ref[0]) < 1e-13
    assert oracle.max_rel_err(S, ref[1]) < 1e-13
    assert oracle.max_rel_err(z, ref[2]) < 1e-13


@pytest.mark.parametrize("blen", [12, 24, 48])
def test_matches_bruteforce_with_dense_rotations(blen):
    q, k, v = _qkv((1, 2, 48, 12), 9)
    pos = R.token_positions(48, 2, 3, frame0=2)  # 6 tokens per frame, frames 2..9
    ang = R.rope3d_angles(pos, (2, 2, 2))
    o, _, _ = R.block_causal_attn_rope(q, k, v, blen, EPS, ang)
    assert oracle.max_rel_err(o, R.bruteforce_rope(q, k, v, blen, EPS, ang)) < 1e-12


@pytest.mark.parametrize("blen,pairs", [(12, (2, 2, 2)), (30, (1, 0, 5)), (1000, (6, 0, 0))])
def test_matches_c_bruteforce_through_relative_angles(blen, pairs):
    # a second brute force, in plain C, that never turns a vector: each pair's score is written
    # with the cosine and sine of the angle difference (oracle/bruteforce.c)
    from oracle.bruteforce import bruteforce_rope_c

    q, k, v = _qkv((2, 1, 60, 12), 23)
    ang = R.rope3d_angles(R.token_positions(60, 2, 5, frame0=4), pairs)
    o, _, _ = R.block_causal_attn_rope(q, k, v, blen, EPS, ang)
    assert oracle.max_rel_err(o, bruteforce_rope_c(q, k, v, blen, EPS, ang)) < 1e-12


@pytest.mark.parametrize("blen", [18, 1000])
def test_output_depends_on_relative_positions_only(blen):
    # every score of the numerator is phi(q_i)^T R(angle_j - angle_i) phi(k_j): moving every token
    # by the same number of frames changes no output (the cache, absolute, does change)
    q, k, v = _qkv((1, 1, 54, 8), 11)
    pairs = (2, 1, 1)
    a0 = R.rope3d_angles(R.token_positions(54, 3, 3, frame0=0), pairs)
    a5 = R.rope3d_angles(R.token_positions(54, 3, 3, frame0=37), pairs)
    o0, S0, _ = R.block_causal_attn_rope(q, k, v, blen, EPS, a0)
    o5, S5, _ = R.block_causal_attn_rope(q, k, v, blen, EPS, a5)
    assert oracle.max_rel_err(o5, o0) < 1e-12
    assert oracle.max_rel_err(S5, S0) > 1e-3


def _hand_case():
    # D = 4, pairs (frame, row, column) = (1, 0, 1): pair 0 turns by the frame index, pair 1 by the
    # column index, each by 1 radian per step (the first pair of a group has theta = base^0).
    # Grid: 1 row x 2 columns per frame, 2 frames -> tokens (f, x) = (0,0), (0,1), (1,0), (1,1).
    # q_i = k_j = (1, 0, 1, 0): R phi = (cos f, sin f, cos x, sin x), so the numerator score is
    # cos(f_i - f_j) + cos(x_i - x_j) and the denominator score phi(q).phi(k) = 2.
    # v_j = (j + 1, 0, 0, 0).
    q = np.tile(np.array([1.0, 0.0, 1.0, 0.0]), (1, 1, 4, 1))
    k = q.copy()
    v = np.zeros((1, 1, 4, 4))
    v[0, 0, :, 0] = [1.0, 2.0, 3.0, 4.0]
    ang = R.rope3d_angles(R.token_positions(4, 1, 2), (1, 0, 1))
    return q, k, v, ang


def test_hand_worked_d4_closed_forms():
    q, k, v, ang = _hand_case()
    c1 = math.cos(1.0)
    # bidirectional, token 0 (f=0, x=0): sum_j [cos f_j + cos x_j] (j+1) over all four tokens
    #   = 2*1 + (1 + c1)*2 + (c1 + 1)*3 + 2 c1*4 = 7 + 13 c1, over 4 tokens x 2 = 8
    o, S, z = R.block_causal_attn_rope(q, k, v, 4, 0.0, ang)
    assert math.isclose(o[0, 0, 0, 0], (7 + 13 * c1) / 8, rel_tol=1e-14)
    # token 3 (f=1, x=1): 2 c1*1 + (c1 + 1)*2 + (1 + c1)*3 + 2*4 = 13 + 7 c1
    assert math.isclose(o[0, 0, 3, 0], (13 + 7 * c1) / 8, rel_tol=1e-14)
    assert np.all(o[0, 0, :, 1:] == 0.0)
    # block-causal with blocks of 2 tokens: token 0 sees tokens 0, 1: (2*1 + (1 + c1)*2) / 4
    ob, _, _ = R.block_causal_attn_rope(q, k, v, 2, 0.0, ang)
    assert math.isclose(ob[0, 0, 0, 0], (4 + 2 * c1) / 4, rel_tol=1e-14)
    assert math.isclose(ob[0, 0, 3, 0], (13 + 7 * c1) / 8, rel_tol=1e-14)
    # the cache: unrotated key sum (4 tokens of (1,0,1,0)) and the rotated-key state's first
    # column sum_j (j+1) (cos f_j, sin f_j, cos x_j, sin x_j)
    np.testing.assert_allclose(z[0, 0], [4.0, 0.0, 4.0, 0.0], rtol=0, atol=0)
    s1 = math.sin(1.0)
    np.testing.assert_allclose(S[0, 0, :, 0], [1 + 2 + 3 * c1 + 4 * c1, 3 * s1 + 4 * s1, 1 + 2 * c1 + 3 + 4 * c1,
                                               2 * s1 + 4 * s1], rtol=1e-14)


def test_streaming_through_the_cache_equals_prefill():
    q, k, v = _qkv((1, 2, 72, 8), 13)
    Hh, W, fpb = 2, 3, 4  # 6 tokens per frame, blocks of 4 frames = 24 tokens
    L = fpb * Hh * W
    pairs = (2, 1, 1)
    ang = R.rope3d_angles(R.token_positions(72, Hh, W), pairs)
    o, S, z = R.block_causal_attn_rope(q, k, v, L, EPS, ang)
    Sc, zc = np.zeros((1, 2, 8, 8)), np.zeros((1, 2, 8))
    for c in range(3):
        sl = slice(c * L, (c + 1) * L)
        a_c = R.rope3d_angles(R.token_positions(L, Hh, W, frame0=c * fpb), pairs)
        oc, Sc, zc = R.block_causal_attn_rope(q[:, :, sl], k[:, :, sl], v[:, :, sl], L, EPS, a_c, Sc, zc)
        assert oracle.max_rel_err(oc, o[:, :, sl]) < 1e-12
    assert oracle.max_rel_err(Sc, S) < 1e-12
    assert oracle.max_rel_err(zc, z) < 1e-12
    assert Sc.nbytes == 2 * 8 * 8 * 8  # the cache does not grow with the number of blocks


# ---- planted mistakes: each one must fail the brute force and the hand-worked closed forms ----
def _mutant(kind, q, k, v, blen, eps, ang):
    fq, fk = oracle.phi(q), oracle.phi(k)
    if kind == "half_split_pairs":  # pairs (p, p + D/2) instead of (2p, 2p + 1)
        D = q.shape[-1]
        perm = np.empty(D, dtype=np.int64)
        perm[0::2], perm[1::2] = np.arange(D // 2), np.arange(D // 2) + D // 2
        inv = np.argsort(perm)
        rq = R.rotate_pairs(fq[..., perm], ang)[..., inv]
        rk = R.rotate_pairs(fk[..., perm], ang)[..., inv]
    elif kind == "q_turned_back":
        rq, rk = R.rotate_pairs(fq, -ang), R.rotate_pairs(fk, ang)
    else:
        rq, rk = R.rotate_pairs(fq, ang), R.rotate_pairs(fk, ang)
    dq, dk = (rq, rk) if kind == "rotated_denominator" else (fq, fk)
    N = q.shape[2]
    o = np.empty_like(q)
    P = np.zeros(q.shape[:2] + (q.shape[-1], v.shape[-1]))
    zP = np.zeros(q.shape[:2] + (q.shape[-1],))
    for c in range(oracle.num_blocks(N, blen)):
        sl = slice(c * blen, min(N, (c + 1) * blen))
        P = P + np.matmul(np.swapaxes(rk[:, :, sl], -1, -2), v[:, :, sl])
        zP = zP + dk[:, :, sl].sum(axis=2)
        o[:, :, sl] = np.matmul(rq[:, :, sl], P) / (np.einsum("bhnd,bhd->bhn", dq[:, :, sl], zP) + eps)[..., None]
    return o


@pytest.mark.parametrize("kind", ["rotated_denominator", "q_turned_back", "half_split_pairs"])
def test_planted_mistake_is_caught(kind):
    q, k, v = _qkv((1, 1, 36, 8), 17)
    ang = R.rope3d_angles(R.token_positions(36, 2, 3), (2, 1, 1))
    ref = R.bruteforce_rope(q, k, v, 12, EPS, ang)
    assert oracle.max_rel_err(_mutant("none", q, k, v, 12, EPS, ang), ref) < 1e-12
    assert oracle.max_rel_err(_mutant(kind, q, k, v, 12, EPS, ang), ref) > 1e-3
    from oracle.bruteforce import bruteforce_rope_c
    assert oracle.max_rel_err(_mutant(kind, q, k, v, 12, EPS, ang), bruteforce_rope_c(q, k, v, 12, EPS, ang)) > 1e-3
    qh, kh, vh, angh = _hand_case()
    good = (13 + 7 * math.cos(1.0)) / 8  # token 3 (frame 1, column 1), bidirectional
    if kind != "half_split_pairs":  # the hand case's features sit on the interleaved pairs only
        assert not math.isclose(_mutant(kind, qh, kh, vh, 4, 0.0, angh)[0, 0, 3, 0], good, rel_tol=1e-6)
