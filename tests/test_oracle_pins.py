"""Pins of the fp64 oracle against things other than itself.

Each check is chosen so that a plausible slip in the oracle (a transposed state, an exclusive
instead of inclusive prefix, an off-by-one block index, a dropped eps or normaliser, a wrong
sign in the feature map) fails at least one of them:

* two independent quadratic brute forces (numpy explicit matrix, plain C loops);
* the token recurrence of causal linear attention (Katharopoulos et al. 2020) for L = 1;
* closed forms: a hand-worked 4-token example, uniform attention, constant v, non-positive q;
* invariants: one-hot state orientation, streaming == prefill, constant cache bytes,
  permutation inside a block, linearity in v.
"""

import numpy as np
import pytest

import golden
import oracle
from oracle.bruteforce import bruteforce_c
from block_causal_linear_relu_b200.inputs import draw_qkv, to_f64

EPS = 1e-6


def _c0(dtype="f32"):
    q, k, v = draw_qkv((1, 2, 256, 32), 0, dtype)
    return to_f64(q, dtype), to_f64(k, dtype), to_f64(v, dtype)


@pytest.mark.parametrize("L", [64, 256, 1000])
def test_linear_form_matches_numpy_bruteforce_c0(L):
    # config 0: B=1, H=2, D=32, 4 blocks x 64 tokens, fp32 inputs, eps=1e-6; L=256/1000: bidirectional
    q, k, v = _c0()
    got = oracle.block_causal_attn(q, k, v, L, EPS)[0]
    ref = oracle.bruteforce_masked(q, k, v, L, EPS)
    assert oracle.max_rel_err(got, ref) < 1e-12


@pytest.mark.parametrize("L", [64, 256])
def test_linear_form_matches_c_bruteforce_c0(L):
    q, k, v = _c0()
    got = oracle.block_causal_attn(q, k, v, L, EPS)[0]
    ref = bruteforce_c(q, k, v, L, EPS)
    assert oracle.max_rel_err(got, ref) < 1e-12


@pytest.mark.parametrize("N,L", [(250, 64), (77, 10), (5, 7), (1, 1), (130, 129)])
def test_ragged_blocks_match_c_bruteforce(N, L):
    q, k, v = draw_qkv((2, 1, N, 8), 3, "f32")
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    got = oracle.block_causal_attn(q, k, v, L, EPS)[0]
    ref = bruteforce_c(q, k, v, L, EPS)
    assert oracle.max_rel_err(got, ref) < 1e-12


def test_value_dim_differs_from_key_dim():
    # S is D x E: rows are key features, columns value features
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 40, 6))
    k = rng.standard_normal((1, 1, 40, 6))
    v = rng.standard_normal((1, 1, 40, 3))
    got = oracle.block_causal_attn(q, k, v, 16, EPS)[0]
    assert got.shape == (1, 1, 40, 3)
    assert oracle.max_rel_err(got, bruteforce_c(q, k, v, 16, EPS)) < 1e-12


def test_block_len_one_is_token_causal_recurrence():
    q, k, v = draw_qkv((1, 2, 12, 4), 11, "f32")
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    got = oracle.block_causal_attn(q, k, v, 1, EPS)[0]
    ref = oracle.causal_recurrence(q, k, v, EPS)
    assert oracle.max_rel_err(got, ref) < 1e-12


def test_block_len_at_least_n_is_bidirectional():
    q, k, v = _c0()
    a = oracle.block_causal_attn(q, k, v, 256, EPS)[0]
    b = oracle.block_causal_attn(q, k, v, 10_000, EPS)[0]
    c = oracle.linattn_fwd(q, k, v, EPS)
    assert np.array_equal(a, b) and np.array_equal(a, c)


@pytest.mark.parametrize("name", golden.FIXTURES)
def test_hand_worked_fixtures(name):
    # tests/golden: small cases worked by hand from the definition (the derivations are in the files)
    g = golden.load(name)
    S_in, z_in = g.get("S_in"), g.get("z_in")
    o, S_out, z_out = oracle.block_causal_attn(g["q"], g["k"], g["v"], g["block_len"], g["eps"], S_in, z_in)
    assert np.allclose(o, g["o_block_causal"], rtol=1e-15, atol=1e-15)
    if S_in is not None:
        assert np.allclose(S_out, g["S_out"], rtol=0, atol=1e-15)
        assert np.allclose(z_out, g["z_out"], rtol=0, atol=1e-15)
    n = g["q"].shape[2]
    ob = oracle.block_causal_attn(g["q"], g["k"], g["v"], n, g["eps"], S_in, z_in)[0]
    assert np.allclose(ob, g["o_bidirectional"], rtol=1e-15, atol=1e-15)
    if S_in is None:
        assert np.allclose(oracle.linattn_fwd(g["q"], g["k"], g["v"], g["eps"]), g["o_bidirectional"], rtol=1e-15,
                           atol=1e-15)


def test_uniform_attention_is_running_mean():
    # q_i = a*1, k_j = b*1 (positive): every visible key gets the same weight D*a*b, so the output
    # is the mean of the visible v_j scaled by den/(den+eps), den = D*a*b*(#visible).
    B, H, N, D, E, L = 1, 2, 50, 4, 3, 8
    a, b = 0.5, 0.25
    q = np.full((B, H, N, D), a)
    k = np.full((B, H, N, D), b)
    v = np.random.default_rng(2).standard_normal((B, H, N, E))
    eps = 1e-2
    got = oracle.block_causal_attn(q, k, v, L, eps)[0]
    for i in range(N):
        vis = min(N, (i // L + 1) * L)
        den = D * a * b * vis
        exp = v[:, :, :vis].mean(axis=2) * den / (den + eps)
        assert np.allclose(got[:, :, i], exp, rtol=1e-13, atol=1e-15)


def test_constant_v_closed_form():
    q, k, _ = _c0()
    c = -1.75
    v = np.full((1, 2, 256, 32), c)
    eps = 0.5  # large enough that the eps term is visible
    got = oracle.block_causal_attn(q, k, v, 64, eps)[0]
    A = np.matmul(np.maximum(q, 0), np.swapaxes(np.maximum(k, 0), -1, -2))
    blk = np.arange(256) // 64
    den = (A * (blk[None, :] <= blk[:, None])).sum(-1)
    assert np.allclose(got, (c * den / (den + eps))[..., None], rtol=1e-12, atol=1e-14)


def test_nonpositive_query_row_gives_zero():
    q, k, v = _c0()
    q[0, 1, 17] = -np.abs(q[0, 1, 17])
    q[0, 0, 200] = 0.0
    got = oracle.block_causal_attn(q, k, v, 64, EPS)[0]
    assert np.all(got[0, 1, 17] == 0.0) and np.all(got[0, 0, 200] == 0.0)


def test_one_hot_state_orientation():
    # a single token with k = 2 e_1, v = 3 e_2 gives S[1, 2] = 6 (row = key feature), z = 2 e_1
    k = np.zeros((1, 1, 1, 4)); k[0, 0, 0, 1] = 2.0
    v = np.zeros((1, 1, 1, 4)); v[0, 0, 0, 2] = 3.0
    S, z = oracle.block_states(k, v, 1)
    exp = np.zeros((4, 4)); exp[1, 2] = 6.0
    assert np.array_equal(S[0, 0, 0], exp)
    assert np.array_equal(z[0, 0, 0], [0, 2.0, 0, 0])
    # a negative key feature contributes nothing (ReLU, not abs or identity)
    k[0, 0, 0, 1] = -2.0
    S, z = oracle.block_states(k, v, 1)
    assert not S.any() and not z.any()


def test_streaming_equals_prefill_and_cache_is_constant():
    B, H, D, L, nb = 1, 3, 16, 20, 7
    q, k, v = draw_qkv((B, H, nb * L, D), 4, "bf16")
    q, k, v = to_f64(q, "bf16"), to_f64(k, "bf16"), to_f64(v, "bf16")
    ref, S_ref, z_ref = oracle.block_causal_attn(q, k, v, L, EPS)
    S = np.zeros((B, H, D, D)); z = np.zeros((B, H, D))
    nbytes0 = S.nbytes + z.nbytes
    outs = []
    for c in range(nb):
        sl = slice(c * L, (c + 1) * L)
        # a non-committing denoising call leaves the cache untouched and gives the same output
        o0, S0, z0 = oracle.cache_step(q[:, :, sl], k[:, :, sl], v[:, :, sl], S, z, EPS, commit=False)
        assert np.array_equal(S0, S) and np.array_equal(z0, z)
        o, S, z = oracle.cache_step(q[:, :, sl], k[:, :, sl], v[:, :, sl], S, z, EPS, commit=True)
        assert np.array_equal(o, o0)
        assert S.nbytes + z.nbytes == nbytes0 == B * H * D * (D + 1) * 8
        outs.append(o)
    assert oracle.max_rel_err(np.concatenate(outs, axis=2), ref) < 1e-12
    assert oracle.max_rel_err(S, S_ref) < 1e-12 and oracle.max_rel_err(z, z_ref) < 1e-12


def test_state_update_accumulates():
    _, k, v = draw_qkv((2, 2, 30, 8), 9, "f32")
    k, v = k.astype(np.float64), v.astype(np.float64)
    S1, z1 = oracle.block_state_update(k[:, :, :13], v[:, :, :13], np.zeros((2, 2, 8, 8)), np.zeros((2, 2, 8)))
    S2, z2 = oracle.block_state_update(k[:, :, 13:], v[:, :, 13:], S1, z1)
    Sa, za = oracle.block_state_update(k, v, np.zeros((2, 2, 8, 8)), np.zeros((2, 2, 8)))
    assert np.allclose(S2, Sa, rtol=1e-13, atol=1e-13) and np.allclose(z2, za, rtol=1e-13, atol=1e-13)
    # and it is the same state that a prefill with one block reports as its final cache
    _, Sp, zp = oracle.block_causal_attn(k, k, v, 30, EPS)
    assert np.allclose(Sp, Sa, rtol=1e-13, atol=1e-13) and np.allclose(zp, za, rtol=1e-13, atol=1e-13)


def test_incoming_cache_is_added_to_every_block():
    q, k, v = draw_qkv((1, 2, 60, 8), 8, "f32")
    q, k, v = (x.astype(np.float64) for x in (q, k, v))
    # the cache equals the state of a previous 40-token segment: prefill over the concatenation
    # must give the same outputs for the last 60 tokens
    pq, pk, pv = (x.astype(np.float64) for x in draw_qkv((1, 2, 40, 8), 12, "f32"))
    _, S_in, z_in = oracle.block_causal_attn(pq, pk, pv, 40, EPS)
    got = oracle.block_causal_attn(q, k, v, 20, EPS, S_in, z_in)[0]
    full = oracle.block_causal_attn(np.concatenate([pq, q], 2), np.concatenate([pk, k], 2),
                                    np.concatenate([pv, v], 2), 20, EPS)[0][:, :, 40:]
    assert oracle.max_rel_err(got, full) < 1e-12


def test_permutation_inside_a_block():
    q, k, v = _c0()
    base = oracle.block_causal_attn(q, k, v, 64, EPS)[0]
    perm = np.random.default_rng(1).permutation(64) + 128  # shuffle block 2's keys/values
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 128:192] = k[:, :, perm]
    v2[:, :, 128:192] = v[:, :, perm]
    assert oracle.max_rel_err(oracle.block_causal_attn(q, k2, v2, 64, EPS)[0], base) < 1e-12
    # moving a key/value pair across a block boundary changes the outputs of the earlier block
    k3, v3 = k.copy(), v.copy()
    k3[:, :, [127, 128]] = k[:, :, [128, 127]]
    v3[:, :, [127, 128]] = v[:, :, [128, 127]]
    moved = oracle.block_causal_attn(q, k3, v3, 64, EPS)[0]
    assert oracle.max_rel_err(moved[:, :, 64:128], base[:, :, 64:128]) > 1e-6


def test_linear_in_v():
    q, k, v = _c0()
    v2 = np.random.default_rng(3).standard_normal(v.shape)
    a = oracle.block_causal_attn(q, k, v, 64, EPS)[0]
    b = oracle.block_causal_attn(q, k, v2, 64, EPS)[0]
    c = oracle.block_causal_attn(q, k, 2.5 * v - v2, 64, EPS)[0]
    assert oracle.max_rel_err(c, 2.5 * a - b) < 1e-12


def test_rows_from_states_matches_full():
    q, k, v = _c0()
    S, z = oracle.block_states(k, v, 64)
    P, zP = oracle.prefix_states(S, z)
    full = oracle.apply_states(q, P, zP, 64, EPS)
    rows = [0, 63, 64, 200, 255]
    blk = np.array(rows) // 64
    got = oracle.rows_from_states(q[0, 1, rows], P[0, 1, blk], zP[0, 1, blk], EPS)
    assert oracle.max_rel_err(got, full[0, 1, rows]) < 1e-14


def test_metric_is_normwise():
    assert oracle.max_rel_err([1.0, -2.0], [1.0, -2.0]) == 0.0
    assert abs(oracle.max_rel_err([1.1, -2.0], [1.0, -2.0]) - 0.05) < 1e-12
