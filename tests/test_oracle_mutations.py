"""Planted mistakes in the oracle's linear form, on the CPU: each must be caught by the brute force
pin, which shows that the pins in test_oracle_pins.py have teeth."""

import numpy as np
import pytest

import oracle
from oracle import linattn as L
from oracle.bruteforce import bruteforce_c
from block_causal_linear_relu_b200.inputs import draw_qkv

EPS = 1e-6


def _mutant(kind, q, k, v, blen, eps):
    S, z = L.block_states(k, v, blen)
    if kind == "transposed_state":
        S = np.swapaxes(S, -1, -2)
    if kind == "identity_feature_map":
        S, z = L.block_states(np.abs(k) * np.sign(k) + 0.0 * k, v, blen)  # no ReLU on k
        S2 = []
        for c in range(S.shape[2]):
            a, b = c * blen, min(k.shape[2], (c + 1) * blen)
            S2.append(np.matmul(np.swapaxes(k[:, :, a:b], -1, -2), v[:, :, a:b]))
        S = np.stack(S2, axis=2)
    P, zP = L.prefix_states(S, z)
    if kind == "exclusive_prefix":
        P = P - S
        zP = zP - z
    if kind == "block_off_by_one":
        P = np.concatenate([P[:, :, 1:], P[:, :, -1:]], axis=2)
        zP = np.concatenate([zP[:, :, 1:], zP[:, :, -1:]], axis=2)
    if kind == "no_normaliser":
        zP = np.zeros_like(zP)
        return L.apply_states(q, P, zP, blen, 1.0)
    if kind == "eps_in_numerator":
        return L.apply_states(q, P, zP, blen, eps) + eps
    return L.apply_states(q, P, zP, blen, eps)


@pytest.mark.parametrize("kind", ["transposed_state", "identity_feature_map", "exclusive_prefix",
                                  "block_off_by_one", "no_normaliser"])
def test_planted_mistake_is_caught(kind):
    q, k, v = (x.astype(np.float64) for x in draw_qkv((1, 2, 96, 8), 21, "f32"))
    ref = bruteforce_c(q, k, v, 32, EPS)
    assert oracle.max_rel_err(_mutant("none", q, k, v, 32, EPS), ref) < 1e-12
    assert oracle.max_rel_err(_mutant(kind, q, k, v, 32, EPS), ref) > 1e-3


def test_planted_eps_in_numerator_is_caught_by_zero_row():
    q, k, v = (x.astype(np.float64) for x in draw_qkv((1, 1, 32, 8), 22, "f32"))
    q[0, 0, 5] = -1.0  # a non-positive query row must give exactly zero
    out = _mutant("eps_in_numerator", q, k, v, 8, 1e-3)
    assert np.any(out[0, 0, 5] != 0.0)


@pytest.mark.parametrize("kind", ["cache_ignored", "cache_twice", "cache_z_dropped"])
def test_planted_cache_mistake_is_caught_by_hand_worked_fixture(kind):
    # the incoming cache's handling, against the hand-worked fixture with a cache (tests/golden)
    import golden

    g = golden.load("hand_worked_cache_d1_n3.txt")
    S, z = L.block_states(g["k"], g["v"], g["block_len"])
    S_in, z_in = g["S_in"], g["z_in"]
    if kind == "cache_ignored":
        S_in, z_in = None, None
    elif kind == "cache_twice":
        S_in, z_in = 2 * S_in, 2 * z_in
    elif kind == "cache_z_dropped":
        z_in = None
    P, zP = L.prefix_states(S, z, S_in, z_in)
    got = L.apply_states(g["q"], P, zP, g["block_len"], g["eps"])
    assert not np.allclose(got, g["o_block_causal"], rtol=1e-6, atol=1e-9)
    P0, zP0 = L.prefix_states(S, z, g["S_in"], g["z_in"])
    assert np.allclose(L.apply_states(g["q"], P0, zP0, g["block_len"], g["eps"]), g["o_block_causal"], rtol=1e-15,
                       atol=1e-15)


# ---------------------------------------------------------------------------------------------
# the projection and temporal-convolution oracles: planted mistakes against their pins
# ---------------------------------------------------------------------------------------------
def _proj_mutant(kind, x, w, H, D):
    from oracle import projection as P
    if kind == "head_feature_swapped":   # rows read as feature-major, head-minor
        B, N, C = x.shape
        y = np.matmul(x, w.T).reshape(B, N, 3, D, H).transpose(2, 0, 4, 1, 3)
        return np.maximum(y[0], 0), np.maximum(y[1], 0), y[2]
    if kind == "relu_on_v":
        q, k, v = P.qkv_projection(x, w, H, D)
        return q, k, np.maximum(v, 0)
    if kind == "no_relu_on_k":
        q, _, v = P.qkv_projection(x, w, H, D)
        F = H * D
        _, _, k_lin = P.qkv_projection(x, np.concatenate([w[:F], w[2 * F:], w[F:2 * F]]), H, D)
        return q, k_lin, v
    if kind == "w_not_transposed":       # x W instead of x W^T (square blocks only)
        B, N, C = x.shape
        F = H * D
        ys = [np.matmul(x, w[i * F:(i + 1) * F]) for i in range(3)]
        out = [y.reshape(B, N, H, D).transpose(0, 2, 1, 3) for y in ys]
        return np.maximum(out[0], 0), np.maximum(out[1], 0), out[2]
    return P.qkv_projection(x, w, H, D)


@pytest.mark.parametrize("kind", ["head_feature_swapped", "relu_on_v", "no_relu_on_k", "w_not_transposed"])
def test_planted_projection_mistake_is_caught(kind):
    import golden

    g = golden.load_values("hand_worked_projection.txt")
    H, D = int(g["H"][0]), int(g["D"][0])
    x, w = g["x"].reshape(1, 2, H * D), g["w_qkv"].reshape(3 * H * D, H * D)
    want = (g["q"].reshape(1, H, 2, D), g["k"].reshape(1, H, 2, D), g["v"].reshape(1, H, 2, D))
    assert all(np.array_equal(a, b) for a, b in zip(_proj_mutant("none", x, w, H, D), want))
    caught_by_fixture = not all(np.array_equal(a, b) for a, b in zip(_proj_mutant(kind, x, w, H, D), want))
    # the fixture has one head, so the head layout is pinned by the one-hot weights instead
    Hh, Dh, C = 3, 4, 12
    xh = np.abs(np.random.default_rng(1).standard_normal((1, 5, C))) + 0.1
    wh = np.zeros((3 * Hh * Dh, C))
    f = Hh * Dh + 1 * Dh + 2           # K output, head 1, feature 2
    wh[f, 3] = 1.0
    _, k, _ = _proj_mutant(kind, xh, wh, Hh, Dh)
    caught_by_one_hot = not np.array_equal(k[:, 1, :, 2], xh[:, :, 3])
    assert caught_by_fixture or caught_by_one_hot


def _conv_mutant(kind, x, w, b, L):
    from oracle import temporal_conv as T
    if kind == "no_padding_token":       # a plain centred conv over the whole sequence
        return T.centred_conv(x, w, b)
    if kind == "no_carried_token":       # blocks convolved in isolation
        return np.concatenate([T.centred_conv(x[:, a:a + L], w, b) for a in range(0, x.shape[1], L)], axis=1)
    if kind == "flipped_kernel":         # convolution instead of correlation
        return T.temporal_conv_block_causal(x, w[:, ::-1], b, L)
    if kind == "carry_first_frame":      # the block's first frame carried instead of its last
        outs, carry = [], None
        for a in range(0, x.shape[1], L):
            y, _ = T.temporal_conv_step(x[:, a:a + L], w, b, carry)
            outs.append(y)
            carry = x[:, a:a + 1]
        return np.concatenate(outs, axis=1)
    return T.temporal_conv_block_causal(x, w, b, L)


@pytest.mark.parametrize("kind", ["no_padding_token", "no_carried_token", "flipped_kernel", "carry_first_frame"])
def test_planted_temporal_conv_mistake_is_caught_by_hand_worked_fixture(kind):
    import golden

    g = golden.load_values("hand_worked_temporal_conv.txt")
    x, w, b = g["x"].reshape(1, 4, 1, 2), g["w"].reshape(2, 3), g["b"]
    want = g["y_block_causal"].reshape(1, 4, 1, 2)
    assert np.array_equal(_conv_mutant("none", x, w, b, 2), want)
    assert not np.allclose(_conv_mutant(kind, x, w, b, 2), want)
