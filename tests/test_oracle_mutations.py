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
