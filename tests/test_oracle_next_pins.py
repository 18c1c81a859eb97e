"""Pins of the projection and temporal-convolution oracles against things other than themselves.

Projection (oracle/projection.py): a hand-worked case; one-hot weights that fix where each output
feature of the fused [3*H*D, C] weight lands (tensor, head, feature); ReLU on Q and K only (the sign
of a negated input); the output projection against its decomposition into a sum over heads.

Temporal convolution (oracle/temporal_conv.py): a hand-worked case (padding token and carried token
of the talk's causal-FFN passage); one block against scipy's zero-padded centred correlation;
streaming block by block with the carried frames against the one-shot construction (the invariant
the passage states); causality; the block-boundary closed form.
"""

import numpy as np
import pytest
import scipy.signal

import golden
from oracle.projection import out_projection, qkv_projection
from oracle.temporal_conv import centred_conv, temporal_conv_block_causal, temporal_conv_step


# ---------------------------------------------------------------------------------------------
# projection
# ---------------------------------------------------------------------------------------------
def test_projection_hand_worked():
    g = golden.load_values("hand_worked_projection.txt")
    H, D = int(g["H"][0]), int(g["D"][0])
    x = g["x"].reshape(1, 2, H * D)
    q, k, v = qkv_projection(x, g["w_qkv"].reshape(3 * H * D, H * D), H, D)
    assert np.array_equal(q, g["q"].reshape(1, H, 2, D))
    assert np.array_equal(k, g["k"].reshape(1, H, 2, D))
    assert np.array_equal(v, g["v"].reshape(1, H, 2, D))
    o = g["o_heads"].reshape(1, 2, 2, 1)
    y = out_projection(o, g["w_o"].reshape(2, 2))
    assert np.array_equal(y, g["y"].reshape(1, 2, 2))


@pytest.mark.parametrize("f,c", [(0, 0), (5, 3), (2 * 3 * 4 - 1, 7), (3 * 4 + 6, 2), (2 * 3 * 4 + 9, 5)])
def test_projection_one_hot_weight_lands_on_its_feature(f, c):
    # H = 3 heads of D = 4 features, C = 8: a single 1 at row f, column c of w_qkv sends input
    # feature c to output feature f: tensor f // (H*D), head (f % (H*D)) // D, feature f % D
    H, D, C = 3, 4, 8
    rng = np.random.default_rng(f * 31 + c)
    x = np.abs(rng.standard_normal((2, 5, C))) + 0.1   # positive: ReLU passes it
    w = np.zeros((3 * H * D, C))
    w[f, c] = 1.0
    outs = qkv_projection(x, w, H, D)
    t, h, d = f // (H * D), (f % (H * D)) // D, f % D
    for i, o in enumerate(outs):
        want = np.zeros((2, H, 5, D))
        if i == t:
            want[:, h, :, d] = x[:, :, c]
        assert np.array_equal(o, want), (i, t, h, d)


def test_projection_relu_on_q_k_only():
    # ReLU(a) - ReLU(-a) = a: the Q and K outputs of x and -x differ by the linear projection, which
    # the V slot gives when the weight blocks are swapped; V of -x is minus V of x
    rng = np.random.default_rng(2)
    H, D, C = 2, 3, 6
    F = H * D
    x = rng.standard_normal((1, 7, C))
    w = rng.standard_normal((3 * F, C))
    q, k, v = qkv_projection(x, w, H, D)
    qn, kn, vn = qkv_projection(-x, w, H, D)
    _, _, q_lin = qkv_projection(x, np.concatenate([w[2 * F:], w[F:2 * F], w[:F]]), H, D)
    _, _, k_lin = qkv_projection(x, np.concatenate([w[:F], w[2 * F:], w[F:2 * F]]), H, D)
    assert np.allclose(vn, -v, rtol=0, atol=1e-14)
    assert np.allclose(q - qn, q_lin, rtol=0, atol=1e-14) and np.allclose(k - kn, k_lin, rtol=0, atol=1e-14)
    assert np.all(q >= 0) and np.all(k >= 0) and np.all((q == 0) | (qn == 0))
    assert np.any(q > 0) and np.any(qn > 0)


def test_out_projection_is_a_sum_over_heads():
    rng = np.random.default_rng(3)
    B, H, N, D, Co = 2, 3, 9, 4, 5
    o = rng.standard_normal((B, H, N, D))
    w = rng.standard_normal((Co, H * D))
    y = out_projection(o, w)
    want = sum(np.einsum("bnd,cd->bnc", o[:, h], w[:, h * D:(h + 1) * D]) for h in range(H))
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# temporal convolution
# ---------------------------------------------------------------------------------------------
def _conv_fixture():
    g = golden.load_values("hand_worked_temporal_conv.txt")
    x = g["x"].reshape(1, 4, 1, 2)
    return g, x, g["w"].reshape(2, 3), g["b"]


def test_temporal_conv_hand_worked():
    g, x, w, b = _conv_fixture()
    L = int(g["frames_per_block"][0])
    y = temporal_conv_block_causal(x, w, b, L)
    assert np.array_equal(y, g["y_block_causal"].reshape(1, 4, 1, 2))
    assert np.array_equal(temporal_conv_block_causal(x, w, b, 4), g["y_one_block"].reshape(1, 4, 1, 2))
    # the same two blocks streamed with the carried frame
    y0, carry = temporal_conv_step(x[:, :2], w, b)
    y1, _ = temporal_conv_step(x[:, 2:], w, b, carry)
    assert np.array_equal(np.concatenate([y0, y1], axis=1), y)


@pytest.mark.parametrize("K", [3, 5])
def test_one_block_is_a_zero_padded_centred_correlation(K):
    rng = np.random.default_rng(K)
    B, T, S, C = 2, 11, 3, 4
    x = rng.standard_normal((B, T, S, C))
    w = rng.standard_normal((C, K))
    bias = rng.standard_normal(C)
    y = temporal_conv_block_causal(x, w, bias, T)
    want = np.zeros_like(x)
    for b in range(B):
        for s in range(S):
            for c in range(C):
                want[b, :, s, c] = scipy.signal.correlate(x[b, :, s, c], w[c], mode="same") + bias[c]
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    assert np.allclose(centred_conv(x, w, bias), want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,L,K", [(60, 3, 3), (10, 3, 3), (7, 7, 3), (12, 4, 5), (9, 2, 3)])
def test_streaming_with_carry_equals_one_shot(T, L, K):
    rng = np.random.default_rng(T + L)
    B, S, C = 1, 5, 6
    x = rng.standard_normal((B, T, S, C))
    w = rng.standard_normal((C, K))
    bias = rng.standard_normal(C)
    one = temporal_conv_block_causal(x, w, bias, L)
    carry, outs = None, []
    for a in range(0, T, L):
        y, carry = temporal_conv_step(x[:, a:a + L], w, bias, carry)
        outs.append(y)
        assert carry.shape == (B, K // 2, S, C)        # constant memory: r frames, whatever the length
    assert np.allclose(np.concatenate(outs, axis=1), one, rtol=1e-12, atol=1e-12)


def test_causality_and_block_boundary_closed_form():
    rng = np.random.default_rng(9)
    B, T, S, C, L = 1, 12, 2, 3, 3
    x = rng.standard_normal((B, T, S, C))
    w = rng.standard_normal((C, 3))
    y = temporal_conv_block_causal(x, w, None, L)
    x2 = x.copy()
    x2[:, 6:] = rng.standard_normal((B, T - 6, S, C))   # change blocks 2 and 3
    y2 = temporal_conv_block_causal(x2, w, None, L)
    assert np.array_equal(y[:, :6], y2[:, :6])          # blocks 0 and 1 cannot see them
    assert not np.allclose(y[:, 6:], y2[:, 6:])
    # last frame of a block: the right neighbour is the padding zero; first frame of a block: the
    # left neighbour is the previous block's last frame
    for t in (2, 5, 8):
        assert np.allclose(y[:, t], w[:, 0] * x[:, t - 1] + w[:, 1] * x[:, t], atol=1e-14)
    for t in (3, 6, 9):
        assert np.allclose(y[:, t], w[:, 0] * x[:, t - 1] + w[:, 1] * x[:, t] + w[:, 2] * x[:, t + 1], atol=1e-14)
