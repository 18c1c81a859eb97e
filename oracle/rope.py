"""fp64 CPU oracle for 3D rotary position embedding inside ReLU linear attention.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path never imports or calls it.

Sources. The SANA-Video talk ("SANA-Video: Efficient Video Generation with Block Linear Diffusion
Transformer", passage on the two video adaptations of the Linear DiT: 3D RoPE for the linear
attention, and the temporal convolution) says that the linear attention gets a 3D rotary position
embedding. The model-family page (comfyui-wiki, architecture paragraph) adds rotary position
embeddings to the architecture. Neither page prints a formula, so the form below is a reading,
the plainest one that keeps the rest of the method intact:

1. Order: the feature map first, then the rotation: phi(x) = max(x, 0) as in the rest of the path,
   and the rotation acts on phi(q) and phi(k) ("RoPE on phi(q), phi(k)").
2. Numerator only. The normaliser phi(q_i) . z must stay positive, and a rotation keeps lengths
   but not signs, so the denominator keeps the unrotated features:
       o_i = R_i phi(q_i) . P / (phi(q_i) . zP + eps),
       P   = S_in + sum_j (R_j phi(k_j)) v_j^T,   zP = z_in + sum_j phi(k_j)   (over the visible j).
   The numerator's score is phi(q_i)^T R_i^T R_j phi(k_j), which depends on the positions only
   through their difference (rotations about the same planes commute).
3. Rotation: the RoFormer form (Su et al. 2021): feature pairs (2p, 2p+1) turn by the angle
   pos * theta_p. "3D": the D/2 pairs are split into three consecutive groups of pairs_t, pairs_h,
   pairs_w pairs, which take the token's frame, row and column index as pos; inside a group of
   P pairs, pair p' (0-based within the group) has theta = base^(-p' / P) (RoFormer's
   base^(-2i/d) with d = 2P features), base = 10000.
4. Positions: tokens are flattened frame-major, then row, then column, on a grid of
   height x width tokens per frame; token n of a (batch, head) sequence sits at frame
   frame0 + n // (height * width), row (n // width) % height, column n % width. frame0 lets a
   streamed block carry its absolute frame index, so streaming through the cache equals the
   one-shot prefill.
5. The cache of the block-causal form is (P, zP) above: the rotated-key state and the unrotated
   key sum.

Pins (tests/test_oracle_rope.py): zero angles reduce it to the pinned plain oracle; an
independent brute force builds every rotation as a dense block-diagonal D x D matrix and the
explicit masked N x N score matrices; a second one, in plain C (bruteforce.c), never turns a
vector and writes each pair's score through the cosine and sine of the angle difference;
shifting frame0 leaves the bidirectional output unchanged (relative positions); a D = 4 case
whose angles are whole radians checked against closed forms; streaming through the cache equals
the prefill; planted mistakes (rotated denominator, q turned the other way, half-split pairs)
each fail a pin. The pages fix none of this form, so parity of
this function is pinned to the mathematics of the reading above, not to the pages ("parity
unpinned" with respect to the pages).
"""

from __future__ import annotations

import math

import numpy as np

from .linattn import num_blocks, phi


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def default_pairs(D: int):
    """Default split of the D/2 rotation pairs over (frame, row, column): row and column get
    floor(D/6) pairs each, the frame axis the rest (for D = 128: 22, 21, 21)."""
    if D % 2 != 0:
        raise ValueError("D must be even for rotation pairs")
    ph = D // 6
    return (D // 2 - 2 * ph, ph, ph)


def token_positions(n_tokens: int, height: int, width: int, frame0: int = 0) -> np.ndarray:
    """(frame, row, column) of tokens 0..n_tokens-1, frame-major flattening (reading 4)."""
    n = np.arange(n_tokens, dtype=np.int64)
    hw = height * width
    return np.stack([frame0 + n // hw, (n // width) % height, n % width], axis=1)


def rope3d_angles(positions: np.ndarray, pairs, base: float = 10000.0) -> np.ndarray:
    """Angle of every rotation pair for every token: [n, D/2] (reading 3).

    Pairs [0, pairs_t) use the frame index, the next pairs_h the row, the last pairs_w the column;
    pair p' of a group of P pairs turns by pos * base^(-p' / P)."""
    positions = np.asarray(positions, dtype=np.int64)
    cols = []
    for axis, P in enumerate(pairs):
        if P == 0:
            continue
        freq = np.power(float(base), -np.arange(P, dtype=np.float64) / P)
        cols.append(positions[:, axis:axis + 1].astype(np.float64) * freq[None, :])
    return np.concatenate(cols, axis=1)


def rotate_pairs(x, angles) -> np.ndarray:
    """Turn each feature pair (2p, 2p+1) of x [..., n, D] by angles [n, D/2]:
    (a, b) -> (a cos - b sin, a sin + b cos)."""
    x = _f64(x)
    c = np.cos(angles)
    s = np.sin(angles)
    a = x[..., 0::2]
    b = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def block_causal_attn_rope(q, k, v, block_len: int, eps: float, angles, S_in=None, z_in=None):
    """Block-causal ReLU linear attention with the rotation on the numerator (readings 1-5).

    q, k, v: [B, H, N, D]; angles: [N, D/2] (the same for every batch and head). Returns
    (o [B,H,N,D], S_out [B,H,D,D], z_out [B,H,D]); S_out holds the rotated-key state, z_out the
    unrotated key sum. block_len >= N is the bidirectional form."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = q.shape
    L = int(block_len)
    fq, fk = phi(q), phi(k)
    rq, rk = rotate_pairs(fq, angles), rotate_pairs(fk, angles)
    P = np.zeros((B, H, D, v.shape[-1])) if S_in is None else _f64(S_in).copy()
    zP = np.zeros((B, H, D)) if z_in is None else _f64(z_in).copy()
    o = np.empty((B, H, N, v.shape[-1]))
    for c in range(num_blocks(N, L)):
        a, b = c * L, min(N, (c + 1) * L)
        P = P + np.matmul(np.swapaxes(rk[:, :, a:b], -1, -2), v[:, :, a:b])
        zP = zP + fk[:, :, a:b].sum(axis=2)
        num = np.matmul(rq[:, :, a:b], P)
        den = np.einsum("bhnd,bhd->bhn", fq[:, :, a:b], zP) + eps
        o[:, :, a:b] = num / den[..., None]
    return o, P, zP


def bruteforce_rope(q, k, v, block_len: int, eps: float, angles) -> np.ndarray:
    """The same result from the explicit masked score matrices: every rotation is a dense
    block-diagonal D x D matrix R_n (2x2 blocks [[cos, -sin], [sin, cos]]); the numerator scores
    are (R_i phi(q_i)) . (R_j phi(k_j)), the denominator scores phi(q_i) . phi(k_j), both masked by
    blk(j) <= blk(i). No cache."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = q.shape
    R = np.zeros((N, D, D))
    for n in range(N):
        for p in range(D // 2):
            c, s = math.cos(angles[n, p]), math.sin(angles[n, p])
            R[n, 2 * p, 2 * p], R[n, 2 * p, 2 * p + 1] = c, -s
            R[n, 2 * p + 1, 2 * p], R[n, 2 * p + 1, 2 * p + 1] = s, c
    blk = np.arange(N) // int(block_len)
    mask = (blk[None, :] <= blk[:, None]).astype(np.float64)
    o = np.empty((B, H, N, v.shape[-1]))
    for bb in range(B):
        for hh in range(H):
            fq, fk = phi(q[bb, hh]), phi(k[bb, hh])
            rq = np.einsum("nde,ne->nd", R, fq)
            rk = np.einsum("nde,ne->nd", R, fk)
            num_scores = (rq @ rk.T) * mask
            den_scores = (fq @ fk.T) * mask
            o[bb, hh] = (num_scores @ v[bb, hh]) / (den_scores.sum(axis=1) + eps)[:, None]
    return o
