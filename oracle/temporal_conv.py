"""fp64 CPU oracle for the block-causal temporal convolution of SANA-Video's causal Mix-FFN.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. It shares no code with the CUDA path.

Sources (SANA-Video pages):

* "SANA-Video: Efficient Video Generation with Block Linear Diffusion Transformer" (ICLR 2026 oral,
  talk transcript), causal FFN with temporal conv passage: with two blocks, block 1 must not see
  block 2, so a zero token is padded between the two blocks; block 2 must see block 1, so the last
  token of block 1 is carried in as the first token of block 2; the padding token (and the carried
  token) are removed after the convolution.
* The SANA-Video model-family page: a one-dimensional temporal convolution inside the Mix-FFN.

Readings (the pages give neither the kernel width nor the weights):

* The convolution runs along the time axis (latent frames), depthwise: one kernel of width
  K = 2r + 1 per channel, centred (y_t = sum_j w[c, j] x_{t + j - r} + b[c], cross-correlation
  order, zero padding at the sequence ends). A centred kernel is what the passage implies: a kernel
  that only looked back would need no padding token between the blocks. The single padding token
  and the single carried token of the passage make r = 1 (K = 3); the construction below takes r
  padding and r carried tokens for a general r.
* A "token" of the passage is one latent frame: every spatial position of a frame is convolved
  along time independently ([B, T, S, C] with T frames of S tokens and C channels).
* Blocks hold ``frames_per_block`` frames (the last one may be shorter), as in the attention.

Pins (tests/test_oracle_next_pins.py): a case worked by hand (tests/golden); one block equals a
plain zero-padded centred correlation (scipy); block-by-block streaming with the carried frames
equals the one-shot construction (the invariant the passage states); causality (a later block
never changes an earlier block's output).
"""

from __future__ import annotations

import math

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def centred_conv(x, w, bias=None):
    """Zero-padded centred depthwise correlation along axis 1 (time): x [B, T, S, C], w [C, K] with K
    odd; y_t = sum_j w[:, j] x_{t + j - r} (+ bias), x outside [0, T) read as zero."""
    x = _f64(x)
    w = _f64(w)
    B, T, S, C = x.shape
    K = w.shape[1]
    assert K % 2 == 1 and w.shape[0] == C
    r = K // 2
    xp = np.zeros((B, T + 2 * r, S, C))
    xp[:, r:r + T] = x
    y = np.zeros((B, T, S, C))
    for j in range(K):
        y += xp[:, j:j + T] * w[:, j]
    if bias is not None:
        y += _f64(bias)
    return y


def temporal_conv_block_causal(x, w, bias, frames_per_block: int):
    """The talk's construction over a whole sequence: between consecutive blocks insert r zero
    padding frames (block c cannot see block c + 1) followed by block c's last r frames carried
    into block c + 1 (block c + 1 sees block c); convolve the padded sequence; keep the outputs of
    the original frames only."""
    x = _f64(x)
    B, T, S, C = x.shape
    r = _f64(w).shape[1] // 2
    L = int(frames_per_block)
    nb = max(1, math.ceil(T / L))
    pieces, keep = [], []
    for c in range(nb):
        a, b = c * L, min(T, (c + 1) * L)
        if c > 0:
            assert a >= r, "a block needs at least r frames before it to carry"
            pieces.append(x[:, a - r:a])            # carried: the previous block's last r frames
            keep += [False] * r
        pieces.append(x[:, a:b])
        keep += [True] * (b - a)
        if c < nb - 1:
            pieces.append(np.zeros((B, r, S, C)))   # padding: the next block is not visible
            keep += [False] * r
    y = centred_conv(np.concatenate(pieces, axis=1), w, bias)
    return y[:, np.array(keep)]


def temporal_conv_step(x_block, w, bias, carry=None):
    """One block of a stream: the block's frames with the carried frames of the previous block in
    front (zeros for the first block) and r zero frames behind. Returns (y_block, new_carry) with
    new_carry = the block's last r frames. Memory kept between blocks: carry only, [B, r, S, C]."""
    x_block = _f64(x_block)
    B, T, S, C = x_block.shape
    r = _f64(w).shape[1] // 2
    front = np.zeros((B, r, S, C)) if carry is None else _f64(carry)
    xp = np.concatenate([front, x_block, np.zeros((B, r, S, C))], axis=1)
    y = centred_conv(xp, w, bias)[:, r:r + T]
    return y, x_block[:, T - r:].copy()
