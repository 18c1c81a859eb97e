"""fp64 CPU oracle for the linear projections around the attention: the fused Q/K/V projection with
the ReLU feature map applied to Q and K, and the output projection.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. It shares no code with the CUDA path.

Sources (SANA-Video pages):

* The SANA-Video model-family page, SANA-Video 2.0 paragraph: hidden size 2560 (the 720p 5B model;
  with 20 heads of 128 features this is the shape of configuration 4), linear-attention layers.
* The Linear DiT of the abstract, design (1): self-attention is replaced by linear attention whose
  feature map is ReLU (the feature map itself comes from the operation this library computes,
  o_i = ReLU(q_i) S / (ReLU(q_i) . z + eps), S = sum ReLU(k_j)^T v_j, z = sum ReLU(k_j)).

Readings (the pages print no projection formula; these are the plainest ones the rest supports):

* Q, K and V are linear maps of the hidden states without bias: y = x W^T with W stored as
  [out_features, in_features] (one row per output feature).
* The three projections are one matrix W_qkv [3 * H * D, C]: rows 0..HD-1 give Q, HD..2HD-1 give K,
  2HD..3HD-1 give V; inside each, head h owns rows h*D .. h*D + D - 1 (feature d of head h is row
  h*D + d). The outputs are laid out [B, H, N, D] as the attention consumes them.
* ReLU is applied to Q and K in the projection's epilogue (the attention applies it again, which
  changes nothing since ReLU(ReLU(x)) = ReLU(x)); V stays linear.
* The output projection concatenates the heads feature-major (o_cat[b, n, h*D + d] = o[b, h, n, d])
  and multiplies by W_o^T, W_o [C_out, H * D], no bias.

Pins (tests/test_oracle_next_pins.py): a case worked by hand (tests/golden), one-hot weights that
fix where every output feature lands, the sign behaviour of ReLU against the linear V, and the
output projection against its sum over heads.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def qkv_projection(x, w_qkv, H: int, D: int):
    """x [B, N, C], w_qkv [3*H*D, C]. Returns (q, k, v), each [B, H, N, D]:
    q = ReLU(x Wq^T), k = ReLU(x Wk^T), v = x Wv^T."""
    x = _f64(x)
    w = _f64(w_qkv)
    B, N, C = x.shape
    assert w.shape == (3 * H * D, C), (w.shape, H, D, C)
    y = np.matmul(x, w.T)                                   # [B, N, 3*H*D]
    y = y.reshape(B, N, 3, H, D).transpose(2, 0, 3, 1, 4)   # [3, B, H, N, D]
    return np.maximum(y[0], 0.0), np.maximum(y[1], 0.0), y[2].copy()


def out_projection(o, w_o):
    """o [B, H, N, D] (attention output), w_o [C_out, H*D]. Returns o_cat W_o^T, [B, N, C_out]."""
    o = _f64(o)
    w = _f64(w_o)
    B, H, N, D = o.shape
    assert w.shape[1] == H * D, (w.shape, H, D)
    o_cat = o.transpose(0, 2, 1, 3).reshape(B, N, H * D)
    return np.matmul(o_cat, w.T)
