"""fp64 CPU oracle for ReLU-kernel linear attention, bidirectional and block-causal.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The product path (the CUDA library and its Python binding)
never imports or calls it, and it shares no code with that path.

What it computes (sources are the SANA-Video pages):

* "SANA-Video: Efficient Video Generation with Block Linear Diffusion Transformer" (ICLR 2026
  oral, talk transcript), block KV cache passage: linear attention keeps a *state* of fixed shape
  D x D whatever the sequence length; a block's state is added to the cache of the previous
  blocks; block-causal linear attention caches the state of block 1, adds block 2's
  contribution, and so on; memory stays constant while the whole history stays visible.
* Same talk, hybrid AR + diffusion passage: video is generated block by block causally and is
  diffused *within* a block, so attention inside a block is bidirectional.
* Same paper's abstract, design (2): the constant-memory state comes from the cumulative
  property of linear attention.
* Feature map ReLU, the normaliser ReLU(q).z + eps and eps itself are not printed on the pages;
  they come from the benchmark spec of this library (out_i = ReLU(q_i).S / (ReLU(q_i).z + eps),
  S = sum ReLU(k_j)^T v_j, z = sum ReLU(k_j)).

Definition (the plain form every function here reaches, up to rounding):

    A_ij = phi(q_i) . phi(k_j),   phi(x) = max(x, 0)
    O_i  = sum_j M_ij A_ij v_j / (sum_j M_ij A_ij + eps)
    M_ij = 1 (bidirectional)   or   [blk(j) <= blk(i)], blk(i) = floor(i / L) (block-causal)

The linear (state) form used below: per block c, S_c = sum_{j in c} phi(k_j) v_j^T (rows: key
feature d, columns: value feature e) and z_c = sum_{j in c} phi(k_j); inclusive prefix
P_c = S_in + sum_{c' <= c} S_c', zP_c = z_in + sum_{c' <= c} z_c'; then
O_i = phi(q_i)^T P_blk(i) / (phi(q_i)^T zP_blk(i) + eps).

Pins (tests/test_oracle_pins.py): two independent brute forces of the explicit masked N x N
matrix (numpy here, plain C in bruteforce.c), the token recurrence of causal linear attention
(Katharopoulos et al. 2020) for L = 1, closed forms (constant v, non-positive q row, one-hot
state), small cases worked by hand from the definition (tests/golden, one of them with an
incoming cache and eps > 0), and invariants (streaming == prefill, constant cache bytes,
permutation within a block). Every function below is pinned; none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np


def phi(x: np.ndarray) -> np.ndarray:
    """ReLU feature map. NaN propagates (numpy maximum semantics)."""
    return np.maximum(x, 0.0)


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def num_blocks(n: int, block_len: int) -> int:
    """Number of blocks; a last block shorter than block_len is allowed (partial)."""
    return max(1, math.ceil(n / block_len)) if n > 0 else 0


def block_states(k, v, block_len: int):
    """Per-block states: S_c = sum_{j in c} phi(k_j) v_j^T  [B,H,nblk,D,D],  z_c = sum phi(k_j)  [B,H,nblk,D].

    The additive update of the talk's block KV cache passage: each block contributes its own
    K^T V (with the ReLU feature map on K) and its own sum of features.
    """
    k = _f64(k)
    v = _f64(v)
    B, H, N, D = k.shape
    L = int(block_len)
    nb = num_blocks(N, L)
    S = np.zeros((B, H, nb, D, v.shape[-1]), dtype=np.float64)
    z = np.zeros((B, H, nb, D), dtype=np.float64)
    for c in range(nb):
        a, b = c * L, min(N, (c + 1) * L)
        fk = phi(k[:, :, a:b, :])
        S[:, :, c] = np.matmul(np.swapaxes(fk, -1, -2), v[:, :, a:b, :])
        z[:, :, c] = fk.sum(axis=2)
    return S, z


def prefix_states(S, z, S_in=None, z_in=None):
    """Inclusive prefix over blocks: P_c = S_in + sum_{c'<=c} S_c' (same for z).

    Inclusive because a block diffuses within itself (sees its own block) and sees the cache of
    all previous blocks.
    """
    P = np.cumsum(S, axis=2)
    zP = np.cumsum(z, axis=2)
    if S_in is not None:
        P = P + _f64(S_in)[:, :, None]
    if z_in is not None:
        zP = zP + _f64(z_in)[:, :, None]
    return P, zP


def apply_states(q, P, zP, block_len: int, eps: float):
    """O_i = phi(q_i)^T P_blk(i) / (phi(q_i)^T zP_blk(i) + eps) for every token."""
    q = _f64(q)
    B, H, N, D = q.shape
    L = int(block_len)
    out = np.zeros((B, H, N, P.shape[-1]), dtype=np.float64)
    for c in range(num_blocks(N, L)):
        a, b = c * L, min(N, (c + 1) * L)
        fq = phi(q[:, :, a:b, :])
        num = np.matmul(fq, P[:, :, c])
        den = np.matmul(fq, zP[:, :, c][..., None])
        out[:, :, a:b] = num / (den + eps)
    return out


def block_causal_attn(q, k, v, block_len: int, eps: float, S_in=None, z_in=None):
    """Block-causal prefill. Returns (O, S_out, z_out) with S_out/z_out the final cache.

    Each block attends to itself (bidirectionally) plus the summed state of all previous blocks
    and of the incoming cache (S_in, z_in), as in the talk's block-causal walkthrough.
    """
    S, z = block_states(k, v, block_len)
    P, zP = prefix_states(S, z, S_in, z_in)
    O = apply_states(q, P, zP, block_len, eps)
    return O, P[:, :, -1].copy(), zP[:, :, -1].copy()


def linattn_fwd(q, k, v, eps: float):
    """Bidirectional full-sequence form: one block holding the whole sequence."""
    N = np.shape(q)[2]
    O, _, _ = block_causal_attn(q, k, v, max(N, 1), eps)
    return O


def block_state_update(k, v, S, z):
    """Cache update without output: S + phi(K)^T V, z + sum phi(K) over all tokens given."""
    N = np.shape(k)[2]
    Sb, zb = block_states(k, v, max(N, 1))
    return _f64(S) + Sb[:, :, 0], _f64(z) + zb[:, :, 0]


def cache_step(q, k, v, S, z, eps: float, commit: bool = True):
    """One streaming step: the block attends to itself plus the cache; the cache then takes the
    block's state if ``commit``. Memory held between steps is (S, z) only, whatever the length."""
    N = np.shape(q)[2]
    O, S_new, z_new = block_causal_attn(q, k, v, max(N, 1), eps, S, z)
    if commit:
        return O, S_new, z_new
    return O, _f64(S).copy(), _f64(z).copy()


def rows_from_states(q_rows, P_rows, zP_rows, eps: float):
    """Output of selected tokens given each token's prefix state: used for sampled checks at sizes
    where the whole output is not needed. q_rows [R,D]; P_rows [R,D,E]; zP_rows [R,D]."""
    fq = phi(_f64(q_rows))
    num = np.einsum("rd,rde->re", fq, _f64(P_rows))
    den = np.einsum("rd,rd->r", fq, _f64(zP_rows))
    return num / (den[:, None] + eps)


# ----------------------------------------------------------------------------------------------
# Brute force (quadratic) form, used only to pin the linear form above.
# ----------------------------------------------------------------------------------------------

def bruteforce_masked(q, k, v, block_len: int, eps: float):
    """Explicit N x N kernel-attention matrix with the block-causal mask, in fp64.

    A = phi(Q) phi(K)^T;  M_ij = [floor(j/L) <= floor(i/L)];  O = (A*M) V / ((A*M) 1 + eps).
    ``block_len >= N`` gives the all-ones mask (bidirectional).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    N = q.shape[2]
    idx = np.arange(N)
    blk = idx // int(block_len)
    M = (blk[None, :] <= blk[:, None]).astype(np.float64)
    A = np.matmul(phi(q), np.swapaxes(phi(k), -1, -2)) * M
    num = np.matmul(A, v)
    den = A.sum(axis=-1, keepdims=True)
    return num / (den + eps)


def causal_recurrence(q, k, v, eps: float, S0=None, z0=None):
    """Token-level recurrence of causal linear attention (Katharopoulos et al. 2020,
    "Transformers are RNNs"): s_i = s_{i-1} + phi(k_i) v_i^T, z_i = z_{i-1} + phi(k_i),
    o_i = phi(q_i)^T s_i / (phi(q_i)^T z_i + eps). Pure Python loops: tiny inputs only."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    out = np.zeros((B, H, N, E))
    for b in range(B):
        for h in range(H):
            s = [[0.0] * E for _ in range(D)] if S0 is None else [list(map(float, r)) for r in _f64(S0)[b, h]]
            zz = [0.0] * D if z0 is None else list(map(float, _f64(z0)[b, h]))
            for i in range(N):
                fk = [max(float(x), 0.0) for x in k[b, h, i]]
                for d in range(D):
                    zz[d] += fk[d]
                    for e in range(E):
                        s[d][e] += fk[d] * float(v[b, h, i, e])
                fq = [max(float(x), 0.0) for x in q[b, h, i]]
                den = sum(fq[d] * zz[d] for d in range(D))
                for e in range(E):
                    out[b, h, i, e] = sum(fq[d] * s[d][e] for d in range(D)) / (den + eps)
    return out


# ----------------------------------------------------------------------------------------------
# Error metric used by every parity check.
# ----------------------------------------------------------------------------------------------

def max_rel_err(got, ref) -> float:
    """Normwise max relative error: max_i |g_i - r_i| / max_i |r_i| (0 when both are all zero).

    Outputs are zero-mean sums that cross zero, so an elementwise ratio is unbounded; the error
    is read relative to the largest reference magnitude of the tensor.
    """
    g = _f64(got)
    r = _f64(ref)
    if r.size == 0:
        return 0.0
    scale = float(np.max(np.abs(r)))
    diff = float(np.max(np.abs(g - r)))
    if scale == 0.0:
        return diff
    return diff / scale
