"""Chunked form of the Gated Delta Rule forward in numpy fp64 (test infrastructure only).

Written from the page "Qwen3Next Samples" (chunk_gated_delta_rule,
"Mathematical Formulas"), step by step in that page's order and names:
gate cumulative sum -> decay mask -> pre-attention matrix A -> matrix
inversion -> value and key cumulative decay -> recurrent state attention ->
state update.  The chunk size C is a parameter (on the LinearAttention
operator page the chunk size is an attribute with no effect on the output), so
C = 1 reduces to the token recurrence and any C must agree with it.

Readings where the page is silent or garbled (each also listed with the design notes):
* The state is kept as S[Dk, Dv] (the decode page's layout); the page's
  ``S^T`` products therefore appear here as plain products with S.
* M_mask (described on the page as a negative mask on the lower triangle) is
  -1 strictly below the diagonal and 0 elsewhere, so the inverse is (I - A)^-1 of a strictly lower
  triangular A; T_tril (lower triangle of ones) includes the diagonal.
* The garbled row recurrence of "Matrix Inversion" is read as forward
  substitution: X[i, :i] = A[i, :i] + A[i, :i] X[:i, :i], inverse = I + X.
* g_last is the cumulative gate at the last valid row of a (possibly partial)
  chunk, and the g in k_gexp = k * exp(g_last - g) is the cumulative gate.
* A chunk never crosses a sequence start; the last chunk of a sequence holds
  the remaining len mod C tokens.
"""
from __future__ import annotations

import math

import numpy as np


def l2norm(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(sum(x^2) + eps) over the last axis ("L2 Normalization")."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def forward_substitution_inverse(A: np.ndarray) -> np.ndarray:
    """(I - A)^-1 for strictly lower-triangular A, one row at a time."""
    n = A.shape[0]
    X = np.zeros_like(A)
    for i in range(n):
        X[i, :i] = A[i, :i] + A[i, :i] @ X[:i, :i]
    return np.eye(n) + X


def inverse_by_block_merge(A: np.ndarray, base: int = 16) -> np.ndarray:
    """(I - A)^-1 from inverses of the diagonal blocks, merged two at a time.

    Follows the page's inverse_pto / inverse_matmul description: the inverse of
    [[M11, 0], [M21, M22]] is [[M11^-1, 0], [-M22^-1 M21 M11^-1, M22^-1]], with
    M = I - A.  Block sizes double from ``base`` up to n (n = base * 2^j)."""
    n = A.shape[0]
    M = np.eye(n) - A
    inv = np.zeros_like(A)
    for s in range(0, n, base):
        inv[s:s + base, s:s + base] = forward_substitution_inverse(A[s:s + base, s:s + base])
    size = base
    while size < n:
        for s in range(0, n, 2 * size):
            i11 = inv[s:s + size, s:s + size]
            i22 = inv[s + size:s + 2 * size, s + size:s + 2 * size]
            m21 = M[s + size:s + 2 * size, s:s + size]
            inv[s + size:s + 2 * size, s:s + size] = -(i22 @ m21 @ i11)
        size *= 2
    return inv


def chunk_intermediates(qn: np.ndarray, kn: np.ndarray, v: np.ndarray, g: np.ndarray,
                        beta: np.ndarray, S: np.ndarray) -> dict:
    """One chunk of one (sequence, v-head).

    qn, kn: normalised (and, for q, scaled) rows [n, Dk]; v [n, Dv]; g, beta [n];
    S [Dk, Dv] the state entering the chunk.  Returns every named intermediate."""
    n = qn.shape[0]
    tril = np.tril(np.ones((n, n)))                      # T_tril, diagonal included
    mask = -np.tril(np.ones((n, n)), k=-1)               # M_mask, strictly lower, negative
    g_cum = tril @ g                                     # Gate Cumulative Sum
    decay = np.exp((g_cum[:, None] - g_cum[None, :]) * tril)   # Decay Mask
    k_beta = kn * beta[:, None]                          # k_beta = k (.) beta
    A = (k_beta @ kn.T) * decay * mask                   # Pre-Attention Matrix
    A_inv = forward_substitution_inverse(A)              # (I - A)^-1
    v_out = A_inv @ (v * beta[:, None])                  # value output
    k_cumdecay = A_inv @ (k_beta * np.exp(g_cum)[:, None])
    v_prime = k_cumdecay @ S                             # v' (state read by the chunk)
    o_inter = (qn * np.exp(g_cum)[:, None]) @ S
    v_new = v_out - v_prime
    o = o_inter + ((qn @ kn.T) * decay * tril) @ v_new
    g_last = g_cum[-1]
    k_gexp = kn * np.exp(g_last - g_cum)[:, None]
    S_new = S * math.exp(g_last) + k_gexp.T @ v_new      # State Update
    return dict(g_cum=g_cum, decay=decay, A=A, A_inv=A_inv, v_out=v_out, k_cumdecay=k_cumdecay,
                v_prime=v_prime, v_new=v_new, o=o, S_in=S, S_new=S_new)


def chunked(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None,
            eps=1e-6, C=128, heads=None, keep=False):
    """Chunked forward over a packed varlen batch (float64 numpy inputs).

    Same shapes and defaults as ``oracle.recurrent``.  With keep=True also
    returns {(b, h, chunk): intermediates}."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, Nqk, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[2]
    B = cu.shape[0] - 1
    G = Nv // Nqk
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(Dk)
    hl = list(range(Nv)) if heads is None else list(heads)
    out = np.zeros((T, len(hl), Dv))
    fin = np.zeros((B, len(hl), Dk, Dv))
    kept = {}
    for b in range(B):
        for slot, h in enumerate(hl):
            hq = h // G
            if state_pool is None:
                S = np.zeros((Dk, Dv))
            else:
                s = b if state_indices is None else int(state_indices[b])
                S = np.asarray(state_pool[s, h], dtype=np.float64).copy()
            start, end = int(cu[b]), int(cu[b + 1])
            for ci, c0 in enumerate(range(start, end, C)):
                c1 = min(c0 + C, end)
                qn = scale * l2norm(q[c0:c1, hq], eps)
                kn = l2norm(k[c0:c1, hq], eps)
                r = chunk_intermediates(qn, kn, v[c0:c1, h], g[c0:c1, h], beta[c0:c1, h], S)
                if keep:
                    r["qn"], r["kn"] = qn, kn
                out[c0:c1, slot] = r["o"]
                S = r["S_new"]
                if keep:
                    kept[(b, h, ci)] = r
            fin[b, slot] = S
    if keep:
        return out, fin, kept
    return out, fin
