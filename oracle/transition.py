"""Brute-force transition-matrix form of the Gated Delta Rule (test infrastructure only).

Each token is an affine map of the state, S_t = M_t S_{t-1} + beta_t kh_t v_t^T
with the dense Dk x Dk matrix M_t = exp(g_t) (I - beta_t kh_t kh_t^T).  This is
the decode page's recurrence ("lite_boost.ops.recurrent_gated_delta_rule",
algorithm flow) with the retrieval substituted into the update, evaluated with
explicit matrices instead of the retrieval vector.  Meant for tiny Dk only.
"""
from __future__ import annotations

import math

import numpy as np


def transition(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None,
               eps=1e-6):
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
    out = np.zeros((T, Nv, Dv))
    fin = np.zeros((B, Nv, Dk, Dv))
    eye = np.eye(Dk)
    for b in range(B):
        for h in range(Nv):
            hq = h // G
            if state_pool is None:
                S = np.zeros((Dk, Dv))
            else:
                s = b if state_indices is None else int(state_indices[b])
                S = np.asarray(state_pool[s, h], dtype=np.float64).copy()
            for t in range(int(cu[b]), int(cu[b + 1])):
                kh = k[t, hq] / math.sqrt(float(k[t, hq] @ k[t, hq]) + eps)
                qh = scale * (q[t, hq] / math.sqrt(float(q[t, hq] @ q[t, hq]) + eps))
                M = math.exp(g[t, h]) * (eye - beta[t, h] * np.outer(kh, kh))
                S = M @ S + beta[t, h] * np.outer(kh, v[t, h])
                out[t, h] = S.T @ qh
            fin[b, h] = S
    return out, fin
