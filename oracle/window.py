"""fp64 oracle of the token recurrence with a window of recent states.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the CUDA path
imports it.

Page "com.microsoft.LinearAttention", attribute ``state_window`` and the shapes
of ``past_state`` / ``present_state``: with ``state_window = W > 0`` both state
tensors carry a leading window axis, (W, B, H_kv, d_k, d_v), holding the W
most recent recurrent states (W from 1 to 8), so that a caller can roll back
to an earlier one; W = 0 keeps only the current state.  The page fixes neither
the order of the window nor where a step starts.  The reading taken here is a
first-in-first-out window in time order:

* entry W - 1 is the most recent state and the step continues from it
  (entry W - 1 of ``past``);
* after each token of the sequence the new state is appended at the end and
  the oldest entry leaves, so after n tokens the window is the last W
  entries of [past[0], ..., past[W - 1], S_1, ..., S_n];
* a sequence shorter than the window therefore keeps its W - n most recent
  past states, moved n places towards entry 0; a sequence with no tokens
  keeps its window unchanged;
* an absent ``past_state`` is W zero states (the page: past_state defaults
  to zeros).

Rolling back r tokens of the last step is then reading entry W - 1 - r.  The
token loop is the one of ``oracle.pool`` (decode page order: decay, retrieval,
update, output from the updated state) under the page's four update rules,
with q and k normalised as in "Qwen3Next Samples", equation "L2
Normalization", and q scaled after the normalisation.  Plain numpy, per token,
for the small shapes of the tests.
"""
from __future__ import annotations

import math

import numpy as np

from . import as_numpy_exact

RULES = ("gated_delta", "delta", "gated", "linear")
MAX_WINDOW = 8


def recurrent_window(q, k, v, g, beta, cu_seqlens, past_window, window, scale=None, eps=1e-6, gk=None,
                     rule="gated_delta"):
    """Token recurrence of every (sequence, v-head) keeping the ``window`` most recent states, in fp64.

    Shapes: q, k [T, Nqk, Dk]; v [T, Nv, Dv]; g, beta [T, Nv]; cu_seqlens [B+1];
    past_window [W, B, Nv, Dk, Dv] or None (zeros); gk [T, Nv, Dk] or None.
    Returns (out [T, Nv, Dv], present_window [W, B, Nv, Dk, Dv]) as float64.
    """
    if rule not in RULES:
        raise ValueError(f"unknown update rule {rule}")
    W = int(window)
    if not 1 <= W <= MAX_WINDOW:
        raise ValueError(f"state window {W} outside 1..{MAX_WINDOW}")
    decay, delta = rule in ("gated_delta", "gated"), rule in ("gated_delta", "delta")
    Q, K, V = as_numpy_exact(q), as_numpy_exact(k), as_numpy_exact(v)
    G = as_numpy_exact(g) if decay else None
    Bt = as_numpy_exact(beta) if delta else None
    GK = None if gk is None else as_numpy_exact(gk)
    cu = np.asarray(cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
    T, Nqk, Dk = Q.shape
    Nv, Dv = V.shape[1], V.shape[2]
    B = cu.shape[0] - 1
    past = np.zeros((W, B, Nv, Dk, Dv)) if past_window is None else as_numpy_exact(past_window)
    if past.shape != (W, B, Nv, Dk, Dv):
        raise ValueError(f"past window of shape {past.shape}, expected {(W, B, Nv, Dk, Dv)}")
    group = Nv // Nqk
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(Dk)
    out = np.zeros((T, Nv, Dv))
    present = np.zeros_like(past)
    for b in range(B):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        for h in range(Nv):
            hq = h // group
            states = [past[w, b, h].copy() for w in range(W)]  # oldest first
            S = states[-1].copy()
            for t in range(t0, t1):
                kh = K[t, hq] / math.sqrt(float(np.dot(K[t, hq], K[t, hq])) + eps)
                qh = scale * Q[t, hq] / math.sqrt(float(np.dot(Q[t, hq], Q[t, hq])) + eps)
                if decay:
                    S = S * math.exp(G[t, h])
                    if GK is not None:
                        S = S * np.exp(GK[t, h])[:, None]
                if delta:
                    kv_mem = S.T @ kh
                    S = S + np.outer(kh, (V[t, h] - kv_mem) * Bt[t, h])
                else:
                    S = S + np.outer(kh, V[t, h])
                out[t, h] = S.T @ qh
                states.append(S.copy())
                states.pop(0)
            for w in range(W):
                present[w, b, h] = states[w]
    return out, present
