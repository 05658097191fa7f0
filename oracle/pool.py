"""fp64 oracle of the token recurrence on a state pool with one slot index per token.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing on the CUDA path
imports it.

Page "lite_boost.ops.recurrent_gated_delta_rule" (parameters ``state``,
``ssm_state_indices``, ``num_accepted_tokens``; return value ``state_out``):
every token selects a slot of the state pool through its own index, the
updated pool is returned, and ``num_accepted_tokens`` marks how many tokens of
a speculative step were accepted (equal to the sequence length in ordinary
decoding).  The page leaves open which slot a sequence starts from; the reading
taken here is the one under which speculative decoding works: the slots of a
sequence's tokens hold the states after those tokens, so the state to continue
from is the one after the last accepted token,

    S_0 = pool[slots[t0 + a - 1]],   a = num_accepted[b] (or the sequence length),

and after each token j of the sequence the state is written to pool[slots[t0 + j]]
(later writes to a slot supersede earlier ones).  Every initial state is read
before any write of the call.  Per token, in the page's order:

    S = S * exp(g) * exp(gk);  kv_mem = S^T k;  S = S + k ((v - kv_mem) * beta)^T;  o = S^T q

with q and k normalised as in "Qwen3Next Samples", equation "L2 Normalization"
(eps inside the square root) and q scaled after the normalisation.  gk, when
given, is the page's key-dimension gate: exp(gk) decays each key row of S (S is
[Dk, Dv]) by its own factor; without gk that factor is 1.  Plain numpy, per
token, for the small shapes of the tests.

``rule`` selects one of the four update rules of the page "com.microsoft.
LinearAttention" (attribute update_rule): ``gated_delta`` (the rule above),
``delta`` (no decay: the gates are not used), ``gated`` (S = S exp(g) exp(gk)
+ k v^T: no retrieval, beta not used) and ``linear`` (S = S + k v^T).  q and k
are normalised in every rule, as this operator defines them.
"""
from __future__ import annotations

import math

import numpy as np

from . import as_numpy_exact


def _ints(x) -> np.ndarray:
    if hasattr(x, "cpu"):
        x = x.cpu().numpy()
    return np.asarray(x, dtype=np.int64)


RULES = ("gated_delta", "delta", "gated", "linear")


def recurrent_pool(q, k, v, g, beta, cu_seqlens, state_pool, token_slots, num_accepted=None, scale=None,
                   eps=1e-6, gk=None, rule="gated_delta"):
    """Token recurrence with per-token pool slots, in fp64.

    Shapes: q, k [T, Nqk, Dk]; v [T, Nv, Dv]; g, beta [T, Nv]; cu_seqlens [B+1];
    state_pool [P, Nv, Dk, Dv]; token_slots [T]; num_accepted [B] or None;
    gk [T, Nv, Dk] or None.
    Returns (out [T, Nv, Dv], pool_out [P, Nv, Dk, Dv]) as float64; pool_out is a
    copy of state_pool with the written slots replaced.
    """
    if rule not in RULES:
        raise ValueError(f"unknown update rule {rule}")
    decay, delta = rule in ("gated_delta", "gated"), rule in ("gated_delta", "delta")
    Q, K, V = as_numpy_exact(q), as_numpy_exact(k), as_numpy_exact(v)
    G = as_numpy_exact(g) if decay else None
    Bt = as_numpy_exact(beta) if delta else None
    GK = None if gk is None else as_numpy_exact(gk)
    pool = as_numpy_exact(state_pool)
    cu, slots = _ints(cu_seqlens), _ints(token_slots)
    acc = None if num_accepted is None else _ints(num_accepted)
    T, Nqk, Dk = Q.shape
    Nv, Dv = V.shape[1], V.shape[2]
    group = Nv // Nqk
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(Dk)
    out = np.zeros((T, Nv, Dv))
    pool_out = pool.copy()
    B = cu.shape[0] - 1
    starts = []
    for b in range(B):  # every initial state comes from the pool as it was before the call
        t0, t1 = int(cu[b]), int(cu[b + 1])
        n = t1 - t0
        if n == 0:
            starts.append(None)
            continue
        a = n if acc is None else int(acc[b])
        if not 1 <= a <= n:
            raise ValueError(f"num_accepted[{b}] = {a} outside 1..{n}")
        starts.append(pool[slots[t0 + a - 1]].copy())
    for b in range(B):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        if starts[b] is None:
            continue
        for h in range(Nv):
            hq = h // group
            S = starts[b][h].copy()  # [Dk, Dv]
            for t in range(t0, t1):
                kh = K[t, hq] / math.sqrt(float(np.dot(K[t, hq], K[t, hq])) + eps)
                qh = scale * Q[t, hq] / math.sqrt(float(np.dot(Q[t, hq], Q[t, hq])) + eps)
                if decay:
                    S = S * math.exp(G[t, h])
                    if GK is not None:
                        S = S * np.exp(GK[t, h])[:, None]  # row i of S (key dimension i)
                if delta:
                    kv_mem = S.T @ kh
                    S = S + np.outer(kh, (V[t, h] - kv_mem) * Bt[t, h])
                else:
                    S = S + np.outer(kh, V[t, h])
                out[t, h] = S.T @ qh
                pool_out[slots[t], h] = S
    return out, pool_out
