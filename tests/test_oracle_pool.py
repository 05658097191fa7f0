"""Pins of the per-token-slot pool oracle (``oracle.pool.recurrent_pool``) to the
independent C token recurrence (CPU only).

The pool oracle restates the decode page's token loop in numpy with the slot
semantics of "lite_boost.ops.recurrent_gated_delta_rule" (``ssm_state_indices``
per token, ``num_accepted_tokens``, the updated pool ``state_out``).  It is
checked against ``oracle.recurrent`` (C, pinned in test_oracle_pins.py) on the
three cases that fix the semantics:

* one slot per sequence, every token accepted: the plain recurrence with the
  final state written back into that slot, every other slot untouched;
* a distinct slot per token: slot j holds the recurrence's state after token j
  (a prefix run of the C oracle);
* ``num_accepted = a``: the sequence starts from the slot of its token a - 1.

Planted mistakes in a copy of the pool oracle's source must each fail a pin.
"""
from __future__ import annotations

import importlib.util
import os
import sys

import numpy as np
import pytest

import oracle
from oracle import pool as pool_oracle

TOL = 1e-12
POOL_SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "pool.py")


def _problem(seed, lens, Nqk=1, Nv=2, D=6, P=12):
    r = np.random.default_rng(seed)
    T = sum(lens)
    return dict(q=r.standard_normal((T, Nqk, D)), k=r.standard_normal((T, Nqk, D)),
                v=r.standard_normal((T, Nv, D)), g=-(r.random((T, Nv)) * 0.5 + 0.01),
                beta=r.random((T, Nv)) * 0.9 + 0.05,
                cu_seqlens=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32),
                state_pool=r.standard_normal((P, Nv, D, D)) * 0.3)


def _close(a, b, what):
    a, b = np.asarray(a), np.asarray(b)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= TOL * scale, f"{what}: max abs diff {err:.3e}"


def _plain(p, lo, hi, init):
    """C recurrence of tokens [lo, hi) of the problem as one sequence from state `init` [Nv, D, D]."""
    sl = lambda x: x[lo:hi]
    return oracle.recurrent(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["g"]), sl(p["beta"]),
                            np.array([0, hi - lo], np.int32), state_pool=init[None])


def pin_one_slot_per_sequence(fn):
    lens = [3, 1, 5, 0, 2]
    p = _problem(31, lens)
    seq_slot = [7, 2, 10, 4, 0]
    slots = np.concatenate([[s] * n for s, n in zip(seq_slot, lens)]).astype(np.int32)
    out, pool = fn(**p, token_slots=slots)
    ref_o, ref_f = oracle.recurrent(p["q"], p["k"], p["v"], p["g"], p["beta"], p["cu_seqlens"],
                                    state_pool=p["state_pool"], state_indices=np.array(seq_slot, np.int32))
    _close(out, ref_o, "one slot: out")
    for b, (s, n) in enumerate(zip(seq_slot, lens)):
        _close(pool[s], ref_f[b] if n else p["state_pool"][s], f"one slot: slot {s}")
    untouched = [s for s in range(p["state_pool"].shape[0]) if s not in seq_slot]
    _close(pool[untouched], p["state_pool"][untouched], "one slot: other slots")


def pin_slot_per_token(fn):
    lens = [4, 3]
    p = _problem(32, lens)
    slots = np.array([5, 9, 1, 3, 11, 6, 2], np.int32)
    out, pool = fn(**p, token_slots=slots, num_accepted=np.array([2, 3], np.int32))
    cu = p["cu_seqlens"]
    for b in range(2):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        init = p["state_pool"][slots[t0 + (2 if b == 0 else 3) - 1]]
        ref_o, _ = _plain(p, t0, t1, init)
        _close(out[t0:t1], ref_o, f"per token: out of sequence {b}")
        for j in range(t1 - t0):
            _, f = _plain(p, t0, t0 + j + 1, init)
            _close(pool[slots[t0 + j]], f[0], f"per token: slot of token {t0 + j}")


def pin_accepted_selects_start(fn):
    lens = [5]
    p = _problem(33, lens, Nv=1)
    slots = np.array([0, 1, 2, 3, 4], np.int32)
    for a in (1, 3, 5):
        out, _ = fn(**p, token_slots=slots, num_accepted=np.array([a], np.int32))
        ref_o, _ = _plain(p, 0, 5, p["state_pool"][a - 1])
        _close(out, ref_o, f"accepted {a}: out")
    # the start must matter
    o1, _ = fn(**p, token_slots=slots, num_accepted=np.array([1], np.int32))
    o5, _ = fn(**p, token_slots=slots, num_accepted=np.array([5], np.int32))
    assert np.max(np.abs(o1 - o5)) > 1e-6


def pin_key_gate_zero(fn):
    """gk = 0 is the recurrence without a key gate."""
    lens = [3, 4]
    p = _problem(34, lens)
    slots = np.array([0, 0, 0, 5, 5, 5, 5], np.int32)
    o1, p1 = fn(**p, token_slots=slots)
    o2, p2 = fn(**p, token_slots=slots, gk=np.zeros(p["k"].shape[:1] + (2, 6)))
    _close(o2, o1, "gk = 0: out")
    _close(p2, p1, "gk = 0: pool")


def pin_key_gate_constant(fn):
    """A gk equal to c in every key dimension is the recurrence with g + c (C oracle)."""
    lens = [5]
    p = _problem(35, lens)
    slots = np.zeros(5, np.int32)
    c = -0.3
    out, pool = fn(**p, token_slots=slots, gk=np.full((5, 2, 6), c))
    shifted = dict(p)
    shifted["g"] = p["g"] + c
    ref_o, ref_f = _plain(shifted, 0, 5, p["state_pool"][0])
    _close(out, ref_o, "gk = c: out")
    _close(pool[0], ref_f[0], "gk = c: state")


def pin_key_gate_rows_closed_form(fn):
    """beta = 0: S_t = diag(exp(sum (g + gk))) S_0 row by row, o_t = S_t^T qh (Dk = 3, Dv = 5)."""
    r = np.random.default_rng(36)
    T, Dk, Dv = 4, 3, 5
    q, k = r.standard_normal((T, 1, Dk)), r.standard_normal((T, 1, Dk))
    v = r.standard_normal((T, 1, Dv))
    g = -(r.random((T, 1)) * 0.5 + 0.01)
    gk = -(r.random((T, 1, Dk)) * 0.7 + 0.01)
    S0 = r.standard_normal((1, 1, Dk, Dv))
    out, pool = fn(q, k, v, g, np.zeros((T, 1)), np.array([0, T], np.int32), S0, np.zeros(T, np.int32), gk=gk)
    scale = 1.0 / np.sqrt(Dk)
    for t in range(T):
        rows = np.exp(np.cumsum(g[:t + 1, 0])[-1] + np.cumsum(gk[:t + 1, 0], axis=0)[-1])
        St = rows[:, None] * S0[0, 0]
        qh = scale * q[t, 0] / np.sqrt(np.dot(q[t, 0], q[t, 0]) + 1e-6)
        _close(out[t, 0], St.T @ qh, f"closed form: out {t}")
    _close(pool[0, 0], St, "closed form: state")


def _sum_closed_form(p, T, decay):
    """The gated / linear rules summed out: S_t = D_t S_0 + sum_{j <= t} D_t D_j^-1 kh_j v_j^T, with
    D_t = diag(exp(sum_{i <= t} (g_i + gk_i))) (identity for the linear rule); o_t = S_t^T qh_t."""
    q, k, v, g, gk = p["q"][:, 0], p["k"][:, 0], p["v"][:, 0], p["g"][:, 0], p["gk"][:, 0]
    S0 = p["state_pool"][0, 0]
    cum = np.cumsum(g[:, None] + gk, axis=0) if decay else np.zeros_like(gk)
    kh = k / np.sqrt(np.sum(k * k, axis=1, keepdims=True) + 1e-6)
    qh = (q / np.sqrt(np.sum(q * q, axis=1, keepdims=True) + 1e-6)) / np.sqrt(q.shape[1])
    outs, S = [], None
    for t in range(T):
        S = np.exp(cum[t])[:, None] * S0
        for j in range(t + 1):
            S = S + np.exp(cum[t] - cum[j])[:, None] * np.outer(kh[j], v[j])
        outs.append(S.T @ qh[t])
    return np.array(outs), S


def _rule_problem(seed):
    r = np.random.default_rng(seed)
    T, Dk, Dv = 5, 3, 4
    return dict(q=r.standard_normal((T, 1, Dk)), k=r.standard_normal((T, 1, Dk)), v=r.standard_normal((T, 1, Dv)),
                g=-(r.random((T, 1)) * 0.5 + 0.01), beta=r.random((T, 1)) * 0.9 + 0.05,
                cu_seqlens=np.array([0, T], np.int32), state_pool=r.standard_normal((1, 1, Dk, Dv)),
                gk=-(r.random((T, 1, Dk)) * 0.4 + 0.01))


def pin_rule_gated_closed_form(fn):
    p = _rule_problem(37)
    out, pool = fn(**p, token_slots=np.zeros(5, np.int32), rule="gated")
    ro, rs = _sum_closed_form(p, 5, decay=True)
    _close(out[:, 0], ro, "gated: out")
    _close(pool[0, 0], rs, "gated: state")


def pin_rule_linear_closed_form(fn):
    p = _rule_problem(38)
    out, pool = fn(**p, token_slots=np.zeros(5, np.int32), rule="linear")
    ro, rs = _sum_closed_form(p, 5, decay=False)
    _close(out[:, 0], ro, "linear: out")
    _close(pool[0, 0], rs, "linear: state")


def pin_rule_delta_is_zero_gate(fn):
    """The delta rule is the C recurrence with g = 0 (the gates given are not used)."""
    p = _problem(39, [6])
    slots = np.zeros(6, np.int32)
    out, pool = fn(**p, token_slots=slots, gk=np.full((6, 2, 6), -0.7), rule="delta")
    zero = dict(p)
    zero["g"] = np.zeros_like(p["g"])
    ro, rf = _plain(zero, 0, 6, p["state_pool"][0])
    _close(out, ro, "delta: out")
    _close(pool[0], rf[0], "delta: state")


PINS = [pin_one_slot_per_sequence, pin_slot_per_token, pin_accepted_selects_start, pin_key_gate_zero,
        pin_key_gate_constant, pin_key_gate_rows_closed_form, pin_rule_gated_closed_form,
        pin_rule_linear_closed_form, pin_rule_delta_is_zero_gate]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pool_oracle_pin(pin):
    pin(pool_oracle.recurrent_pool)


MUTANTS = [
    ("start_from_first_token_slot", "starts.append(pool[slots[t0 + a - 1]].copy())",
     "starts.append(pool[slots[t0]].copy())"),
    ("start_from_last_token_slot", "starts.append(pool[slots[t0 + a - 1]].copy())",
     "starts.append(pool[slots[t1 - 1]].copy())"),
    ("write_to_sequence_start_slot", "pool_out[slots[t], h] = S", "pool_out[slots[t0], h] = S"),
    ("no_decay", "S = S * math.exp(G[t, h])", "S = S"),
    ("write_before_update", "                pool_out[slots[t], h] = S\n",
     "                pool_out[slots[t], h] = starts[b][h]\n"),
    ("key_gate_on_columns", "S = S * np.exp(GK[t, h])[:, None]", "S = S * np.exp(GK[t, h])[:S.shape[1]][None, :]"),
    ("key_gate_sign", "S = S * np.exp(GK[t, h])[:, None]", "S = S * np.exp(-GK[t, h])[:, None]"),
    ("key_gate_ignored", "S = S * np.exp(GK[t, h])[:, None]", "S = S"),
    ("gated_rule_without_decay", 'decay, delta = rule in ("gated_delta", "gated")', 'decay, delta = rule in ("gated_delta",)'),
    ("delta_rule_with_decay", 'decay, delta = rule in ("gated_delta", "gated")', 'decay, delta = rule in ("gated_delta", "gated", "delta")'),
    ("linear_rule_uses_beta", "S = S + np.outer(kh, V[t, h])", "S = S + np.outer(kh, V[t, h] * 0.5)"),
    ("rules_without_retrieval_retrieve", 'rule in ("gated_delta", "delta")\n', 'rule in ("gated_delta", "delta", "gated")\n'),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_pool_mistake_is_caught(name, old, new):
    src = open(POOL_SRC).read()
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader(f"oracle._pool_mutant_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__dict__["__package__"] = "oracle"
    sys.modules[spec.name] = mod
    try:
        exec(compile(src.replace(old, new), POOL_SRC, "exec"), mod.__dict__)
        caught = 0
        for pin in PINS:
            try:
                pin(mod.recurrent_pool)
            except Exception:  # a wrong value or a shape the mistake cannot handle
                caught += 1
        assert caught >= 1, f"no pin fails for the planted mistake {name}"
    finally:
        del sys.modules[spec.name]


def test_fp16_inputs_widen_exactly():
    """fp16 activations and states enter the oracle exactly: the smallest subnormal, the smallest normal,
    the largest finite value and a rounded decimal keep their exact binary values."""
    import torch
    x = torch.tensor([2.0 ** -24, -(2.0 ** -14), 65504.0, 0.1], dtype=torch.float16)
    got = oracle.as_numpy_exact(x)
    assert got.dtype == np.float64
    assert list(got) == [2.0 ** -24, -(2.0 ** -14), 65504.0, 1638.0 / 16384.0]  # 0.1 rounds to 1638 * 2^-14
