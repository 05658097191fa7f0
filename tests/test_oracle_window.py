"""Pins of the state-window oracle (``oracle.window.recurrent_window``) (CPU only).

The window oracle restates the token loop with the LinearAttention page's
``state_window``: the W most recent states, oldest first, the step continuing
from the newest.  It is checked against two independent statements:

* the C token recurrence (``oracle.recurrent``, pinned in test_oracle_pins.py):
  every window entry is the final state of a prefix run, W = 1 is the plain
  recurrence, an absent past window is the zero initial state;
* the per-token-slot pool oracle (``oracle.pool``, pinned in
  test_oracle_pool.py) for the four update rules and the key gate: a window of
  W entries is a pool whose last W tokens of each sequence write W slots.

Planted mistakes in a copy of the window oracle's source must each fail a pin.
"""
from __future__ import annotations

import importlib.util
import os
import sys

import numpy as np
import pytest

import oracle
from oracle import pool as pool_oracle
from oracle import window as window_oracle

TOL = 1e-12
WINDOW_SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "window.py")


def _problem(seed, lens, W, Nqk=1, Nv=2, Dk=5, Dv=7):
    r = np.random.default_rng(seed)
    T, B = sum(lens), len(lens)
    return dict(q=r.standard_normal((T, Nqk, Dk)), k=r.standard_normal((T, Nqk, Dk)),
                v=r.standard_normal((T, Nv, Dv)), g=-(r.random((T, Nv)) * 0.5 + 0.01),
                beta=r.random((T, Nv)) * 0.9 + 0.05,
                cu_seqlens=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32),
                past_window=r.standard_normal((W, B, Nv, Dk, Dv)) * 0.3, window=W)


def _close(a, b, what):
    a, b = np.asarray(a), np.asarray(b)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= TOL * scale, f"{what}: max abs diff {err:.3e}"


def _prefix(p, b, m, init):
    """C recurrence of the first m tokens of sequence b from state `init` [Nv, Dk, Dv]: (out, final)."""
    t0 = int(p["cu_seqlens"][b])
    sl = lambda x: x[t0:t0 + m]
    o, f = oracle.recurrent(sl(p["q"]), sl(p["k"]), sl(p["v"]), sl(p["g"]), sl(p["beta"]),
                            np.array([0, m], np.int32), state_pool=init[None])
    return o, f[0]


def pin_window_one_is_the_recurrence(fn):
    lens = [4, 1, 3]
    p = _problem(51, lens, 1)
    out, present = fn(**p)
    ref_o, ref_f = oracle.recurrent(p["q"], p["k"], p["v"], p["g"], p["beta"], p["cu_seqlens"],
                                    state_pool=p["past_window"][0])
    _close(out, ref_o, "W = 1: out")
    _close(present[0], ref_f, "W = 1: state")


def pin_window_holds_prefix_states(fn):
    """n >= W: entry w is the state after token n - W + w (0-based), the step starting from entry W - 1."""
    lens, W = [6, 4], 4
    p = _problem(52, lens, W)
    out, present = fn(**p)
    cu = p["cu_seqlens"]
    for b, n in enumerate(lens):
        init = p["past_window"][W - 1, b]
        ref_o, _ = _prefix(p, b, n, init)
        _close(out[cu[b]:cu[b + 1]], ref_o, f"prefix: out of sequence {b}")
        for w in range(W):
            _, f = _prefix(p, b, n - W + 1 + w, init)
            _close(present[w, b], f, f"prefix: entry {w} of sequence {b}")


def pin_short_sequence_shifts_the_window(fn):
    """n < W: the W - n newest past states move n places towards entry 0, then the n new states."""
    lens, W = [2, 1, 3], 5
    p = _problem(53, lens, W)
    out, present = fn(**p)
    for b, n in enumerate(lens):
        past = p["past_window"][:, b]
        for w in range(W - n):
            _close(present[w, b], past[w + n], f"shift: entry {w} of sequence {b}")
        for j in range(n):
            _, f = _prefix(p, b, j + 1, past[W - 1])
            _close(present[W - n + j, b], f, f"shift: new entry {W - n + j} of sequence {b}")


def pin_empty_sequence_keeps_its_window(fn):
    lens, W = [0, 3, 0], 3
    p = _problem(54, lens, W)
    out, present = fn(**p)
    for b in (0, 2):
        _close(present[:, b], p["past_window"][:, b], f"empty sequence {b}")
    assert out.shape == (3, 2, 7)


def pin_absent_past_is_zero(fn):
    lens, W = [3, 1], 2
    p = _problem(55, lens, W)
    p["past_window"] = None
    out, present = fn(**p)
    ref_o, ref_f = oracle.recurrent(p["q"], p["k"], p["v"], p["g"], p["beta"], p["cu_seqlens"])
    _close(out, ref_o, "no past: out")
    _close(present[W - 1], ref_f, "no past: newest entry")
    _, f = _prefix(p, 0, 2, np.zeros((2, 5, 7)))
    _close(present[0, 0], f, "no past: older entry")
    _close(present[0, 1], np.zeros((2, 5, 7)), "no past: zero entry of a 1-token sequence")


def pin_rules_match_the_pool_oracle(fn):
    """Sequences of n >= W tokens: token j writes pool slot (W - n + j) * B + b when j >= n - W, a scratch
    slot otherwise; the pool oracle then starts every sequence from slot (W - 1) * B + b."""
    lens, W = [5, 3, 4], 3
    base = _problem(56, lens, W)
    B, Nv, Dk, Dv = 3, 2, 5, 7
    gk = -(np.random.default_rng(57).random((sum(lens), Nv, Dk)) * 0.3 + 0.01)
    slots = []
    for b, n in enumerate(lens):
        slots += [(W - n + j) * B + b if j >= n - W else W * B + b for j in range(n)]
    pool = np.concatenate([base["past_window"].reshape(W * B, Nv, Dk, Dv), np.zeros((B, Nv, Dk, Dv))])
    for rule in pool_oracle.RULES:
        for key_gate in (None, gk):
            out, present = fn(**base, gk=key_gate, rule=rule)
            ro, rpool = pool_oracle.recurrent_pool(base["q"], base["k"], base["v"], base["g"], base["beta"],
                                                   base["cu_seqlens"], pool, np.array(slots, np.int32),
                                                   gk=key_gate, rule=rule)
            what = f"rule {rule}{' with gk' if key_gate is not None else ''}"
            _close(out, ro, f"{what}: out")
            _close(present, rpool[:W * B].reshape(W, B, Nv, Dk, Dv), f"{what}: window")


PINS = [pin_window_one_is_the_recurrence, pin_window_holds_prefix_states, pin_short_sequence_shifts_the_window,
        pin_empty_sequence_keeps_its_window, pin_absent_past_is_zero, pin_rules_match_the_pool_oracle]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_window_oracle_pin(pin):
    pin(window_oracle.recurrent_window)


def test_window_bounds():
    p = _problem(58, [2], 1)
    for W in (0, 9):
        p.update(window=W, past_window=None)
        with pytest.raises(ValueError):
            window_oracle.recurrent_window(**p)


MUTANTS = [
    ("newest_first", "present[w, b, h] = states[w]", "present[w, b, h] = states[W - 1 - w]"),
    ("start_from_oldest", "S = states[-1].copy()", "S = states[0].copy()"),
    ("drops_the_previous_state", "states.pop(0)", "states.pop(-2)"),
    ("window_left_as_past", "present[w, b, h] = states[w]", "present[w, b, h] = past[w, b, h]"),
    ("output_from_state_before_token", "out[t, h] = S.T @ qh", "out[t, h] = states[-1].T @ qh"),
    ("no_decay", "S = S * math.exp(G[t, h])", "S = S"),
    ("key_gate_on_columns", "S = S * np.exp(GK[t, h])[:, None]", "S = S * np.exp(GK[t, h])[:S.shape[1]][None, :]"),
    ("gated_rule_retrieves", 'rule in ("gated_delta", "delta")\n', 'rule in ("gated_delta", "delta", "gated")\n'),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_window_mistake_is_caught(name, old, new):
    src = open(WINDOW_SRC).read()
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader(f"oracle._window_mutant_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__dict__["__package__"] = "oracle"
    sys.modules[spec.name] = mod
    try:
        exec(compile(src.replace(old, new), WINDOW_SRC, "exec"), mod.__dict__)
        caught = 0
        for pin in PINS:
            try:
                pin(mod.recurrent_window)
            except Exception:  # a wrong value or a shape the mistake cannot handle
                caught += 1
        assert caught >= 1, f"no pin fails for the planted mistake {name}"
    finally:
        del sys.modules[spec.name]
