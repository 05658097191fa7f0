"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each ``pin_*`` takes a recurrence callable with the signature of
``oracle.recurrent`` and raises AssertionError when it disagrees with a value
fixed by the pages or by the mathematics: a hand-worked example, closed forms
of special cases, an independent brute-force evaluation, and structural
invariants (head grouping, packing, slot selection, split-and-resume).  The
pins run against the oracle (all must hold) and against copies of the oracle
source with one planted mistake each (at least one pin must fail for every
mistake), which shows that the pin set can see the mistakes that matter.
"""
from __future__ import annotations

import functools
import math
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _random_problem(seed, lens, Nqk=1, Nv=1, D=6, with_pool=False, P=None):
    r = _rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = r.standard_normal((T, Nqk, D))
    k = r.standard_normal((T, Nqk, D))
    v = r.standard_normal((T, Nv, D))
    g = -(r.random((T, Nv)) * 0.5 + 0.01)
    beta = r.random((T, Nv)) * 0.9 + 0.05
    pool = idx = None
    if with_pool:
        P = P or len(lens)
        pool = r.standard_normal((P, Nv, D, D)) * 0.3
        idx = r.permutation(P)[:len(lens)].astype(np.int32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=cu, state_pool=pool, state_indices=idx)


def _close(a, b, tol=TOL, what=""):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs diff {err:.3e} (scale {scale:.3e})"


# ----------------------------------------------------------------------------- pins

def pin_golden(rec):
    """Hand-worked three-token example (tests/golden/hand_d2_three_tokens.txt)."""
    rows = {}
    with open(os.path.join(HERE, "golden", "hand_d2_three_tokens.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            key, val = line.split(":", 1)
            rows[key.strip()] = [[float(x) for x in part.split()] for part in val.split(";")]
    k = np.array(rows["k"])[:, None, :]
    q = np.array(rows["q"])[:, None, :]
    v = np.array(rows["v"])[:, None, :]
    beta = np.array(rows["beta"]).reshape(3, 1)
    g = np.full((3, 1), math.log(0.5))
    out, fin = rec(q, k, v, g, beta, np.array([0, 3], np.int32), scale=1.0, eps=0.0)
    _close(out[:, 0, :], np.array(rows["out"]), 1e-14, "golden out")
    _close(fin[0, 0], np.array(rows["final_state"]), 1e-14, "golden final state")


def pin_beta_zero_zero_state(rec):
    """beta = 0 with no initial state: nothing is ever written, output and state are exactly 0."""
    p = _random_problem(1, [5, 9], Nqk=2, Nv=4)
    p["beta"][:] = 0.0
    out, fin = rec(**p)
    assert np.all(out == 0.0) and np.all(fin == 0.0)


def pin_beta_zero_closed_form(rec):
    """beta = 0: S_t = exp(sum of gates so far) S0, o_t = S_t^T qh_t (pure decay)."""
    p = _random_problem(2, [4, 7], Nqk=1, Nv=2, with_pool=True, P=5)
    p["beta"][:] = 0.0
    p["q"] = _unit_rows(p["q"])
    scale = 0.7
    out, fin = rec(**p, scale=scale, eps=0.0)
    cu = p["cu_seqlens"]
    for b in range(2):
        for h in range(2):
            S0 = p["state_pool"][p["state_indices"][b], h]
            acc = 0.0
            for t in range(cu[b], cu[b + 1]):
                acc += p["g"][t, h]
                _close(out[t, h], math.exp(acc) * S0.T @ (scale * p["q"][t, 0]), 1e-12, "decay-only o")
            _close(fin[b, h], math.exp(acc) * S0, 1e-12, "decay-only state")


def pin_orthonormal_retrieval(rec):
    """g = 0, beta = 1, orthonormal keys: each write sees kv = 0, queries return stored values."""
    r = _rng(3)
    D, n = 16, 12
    Qm, _ = np.linalg.qr(r.standard_normal((D, D)))
    keys = Qm.T[:n]                              # orthonormal rows
    vals = r.standard_normal((n, D))
    sigma = [int(r.integers(0, t + 1)) for t in range(n)]   # query a key already written
    q = keys[sigma][:, None, :]
    k = keys[:, None, :]
    v = vals[:, None, :]
    out, fin = rec(q, k, v, np.zeros((n, 1)), np.ones((n, 1)), np.array([0, n], np.int32),
                   scale=1.0, eps=0.0)
    for t in range(n):
        _close(out[t, 0], vals[sigma[t]], 1e-12, "retrieval o")
    for j in range(n):
        _close(fin[0, 0].T @ keys[j], vals[j], 1e-12, "retrieval state")


def pin_delta_overwrite(rec):
    """beta = 1, g = 0: writing (k, v1) then (k, v2) leaves S^T kh = v2, whatever S0 was."""
    r = _rng(4)
    D = 8
    kk = r.standard_normal(D)
    kh = kk / np.linalg.norm(kk)
    v1, v2 = r.standard_normal(D), r.standard_normal(D)
    q = np.stack([kk, kk])[:, None, :]
    k = np.stack([kk, 2.5 * kk])[:, None, :]
    v = np.stack([v1, v2])[:, None, :]
    pool = r.standard_normal((1, 1, D, D))
    out, fin = rec(q, k, v, np.zeros((2, 1)), np.ones((2, 1)), np.array([0, 2], np.int32),
                   state_pool=pool, scale=1.0, eps=0.0)
    _close(fin[0, 0].T @ kh, v2, 1e-12, "overwrite state")
    _close(out[1, 0], v2, 1e-12, "overwrite o")
    _close(out[0, 0], v1, 1e-12, "first write o")


def pin_single_token(rec):
    """One token: S1 = e^g S0 + beta kh (v - e^g S0^T kh)^T and o = S1^T qh."""
    r = _rng(5)
    D = 6
    kh = _unit_rows(r.standard_normal(D))
    qh = _unit_rows(r.standard_normal(D))
    v = r.standard_normal(D)
    S0 = r.standard_normal((D, D))
    g, b, scale = -0.37, 0.61, 1.3
    S1 = math.exp(g) * S0 + b * np.outer(kh, v - math.exp(g) * S0.T @ kh)
    out, fin = rec(qh[None, None], kh[None, None], v[None, None], np.array([[g]]), np.array([[b]]),
                   np.array([0, 1], np.int32), state_pool=S0[None, None], scale=scale, eps=0.0)
    _close(fin[0, 0], S1, 1e-13, "single-token state")
    _close(out[0, 0], S1.T @ (scale * qh), 1e-13, "single-token o")


def pin_eps_inside_sqrt(rec):
    """eps sits inside the square root: a key with |k|^2 = 3 eps normalises to length sqrt(3)/2."""
    D, eps = 4, 1e-4
    k = np.zeros((1, 1, D))
    k[0, 0, 0] = math.sqrt(3 * eps)
    q = np.zeros((1, 1, D))
    q[0, 0, 0] = 1e4                                 # |q|^2 >> eps: qh = e1 to ~1e-16
    v = np.array([[[1.0, -2.0, 0.5, 3.0]]])
    out, fin = rec(q, k, v, np.zeros((1, 1)), np.ones((1, 1)), np.array([0, 1], np.int32),
                   scale=1.0, eps=eps)
    c = math.sqrt(3.0) / 2.0
    _close(fin[0, 0, 0], c * v[0, 0], 1e-12, "eps state")
    _close(out[0, 0], c * v[0, 0], 1e-12, "eps o")


def pin_gqa_grouping(rec):
    """v-head h reads qk-head h // (Nv/Nqk): each v-head equals a one-head run on its group's q, k."""
    p = _random_problem(6, [6, 3], Nqk=2, Nv=4)
    out, fin = rec(**p)
    for h in range(4):
        hq = h // 2
        o1, f1 = rec(p["q"][:, hq:hq + 1], p["k"][:, hq:hq + 1], p["v"][:, h:h + 1],
                     p["g"][:, h:h + 1], p["beta"][:, h:h + 1], p["cu_seqlens"])
        _close(out[:, h], o1[:, 0], 1e-14, "gqa o")
        _close(fin[:, h], f1[:, 0], 1e-14, "gqa state")


def pin_packing(rec):
    """A packed batch equals each sequence run on its own (sequences never interact)."""
    p = _random_problem(7, [5, 1, 8], Nqk=1, Nv=2, with_pool=True, P=6)
    out, fin = rec(**p)
    cu = p["cu_seqlens"]
    for b in range(3):
        s, e = cu[b], cu[b + 1]
        ob, fb = rec(p["q"][s:e], p["k"][s:e], p["v"][s:e], p["g"][s:e], p["beta"][s:e],
                     np.array([0, e - s], np.int32),
                     state_pool=p["state_pool"][p["state_indices"][b]][None])
        _close(out[s:e], ob, 1e-14, "packed o")
        _close(fin[b], fb[0], 1e-14, "packed state")


def pin_slots(rec):
    """Sequence b starts from pool[state_indices[b]], or pool[b] without indices."""
    p = _random_problem(8, [3, 4], Nqk=1, Nv=1, with_pool=True, P=4)
    p["state_indices"] = np.array([3, 1], np.int32)
    out, fin = rec(**p)
    swapped = dict(p)
    swapped["state_pool"] = p["state_pool"][[3, 1]]
    swapped["state_indices"] = None
    o2, f2 = rec(**swapped)
    _close(out, o2, 1e-14, "slot o")
    _close(fin, f2, 1e-14, "slot state")
    # a different slot must change the answer
    p["state_indices"] = np.array([0, 1], np.int32)
    o3, _ = rec(**p)
    assert np.max(np.abs(o3 - out)) > 1e-6


def pin_split_resume(rec):
    """Running [0, a) then [a, n) from the carried state equals one run over [0, n)."""
    p = _random_problem(9, [11], Nqk=1, Nv=2)
    out, fin = rec(**p)
    a = 4
    cut = lambda x, s, e: x[s:e]
    o1, f1 = rec(*(cut(p[n], 0, a) for n in ("q", "k", "v", "g", "beta")), np.array([0, a], np.int32))
    o2, f2 = rec(*(cut(p[n], a, 11) for n in ("q", "k", "v", "g", "beta")),
                 np.array([0, 11 - a], np.int32), state_pool=f1)
    _close(np.concatenate([o1, o2]), out, 1e-13, "split o")
    _close(f2, fin, 1e-13, "split state")


def pin_transition_bruteforce(rec):
    """Brute force with explicit Dk x Dk transition matrices on tiny shapes."""
    for seed, D in ((10, 2), (11, 3), (12, 4)):
        p = _random_problem(seed, [7, 13], Nqk=1, Nv=2, D=D, with_pool=True, P=3)
        out, fin = rec(**p, scale=0.9, eps=1e-3)
        o2, f2 = oracle.transition(**p, scale=0.9, eps=1e-3)
        _close(out, o2, 1e-12, f"transition o D={D}")
        _close(fin, f2, 1e-12, f"transition state D={D}")


PINS = [pin_golden, pin_beta_zero_zero_state, pin_beta_zero_closed_form, pin_orthonormal_retrieval,
        pin_delta_overwrite, pin_single_token, pin_eps_inside_sqrt, pin_gqa_grouping, pin_packing,
        pin_slots, pin_split_resume, pin_transition_bruteforce]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.recurrent)


# --------------------------------------------------------------- planted mistakes

# (name, original text, replacement) applied once to a copy of the oracle source
MUTANTS = [
    ("decay_sign", "exp(ld(J->g, J->dt_g, gh))", "exp(-ld(J->g, J->dt_g, gh))"),
    ("no_decay", "S[i] = decay * S[i];", "S[i] = S[i];"),
    ("eps_outside_sqrt", "sqrt(ssk + J->eps)", "(sqrt(ssk) + J->eps)"),
    ("beta_misplaced", "u[j] = bt * (ld(J->v, J->dt_v, v_base + j) - kv[j]);",
     "u[j] = ld(J->v, J->dt_v, v_base + j) - bt * kv[j];"),
    ("retrieval_transposed", "acc += S[(int64_t)d * Dv + j] * kh[d];",
     "acc += S[(int64_t)j * Dv + d] * kh[d];"),
    ("output_reads_key", "acc += S[(int64_t)d * Dv + j] * qh[d];", "acc += S[(int64_t)d * Dv + j] * kh[d];"),
    ("gqa_modulo", "const int32_t hq = h / G;", "const int32_t hq = h % J->Nqk;"),
    ("no_scale", "qh[d] = J->scale * (", "qh[d] = ("),
    ("q_not_normalised", "qh[d] = J->scale * (ld(J->q, J->dt_q, qk_base + d) / qden);",
     "qh[d] = J->scale * ld(J->q, J->dt_q, qk_base + d);"),
    ("slot_ignored", "J->state_indices ? J->state_indices[b] : b", "b"),
    ("update_sign", "+= kh[d] * u[j];", "-= kh[d] * u[j];"),
    ("no_retrieval", "kv[j] = acc;", "kv[j] = 0.0 * acc;"),
]


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="gdn_oracle_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(mutant_dir, name, old, new):
    src = open(oracle_build.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = os.path.join(mutant_dir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.load(oracle_build.build(src=path, out=os.path.join(mutant_dir, f"{name}.so"), force=True))
    rec = functools.partial(oracle.recurrent, lib=lib)
    caught = []
    for pin in PINS:
        try:
            pin(rec)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"


# ------------------------------------------------------------ chunked form pins

@pytest.mark.parametrize("C", [1, 2, 7, 16, 64, 128])
def test_chunked_equals_recurrence(C):
    """Chunk size does not change the result; C = 1 is the recurrence itself."""
    p = _random_problem(20, [150, 1, 129, 40], Nqk=2, Nv=4, D=8, with_pool=True, P=6)
    o1, f1 = oracle.recurrent(**p, scale=0.5, eps=1e-6)
    o2, f2 = oracle.chunked(**p, scale=0.5, eps=1e-6, C=C)
    _close(o2, o1, 1e-10, f"chunked o C={C}")
    _close(f2, f1, 1e-10, f"chunked state C={C}")


def test_chunk_inverse_is_inverse():
    """(I - A) (I - A)^-1 = I for the chunk matrix, and the block merge equals forward substitution."""
    p = _random_problem(21, [128], Nqk=1, Nv=1, D=16)
    _, _, kept = oracle.chunked(**p, C=128, keep=True)
    r = kept[(0, 0, 0)]
    A, Ainv = r["A"], r["A_inv"]
    assert np.allclose(np.triu(A), 0.0)             # strictly lower triangular
    assert np.max(np.abs((np.eye(128) - A) @ Ainv - np.eye(128))) < 1e-12
    for base in (8, 16, 32):
        assert np.max(np.abs(oracle.inverse_by_block_merge(A, base) - Ainv)) < 1e-12


def test_chunk_intermediates_identities():
    """U' = v_out - W S, o restricted to the chunk, and the state update close the chunk exactly."""
    p = _random_problem(22, [100], Nqk=1, Nv=1, D=8, with_pool=True, P=1)
    _, _, kept = oracle.chunked(**p, C=32, keep=True)
    o_rec, _ = oracle.recurrent(**p)
    for (b, h, c), r in kept.items():
        _close(r["v_new"], r["v_out"] - r["k_cumdecay"] @ r["S_in"], 1e-12, "v_new")
        n = r["o"].shape[0]
        _close(r["o"], o_rec[c * 32:c * 32 + n, 0], 1e-10, "chunk o")


def test_state_update_split_into_state_free_parts():
    """The state update regrouped as e^{g_last} S + N - Mk S, with N = k_gexp^T v_out and
    Mk = k_gexp^T k_cumdecay (the form the GPU state pass iterates), closes each chunk
    exactly as the page's update does, partial last chunk included."""
    p = _random_problem(23, [75, 32], Nqk=1, Nv=2, D=8, with_pool=True, P=2)
    _, _, kept = oracle.chunked(**p, C=32, keep=True)
    assert any(r["o"].shape[0] < 32 for r in kept.values())
    for r in kept.values():
        k_gexp = r["kn"] * np.exp(r["g_cum"][-1] - r["g_cum"])[:, None]
        N = k_gexp.T @ r["v_out"]
        Mk = k_gexp.T @ r["k_cumdecay"]
        S = r["S_in"]
        _close(np.exp(r["g_cum"][-1]) * S + N - Mk @ S, r["S_new"], 1e-12, "regrouped state update")


def _unequal_problem(seed, lens, Dk, Dv, Nqk=1, Nv=2, P=3):
    r = _rng(seed)
    T = sum(lens)
    return dict(q=r.standard_normal((T, Nqk, Dk)), k=r.standard_normal((T, Nqk, Dk)),
                v=r.standard_normal((T, Nv, Dv)), g=-(r.random((T, Nv)) * 0.5 + 0.01),
                beta=r.random((T, Nv)) * 0.9 + 0.05,
                cu_seqlens=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32),
                state_pool=r.standard_normal((P, Nv, Dk, Dv)) * 0.3,
                state_indices=r.permutation(P)[:len(lens)].astype(np.int32))


@pytest.mark.parametrize("Dk,Dv", [(3, 5), (6, 2), (4, 16)])
def test_unequal_head_dims_three_forms_agree(Dk, Dv):
    """Dk != Dv (the decode page's example shape has Dk = 64, Dv = 512): the C recurrence, the chunked
    form at several chunk sizes and the dense transition matrices give one result, the state kept as
    [Dk, Dv] (a transposed state or a swapped head dimension cannot pass with Dk != Dv)."""
    p = _unequal_problem(24, [9, 1, 20], Dk, Dv)
    o1, f1 = oracle.recurrent(**p, scale=0.7, eps=1e-4)
    assert o1.shape == (30, 2, Dv) and f1.shape == (3, 2, Dk, Dv)
    o2, f2 = oracle.transition(**p, scale=0.7, eps=1e-4)
    _close(o1, o2, 1e-12, "transition o")
    _close(f1, f2, 1e-12, "transition state")
    for C in (1, 4, 16):
        o3, f3 = oracle.chunked(**p, scale=0.7, eps=1e-4, C=C)
        _close(o3, o1, 1e-10, f"chunked o C={C}")
        _close(f3, f1, 1e-10, f"chunked state C={C}")


def test_unequal_head_dims_beta_zero_closed_form():
    """beta = 0 with Dk != Dv: S_t = e^{sum g} S_0 and o_t = S_t^T qh_t, in both the C recurrence and
    the chunked form."""
    p = _unequal_problem(25, [7], 4, 9, Nv=1, P=1)
    p["beta"] = np.zeros_like(p["beta"])
    S0 = p["state_pool"][0, 0]
    cum = np.cumsum(p["g"][:, 0])
    q = p["q"][:, 0]
    qh = 0.5 * q / np.sqrt(np.sum(q * q, axis=1, keepdims=True) + 1e-6)
    ref = np.stack([(math.exp(cum[t]) * S0).T @ qh[t] for t in range(7)])
    for name, fn in (("recurrence", oracle.recurrent), ("chunked", functools.partial(oracle.chunked, C=4))):
        o, f = fn(**p, scale=0.5, eps=1e-6)
        _close(o[:, 0], ref, 1e-12, f"{name}: o")
        _close(f[0, 0], math.exp(cum[-1]) * S0, 1e-12, f"{name}: state")
