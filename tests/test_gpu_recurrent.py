"""GPU parity of gdn_recurrent_fwd (token recurrence on a pool updated in place,
one slot per token) against the fp64 pool oracle.

Tolerances as for the forward pass (relative L2 <= 1e-2, max-abs <= 2e-2 RMS,
see helpers.assert_close); slots that no token writes must come back bit-exact.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import inputs
from oracle.pool import recurrent_pool

from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(lens, Nqk, Nv, P, seed, per_token, accepted, Dk=128, Dv=128):
    """Inputs, token slots [T] and accepted counts [B] (None: every token accepted)."""
    inp = inputs.make(lens, Nqk=Nqk, Nv=Nv, state=("normal", 0.02, P, "perm"), seed=seed, Dk=Dk, Dv=Dv)
    r = np.random.default_rng(seed + 1000)
    cu = inp.cu_seqlens.numpy()
    T, B = int(cu[-1]), len(lens)
    if per_token:  # a distinct slot for every token
        slots = r.permutation(P)[:T].astype(np.int32)
    else:  # every token of sequence b on the sequence's slot
        seq_slot = r.permutation(P)[:B]
        slots = np.concatenate([np.full(n, seq_slot[b]) for b, n in enumerate(lens)] + [np.zeros(0)]).astype(np.int32)
    acc = None
    if accepted:
        acc = np.array([r.integers(1, n + 1) if n > 0 else 0 for n in lens], np.int32)
    return inp, slots, acc


def _key_gate(inp, seed):
    return inputs.key_gate(inp, seed)


def _run_and_check(inp, slots, acc, max_seqlen, what, gk=None, bf16_pool=False, rule="gated_delta"):
    pool0 = inp.state_pool.to(torch.bfloat16) if bf16_pool else inp.state_pool
    ro, rpool = recurrent_pool(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, pool0, slots,
                               num_accepted=acc, scale=inp.scale, eps=inp.eps, gk=gk, rule=rule)
    d = inp.to(DEV)
    pool = pool0.to(DEV).clone()
    start = pool.clone()
    ts = torch.from_numpy(slots).to(DEV)
    na = None if acc is None else torch.from_numpy(acc).to(DEV)
    decay, delta = rule in ("gated_delta", "gated"), rule in ("gated_delta", "delta")
    out = gdn.recurrent_fwd(d.q, d.k, d.v, d.g if decay else None, d.beta if delta else None, d.cu_seqlens, pool,
                            ts, num_accepted=na, scale=d.scale, eps=d.eps,
                            gk=None if gk is None or not decay else gk.to(DEV), update_rule=rule,
                            max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    assert_close(out, ro, f"{what} out")
    written = np.unique(slots)
    assert_close(pool[torch.from_numpy(written).to(DEV).long()], rpool[written], f"{what} written slots")
    others = np.setdiff1d(np.arange(pool.shape[0]), written)
    if others.size:
        idx = torch.from_numpy(others).to(DEV).long()
        assert torch.equal(pool[idx], start[idx]), f"{what}: a slot no token names was changed"


@pytest.mark.parametrize("max_seqlen", [4, 0])
def test_recurrent_decode_one_slot_per_sequence(max_seqlen):
    """Ordinary decoding: all tokens of a sequence on its slot, read and written back in place."""
    r = np.random.default_rng(40)
    lens = [int(x) for x in r.integers(1, 5, size=48)]
    inp, slots, acc = _case(lens, Nqk=4, Nv=8, P=64, seed=41, per_token=False, accepted=False)
    _run_and_check(inp, slots, acc, max_seqlen, f"decode max_seqlen={max_seqlen}")


@pytest.mark.parametrize("max_seqlen", [5, 16])
def test_recurrent_speculative_slot_per_token(max_seqlen):
    """Speculative decoding: a slot per token, each sequence starting from its last accepted token's slot."""
    r = np.random.default_rng(42)
    lens = [int(x) for x in r.integers(1, 6, size=40)]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=224, seed=43, per_token=True, accepted=True)
    _run_and_check(inp, slots, acc, max_seqlen, f"speculative max_seqlen={max_seqlen}")


@pytest.mark.parametrize("max_seqlen", [0, 8, 24])
def test_recurrent_long_and_empty_sequences(max_seqlen):
    """Sequences past the staged tokens (read directly), empty ones (nothing read or written)."""
    lens = [0, 20, 3, 0, 17, 9]
    inp, slots, acc = _case(lens, Nqk=1, Nv=2, P=64, seed=44, per_token=True, accepted=True)
    _run_and_check(inp, slots, acc, max_seqlen, f"long/empty max_seqlen={max_seqlen}")


def test_recurrent_runs_of_slots():
    """Runs of tokens sharing a slot inside a sequence (A A B B B C): each slot keeps its run's last state."""
    lens = [6, 4]
    inp, _, _ = _case(lens, Nqk=1, Nv=2, P=16, seed=45, per_token=False, accepted=False)
    slots = np.array([3, 3, 7, 7, 7, 1, 9, 9, 12, 12], np.int32)
    acc = np.array([6, 2], np.int32)
    _run_and_check(inp, slots, acc, 8, "runs of slots")


def test_recurrent_matches_chunk_fwd_final_state():
    """One slot per sequence equals the short path of gdn_chunk_fwd with its final states."""
    lens = [3, 1, 8, 5]
    inp, slots, _ = _case(lens, Nqk=2, Nv=4, P=8, seed=46, per_token=False, accepted=False)
    d = inp.to(DEV)
    cu = inp.cu_seqlens.numpy()
    seq_slot = torch.tensor([int(slots[cu[b]]) for b in range(len(lens))], dtype=torch.int32, device=DEV)
    out_c, fin_c = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, seq_slot, scale=d.scale,
                                 eps=d.eps, max_seqlen=8)
    pool = d.state_pool.clone()
    out_r = gdn.recurrent_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, pool, torch.from_numpy(slots).to(DEV),
                              scale=d.scale, eps=d.eps, max_seqlen=8)
    torch.cuda.synchronize()
    assert torch.equal(out_r, out_c)
    assert torch.equal(pool[seq_slot.long()], fin_c)


@pytest.mark.parametrize("max_seqlen", [4, 0])
def test_recurrent_key_gate(max_seqlen):
    """The decode page's key-dimension gate: each key row of S decays by e^{g + gk_i}."""
    r = np.random.default_rng(47)
    lens = [int(x) for x in r.integers(1, 5, size=32)]
    inp, slots, acc = _case(lens, Nqk=4, Nv=8, P=48, seed=48, per_token=False, accepted=False)
    _run_and_check(inp, slots, acc, max_seqlen, f"key gate max_seqlen={max_seqlen}", gk=_key_gate(inp, 49))


@pytest.mark.parametrize("max_seqlen", [8, 16])
def test_recurrent_bf16_pool(max_seqlen):
    """A bf16 state pool: widened on load, the fp32 state rounded when written."""
    r = np.random.default_rng(50)
    lens = [int(x) for x in r.integers(1, 9, size=32)]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=40, seed=51, per_token=False, accepted=False)
    _run_and_check(inp, slots, acc, max_seqlen, f"bf16 pool max_seqlen={max_seqlen}", bf16_pool=True)


def test_recurrent_decode_page_operator():
    """Everything of the decode page at once: bf16 pool, key gate, a slot per token, accepted counts."""
    r = np.random.default_rng(52)
    lens = [int(x) for x in r.integers(1, 6, size=36)]
    inp, slots, acc = _case(lens, Nqk=4, Nv=8, P=224, seed=53, per_token=True, accepted=True)
    _run_and_check(inp, slots, acc, 5, "decode page operator", gk=_key_gate(inp, 54), bf16_pool=True)


@pytest.mark.parametrize("max_seqlen", [0, 8])
def test_recurrent_key_gate_past_staged_tokens(max_seqlen):
    """Key gate on tokens read directly (past the staged ones), fp32 and bf16 pools."""
    lens = [19, 2, 11]
    inp, slots, acc = _case(lens, Nqk=1, Nv=2, P=40, seed=55, per_token=True, accepted=True)
    gk = _key_gate(inp, 56)
    _run_and_check(inp, slots, acc, max_seqlen, f"key gate, long, max_seqlen={max_seqlen}", gk=gk)
    _run_and_check(inp, slots, acc, max_seqlen, f"key gate, long, bf16, max_seqlen={max_seqlen}", gk=gk,
                   bf16_pool=True)


@pytest.mark.parametrize("rule", ["delta", "gated", "linear"])
@pytest.mark.parametrize("max_seqlen", [8, 0])
def test_recurrent_update_rules(rule, max_seqlen):
    """The LinearAttention page's other update rules, a slot per token, staged and direct-read tokens."""
    lens = [3, 1, 6, 0, 18, 2]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=40, seed=57, per_token=True, accepted=True)
    _run_and_check(inp, slots, acc, max_seqlen, f"rule {rule} max_seqlen={max_seqlen}", rule=rule)


def test_recurrent_gated_rule_key_gate_bf16():
    """The gated rule with the key-dimension gate on a bf16 pool (ordinary decoding)."""
    r = np.random.default_rng(58)
    lens = [int(x) for x in r.integers(1, 5, size=24)]
    inp, slots, acc = _case(lens, Nqk=4, Nv=8, P=32, seed=59, per_token=False, accepted=False)
    _run_and_check(inp, slots, acc, 4, "gated rule, gk, bf16", gk=_key_gate(inp, 60), bf16_pool=True, rule="gated")


@pytest.mark.parametrize("Dk,Dv", [(64, 512), (64, 64), (128, 64), (128, 256)])
def test_recurrent_head_dimensions(Dk, Dv):
    """Key and value dimensions other than 128 (the decode page's example: Dk = 64, Dv = 512), with the
    key gate, a bf16 pool, a slot per token and a sequence past the staged tokens."""
    lens = [1, 4, 2, 19, 3]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=40, seed=61, per_token=True, accepted=True, Dk=Dk, Dv=Dv)
    _run_and_check(inp, slots, acc, 0, f"Dk={Dk} Dv={Dv}", gk=_key_gate(inp, 62), bf16_pool=True)
    _run_and_check(inp, slots, acc, 4, f"Dk={Dk} Dv={Dv} fp32 delta", rule="delta")


@pytest.mark.parametrize("act,state", [(torch.float16, torch.float32), (torch.float16, torch.float16),
                                       (torch.float32, torch.float32), (torch.float32, torch.float16)])
def test_recurrent_linear_attention_types(act, state):
    """The LinearAttention page's element types: activations and state each fp16 or fp32, with the key
    gate, a slot per token, accepted counts and tokens past the staged ones.  The activations carry bits
    beyond bf16 (a small fp32 perturbation), so a narrowed path would show."""
    lens = [3, 1, 6, 19, 2]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=40, seed=63, per_token=True, accepted=True)
    gen = torch.Generator().manual_seed(64)
    widen = lambda x: (x.float() + 1e-3 * torch.randn(x.shape, generator=gen)).to(act)
    q, k, v = widen(inp.q), widen(inp.k), widen(inp.v)
    pool0 = inp.state_pool.to(state)
    gk = _key_gate(inp, 65)
    ro, rpool = recurrent_pool(q, k, v, inp.g, inp.beta, inp.cu_seqlens, pool0, slots, num_accepted=acc,
                               scale=inp.scale, eps=inp.eps, gk=gk)
    d = inp.to(DEV)
    pool = pool0.to(DEV).clone()
    start = pool.clone()
    out = gdn.recurrent_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, pool,
                            torch.from_numpy(slots).to(DEV), num_accepted=torch.from_numpy(acc).to(DEV),
                            scale=d.scale, eps=d.eps, gk=gk.to(DEV), max_seqlen=0)
    torch.cuda.synchronize()
    what = f"act {act} state {state}"
    assert out.dtype == act
    assert_close(out, ro, f"{what} out")
    written = np.unique(slots)
    assert_close(pool[torch.from_numpy(written).to(DEV).long()], rpool[written], f"{what} written slots")
    others = torch.from_numpy(np.setdiff1d(np.arange(pool.shape[0]), written)).to(DEV).long()
    assert torch.equal(pool[others], start[others])


@pytest.mark.parametrize("bf16_pool", [False, True])
@pytest.mark.parametrize("rule", ["gated_delta", "delta", "gated", "linear"])
def test_recurrent_one_token_decode_kernel(bf16_pool, rule):
    """max_seqlen = 1 (one token per sequence, the decode page's common call) takes the streaming decode
    kernel: a token per sequence, empty sequences, some sequences moved to another slot, the key gate on
    the decaying rules."""
    r = np.random.default_rng(110)
    lens = [int(x) for x in r.choice([0, 1, 1, 1], size=70)]
    inp, slots, acc = _case(lens, Nqk=4, Nv=8, P=160, seed=111, per_token=True, accepted=False)
    gk = _key_gate(inp, 112) if rule in ("gated_delta", "gated") else None
    _run_and_check(inp, slots, acc, 1, f"decode kernel {rule} bf16_pool={bf16_pool}", gk=gk, bf16_pool=bf16_pool,
                   rule=rule)


@pytest.mark.parametrize("Dk,Dv", [(64, 512), (64, 64), (128, 256)])
def test_recurrent_one_token_decode_head_dimensions(Dk, Dv):
    r = np.random.default_rng(113)
    lens = [int(x) for x in r.choice([0, 1], size=40, p=[0.1, 0.9])]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=60, seed=114, per_token=False, accepted=False, Dk=Dk, Dv=Dv)
    _run_and_check(inp, slots, acc, 1, f"decode kernel Dk={Dk} Dv={Dv} bf16", gk=_key_gate(inp, 115), bf16_pool=True)
    _run_and_check(inp, slots, acc, 1, f"decode kernel Dk={Dk} Dv={Dv} fp32")


@pytest.mark.parametrize("bf16_pool", [False, True])
def test_recurrent_decode_hint_too_small_stays_exact(bf16_pool):
    """max_seqlen = 1 understated: sequences of 2..6 tokens with per-token slots and accepted counts run
    the decode kernel's fp32 register path and still match the oracle."""
    lens = [1, 3, 0, 6, 1, 2, 5]
    inp, slots, acc = _case(lens, Nqk=2, Nv=4, P=40, seed=116, per_token=True, accepted=True)
    _run_and_check(inp, slots, acc, 1, f"decode kernel understated hint bf16_pool={bf16_pool}",
                   gk=_key_gate(inp, 117), bf16_pool=bf16_pool)
