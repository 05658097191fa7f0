"""GPU parity of gdn_recurrent_window_fwd (the LinearAttention page's state_window: the W most recent
states per (sequence, head), updated in place) against the fp64 window oracle ``oracle.window``.

Tolerances as for the forward pass (helpers.assert_close).  The window entries are checked for every
sequence -- shorter than the window (kept past entries moved down), longer than it (only the last W
states), empty (the window left as it was, bit for bit) -- under the four update rules, with and
without the key gate, for fp32 and 16-bit windows and for window sizes 0 (no window axis), 1, 4 and 8.
"""
from __future__ import annotations

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import inputs
from oracle.window import recurrent_window

from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _past(W, B, Nv, Dk, Dv, seed, dtype):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(W, B, Nv, Dk, Dv, generator=gen) * 0.02).to(dtype)


def _run(lens, W, rule="gated_delta", gk=False, state=torch.float32, act=torch.bfloat16, Dk=128, Dv=128,
         max_seqlen=0, seed=70, zero_past=False):
    inp = inputs.make(lens, Nqk=2, Nv=4, seed=seed, Dk=Dk, Dv=Dv)
    Wd = max(W, 1)
    past = torch.zeros(Wd, inp.B, inp.Nv, Dk, Dv, dtype=state) if zero_past else \
        _past(Wd, inp.B, inp.Nv, Dk, Dv, seed + 1, state)
    q, k, v = inp.q.to(act), inp.k.to(act), inp.v.to(act)
    key_gate = inputs.key_gate(inp, seed + 2) if gk else None
    ro, rwin = recurrent_window(q, k, v, inp.g, inp.beta, inp.cu_seqlens, past, Wd, scale=inp.scale, eps=inp.eps,
                                gk=key_gate, rule=rule)
    d = inp.to(DEV)
    win = past.to(DEV).clone()
    decay, delta = rule in ("gated_delta", "gated"), rule in ("gated_delta", "delta")
    out = gdn.recurrent_window_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g if decay else None,
                                   d.beta if delta else None, d.cu_seqlens, win, W, scale=d.scale, eps=d.eps,
                                   gk=None if key_gate is None else key_gate.to(DEV), update_rule=rule,
                                   max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    what = f"W={W} {rule} gk={gk} state={state} act={act} lens={lens}"
    if inp.T:
        assert_close(out, ro, f"{what} out")
    for b, n in enumerate(inp.seqlens):
        if n == 0:
            assert torch.equal(win[:, b].cpu(), past[:, b]), f"{what}: the window of an empty sequence changed"
        else:
            assert_close(win[:, b], rwin[:, b], f"{what} window of sequence {b} (n={n})")
    return win


@pytest.mark.parametrize("W", [1, 4, 8])
@pytest.mark.parametrize("max_seqlen", [8, 0])
def test_window_sizes_short_and_long_sequences(W, max_seqlen):
    # lengths below, at and above each window, an empty sequence, and one past the staged tokens
    _run([1, 3, 0, 4, 8, 2, 7, 5, 20][: 9 if max_seqlen == 0 else 8], W, max_seqlen=max_seqlen)


@pytest.mark.parametrize("rule", ["gated_delta", "delta", "gated", "linear"])
def test_window_update_rules_with_key_gate(rule):
    _run([2, 6, 1, 5, 0, 3], 4, rule=rule, gk=rule in ("gated_delta", "gated"))


def test_window_zero_means_current_state_only():
    """window = 0 (no window axis): the buffer is the current state, the same as a window of one entry."""
    a = _run([3, 1, 0, 6], 0, seed=80)
    b = _run([3, 1, 0, 6], 1, seed=80)
    assert torch.equal(a, b)


def test_window_absent_past_is_zeros():
    _run([2, 5, 1], 4, zero_past=True)


@pytest.mark.parametrize("state,act", [(torch.bfloat16, torch.bfloat16), (torch.float16, torch.float16),
                                       (torch.float32, torch.float32)])
def test_window_element_types(state, act):
    _run([2, 4, 1, 9], 3, state=state, act=act, gk=True)


def test_window_decode_page_head_dimensions():
    _run([1, 2, 1, 3], 4, state=torch.bfloat16, Dk=64, Dv=512, gk=True)


def test_window_rollback_reads_earlier_states():
    """Rolling back r tokens is reading entry W - 1 - r: a second step from the rolled-back state
    equals a step over the shortened sequence."""
    W = 4
    lens = [4, 4]
    inp = inputs.make(lens, Nqk=2, Nv=4, seed=90)
    d = inp.to(DEV)
    win = torch.zeros(W, inp.B, inp.Nv, 128, 128, device=DEV)
    gdn.recurrent_window_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, win, W, scale=d.scale, eps=d.eps)
    # the same batch with only the first two tokens of each sequence, on a fresh window
    keep = torch.cat([torch.arange(0, 2), torch.arange(4, 6)])
    sd = inputs.GdnInputs("short", inp.q[keep], inp.k[keep], inp.v[keep], inp.g[keep], inp.beta[keep],
                          torch.tensor([0, 2, 4], dtype=torch.int32), None, None, inp.scale, inp.eps,
                          [2, 2]).to(DEV)
    win2 = torch.zeros(W, inp.B, inp.Nv, 128, 128, device=DEV)
    gdn.recurrent_window_fwd(sd.q, sd.k, sd.v, sd.g, sd.beta, sd.cu_seqlens, win2, W, scale=sd.scale, eps=sd.eps)
    torch.cuda.synchronize()
    # two tokens rolled back: entry W - 1 - 2 of the long run is the newest entry of the short run
    assert torch.equal(win[W - 3], win2[W - 1])
