"""GPU parity of gdn_chunk_fwd_rule (the LinearAttention page's update rules in the
chunked path and in the fused short path) against the fp64 pool oracle.

Each sequence starts from its pool slot and the oracle's updated slot is the
sequence's final state.  Tolerances as for the forward pass (helpers.assert_close).
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


def _check_rule(lens, rule, max_seqlen, seed, Nqk=2, Nv=4):
    inp = inputs.make(lens, Nqk=Nqk, Nv=Nv, state=("normal", 0.02, len(lens) + 3, "perm"), seed=seed)
    cu = inp.cu_seqlens.numpy()
    idx = inp.state_indices.numpy()
    slots = np.concatenate([np.full(n, idx[b]) for b, n in enumerate(lens)] + [np.zeros(0)]).astype(np.int32)
    ro, rpool = recurrent_pool(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.state_pool, slots,
                               scale=inp.scale, eps=inp.eps, rule=rule)
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices, scale=d.scale,
                             eps=d.eps, max_seqlen=max_seqlen, update_rule=rule)
    torch.cuda.synchronize()
    what = f"rule {rule} max_seqlen={max_seqlen}"
    assert_close(out, ro, f"{what} out")
    ref_fin = np.stack([rpool[idx[b]] for b in range(len(lens))])  # empty sequences keep their start
    assert_close(fin, ref_fin, f"{what} final_state")


@pytest.mark.parametrize("rule", ["delta", "gated", "linear"])
def test_chunked_path_update_rules(rule):
    """Varlen batch through the chunk kernels: full chunks, ragged tails, a 1-token and an empty sequence."""
    _check_rule([1000, 513, 128, 300, 0, 1], rule, 0, seed=71)


@pytest.mark.parametrize("rule", ["delta", "gated", "linear"])
def test_chunked_path_update_rules_two_ranges(rule):
    """Enough chunks for the two pipelined ranges (a sequence crossing the range boundary)."""
    _check_rule([2600, 1900], rule, 0, seed=72, Nqk=1, Nv=2)


@pytest.mark.parametrize("rule", ["delta", "gated", "linear"])
@pytest.mark.parametrize("max_seqlen", [8, 16])
def test_short_path_update_rules(rule, max_seqlen):
    lens = [3, 8, 1, 0, 5] if max_seqlen == 8 else [16, 9, 2, 12]
    _check_rule(lens, rule, max_seqlen, seed=73)


def test_delta_rule_is_gated_delta_with_zero_gate():
    """The delta rule equals the gated delta rule with g = 0 through the chunk kernels (bit for bit)."""
    inp = inputs.make([700, 129], Nqk=2, Nv=4, seed=74)
    d = inp.to(DEV)
    o1, f1 = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, update_rule="delta")
    o2, f2 = gdn.chunk_fwd(d.q, d.k, d.v, torch.zeros_like(d.g), d.beta, d.cu_seqlens)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)
