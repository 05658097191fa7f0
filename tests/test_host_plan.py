"""The cut of gdn_chunk_fwd_host into pieces, checked on the host (CPU only).

gdn_chunk_fwd_host streams a batch through the GPU in pieces and resumes a
sequence cut between two pieces from its carried state.  That is exact only
if every cut falls on a chunk start of its sequence (the prefill page's
chunks of L = 128 tokens start at each sequence's first token), every token
is computed once, and the carried state is handed from a piece to the next
piece of the same sequence.  These properties are checked here on random
batches through the library's own planner (gdn_testing_host_plan).
"""
from __future__ import annotations

import os
import random

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import _binding as B


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("libgdn.so not built")


def _check_plan(lens, segments):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1]
    rows = gdn.host_plan(torch.tensor(cu, dtype=torch.int32), segments)
    covered = []
    finals = []
    prev = None
    nseg = 0
    for seg, b0, nb, t0, t1, src, dst in rows:
        assert prev is None or seg >= prev[0]
        nseg = max(nseg, seg + 1)
        assert 0 <= b0 and b0 + nb <= len(lens) and nb >= 1 and 0 <= t0 <= t1 <= T
        covered.append((t0, t1))
        if src == 2 or dst == 1:  # a piece of one sequence whose state crosses a cut
            assert nb == 1
        s, e = cu[b0], cu[b0 + nb]
        if src == 2:
            assert t0 > s and (t0 - s) % 128 == 0            # resumes at a chunk start
            assert prev is not None and prev[6] == 1 and prev[1] == b0 and prev[4] == t0  # from the previous piece
        else:
            assert t0 == s
        if dst == 1:
            assert t1 < e and (t1 - cu[b0]) % 128 == 0       # stops at a chunk start
        else:
            assert t1 == e
            finals.extend(range(b0, b0 + nb))
        if prev is not None and prev[6] == 1:
            assert src == 2                                   # the carried state is taken up at once
        prev = (seg, b0, nb, t0, t1, src, dst)
    assert prev is None or prev[6] == 0
    assert sorted(finals) == list(range(len(lens)))           # every sequence ends exactly once
    covered.sort()
    pos = 0
    for t0, t1 in covered:                                    # every token exactly once
        assert t0 == pos or t0 == t1 == pos
        pos = t1
    assert pos == T
    assert nseg <= max(segments, 1)
    return rows


def test_long_sequence_cut_at_chunk_starts():
    rows = _check_plan([32768], 8)
    assert len(rows) == 8 and all(r[4] - r[3] == 4096 for r in rows)


def test_plan_properties_on_random_batches():
    r = random.Random(7)
    for _ in range(400):
        nb = r.randint(1, 20)
        lens = [r.choice([0, 1, 127, 128, 129, 255, 256, 257, r.randint(0, 3000)]) for _ in range(nb)]
        _check_plan(lens, r.randint(1, 12))


def test_all_empty_and_invalid():
    assert _check_plan([0, 0, 0], 4) == [[0, 0, 3, 0, 0, 1, 0]]
    with pytest.raises(ValueError):
        gdn.host_plan(torch.tensor([0, 5, 3], dtype=torch.int32))  # decreasing
