"""The allocation-free entry point, gdn_chunk_fwd_noalloc, through the C ABI.

Some callers may not allocate device memory at all while they run (a plugin
or custom op inside an engine that owns the whole GPU's memory, an interface
with no room for a workspace).  For them the library runs the chunked path on
a static per-GPU scratch buffer of its own.  This file checks, on a GPU, that
calls in a row -- each one finding the previous one's leftovers in the
shared scratch -- give the same results as the allocating entry point
gdn_chunk_fwd bit for bit (both run the same kernels on the same inputs), also
for a batch long enough that the chunked pass is split into pipelined chunk
ranges, that the scratch's device status words can be read back without an
allocation, and that sizes needing more scratch than the buffer holds are
refused before anything runs.

The file sorts last so that a run stopping at its first failure has already
run every other test; it also passes on its own in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import _binding as B
from gated_deltanet_linear_17_b200 import inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(d, out, fin, max_seqlen=0):
    """One call of gdn_chunk_fwd_noalloc through the C ABI on the current stream."""
    rc = gdn.lib().gdn_chunk_fwd_noalloc(
        _p(d.q), _p(d.k), _p(d.v), _p(d.g), _p(d.beta), _p(d.cu_seqlens), _p(d.state_pool), _p(d.state_indices),
        d.scale, d.eps, _p(out), _p(fin), d.T, d.B, d.Nqk, d.Nv, d.P, max_seqlen,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


def test_calls_in_a_row_match_allocating_entry():
    first = inputs.make([300, 129, 1, 64], Nqk=2, Nv=4, state=("normal", 0.02, 6, "perm"), seed=31).to("cuda")
    second = inputs.make([257, 40], Nqk=4, Nv=8, state=("normal", 0.02, 2, "identity"), seed=32).to("cuda")
    # 43 chunks: the chunked pass runs as two pipelined ranges (side streams, a carried state)
    third = inputs.make([3000, 2100, 129], Nqk=2, Nv=4, state=("normal", 0.02, 5, "perm"), seed=33).to("cuda")
    assert gdn.pipeline_ranges(third.T, third.B, third.Nqk, third.Nv) == 2
    assert gdn.workspace_bytes(third.T, third.B, third.Nqk, third.Nv) <= B.NOALLOC_SCRATCH_BYTES
    for d in (first, second, third, first):
        ref_out, ref_fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                                         scale=d.scale, eps=d.eps)
        out = torch.full_like(ref_out, float("nan"))
        fin = torch.full_like(ref_fin, float("nan"))
        assert _noalloc(d, out, fin) == B.GDN_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), "noalloc out differs from gdn_chunk_fwd"
        assert torch.equal(fin, ref_fin), "noalloc final_state differs from gdn_chunk_fwd"
        # the scratch's status words, copied out without an allocation: clean, with the chunk count
        words = gdn.noalloc_status()
        assert words == [0, sum((n + 127) // 128 for n in d.seqlens), 0, 0]


def test_sizes_beyond_the_scratch_are_refused():
    # a 32K-token prefill at 16/32 heads needs ~1 GiB of workspace; nothing is enqueued
    need = gdn.workspace_bytes(32768, 1, 16, 32)
    assert need > B.NOALLOC_SCRATCH_BYTES
    M = 1 << 20
    vp = ctypes.c_void_p
    rc = gdn.lib().gdn_chunk_fwd_noalloc(vp(M), vp(2 * M), vp(3 * M), vp(4 * M), vp(5 * M), vp(6 * M), None, None,
                                         0.0, 1e-6, vp(7 * M), None, 32768, 1, 16, 32, 0, 0, None)
    assert rc == B.GDN_ERR_SCRATCH_LIMIT
    assert "SCRATCH" in gdn.status_string(rc)
