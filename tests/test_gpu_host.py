"""gdn_chunk_fwd_host (host buffers in and out, copies overlapped with the compute) against
gdn_chunk_fwd on the device, bit for bit (GPU).

The host entry streams the batch through the GPU in pieces cut at chunk starts and carries each cut
sequence's fp32 state to its next piece, so its results must equal one device call exactly, whatever
the number of pieces.
"""
from __future__ import annotations

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _device_call(inp):
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                             scale=d.scale, eps=d.eps)
    torch.cuda.synchronize()
    return out.cpu(), fin.cpu()


def _pinned(inp):
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    return [pin(getattr(inp, n)) for n in ("q", "k", "v", "g", "beta", "cu_seqlens", "state_pool", "state_indices")]


@pytest.mark.parametrize("lens,state,segments", [
    ([1000, 513, 128, 2407], ("normal", 0.02, 6, "perm"), 4),     # cuts inside sequences, a pool
    ([1000, 513, 128, 2407], None, 1),                            # one piece
    ([5000], ("normal", 0.02, 1, "identity"), 7),                 # one sequence in 7 pieces (a state carried 6 times)
    ([0, 300, 0, 129, 1, 2200, 0], ("normal", 0.02, 9, "perm"), 3),  # empty sequences between and at the end
])
def test_host_entry_equals_device_call(lens, state, segments):
    inp = inputs.make(lens, Nqk=2, Nv=4, state=state, seed=61)
    ref_out, ref_fin = _device_call(inp)
    q, k, v, g, beta, cu, pool, idx = _pinned(inp)
    for _ in range(2):  # the second call reuses the device buffer and the copy streams
        out, fin, h2d, d2h = gdn.chunk_fwd_host(q, k, v, g, beta, cu, pool, idx, scale=inp.scale, eps=inp.eps,
                                                device=DEV, segments=segments)
        assert torch.equal(out, ref_out)
        assert torch.equal(fin, ref_fin)
    assert d2h == out.numel() * 2 + fin.numel() * 4


def test_host_entry_full_prefill_workload():
    """The bench's one-layer prefill (T = 32768, Nqk = 16, Nv = 32) through the host entry, 8 pieces."""
    inp = inputs.config("prefill_s32k")
    ref_out, ref_fin = _device_call(inp)
    q, k, v, g, beta, cu, pool, idx = _pinned(inp)
    out, fin, _, _ = gdn.chunk_fwd_host(q, k, v, g, beta, cu, pool, idx, scale=inp.scale, eps=inp.eps, device=DEV)
    assert torch.equal(out, ref_out)
    assert torch.equal(fin, ref_fin)
