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


def test_host_entry_status_folded_over_pieces():
    """The call's device status words sit at the start of the device buffer, folded over the pieces:
    the chunk counts add up to the batch's, and a value beyond the fp16 range in the first piece is still
    reported after the later, clean pieces have run (each piece's chunk table clears its own words)."""
    lens = [1000, 513, 128, 2407]
    inp = inputs.make(lens, Nqk=2, Nv=4, state=("normal", 0.02, 6, "perm"), seed=63)
    q, k, v, g, beta, cu, pool, idx = _pinned(inp)
    need = gdn.host_buffer_bytes(cu, 2, 4, True, 4)
    buf = torch.empty(need, dtype=torch.uint8, device=DEV)
    gdn.chunk_fwd_host(q, k, v, g, beta, cu, pool, idx, scale=inp.scale, eps=inp.eps, device=DEV, segments=4,
                       device_buffer=buf, check_status=True)
    words = gdn.read_status(buf)
    assert words[0] == 0 and words[2] == 0 and words[3] == 0, words
    assert words[1] == sum((n + 127) // 128 for n in lens)
    rows = gdn.host_plan(inp.cu_seqlens, 4)
    assert len({r[0] for r in rows}) > 1  # the batch really runs in several pieces
    big = v.clone()
    big[:200] *= 2.0 ** 20  # beta v beyond +-65504 in the first sequence, the first piece
    with pytest.raises(RuntimeError, match="fp16 range"):
        gdn.chunk_fwd_host(q, k, big, g, beta, cu, pool, idx, scale=inp.scale, eps=inp.eps, device=DEV,
                           segments=4, device_buffer=buf, check_status=True)
    assert gdn.read_status(buf)[3] & 1
