"""Device-side failure reporting of the chunked path, through the C ABI (GPU).

The decode page's operator raises ValueError on bad arguments and
RuntimeError when execution fails.  Host-visible errors come back as the
return code (tests/test_abi.py); what only the device sees lands in the four
status words of the workspace, read with gdn_read_status:
  - a malformed cu_seqlens (word 0), found by the chunk-table kernel;
  - a bounded wait that gave up (word 2), run out here on purpose through the
    self-test hook, which waits on an mbarrier that nothing arrives on: no
    fault, no trap, no hang, and the bit comes back set;
  - a value beyond the fp16 range in an fp16 intermediate (word 3).
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import _binding as B
from gated_deltanet_linear_17_b200 import inputs
from helpers import assert_close, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
CU_FIRST, CU_DECREASING, CU_TOTAL = 1, 2, 4
WAIT_SELFTEST = 8
RANGE_INTRA, RANGE_STATE, RANGE_OUTPUT = 1, 2, 4


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _poisoned_stages(T, Bn, Nqk=1, Nv=2):
    st = gdn.Stages(T, Bn, Nqk, Nv, DEV)
    st.ws[:16].fill_(0xFF)  # stale words from an imagined earlier call
    return st


@pytest.mark.parametrize("cu,bits", [
    ([0, 100, 60, 300], CU_DECREASING),          # sequence 1 ends before it starts
    ([0, 100, 200, 250], CU_TOTAL),              # cu[B] != T (T = 300)
    ([5, 100, 200, 300], CU_FIRST),              # cu[0] != 0
    ([0, 100, 200, 300], 0),                     # well formed
])
def test_chunk_map_reports_cu_seqlens_errors(cu, bits):
    st = _poisoned_stages(300, 3)
    st.chunk_map(torch.tensor(cu, dtype=torch.int32, device=DEV))
    words = gdn.read_status(st.ws)
    assert words[0] == bits
    assert words[2] == 0 and words[3] == 0  # cleared by the chunk table, which runs first in every call
    info = st.chunk_info.cpu()
    # every chunk row stays inside [0, T), whatever the clamping did
    rows = info[: words[1]]
    assert torch.all(rows[:, 1] >= 0) and torch.all(rows[:, 1] + rows[:, 2] <= 300)


def test_bounded_wait_runs_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    # with the arrival the wait succeeds and nothing is set
    assert gdn.lib().gdn_selftest_wait(64, 1, ctypes.c_void_p(ws.data_ptr()), 256, _stream()) == B.GDN_OK
    assert gdn.read_status(ws) == [0, 0, 0, 0]
    # without it the wait gives up after 64 polls and sets its bit in word 2
    assert gdn.lib().gdn_selftest_wait(64, 0, ctypes.c_void_p(ws.data_ptr()), 256, _stream()) == B.GDN_OK
    words = gdn.read_status(ws)
    assert words[2] == WAIT_SELFTEST and words[0] == 0 and words[3] == 0
    assert gdn.decode_status(words) == ["the self-test wait gave up"]
    # the context is still usable afterwards: a forward pass runs and its status is clean
    inp = inputs.make([300, 40], Nqk=1, Nv=2, seed=40)
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, scale=d.scale, eps=d.eps, check_status=True)
    torch.cuda.synchronize()
    ro, rf = run_oracle(inp)
    assert_close(out, ro, "after the self-test out")
    assert_close(fin, rf, "after the self-test final_state")


def test_forward_status_clean_and_chunk_count():
    inp = inputs.config("varlen_b4")
    d = inp.to(DEV)
    ws = torch.full((gdn.workspace_bytes(d.T, d.B, d.Nqk, d.Nv),), 0xFF, dtype=torch.uint8, device=DEV)
    gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices, scale=d.scale,
                  eps=d.eps, workspace=ws)
    words = gdn.read_status(ws)
    assert words == [0, sum((n + 127) // 128 for n in inp.seqlens), 0, 0]


def _scaled(inp, vs, ss):
    """The same batch with v and the initial states scaled (the operator is linear in both jointly)."""
    v = (inp.v.float() * vs).to(torch.bfloat16)
    pool = None if inp.state_pool is None else inp.state_pool * ss
    return inputs.GdnInputs(inp.name + f"*{vs:g}", inp.q, inp.k, v, inp.g, inp.beta, inp.cu_seqlens, pool,
                            inp.state_indices, inp.scale, inp.eps, list(inp.seqlens))


def test_fp16_range_large_values_match_or_report():
    """v of magnitude ~1e3 and initial states ~20: inside the fp16 range, so the result must match the
    oracle with a clean status; at ~1e6 the fp16 intermediates cannot hold the values and word 3 says so."""
    base = inputs.make([700, 129, 300], Nqk=2, Nv=4, state=("normal", 0.02, 3, "perm"), seed=41)
    inp = _scaled(base, 1024.0, 1024.0)
    d = inp.to(DEV)
    ws = torch.empty(gdn.workspace_bytes(d.T, d.B, d.Nqk, d.Nv), dtype=torch.uint8, device=DEV)
    out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                             scale=d.scale, eps=d.eps, workspace=ws)
    words = gdn.read_status(ws)
    ro, rf = run_oracle(inp)
    assert words[3] == 0, gdn.decode_status(words)
    assert_close(out, ro, "v*1024 out")
    assert_close(fin, rf, "v*1024 final_state")

    big = _scaled(base, 2.0 ** 20, 2.0 ** 20).to(DEV)
    gdn.chunk_fwd(big.q, big.k, big.v, big.g, big.beta, big.cu_seqlens, big.state_pool, big.state_indices,
                  scale=big.scale, eps=big.eps, workspace=ws)
    words = gdn.read_status(ws)
    assert words[3] & RANGE_INTRA and words[3] & RANGE_STATE, words
    with pytest.raises(RuntimeError, match="fp16 range"):
        gdn.chunk_fwd(big.q, big.k, big.v, big.g, big.beta, big.cu_seqlens, big.state_pool, big.state_indices,
                      scale=big.scale, eps=big.eps, workspace=ws, check_status=True)
    # the next call on the same workspace starts from clean words again
    gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices, scale=d.scale,
                  eps=d.eps, workspace=ws)
    assert gdn.read_status(ws)[2:] == [0, 0]
