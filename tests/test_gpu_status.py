"""Device-side failure reporting of the chunked path, through the C ABI (GPU).

The decode page's operator raises ValueError on bad arguments and
RuntimeError when execution fails.  Host-visible errors come back as the
return code (tests/test_abi.py); what only the device sees lands in the four
status words of the workspace, read with gdn_read_status:
  - a malformed cu_seqlens (word 0), found by the chunk-table kernel;
  - a bounded wait that gave up (word 2), run out here on purpose through the
    self-test hook, which waits on an mbarrier that nothing arrives on: no
    fault, no trap, no hang, and the bit comes back set;
  - a value beyond the fp16 range in an fp16 intermediate (word 3);
  - with the value checks switched on, a gate above 0, a beta outside [0, 1]
    or a slot index outside the pool (word 0, GDN_DEV_VAL_*), and the same
    bits from gdn_check_values called on its own.
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


VAL_GATE, VAL_BETA, VAL_INDEX = 8, 16, 32


def _bf16_bits(x):
    return torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()


@pytest.mark.parametrize("plant,bits", [
    (None, 0),
    ("gate_positive", VAL_GATE),
    ("gate_nan", VAL_GATE),
    ("beta_above_one", VAL_BETA),
    ("beta_negative", VAL_BETA),
    ("beta_nan", VAL_BETA),
    ("index_at_P", VAL_INDEX),
    ("index_negative", VAL_INDEX),
])
def test_check_values_finds_each_case(plant, bits):
    inp = inputs.make([300, 129, 1, 700], Nqk=2, Nv=4, state=("normal", 0.02, 6, "perm"), seed=111)
    d = inp.to(DEV)
    g, beta, idx = d.g.clone(), d.beta.clone(), d.state_indices.clone()
    P = inp.state_pool.shape[0]
    if plant == "gate_positive":
        g[777, 3] = 0.25
    elif plant == "gate_nan":
        g[5, 0] = float("nan")
    elif plant == "beta_above_one":
        beta[1000, 2] = 1.5
    elif plant == "beta_negative":
        beta[0, 1] = -0.125
    elif plant == "beta_nan":
        beta.view(torch.int16)[42, 3] = 0x7FC0
    elif plant == "index_at_P":
        idx[2] = P
    elif plant == "index_negative":
        idx[0] = -1
    assert gdn.check_values(g, beta, idx, P) == bits
    assert gdn.check_values(g=g) == bits & VAL_GATE
    assert gdn.check_values(beta=beta) == bits & VAL_BETA
    assert gdn.check_values(state_indices=idx, P=P) == bits & VAL_INDEX


def test_value_checks_switch_reports_through_the_workspace():
    """With the switch on, a chunked call's status word 0 carries the value bits (and its results are
    those of the call without the checks); with it off, nothing is checked."""
    inp = inputs.make([300, 129, 1, 700], Nqk=2, Nv=4, state=("normal", 0.02, 6, "perm"), seed=113)
    d = inp.to(DEV)
    g = d.g.clone()
    g[100, 2] = 0.5  # a gate above 0
    ws = torch.empty(gdn.workspace_bytes(d.T, d.B, d.Nqk, d.Nv), dtype=torch.uint8, device=DEV)
    run = lambda: gdn.chunk_fwd(d.q, d.k, d.v, g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                                scale=d.scale, eps=d.eps, workspace=ws)
    out0, fin0 = run()
    assert gdn.read_status(ws)[0] == 0
    prev = gdn.set_value_checks(True)
    try:
        out1, fin1 = run()
        words = gdn.read_status(ws)
        assert words[0] == VAL_GATE, words
        assert "a gate that is not <= 0" in gdn.decode_status(words)
        # a clean call on the same workspace: the chunk table clears the word first
        gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                                scale=d.scale, eps=d.eps, workspace=ws)
        assert gdn.read_status(ws)[0] == 0
    finally:
        gdn.set_value_checks(prev)
    torch.cuda.synchronize()
    assert torch.equal(out0, out1) and torch.equal(fin0, fin1)
