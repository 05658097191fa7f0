"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance (bf16 inputs/outputs, fp32 accumulation and state), per tensor:
relative L2 <= 1e-2 and max-abs <= 2e-2 * RMS(reference).  Index work (the
chunk table, slot selection, packing) is checked bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import inputs
import helpers
from helpers import assert_close, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _gpu(inp, max_seqlen=0, **kw):
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                             scale=d.scale, eps=d.eps, max_seqlen=max_seqlen, **kw)
    torch.cuda.synchronize()
    return out, fin


def _check(inp, out, fin, heads=None, what=""):
    ro, rf = run_oracle(inp, heads=heads)
    if heads is not None:
        out, fin = out[:, heads], fin[:, heads]
    assert_close(out, ro, f"{what} out")
    assert_close(fin, rf, f"{what} final_state")


# ------------------------------------------------------------------ named workloads

@pytest.mark.parametrize("name", ["single_s256", "varlen_b4"])
def test_small_configs_all_heads(name):
    inp = inputs.config(name)
    out, fin = _gpu(inp)
    _check(inp, out, fin, what=name)


def test_prefill_s32k_sampled_heads():
    """Full-size one-layer prefill (T = 32768, Nqk = 16, Nv = 32), oracle on three v-heads."""
    inp = inputs.config("prefill_s32k")
    out, fin = _gpu(inp)
    _check(inp, out, fin, heads=[0, 13, 31], what="prefill_s32k")


def test_short_pool_b256_both_paths():
    """256 sequences of 1..8 tokens from a 512-slot pool: fused short kernel and chunked kernels."""
    inp = inputs.config("short_pool_b256")
    ro, rf = run_oracle(inp)
    for ms in (inp.max_seqlen, 0):
        out, fin = _gpu(inp, max_seqlen=ms)
        assert_close(out, ro, f"short max_seqlen={ms} out")
        assert_close(fin, rf, f"short max_seqlen={ms} final_state")


def test_short_path_staging_depths():
    """Sequences of 9..16 tokens from a pool: the fused kernel stages 16 tokens when max_seqlen says 16,
    8 when it says 8 (an understated bound: the tokens past the eighth are read directly)."""
    inp = inputs.make([9, 16, 1, 12, 8, 15], Nqk=2, Nv=4, state=("normal", 0.02, 8, "perm"), seed=23)
    ro, rf = run_oracle(inp)
    for ms in (16, 8):
        out, fin = _gpu(inp, max_seqlen=ms)
        assert_close(out, ro, f"short staging max_seqlen={ms} out")
        assert_close(fin, rf, f"short staging max_seqlen={ms} final_state")


def test_short_path_without_pool_two_heads():
    """Fused short kernel with a zero initial state, empty sequences and Nv = 2 (g, beta rows of 8 and 4 bytes)."""
    inp = inputs.make([5, 1, 8, 0, 3, 16, 0], Nqk=1, Nv=2, seed=21)
    out, fin = _gpu(inp, max_seqlen=16)
    _check(inp, out, fin, what="short, no pool")


@pytest.mark.slow
def test_long_s128k_b2_sampled_heads():
    """Two 128K-token sequences with initial states, oracle on v-heads 0, 7, 16, 31."""
    inp = inputs.config("long_s128k_b2")
    out, fin = _gpu(inp)
    _check(inp, out, fin, heads=[0, 7, 16, 31], what="long_s128k_b2")


# ------------------------------------------------------------------ per-kernel intermediates

def test_stages_match_chunked_intermediates():
    """Each kernel's output against the chunked form's named intermediates."""
    inp = inputs.make([200, 129, 1, 128], Nqk=2, Nv=4, state=("normal", 0.02, 6, "perm"), seed=11)
    d = inp.to(DEV)
    st = gdn.Stages(inp.T, inp.B, inp.Nqk, inp.Nv, DEV)
    out = torch.empty(inp.T, inp.Nv, 128, dtype=torch.bfloat16, device=DEV)
    fin = torch.empty(inp.B, inp.Nv, 128, 128, dtype=torch.float32, device=DEV)
    st.chunk_map(d.cu_seqlens)
    st.intra(d.k, d.v, d.g, d.beta, inp.eps)
    st.state(d.k, d.state_pool, d.state_indices, fin)
    st.output(d.q, d.k, d.g, out, inp.scale, inp.eps)
    torch.cuda.synchronize()
    X = {n: oracle.as_numpy_exact(getattr(inp, n)) for n in ("q", "k", "v", "g", "beta")}
    _, _, kept = oracle.chunked(X["q"], X["k"], X["v"], X["g"], X["beta"], inp.cu_seqlens.numpy(),
                                inp.state_pool.double().numpy(), inp.state_indices.numpy(),
                                scale=inp.scale, eps=inp.eps, C=128, keep=True)
    info = st.chunk_info.cpu().numpy()
    seq_first = {}
    for c in range(info.shape[0]):
        if info[c, 0] >= 0 and info[c, 3] == 0:
            seq_first[int(info[c, 0])] = c
    names = {"U": "v_out", "W": "k_cumdecay", "Sc": "S_in", "Mk": None}
    per_token = {"U", "W"}
    got = {n: [] for n in names}
    ref = {n: [] for n in names}
    gam_g, gam_r, kh_g, kh_r, qh_g, qh_r = [], [], [], [], [], []
    rk, rq, gcum = st.rk.cpu().double().numpy(), st.rq.cpu().double().numpy(), st.gcum.cpu().double()
    G = inp.Nv // inp.Nqk
    for (b, h, ci), r in kept.items():
        c = seq_first[b] + ci
        n = r["o"].shape[0]
        t0 = int(info[c, 1])
        assert int(info[c, 2]) == n
        # the factor of the state update that multiplies S ("State Update": k_gexp^T k_cumdecay)
        k_gexp = r["kn"] * np.exp(r["g_cum"][-1] - r["g_cum"])[:, None]
        derived = {"Mk": k_gexp.T @ r["k_cumdecay"]}
        for nm, key in names.items():
            t = getattr(st, nm)[c, h].cpu().double().numpy()
            got[nm].append(t[:n] if nm in per_token else t)
            ref[nm].append(r[key] if key else derived[nm])
        hq = h // G
        gam_g.append(gcum[h, t0:t0 + n].numpy())
        gam_r.append(r["g_cum"])
        kh_g.append(X["k"][t0:t0 + n, hq] * rk[hq, t0:t0 + n, None])
        kh_r.append(r["kn"])
        qh_g.append(X["q"][t0:t0 + n, hq] * rq[hq, t0:t0 + n, None])
        qh_r.append(r["qn"])
    cat = lambda xs: np.concatenate([x.reshape(-1) for x in xs])
    assert_close(cat(gam_g), cat(gam_r), "gcum", rel_l2=1e-5, max_abs_rms=1e-5)
    # fp32 normalisation factors applied to the exact raw rows
    assert_close(cat(kh_g), cat(kh_r), "k normalised", rel_l2=1e-5, max_abs_rms=1e-5)
    assert_close(cat(qh_g), cat(qh_r), "q normalised and scaled", rel_l2=1e-5, max_abs_rms=1e-5)
    for nm in names:  # fp16 intermediates: their own storage rounding is allowed per element
        assert_close(cat(got[nm]), cat(ref[nm]), f"stage {nm}", ulp=helpers.FP16_HALF_ULP)
    assert int(st.status.cpu()[2]) == 0
    _check(inp, out, fin, what="stages")


def test_chunk_table_bit_exact():
    lens = [0, 1, 127, 128, 129, 0, 255, 256, 257, 3]
    inp = inputs.make(lens, Nqk=1, Nv=1, seed=5)
    d = inp.to(DEV)
    st = gdn.Stages(inp.T, inp.B, 1, 1, DEV)
    st.chunk_map(d.cu_seqlens)
    torch.cuda.synchronize()
    rows = []
    t = 0
    for b, n in enumerate(lens):
        for j, s in enumerate(range(0, n, 128)):
            rows.append([b, t + s, min(128, n - s), j])
        t += n
    info = st.chunk_info.cpu().numpy()
    assert np.array_equal(info[:len(rows)], np.array(rows, dtype=np.int32))
    assert np.all(info[len(rows):, 0] == -1)
    status = st.status.cpu().numpy()
    assert status[0] == 0 and status[1] == len(rows)


# ------------------------------------------------------------------ edge cases and invariants

def test_ragged_lengths_with_empty_sequences():
    lens = [0, 1, 127, 128, 129, 0, 255, 256, 257, 2]
    inp = inputs.make(lens, Nqk=2, Nv=4, state=("normal", 0.02, 12, "perm"), seed=6)
    out, fin = _gpu(inp)
    _check(inp, out, fin, what="ragged")
    # zero-length sequences keep their initial state
    for b in (0, 5):
        assert torch.equal(fin[b].cpu(), inp.state_pool[inp.state_indices[b]])


def test_largest_head_counts():
    """The largest head counts the boundary accepts (Nqk = 64, Nv = 256, GQA group 4) on ragged sequences
    that span several chunks, with a pool: the kernels' head indexing at their widest grid; the oracle on a
    spread of v-heads, the first and last of qk-head groups among them."""
    inp = inputs.make([300, 129, 1, 260], Nqk=64, Nv=256, state=("normal", 0.02, 5, "perm"), seed=121)
    for ms in (0, inp.max_seqlen):  # the chunked kernels, then the same call with a length hint
        out, fin = _gpu(inp, max_seqlen=ms)
        _check(inp, out, fin, heads=[0, 3, 4, 127, 128, 200, 255], what=f"Nqk=64 Nv=256 max_seqlen={ms}")
    short = inputs.make([3, 1, 8, 5], Nqk=64, Nv=256, state=("normal", 0.02, 6, "perm"), seed=122)
    out, fin = _gpu(short, max_seqlen=short.max_seqlen)  # the fused short-sequence kernel
    _check(short, out, fin, heads=[0, 63, 64, 255], what="short Nqk=64 Nv=256")


def test_all_sequences_empty():
    inp = inputs.make([0, 0, 0], Nqk=1, Nv=2, state=("normal", 0.02, 3, "perm"), seed=7)
    out, fin = _gpu(inp)
    assert out.shape[0] == 0
    assert torch.equal(fin.cpu(), inp.state_pool[inp.state_indices.long()])


def test_beta_zero_gives_exact_zeros():
    inp = inputs.make([300, 5], Nqk=2, Nv=4, beta=("const", 0.0), seed=8)
    out, fin = _gpu(inp)
    assert torch.count_nonzero(out) == 0 and torch.count_nonzero(fin) == 0


@pytest.mark.parametrize("gate", [("uniform_neg", 30.0, 5.0), ("uniform_neg", 1.5, 3.5), ("zero",)],
                         ids=["strong_decay", "span_near_64", "no_decay"])
def test_gate_extremes(gate):
    """Gates far below zero (e^gamma underflows inside a chunk), gates whose span over a
    16-row block straddles the kernels' switch to element-by-element decays, and gates
    of exactly zero."""
    inp = inputs.make([300, 17, 129], Nqk=2, Nv=4, g=gate, state=("normal", 0.02, 3, "perm"), seed=14)
    out, fin = _gpu(inp)
    assert torch.isfinite(out.float()).all() and torch.isfinite(fin).all()
    _check(inp, out, fin, what=f"gate {gate[0]}")


def test_every_output_written_once_nan_canary():
    inp = inputs.make([130, 0, 77], Nqk=2, Nv=2, seed=9)
    d = inp.to(DEV)
    out = torch.full((inp.T, inp.Nv, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    fin = torch.full((inp.B, inp.Nv, 128, 128), float("nan"), device=DEV)
    big = torch.full((inp.T + 64, inp.Nv, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    out = big[:inp.T]
    gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, out=out, final_state=fin)
    torch.cuda.synchronize()
    assert not torch.isnan(out).any() and not torch.isnan(fin).any()
    assert torch.isnan(big[inp.T:]).all()  # nothing written past T


def test_packed_equals_separate_bit_exact():
    inp = inputs.make([300, 129, 64], Nqk=2, Nv=4, state=("normal", 0.02, 3, "identity"), seed=10)
    out, fin = _gpu(inp)
    cu = inp.cu_seqlens
    for b in range(inp.B):
        s, e = int(cu[b]), int(cu[b + 1])
        one = inputs.GdnInputs("one", inp.q[s:e].contiguous(), inp.k[s:e].contiguous(), inp.v[s:e].contiguous(),
                               inp.g[s:e].contiguous(), inp.beta[s:e].contiguous(),
                               torch.tensor([0, e - s], dtype=torch.int32), inp.state_pool[b:b + 1].contiguous(),
                               None, inp.scale, inp.eps, [e - s])
        o1, f1 = _gpu(one)
        assert torch.equal(o1, out[s:e]) and torch.equal(f1[0], fin[b])


def test_slot_permutation_bit_exact():
    inp = inputs.make([150, 40], Nqk=1, Nv=2, state=("normal", 0.02, 5, "perm"), seed=12)
    out, fin = _gpu(inp)
    perm = torch.tensor([3, 0, 4, 1, 2])
    pool2 = torch.empty_like(inp.state_pool)
    pool2[perm] = inp.state_pool
    inp2 = inputs.GdnInputs("perm", inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, pool2,
                            perm[inp.state_indices.long()].to(torch.int32), inp.scale, inp.eps, inp.seqlens)
    out2, fin2 = _gpu(inp2)
    assert torch.equal(out, out2) and torch.equal(fin, fin2)


def test_gqa_group_heads_agree():
    inp = inputs.make([260], Nqk=2, Nv=4, seed=13)
    for h in (1, 3):  # copy v-head h-1's v, g, beta into v-head h (same qk-head group)
        inp.v[:, h] = inp.v[:, h - 1]
        inp.g[:, h] = inp.g[:, h - 1]
        inp.beta[:, h] = inp.beta[:, h - 1]
    out, fin = _gpu(inp)
    assert torch.equal(out[:, 1], out[:, 0]) and torch.equal(out[:, 3], out[:, 2])
    assert not torch.equal(out[:, 2], out[:, 0])


def test_split_and_resume():
    inp = inputs.make([700], Nqk=2, Nv=4, seed=14)
    out, fin = _gpu(inp)
    a = 333
    first = inputs.GdnInputs("a", inp.q[:a].contiguous(), inp.k[:a].contiguous(), inp.v[:a].contiguous(),
                             inp.g[:a].contiguous(), inp.beta[:a].contiguous(), torch.tensor([0, a], dtype=torch.int32),
                             None, None, inp.scale, inp.eps, [a])
    o1, f1 = _gpu(first)
    second = inputs.GdnInputs("b", inp.q[a:].contiguous(), inp.k[a:].contiguous(), inp.v[a:].contiguous(),
                              inp.g[a:].contiguous(), inp.beta[a:].contiguous(),
                              torch.tensor([0, 700 - a], dtype=torch.int32), f1.cpu(), None, inp.scale, inp.eps,
                              [700 - a])
    o2, f2 = _gpu(second)
    assert_close(torch.cat([o1, o2]), out.double().cpu().numpy(), "split out")
    assert_close(f2, fin.double().cpu().numpy(), "split final_state")


def test_short_kernel_any_length():
    """The fused kernel is the recurrence: exact for long sequences too (just slower)."""
    inp = inputs.make([40, 3, 0, 200], Nqk=2, Nv=4, state=("normal", 0.02, 4, "perm"), seed=15)
    d = inp.to(DEV)
    out, fin = gdn.short_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                             scale=inp.scale, eps=inp.eps)
    torch.cuda.synchronize()
    _check(inp, out, fin, what="short any length")


def test_workspace_given_or_internal_identical():
    inp = inputs.config("varlen_b4")
    d = inp.to(DEV)
    ws = torch.empty(gdn.workspace_bytes(inp.T, inp.B, inp.Nqk, inp.Nv), dtype=torch.uint8, device=DEV)
    o1, f1 = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices, workspace=ws)
    lib = gdn.lib()
    import ctypes
    o2 = torch.empty_like(o1)
    f2 = torch.empty_like(f1)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = lib.gdn_chunk_fwd(p(d.q), p(d.k), p(d.v), p(d.g), p(d.beta), p(d.cu_seqlens), p(d.state_pool),
                           p(d.state_indices), 0.0, 1e-6, p(o2), p(f2), inp.T, inp.B, inp.Nqk, inp.Nv, inp.P, 0,
                           None, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


# ------------------------------------------------------------------ the pipelined forward pass

def _staged(inp):
    d = inp.to(DEV)
    st = gdn.Stages(inp.T, inp.B, inp.Nqk, inp.Nv, DEV)
    out, fin = st.run_all(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                          scale=inp.scale, eps=inp.eps)
    torch.cuda.synchronize()
    return out, fin


@pytest.mark.parametrize("lens", [[32768], [3000, 5000, 129, 0, 2600], [9000, 1, 7000], [2048, 2048]],
                         ids=["one_seq", "boundary_inside_seq", "tiny_seq_between", "boundary_between_seqs"])
def test_pipelined_equals_staged_bit_exact(lens):
    """gdn_chunk_fwd runs chunk ranges as a pipeline over several streams, with the state of a
    sequence that crosses a range boundary carried in fp32: it must equal the kernels run one
    after another over all chunks, bit for bit."""
    inp = inputs.make(lens, Nqk=4, Nv=8, state=("normal", 0.02, len(lens), "perm"), seed=31)
    assert gdn.pipeline_ranges(inp.T, inp.B, inp.Nqk, inp.Nv) > 1
    out, fin = _gpu(inp)
    so, sf = _staged(inp)
    assert torch.equal(out, so) and torch.equal(fin, sf)


def test_pipelined_varlen_against_oracle():
    """A range boundary inside a sequence, an empty sequence and a 2-chunk sequence, through the
    pipelined call, against the oracle on a subset of v-heads."""
    inp = inputs.make([3000, 5000, 129, 0, 2600], Nqk=4, Nv=8, state=("normal", 0.02, 5, "perm"), seed=32)
    out, fin = _gpu(inp)
    _check(inp, out, fin, heads=[0, 3, 5], what="pipelined varlen")
