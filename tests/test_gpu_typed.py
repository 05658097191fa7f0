"""GPU parity of the chunked path with the LinearAttention page's element types (gdn_chunk_fwd_typed):
activations (q, k, v, out) fp16 or fp32 and the state (pool, final state) fp16 or fp32, beside the
decode page's bf16 activations and bf16 state, and with head dimensions other than 128 (Dk 64 or 128,
Dv up to 512), against the fp64 oracle.

The activations carry bits beyond bf16 (a small fp32 perturbation of the seeded values), so a path that
narrowed them to bf16 would show; fp16 rows enter the tensor core exactly, fp32 rows are rounded to
fp16 first (11 significant bits).  Tolerances as for the forward pass (helpers.assert_close: a 16-bit
result also carries its own half-ulp).
"""
from __future__ import annotations

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import inputs
import oracle

from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32, BF16, F16 = torch.float32, torch.bfloat16, torch.float16


def _widen(inp, act, seed):
    gen = torch.Generator().manual_seed(seed)
    return [(x.float() + 1e-3 * torch.randn(x.shape, generator=gen)).to(act) for x in (inp.q, inp.k, inp.v)]


def _oracle(q, k, v, inp, pool, rule="gated_delta"):
    ex = lambda t: None if t is None else oracle.as_numpy_exact(t)
    g = inp.g if rule in ("gated_delta", "gated") else torch.zeros_like(inp.g)
    if rule in ("gated_delta", "delta"):
        return oracle.recurrent(ex(q), ex(k), ex(v), g, inp.beta, inp.cu_seqlens, ex(pool), inp.state_indices,
                                scale=inp.scale, eps=inp.eps)
    from oracle.pool import recurrent_pool  # rules without the retrieval: the pool oracle, one slot per sequence
    P = pool.shape[0] if pool is not None else inp.B
    idx = inp.state_indices if inp.state_indices is not None else torch.arange(inp.B, dtype=torch.int32)
    slots = torch.cat([torch.full((n,), int(idx[b])) for b, n in enumerate(inp.seqlens)]).numpy().astype("int32")
    p0 = pool if pool is not None else torch.zeros(P, inp.Nv, inp.q.shape[2], inp.v.shape[2])
    ro, rpool = recurrent_pool(q, k, v, inp.g, inp.beta, inp.cu_seqlens, p0, slots, scale=inp.scale, eps=inp.eps,
                               rule=rule)
    return ro, rpool[idx.long().numpy()]


@pytest.mark.parametrize("act,state", [(F16, F32), (F16, F16), (F32, F32), (F32, F16), (BF16, BF16), (BF16, F16),
                                       (F16, BF16)])
def test_element_types_varlen_ragged(act, state):
    inp = inputs.make([300, 129, 1, 700, 0, 64], Nqk=2, Nv=4, state=("normal", 0.02, 8, "perm"), seed=95)
    q, k, v = _widen(inp, act, 96) if act != BF16 else (inp.q, inp.k, inp.v)
    pool = inp.state_pool.to(state)
    ro, rf = _oracle(q, k, v, inp, pool)
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, pool.to(DEV),
                             d.state_indices, scale=d.scale, eps=d.eps, check_status=True)
    torch.cuda.synchronize()
    assert out.dtype == act and fin.dtype == state
    assert_close(out, ro, f"{act}/{state} out")
    assert_close(fin, rf, f"{act}/{state} final_state")


def test_fp16_pipelined_ranges_and_short_hint():
    """43 chunks (two pipelined chunk ranges with a carried state); a max_seqlen hint in the short range is
    ignored by the typed path, which runs the chunked kernels."""
    inp = inputs.make([3000, 1100, 257, 5], Nqk=2, Nv=4, state=("normal", 0.02, 5, "perm"), seed=97)
    q, k, v = _widen(inp, F16, 98)
    pool = inp.state_pool.to(F16)
    ro, rf = _oracle(q, k, v, inp, pool)
    d = inp.to(DEV)
    assert gdn.pipeline_ranges(d.T, d.B, d.Nqk, d.Nv) == 2
    for ms in (0, 8):
        out, fin = gdn.chunk_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, pool.to(DEV),
                                 d.state_indices, scale=d.scale, eps=d.eps, max_seqlen=ms)
        torch.cuda.synchronize()
        assert_close(out, ro, f"fp16 pipelined out (max_seqlen={ms})")
        assert_close(fin, rf, f"fp16 pipelined final_state (max_seqlen={ms})")


@pytest.mark.parametrize("rule", ["delta", "gated", "linear"])
def test_fp32_activations_update_rules(rule):
    inp = inputs.make([200, 129, 33], Nqk=1, Nv=2, state=("normal", 0.02, 3, "identity"), seed=99)
    q, k, v = _widen(inp, F32, 100)
    ro, rf = _oracle(q, k, v, inp, inp.state_pool, rule)
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, d.state_pool,
                             d.state_indices, scale=d.scale, eps=d.eps, update_rule=rule)
    torch.cuda.synchronize()
    assert_close(out, ro, f"fp32 {rule} out")
    assert_close(fin, rf, f"fp32 {rule} final_state")


def test_fp32_activation_beyond_fp16_range_is_reported():
    inp = inputs.make([300, 40], Nqk=1, Nv=2, seed=101)
    q, k, v = _widen(inp, F32, 102)
    v[5, 1, 7] = 1.0e6  # cannot be held in fp16
    d = inp.to(DEV)
    ws = torch.empty(gdn.lib().gdn_chunk_fwd_typed_workspace_bytes(d.T, d.B, d.Nqk, d.Nv, 0, 128, 128), dtype=torch.uint8,
                     device=DEV)
    gdn.chunk_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, scale=d.scale, eps=d.eps,
                  workspace=ws)
    words = gdn.read_status(ws)
    assert words[3] & 8, words
    assert "an fp32 activation beyond the fp16 range" in gdn.decode_status(words)


@pytest.mark.parametrize("Dk,Dv,act,state", [(64, 512, BF16, F32), (128, 256, BF16, F32), (64, 128, BF16, F32),
                                             (64, 256, F16, BF16), (128, 384, F32, F16)])
def test_head_dimensions_chunked(Dk, Dv, act, state):
    """Dk != Dv in the chunked path (the decode page's example has Dk = 64, Dv = 512): Dk = 64 runs as 128
    with zero key columns, Dv = 128 m as m sub-heads per v-head sharing q, k, gate and beta."""
    inp = inputs.make([300, 129, 1, 700, 0, 64], Nqk=2, Nv=4, state=("normal", 0.02, 8, "perm"), seed=103,
                      Dk=Dk, Dv=Dv)
    q, k, v = _widen(inp, act, 104) if act != BF16 else (inp.q, inp.k, inp.v)
    pool = inp.state_pool.to(state)
    ro, rf = _oracle(q, k, v, inp, pool)
    d = inp.to(DEV)
    out, fin = gdn.chunk_fwd(q.to(DEV), k.to(DEV), v.to(DEV), d.g, d.beta, d.cu_seqlens, pool.to(DEV),
                             d.state_indices, scale=d.scale, eps=d.eps, check_status=True)
    torch.cuda.synchronize()
    assert out.shape == (inp.T, 4, Dv) and fin.shape == (inp.B, 4, Dk, Dv)
    assert_close(out, ro, f"Dk={Dk} Dv={Dv} {act}/{state} out")
    assert_close(fin, rf, f"Dk={Dk} Dv={Dv} {act}/{state} final_state")


def test_head_dimensions_pipelined_and_rules():
    """Dk = 64, Dv = 512 over two pipelined chunk ranges (a carried state per sub-head), and the gated rule."""
    inp = inputs.make([3000, 1500, 7], Nqk=1, Nv=2, state=("normal", 0.02, 3, "perm"), seed=105, Dk=64, Dv=512)
    d = inp.to(DEV)
    assert gdn.pipeline_ranges(d.T, d.B, d.Nqk, d.Nv * 4) == 2
    for rule in ("gated_delta", "gated"):
        ro, rf = _oracle(inp.q, inp.k, inp.v, inp, inp.state_pool, rule)
        out, fin = gdn.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices,
                                 scale=d.scale, eps=d.eps, update_rule=rule)
        torch.cuda.synchronize()
        assert_close(out, ro, f"Dk=64 Dv=512 {rule} out")
        assert_close(fin, rf, f"Dk=64 Dv=512 {rule} final_state")
