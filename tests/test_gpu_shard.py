"""The multi-GPU split of the forward pass, recombined on one GPU (bit for bit).

The operator has no exchange step: sequences and the v-head groups of the
qk-heads are independent problems.  ``dist.shard_heads`` and
``dist.shard_sequences`` give each rank a contiguous block of them; here each
block runs as its own gdn_chunk_fwd call (what a rank would run) and the
pieces, put back together, must equal the unsharded call exactly -- including
when a piece changes how many chunk ranges the call pipelines.
"""
from __future__ import annotations

import pytest
import torch

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import dist, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run(d, q, k, v, g, beta, cu, pool, idx):
    return gdn.chunk_fwd(q, k, v, g, beta, cu, pool, idx, scale=d.scale, eps=d.eps)


@pytest.mark.parametrize("name,world", [("varlen_b4", 2), ("varlen_b4", 4), ("prefill_s32k", 2)])
def test_head_shards_recombine_exactly(name, world):
    d = inputs.config(name).to(DEV)
    out, fin = _run(d, d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices)
    parts_o, parts_f = [], []
    for r in range(world):
        a, b, va, vb = dist.shard_heads(d.Nqk, d.Nv, world, r)
        pool = None if d.state_pool is None else d.state_pool[:, va:vb].contiguous()
        o, f = _run(d, d.q[:, a:b].contiguous(), d.k[:, a:b].contiguous(), d.v[:, va:vb].contiguous(),
                    d.g[:, va:vb].contiguous(), d.beta[:, va:vb].contiguous(), d.cu_seqlens, pool, d.state_indices)
        parts_o.append(o)
        parts_f.append(f)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts_o, 1), out)
    assert torch.equal(torch.cat(parts_f, 1), fin)


@pytest.mark.parametrize("lens,world", [([1000, 513, 128, 2407], 2), ([3000, 1, 129, 4100, 0, 700], 3)])
def test_sequence_shards_recombine_exactly(lens, world):
    d = inputs.make(lens, Nqk=2, Nv=4, state=("normal", 0.02, len(lens) + 2, "perm"), seed=51).to(DEV)
    out, fin = _run(d, d.q, d.k, d.v, d.g, d.beta, d.cu_seqlens, d.state_pool, d.state_indices)
    cu = d.cu_seqlens.cpu().tolist()
    ranges = set()
    parts_o, parts_f = [], []
    for r in range(world):
        b0, b1 = dist.shard_sequences(lens, world, r)
        t0, t1 = cu[b0], cu[b1]
        sub_cu = torch.tensor([c - t0 for c in cu[b0:b1 + 1]], dtype=torch.int32, device=DEV)
        ranges.add(gdn.pipeline_ranges(t1 - t0, b1 - b0, d.Nqk, d.Nv))
        if b1 == b0:
            continue
        o, f = _run(d, d.q[t0:t1], d.k[t0:t1], d.v[t0:t1], d.g[t0:t1], d.beta[t0:t1], sub_cu, d.state_pool,
                    d.state_indices[b0:b1].contiguous())
        parts_o.append(o)
        parts_f.append(f)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts_o, 0), out)
    assert torch.equal(torch.cat(parts_f, 0), fin)
    # the unsharded call pipelines two chunk ranges; at least one shard runs with another count
    assert gdn.pipeline_ranges(d.T, d.B, d.Nqk, d.Nv) == 2 and ranges != {2}
