"""The C-ABI library loads, exports every symbol its headers declare, and
rejects bad arguments before touching a GPU (CPU only: no call here enqueues work)."""
from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

import gated_deltanet_linear_17_b200 as gdn
from gated_deltanet_linear_17_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"\b(gdn_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("libgdn.so not built")
    return gdn.lib()


def test_headers_declare_entry_points():
    names = _declared()
    for n in ("gdn_chunk_fwd", "gdn_chunk_fwd_workspace_bytes", "gdn_status_string", "gdn_short_fwd",
              "gdn_stage_intra", "gdn_stage_state", "gdn_stage_output", "gdn_read_status",
              "gdn_noalloc_read_status", "gdn_selftest_wait", "gdn_check_values", "gdn_set_value_checks"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings(lib):
    for code in range(0, 9):
        assert gdn.status_string(code).startswith("GDN_")
    assert "UNKNOWN" in gdn.status_string(99)


def test_workspace_layout_regions_disjoint_and_aligned(lib):
    lay = gdn.workspace_layout(4048, 4, 4, 8)
    assert lay["max_chunks"] == (4048 + 127 * 4) // 128
    regions = ["status", "chunk_info", "seq_chunk0", "rq", "rk", "gcum", "betaf", "U", "W", "Mk", "Sc", "fa", "carry"]
    offs = [lay[r] for r in regions]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    tile = 128 * 128 * 2
    assert lay["W"] - lay["U"] == lay["max_chunks"] * 8 * tile
    assert lay["fa"] >= lay["Sc"] + lay["max_chunks"] * 8 * tile
    assert lay["carry"] >= lay["fa"] + lay["max_chunks"] * 8 * 132 * 4
    assert lay["total"] >= lay["carry"]  # few chunks: one range, no carry slots
    big = gdn.workspace_layout(32768, 1, 16, 32)  # 256 chunks: 2 ranges, 1 carry slot
    assert big["total"] >= big["carry"] + 32 * 128 * 128 * 4
    assert gdn.pipeline_ranges(32768, 1, 16, 32) == 2 and gdn.pipeline_ranges(3000, 1, 16, 32) == 1
    assert gdn.workspace_bytes(4048, 4, 4, 8) == lay["total"]


def test_max_chunks_is_an_upper_bound():
    # floor((T + 127 B) / 128) >= sum(ceil(len / 128)) for every packing
    import random
    r = random.Random(0)
    for _ in range(2000):
        Bn = r.randint(1, 12)
        lens = [r.choice([0, 1, 127, 128, 129, r.randint(0, 700)]) for _ in range(Bn)]
        T = sum(lens)
        assert sum((n + 127) // 128 for n in lens) <= (T + 127 * Bn) // 128


def _call(lib, **over):
    M = 1 << 20  # fake, disjoint, 16-byte aligned addresses (never dereferenced)
    a = dict(q=1 * M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, cu=6 * M, pool=None, idx=None, scale=0.0,
             eps=1e-6, out=7 * M, fin=None, T=8, B=1, Nqk=2, Nv=4, P=0, max_seqlen=0, ws=None, wsb=0,
             stream=None)
    a.update(over)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_chunk_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]), vp(a["cu"]),
                             vp(a["pool"]), vp(a["idx"]), a["scale"], a["eps"], vp(a["out"]), vp(a["fin"]),
                             a["T"], a["B"], a["Nqk"], a["Nv"], a["P"], a["max_seqlen"], vp(a["ws"]), a["wsb"],
                             vp(a["stream"]))


def test_argument_errors_before_any_launch(lib):
    # These return before any CUDA call (the fake addresses are never dereferenced).
    assert _call(lib, Nv=3) == B.GDN_ERR_BAD_SHAPE            # Nv not a multiple of Nqk
    assert _call(lib, T=-1) == B.GDN_ERR_BAD_SHAPE
    assert _call(lib, Nqk=0) == B.GDN_ERR_BAD_SHAPE
    assert _call(lib, P=-1) == B.GDN_ERR_BAD_SHAPE
    assert _call(lib, q=None) == B.GDN_ERR_NULL_ARG
    assert _call(lib, cu=None) == B.GDN_ERR_NULL_ARG
    assert _call(lib, q=(1 << 20) + 8) == B.GDN_ERR_ALIGNMENT  # not 16-byte aligned
    assert _call(lib, out=3 << 20) == B.GDN_ERR_OVERLAP           # out aliases v
    assert _call(lib, pool=9 << 20, P=1, B=2) == B.GDN_ERR_BAD_SHAPE   # P < B without indices
    assert _call(lib, pool=9 << 20, P=1, fin=9 << 20) == B.GDN_ERR_OVERLAP
    assert _call(lib, Nqk=128, Nv=128) == B.GDN_ERR_UNSUPPORTED
    assert _call(lib, T=1 << 31) == B.GDN_ERR_UNSUPPORTED
    assert _call(lib, B=0) == B.GDN_OK                        # empty batch: nothing to do
    assert _call(lib, ws=8 << 20, wsb=10) == B.GDN_ERR_WORKSPACE  # caller workspace too small
    assert _call(lib, ws=(8 << 20) + 4, wsb=1 << 40) == B.GDN_ERR_ALIGNMENT


def _call_recurrent(lib, **over):
    M = 1 << 20  # fake, disjoint, aligned addresses; every call below returns before any launch
    a = dict(q=1 * M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, gk=None, cu=6 * M, pool=9 * M, act=1, bf16=0, rule=0,
             slots=10 * M, acc=None, scale=0.0, eps=1e-6, out=7 * M, T=8, B=1, Nqk=2, Nv=4, Dk=128, Dv=128, P=2,
             max_seqlen=0, stream=None)
    a.update(over)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return lib.gdn_recurrent_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]), vp(a["gk"]),
                                 vp(a["cu"]), vp(a["pool"]), a["act"], a["bf16"], a["rule"], vp(a["slots"]), vp(a["acc"]),
                                 a["scale"],
                                 a["eps"], vp(a["out"]), a["T"], a["B"], a["Nqk"], a["Nv"], a["Dk"], a["Dv"], a["P"],
                                 a["max_seqlen"],
                                 vp(a["stream"]))


def test_recurrent_argument_errors_before_any_launch(lib):
    M = 1 << 20
    assert _call_recurrent(lib, pool=None) == B.GDN_ERR_NULL_ARG
    assert _call_recurrent(lib, slots=None) == B.GDN_ERR_NULL_ARG
    assert _call_recurrent(lib, P=0) == B.GDN_ERR_BAD_SHAPE
    assert _call_recurrent(lib, Nv=3) == B.GDN_ERR_BAD_SHAPE
    assert _call_recurrent(lib, bf16=3) == B.GDN_ERR_BAD_SHAPE             # unknown pool type code
    assert _call_recurrent(lib, act=5) == B.GDN_ERR_BAD_SHAPE              # unknown activation type code
    assert _call_recurrent(lib, act=1, bf16=2) == B.GDN_ERR_UNSUPPORTED     # bf16 activations, fp16 pool
    assert _call_recurrent(lib, act=2, bf16=1) == B.GDN_ERR_UNSUPPORTED     # fp16 activations, bf16 pool
    assert _call_recurrent(lib, act=0, Dk=64) == B.GDN_ERR_UNSUPPORTED      # fp32 activations need Dk = 128
    assert _call_recurrent(lib, act=2, bf16=2, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT  # accepted pair
    assert _call_recurrent(lib, rule=4) == B.GDN_ERR_BAD_SHAPE
    assert _call_recurrent(lib, Dk=96) == B.GDN_ERR_UNSUPPORTED
    assert _call_recurrent(lib, Dv=48) == B.GDN_ERR_UNSUPPORTED
    assert _call_recurrent(lib, Dv=96, bf16=1) == B.GDN_ERR_UNSUPPORTED   # a bf16 pool: Dv a multiple of 64
    assert _call_recurrent(lib, Dv=0) == B.GDN_ERR_BAD_SHAPE
    assert _call_recurrent(lib, Dk=64, Dv=512, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT  # accepted sizes
    assert _call_recurrent(lib, g=None) == B.GDN_ERR_NULL_ARG             # the gated delta rule reads g
    # rules that do not read g / beta accept NULL there (each call still stops at a later check)
    assert _call_recurrent(lib, beta=None, rule=2, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, g=None, rule=1, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, g=None, beta=None, rule=3, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, beta=None) == B.GDN_ERR_NULL_ARG          # and beta
    assert _call_recurrent(lib, slots=10 * M + 2) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, acc=11 * M + 1) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, pool=9 * M + 8) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, gk=12 * M + 4) == B.GDN_ERR_ALIGNMENT
    assert _call_recurrent(lib, out=9 * M) == B.GDN_ERR_OVERLAP          # out inside the pool
    assert _call_recurrent(lib, out=9 * M, bf16=1) == B.GDN_ERR_OVERLAP  # also for a bf16 pool
    assert _call_recurrent(lib, out=12 * M, gk=12 * M) == B.GDN_ERR_OVERLAP
    assert _call_recurrent(lib, out=3 * M) == B.GDN_ERR_OVERLAP          # out aliases v
    assert _call_recurrent(lib, B=0) == B.GDN_OK                         # nothing to do
    assert _call_recurrent(lib, T=0, B=1) == B.GDN_OK


def test_stage_argument_errors(lib):
    vp = ctypes.c_void_p
    x = vp(16)
    assert lib.gdn_stage_intra(x, x, x, x, 1e-6, 8, 1, 2, 4, None, 0, None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_stage_intra(x, x, x, x, 1e-6, 8, 1, 2, 4, x, 10, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_stage_output(x, x, x, 0.0, 1e-6, x, 8, 1, 2, 3, x, 1 << 30, None) == B.GDN_ERR_BAD_SHAPE


def test_python_layer_refuses_cpu_tensors():
    import torch
    from gated_deltanet_linear_17_b200 import inputs
    inp = inputs.make([5], 1, 2, seed=0)
    with pytest.raises(RuntimeError):
        gdn.chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens)


def test_value_checks_refuse_cpu_tensors():
    import torch
    from gated_deltanet_linear_17_b200 import inputs
    inp = inputs.make([5, 3], 1, 2, state=("normal", 0.02, 2, "perm"), seed=0)
    with pytest.raises(RuntimeError):
        gdn.check_values(inp.g, inp.beta)
    with pytest.raises(RuntimeError):
        gdn.check_values(state_indices=inp.state_indices, P=2)
    assert gdn.check_values() == 0  # nothing to check


def _noalloc(lib, **over):
    M = 1 << 20  # fake, disjoint, 16-byte aligned addresses; every call below returns before any launch
    a = dict(T=8, B=1, Nqk=2, Nv=4, P=0, max_seqlen=0)
    a.update(over)
    vp = ctypes.c_void_p
    return lib.gdn_chunk_fwd_noalloc(vp(M), vp(2 * M), vp(3 * M), vp(4 * M), vp(5 * M), vp(6 * M), None, None, 0.0,
                                     1e-6, vp(7 * M), None, a["T"], a["B"], a["Nqk"], a["Nv"], a["P"],
                                     a["max_seqlen"], None)


def test_noalloc_refuses_bad_shapes_before_the_scratch_limit(lib):
    # sizes large enough to exceed the scratch, but invalid for gdn_chunk_fwd too: the shape code wins
    assert _noalloc(lib, T=1 << 20, Nqk=2, Nv=3) == B.GDN_ERR_BAD_SHAPE
    assert _noalloc(lib, T=1 << 20, Nqk=128, Nv=128) == B.GDN_ERR_UNSUPPORTED
    assert _noalloc(lib, T=1 << 20, P=-1) == B.GDN_ERR_BAD_SHAPE
    assert _noalloc(lib, T=1 << 20, Nqk=16, Nv=32) == B.GDN_ERR_SCRATCH_LIMIT
    # the stated limit: one sequence of 1920 tokens at Nqk = 16, Nv = 32 fits, 1921 does not
    assert gdn.workspace_bytes(1920, 1, 16, 32) <= B.NOALLOC_SCRATCH_BYTES < gdn.workspace_bytes(1921, 1, 16, 32)
    assert _noalloc(lib, T=1921, Nqk=16, Nv=32) == B.GDN_ERR_SCRATCH_LIMIT
    assert "1920 tokens" in open(os.path.join(ROOT, "include", "gdn.h")).read()


def test_status_entry_argument_errors(lib):
    vp = ctypes.c_void_p
    assert lib.gdn_read_status(None, vp(1 << 20), None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_read_status(vp(1 << 20), None, None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_read_status(vp((1 << 20) + 8), vp(2 << 20), None) == B.GDN_ERR_ALIGNMENT
    assert lib.gdn_read_status(vp(1 << 20), vp((2 << 20) + 2), None) == B.GDN_ERR_ALIGNMENT
    assert lib.gdn_noalloc_read_status(None, None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_selftest_wait(16, 0, None, 16, None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_selftest_wait(16, 0, vp((1 << 20) + 4), 16, None) == B.GDN_ERR_ALIGNMENT
    assert lib.gdn_selftest_wait(16, 0, vp(1 << 20), 8, None) == B.GDN_ERR_WORKSPACE
    assert lib.gdn_selftest_wait(0, 0, vp(1 << 20), 16, None) == B.GDN_ERR_BAD_SHAPE
    assert lib.gdn_selftest_wait((1 << 22) + 1, 0, vp(1 << 20), 16, None) == B.GDN_ERR_BAD_SHAPE


def test_value_check_entry_argument_errors(lib):
    """gdn_check_values refuses bad arguments before it enqueues anything; the switch of the chunked
    entry points is process-wide and returns its previous setting."""
    vp = ctypes.c_void_p
    g, beta, idx, word = vp(1 << 20), vp(2 << 20), vp(3 << 20), vp(4 << 20)
    assert lib.gdn_check_values(g, beta, idx, 100, 2, 4, 8, None, None) == B.GDN_ERR_NULL_ARG
    assert lib.gdn_check_values(g, beta, idx, -1, 2, 4, 8, word, None) == B.GDN_ERR_BAD_SHAPE
    assert lib.gdn_check_values(g, beta, idx, 100, -2, 4, 8, word, None) == B.GDN_ERR_BAD_SHAPE
    assert lib.gdn_check_values(g, beta, idx, 100, 2, 0, 8, word, None) == B.GDN_ERR_BAD_SHAPE
    assert lib.gdn_check_values(g, beta, idx, 100, 2, 4, -1, word, None) == B.GDN_ERR_BAD_SHAPE
    assert lib.gdn_check_values(vp((1 << 20) + 2), beta, idx, 100, 2, 4, 8, word, None) == B.GDN_ERR_ALIGNMENT
    assert lib.gdn_check_values(g, vp((2 << 20) + 1), idx, 100, 2, 4, 8, word, None) == B.GDN_ERR_ALIGNMENT
    assert lib.gdn_check_values(g, beta, idx, 100, 2, 4, 8, vp((4 << 20) + 2), None) == B.GDN_ERR_ALIGNMENT
    # nothing to check: no launch, GDN_OK
    assert lib.gdn_check_values(None, None, None, 100, 0, 4, 8, word, None) == B.GDN_OK
    assert gdn.set_value_checks(True) is False
    assert gdn.set_value_checks(False) is True
    assert gdn.set_value_checks(False) is False


def test_status_bits_match_the_header():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    macros = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define (GDN_DEV_\w+) (\d+)", text)}
    word = {"CU": 0, "VAL": 0, "WAIT": 2, "RANGE": 3}
    for name, bit in macros.items():
        assert bit in B.DEV_BITS[word[name.split("_")[2]]], name
    assert sum(len(v) for v in B.DEV_BITS.values()) == len(macros)
    assert gdn.decode_status([0, 5, 0, 0]) == []
    assert gdn.decode_status([2, 5, 4, 2]) == ["cu_seqlens decreasing", "a wait of the intra-chunk kernel gave up",
                                               "the state beyond the fp16 range"]


def test_window_entry_argument_errors(lib):
    M = 1 << 20  # fake, disjoint, aligned addresses; every call below returns before any launch
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(**over):
        a = dict(q=M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, gk=None, cu=6 * M, win=9 * M, W=4, act=1, sdt=0,
                 rule=0, out=7 * M, T=8, B=1, Nqk=2, Nv=4, Dk=128, Dv=128)
        a.update(over)
        return lib.gdn_recurrent_window_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]),
                                            vp(a["gk"]), vp(a["cu"]), vp(a["win"]), a["W"], a["act"], a["sdt"],
                                            a["rule"], 0.0, 1e-6, vp(a["out"]), a["T"], a["B"], a["Nqk"], a["Nv"],
                                            a["Dk"], a["Dv"], 0, None)
    assert call(W=9) == B.GDN_ERR_BAD_SHAPE and call(W=-1) == B.GDN_ERR_BAD_SHAPE
    assert call(win=None) == B.GDN_ERR_NULL_ARG
    assert call(Nv=3) == B.GDN_ERR_BAD_SHAPE
    assert call(act=2, sdt=1) == B.GDN_ERR_UNSUPPORTED
    assert call(win=9 * M + 8) == B.GDN_ERR_ALIGNMENT
    entry = 1 * 4 * 128 * 128 * 4  # bytes of one window entry at B = 1, Nv = 4, fp32
    assert call(out=9 * M) == B.GDN_ERR_OVERLAP                    # out inside the window buffer
    assert call(out=9 * M + 3 * entry) == B.GDN_ERR_OVERLAP        # inside entry 3 of a 4-entry window
    assert call(out=9 * M + 3 * entry, W=3, g=None) == B.GDN_ERR_NULL_ARG  # past a 3-entry window: later checks
    assert call(B=0) == B.GDN_OK and call(T=0) == B.GDN_OK
    assert call(W=0, g=None) == B.GDN_ERR_NULL_ARG                  # the gated delta rule reads g


def test_typed_entry_argument_errors(lib):
    M = 1 << 20  # fake, disjoint, aligned addresses; every call below returns before any launch
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(**over):
        a = dict(q=M, k=2 * M, v=3 * M, g=4 * M, beta=5 * M, cu=6 * M, pool=None, out=7 * M, fin=None, T=8, B=1,
                 Nqk=2, Nv=4, P=0, rule=0, act=2, sdt=0, Dk=128, Dv=128, ws=None, wsb=0)
        a.update(over)
        return lib.gdn_chunk_fwd_typed(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["g"]), vp(a["beta"]), vp(a["cu"]),
                                       vp(a["pool"]), None, 0.0, 1e-6, vp(a["out"]), vp(a["fin"]), a["T"], a["B"],
                                       a["Nqk"], a["Nv"], a["P"], a["rule"], a["act"], a["sdt"], a["Dk"], a["Dv"], 0,
                                       vp(a["ws"]), a["wsb"], None)
    assert call(act=3) == B.GDN_ERR_BAD_SHAPE and call(sdt=-1) == B.GDN_ERR_BAD_SHAPE
    assert call(rule=4) == B.GDN_ERR_BAD_SHAPE
    assert call(Nv=3) == B.GDN_ERR_BAD_SHAPE
    assert call(q=None) == B.GDN_ERR_NULL_ARG
    # fp32 activations: out (4 bytes per element) overlaps v when 16 KiB apart
    assert call(act=0, out=3 * M + 8 * 4 * 128 * 2) == B.GDN_ERR_OVERLAP
    assert call(ws=8 << 20, wsb=10) == B.GDN_ERR_WORKSPACE
    # the fp32-activation workspace holds their fp16 copies on top of the 16-bit one
    w16 = lib.gdn_chunk_fwd_typed_workspace_bytes(4096, 2, 4, 8, 2, 128, 128)
    w32 = lib.gdn_chunk_fwd_typed_workspace_bytes(4096, 2, 4, 8, 0, 128, 128)
    assert w16 == gdn.workspace_bytes(4096, 2, 4, 8) and w32 >= w16 + (2 * 4 + 8) * 4096 * 128 * 2
    # head dimensions: Dv = 512 runs as four 128-column sub-heads per v-head; Dk 64 or 128 only
    assert lib.gdn_chunk_fwd_typed_workspace_bytes(4096, 2, 4, 8, 2, 64, 512) == gdn.workspace_bytes(4096, 2, 4, 32)
    assert lib.gdn_chunk_fwd_typed_workspace_bytes(4096, 2, 4, 8, 2, 96, 128) == 0
    assert lib.gdn_chunk_fwd_typed_workspace_bytes(4096, 2, 4, 8, 2, 128, 192) == 0
    assert call(Dk=96) == B.GDN_ERR_UNSUPPORTED and call(Dv=640) == B.GDN_ERR_UNSUPPORTED
    assert call(Dv=192) == B.GDN_ERR_UNSUPPORTED and call(Dk=0) == B.GDN_ERR_BAD_SHAPE
    assert call(Nqk=64, Nv=128, Dv=512) == B.GDN_ERR_UNSUPPORTED  # 512 sub-heads of 128 columns
    # out of a Dv = 512 call (4 bytes per fp32 element) overlaps v when 64 KiB apart
    assert call(act=0, Dk=64, Dv=512, out=3 * M + 8 * 4 * 512 * 2) == B.GDN_ERR_OVERLAP
