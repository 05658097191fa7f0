"""ctypes binding of ``libgdn.so`` (include/gdn.h, include/gdn_stages.h).

Argument marshalling only: shapes and dtypes are checked, torch supplies the
device memory and the current stream, and every step of the computation runs
in the library's CUDA kernels.  There is no fallback: if the library is
missing or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")
HEAD_DIM = 128
CHUNK = 128
SHORT_MAX = 16

GDN_OK, GDN_ERR_NULL_ARG, GDN_ERR_BAD_SHAPE, GDN_ERR_UNSUPPORTED = 0, 1, 2, 3
GDN_ERR_ALIGNMENT, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, GDN_ERR_OVERLAP = 4, 5, 6, 7
GDN_ERR_SCRATCH_LIMIT = 8
NOALLOC_SCRATCH_BYTES = 64 << 20
# bits of the device status words (GDN_DEV_* in gdn.h): word 0 cu_seqlens, word 2 waits, word 3 fp16 range
DEV_BITS = {0: {1: "cu[0] != 0", 2: "cu_seqlens decreasing", 4: "cu[B] != T", 8: "a gate that is not <= 0",
                16: "a beta outside [0, 1]", 32: "a state index outside [0, P)"},
            2: {1: "a wait of the state pass gave up", 2: "a wait of the output kernel gave up",
                4: "a wait of the intra-chunk kernel gave up", 8: "the self-test wait gave up"},
            3: {1: "U (or beta v) beyond the fp16 range", 2: "the state beyond the fp16 range",
                4: "the output kernel's fp16 operand beyond the fp16 range",
                8: "an fp32 activation beyond the fp16 range"}}
# update rules of gdn_chunk_fwd_rule and gdn_recurrent_fwd (GDN_RULE_* in gdn.h)
UPDATE_RULES = {"gated_delta": 0, "delta": 1, "gated": 2, "linear": 3}
# element types of gdn_recurrent_fwd (GDN_DTYPE_* in gdn.h)
DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}

_lib = None


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("total", "status", "chunk_info", "seq_chunk0", "rq", "rk", "gcum", "betaf", "U", "W", "Mk", "Sc", "fa",
                 "carry", "act16")] + \
               [("max_chunks", ctypes.c_int64)]


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m gated_deltanet_linear_17_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_version.restype = ctypes.c_int
        L.gdn_chunk_fwd_workspace_bytes.restype = sz
        L.gdn_chunk_fwd_workspace_bytes.argtypes = [i64, i32, i32, i32]
        L.gdn_workspace_layout.restype = ctypes.c_int
        L.gdn_workspace_layout.argtypes = [i64, i32, i32, i32, ctypes.POINTER(_Layout)]
        L.gdn_chunk_fwd.restype = ctypes.c_int
        L.gdn_chunk_fwd.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, i32, p, sz, p]
        L.gdn_chunk_fwd_rule.restype = ctypes.c_int
        L.gdn_chunk_fwd_rule.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, i32, i32, p,
                                         sz, p]
        L.gdn_chunk_fwd_typed_workspace_bytes.restype = sz
        L.gdn_chunk_fwd_typed_workspace_bytes.argtypes = [i64, i32, i32, i32, i32, i32, i32]
        L.gdn_chunk_fwd_typed.restype = ctypes.c_int
        # q k v g beta cu pool idx | scale eps | out final | T B Nqk Nv P | rule act_dtype state_dtype Dk Dv
        # max_seqlen | workspace bytes stream
        L.gdn_chunk_fwd_typed.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, i32, i32,
                                          i32, i32, i32, i32, p, sz, p]
        L.gdn_chunk_fwd_noalloc.restype = ctypes.c_int
        L.gdn_chunk_fwd_noalloc.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, i32, p]
        L.gdn_selftest_umma.restype = ctypes.c_int
        L.gdn_selftest_umma.argtypes = [p, p, p, i32, i32, i32, i32, i32, p, p]
        L.gdn_selftest_wait.restype = ctypes.c_int
        L.gdn_selftest_wait.argtypes = [i32, i32, p, sz, p]
        L.gdn_chunk_fwd_host_bytes.restype = sz
        L.gdn_chunk_fwd_host_bytes.argtypes = [p, i64, i32, i32, i32, i32, i32]
        L.gdn_chunk_fwd_host.restype = ctypes.c_int
        L.gdn_chunk_fwd_host.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, i32, p, sz,
                                         p]
        L.gdn_testing_host_plan.restype = ctypes.c_int
        L.gdn_testing_host_plan.argtypes = [p, i64, i32, i32, p, i32]
        L.gdn_read_status.restype = ctypes.c_int
        L.gdn_read_status.argtypes = [p, p, p]
        L.gdn_check_values.restype = ctypes.c_int
        L.gdn_check_values.argtypes = [p, p, p, i64, i32, i32, i32, p, p]
        L.gdn_set_value_checks.restype = ctypes.c_int
        L.gdn_set_value_checks.argtypes = [ctypes.c_int]
        L.gdn_noalloc_read_status.restype = ctypes.c_int
        L.gdn_noalloc_read_status.argtypes = [p, p]
        L.gdn_short_fwd.restype = ctypes.c_int
        L.gdn_short_fwd.argtypes = [p, p, p, p, p, p, p, p, f32, f32, p, p, i64, i32, i32, i32, i32, p]
        L.gdn_recurrent_fwd.restype = ctypes.c_int
        # q k v g beta gk cu pool | act_dtype state_dtype rule | slots accepted | scale eps | out | T |
        # B Nqk Nv Dk Dv P max_seqlen | stream
        L.gdn_recurrent_fwd.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, p, p, f32, f32, p, i64, i32, i32, i32,
                                        i32, i32, i32, i32, p]
        L.gdn_recurrent_window_fwd.restype = ctypes.c_int
        # q k v g beta gk cu window | W act_dtype state_dtype rule | scale eps | out | T | B Nqk Nv Dk Dv | max_seqlen
        L.gdn_recurrent_window_fwd.argtypes = [p, p, p, p, p, p, p, p, i32, i32, i32, i32, f32, f32, p, i64, i32, i32,
                                               i32, i32, i32, i32, p]
        L.gdn_stage_chunk_map.restype = ctypes.c_int
        L.gdn_stage_chunk_map.argtypes = [p, i64, i32, i32, i32, p, sz, p]
        L.gdn_stage_intra.restype = ctypes.c_int
        L.gdn_stage_intra.argtypes = [p, p, p, p, f32, i64, i32, i32, i32, p, sz, p]
        L.gdn_stage_state.restype = ctypes.c_int
        L.gdn_stage_state.argtypes = [p, p, p, p, i64, i32, i32, i32, i32, p, sz, p]
        L.gdn_stage_output.restype = ctypes.c_int
        L.gdn_stage_output.argtypes = [p, p, p, f32, f32, p, i64, i32, i32, i32, p, sz, p]
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().gdn_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code == GDN_OK:
        return
    msg = f"{what}: {status_string(code)}"
    if code in (GDN_ERR_BAD_SHAPE, GDN_ERR_UNSUPPORTED, GDN_ERR_NULL_ARG, GDN_ERR_OVERLAP, GDN_ERR_WORKSPACE,
                GDN_ERR_ALIGNMENT, GDN_ERR_SCRATCH_LIMIT):
        raise ValueError(msg)
    raise RuntimeError(msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise RuntimeError(f"{name} must be on a CUDA device (got {t.device})")
    if device is not None and t.device != device:
        raise RuntimeError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise RuntimeError(f"{name} must be {dtype} (got {t.dtype})")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_bytes(T: int, B: int, Nqk: int, Nv: int) -> int:
    return int(lib().gdn_chunk_fwd_workspace_bytes(T, B, Nqk, Nv))


def workspace_layout(T: int, B: int, Nqk: int, Nv: int) -> dict:
    lay = _Layout()
    _check(lib().gdn_workspace_layout(T, B, Nqk, Nv, ctypes.byref(lay)), "gdn_workspace_layout")
    return {n: getattr(lay, n) for n, _ in _Layout._fields_}


def _resolve(q, k, v, g, beta, cu_seqlens, state_pool, state_indices, act=torch.bfloat16, state=torch.float32,
             dims=False):
    """Shapes of a chunked call; ``dims`` allows head dimensions other than 128 (the typed entry)."""
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q/k must be [T, Nqk, Dk] and v [T, Nv, Dv]")
    T, Nqk, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[2]
    if not dims and (Dk != HEAD_DIM or Dv != HEAD_DIM):
        raise ValueError(f"head dimension must be {HEAD_DIM}")
    if Nv % Nqk != 0:
        raise ValueError(f"Nv ({Nv}) must be a multiple of Nqk ({Nqk})")
    B = cu_seqlens.shape[0] - 1
    dev = q.device
    _need(q, "q", act, (T, Nqk, Dk), dev)
    _need(k, "k", act, (T, Nqk, Dk), dev)
    _need(v, "v", act, (T, Nv, Dv), dev)
    _need(g, "g", torch.float32, (T, Nv), dev)
    _need(beta, "beta", torch.bfloat16, (T, Nv), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    P = 0
    if state_pool is not None:
        P = state_pool.shape[0]
        _need(state_pool, "state_pool", state, (P, Nv, Dk, Dv), dev)
    if state_indices is not None:
        _need(state_indices, "state_indices", torch.int32, (B,), dev)
    return T, B, Nqk, Nv, P, dev


def chunk_fwd(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None, eps=1e-6,
              max_seqlen: int = 0, out=None, final_state=None, output_final_state=True, workspace=None,
              stream=None, update_rule="gated_delta", check_status=False, state_dtype=None):
    """Gated Delta Rule forward through ``gdn_chunk_fwd`` (``gdn_chunk_fwd_rule`` for another
    ``update_rule``: delta, gated or linear); returns (out, final_state).

    q, k [T, Nqk, 128] bf16; v [T, Nv, 128] bf16; g [T, Nv] fp32; beta [T, Nv]
    bf16; cu_seqlens [B+1] int32; state_pool [P, Nv, 128, 128] fp32 or None;
    state_indices [B] int32 or None.  All on one CUDA device.  ``max_seqlen``
    in 1..16 selects the fused short-sequence kernel.  g is not needed by the
    delta and linear rules, beta not by the gated and linear rules (pass None).
    ``check_status`` waits for the call and raises RuntimeError when the device
    status words of the chunked path report a malformed cu_seqlens, a wait that
    gave up or a value beyond the fp16 range (see ``read_status``).

    Element types (the LinearAttention page: activations and state each fp16 or
    fp32): q, k, v and out share one type, bf16, fp16 or fp32; the state pool and
    final_state share another, fp32, fp16 or bf16 (``state_dtype`` sets it when
    there is no pool; fp32 by default).  Head dimensions: Dk (q, k) 64 or 128,
    Dv (v, out, states [.., Dk, Dv]) a multiple of 128 up to 512.  Anything but
    bf16 activations with an fp32 state and 128 x 128 heads goes through
    ``gdn_chunk_fwd_typed``."""
    if update_rule not in UPDATE_RULES:
        raise ValueError(f"update_rule must be one of {sorted(UPDATE_RULES)}")
    rule = UPDATE_RULES[update_rule]
    if rule in (1, 3):
        g = None
    if rule in (2, 3):
        beta = None
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q/k must be [T, Nqk, 128] and v [T, Nv, 128]")
    act = q.dtype
    state = state_pool.dtype if state_pool is not None else (state_dtype or torch.float32)
    if act not in DTYPES or state not in DTYPES:
        raise RuntimeError(f"activations and states must be bfloat16, float16 or float32 (got {act}, {state})")
    gg = g if g is not None else torch.empty(q.shape[0], v.shape[1], dtype=torch.float32, device=q.device)
    bb = beta if beta is not None else torch.empty(q.shape[0], v.shape[1], dtype=torch.bfloat16, device=q.device)
    T, B, Nqk, Nv, P, dev = _resolve(q, k, v, gg, bb, cu_seqlens, state_pool, state_indices, act, state, dims=True)
    Dk, Dv = q.shape[2], v.shape[2]
    if out is None:
        out = torch.empty(T, Nv, Dv, dtype=act, device=dev)
    else:
        _need(out, "out", act, (T, Nv, Dv), dev)
    if final_state is None and output_final_state:
        final_state = torch.empty(B, Nv, Dk, Dv, dtype=state, device=dev)
    elif final_state is not None:
        _need(final_state, "final_state", state, (B, Nv, Dk, Dv), dev)
    typed = act != torch.bfloat16 or state != torch.float32 or Dk != HEAD_DIM or Dv != HEAD_DIM
    short = 1 <= int(max_seqlen) <= SHORT_MAX and not typed
    if workspace is None and not short and B > 0:
        nbytes = lib().gdn_chunk_fwd_typed_workspace_bytes(T, B, Nqk, Nv, DTYPES[act], Dk, Dv)
        if nbytes == 0:
            raise ValueError(f"unsupported head dimensions Dk={Dk}, Dv={Dv}")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    sc = 0.0 if scale is None else float(scale)
    if typed:
        rc = lib().gdn_chunk_fwd_typed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                       _ptr(state_pool), _ptr(state_indices), sc, float(eps), _ptr(out),
                                       _ptr(final_state), T, B, Nqk, Nv, P, rule, DTYPES[act], DTYPES[state], Dk, Dv,
                                       int(max_seqlen), _ptr(workspace), ws_bytes, _stream(stream))
        _check(rc, "gdn_chunk_fwd_typed")
    elif rule == 0:
        rc = lib().gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), _ptr(state_pool),
                                 _ptr(state_indices), sc, float(eps), _ptr(out), _ptr(final_state), T, B, Nqk, Nv, P,
                                 int(max_seqlen), _ptr(workspace), ws_bytes, _stream(stream))
        _check(rc, "gdn_chunk_fwd")
    else:
        rc = lib().gdn_chunk_fwd_rule(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                      _ptr(state_pool), _ptr(state_indices), sc, float(eps), _ptr(out),
                                      _ptr(final_state), T, B, Nqk, Nv, P, rule, int(max_seqlen), _ptr(workspace),
                                      ws_bytes, _stream(stream))
        _check(rc, "gdn_chunk_fwd_rule")
    if check_status and workspace is not None and not short:
        found = decode_status(read_status(workspace, stream))
        if found:
            raise RuntimeError("gdn_chunk_fwd: " + "; ".join(found))
    return out, final_state


def chunk_fwd_noalloc(q, k, v, g, beta, cu_seqlens, out, final_state=None, state_pool=None, state_indices=None,
                      scale=None, eps=1e-6, max_seqlen: int = 0, stream=None):
    """``gdn_chunk_fwd_noalloc``: the forward pass with no device allocation at all.

    For callers that may not allocate device memory: the caller passes every
    input and output (``out``, and ``final_state`` or None), and the library
    runs on its static per-GPU scratch (64 MiB); sizes that need more raise
    ValueError (GDN_ERR_SCRATCH_LIMIT).  Calls that may overlap on the GPU
    share that scratch and must be ordered on one stream."""
    T, B, Nqk, Nv, P, dev = _resolve(q, k, v, g, beta, cu_seqlens, state_pool, state_indices)
    _need(out, "out", torch.bfloat16, (T, Nv, HEAD_DIM), dev)
    if final_state is not None:
        _need(final_state, "final_state", torch.float32, (B, Nv, HEAD_DIM, HEAD_DIM), dev)
    sc = 0.0 if scale is None else float(scale)
    rc = lib().gdn_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                     _ptr(state_pool), _ptr(state_indices), sc, float(eps), _ptr(out),
                                     _ptr(final_state), T, B, Nqk, Nv, P, int(max_seqlen), _stream(stream))
    _check(rc, "gdn_chunk_fwd_noalloc")
    return out, final_state


def decode_status(words) -> list:
    """Human-readable findings of the four device status words (empty when all is well)."""
    words = [int(w) for w in words]
    return [msg for w, bits in DEV_BITS.items() for b, msg in bits.items() if words[w] & b]


def read_status(workspace, stream=None) -> list:
    """The workspace's four device status words (``gdn_read_status``), after the stream's work is done."""
    st = torch.cuda.current_stream() if stream is None else stream
    dst = torch.zeros(4, dtype=torch.int32, device=workspace.device)
    _check(lib().gdn_read_status(_ptr(workspace), _ptr(dst), _stream(st)), "gdn_read_status")
    st.synchronize()
    return dst.cpu().tolist()


def check_values(g=None, beta=None, state_indices=None, P=0, stream=None) -> int:
    """The value checks of ``gdn_check_values`` on device tensors g [T, Nv] fp32, beta [T, Nv] bf16 and
    state_indices [B] int32 (each optional): the GDN_DEV_VAL_* bits found (0 when every value is in range),
    after the stream's work is done."""
    ref = next((t for t in (g, beta, state_indices) if t is not None), None)
    if ref is None:
        return 0
    T, Nv = (g.shape[0], g.shape[1]) if g is not None else (beta.shape[0], beta.shape[1]) if beta is not None \
        else (0, 1)
    for t, dt in ((g, torch.float32), (beta, torch.bfloat16)):
        if t is not None:
            _need(t, "g" if dt == torch.float32 else "beta", dt, (T, Nv), ref.device)
    B = 0
    if state_indices is not None:
        _need(state_indices, "state_indices", torch.int32, (state_indices.shape[0],), ref.device)
        B = state_indices.shape[0]
    st = torch.cuda.current_stream() if stream is None else stream
    word = torch.zeros(1, dtype=torch.int32, device=ref.device)
    _check(lib().gdn_check_values(_ptr(g), _ptr(beta), _ptr(state_indices), T, B, Nv, int(P), _ptr(word),
                                  _stream(st)), "gdn_check_values")
    st.synchronize()
    return int(word.item())


def set_value_checks(on: bool) -> bool:
    """Switch the value checks of the chunked entry points on or off (``gdn_set_value_checks``); returns the
    previous setting.  With the checks on, a chunked call's status word 0 also carries the GDN_DEV_VAL_* bits."""
    return bool(lib().gdn_set_value_checks(1 if on else 0))


def noalloc_status(stream=None) -> list:
    """The four device status words of the allocation-free entry's scratch (``gdn_noalloc_read_status``),
    copied into pinned host memory without any device allocation."""
    st = torch.cuda.current_stream() if stream is None else stream
    dst = torch.zeros(4, dtype=torch.int32, pin_memory=True)
    _check(lib().gdn_noalloc_read_status(_ptr(dst), _stream(st)), "gdn_noalloc_read_status")
    st.synchronize()
    return dst.tolist()


def pipeline_ranges(T, B, Nqk=1, Nv=1):
    """Number of chunk ranges gdn_chunk_fwd pipelines for these sizes (one carry slot per boundary
    in the workspace layout)."""
    lay = workspace_layout(T, B, Nqk, Nv)
    return 1 + (lay["act16"] - lay["carry"]) // (Nv * HEAD_DIM * HEAD_DIM * 4)


def short_fwd(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None, eps=1e-6,
              out=None, final_state=None, stream=None):
    """The fused short-sequence kernel directly (``gdn_short_fwd``)."""
    T, B, Nqk, Nv, P, dev = _resolve(q, k, v, g, beta, cu_seqlens, state_pool, state_indices)
    if out is None:
        out = torch.empty(T, Nv, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = torch.empty(B, Nv, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev)
    sc = 0.0 if scale is None else float(scale)
    rc = lib().gdn_short_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens), _ptr(state_pool),
                             _ptr(state_indices), sc, float(eps), _ptr(out), _ptr(final_state), T, B, Nqk, Nv, P,
                             _stream(stream))
    _check(rc, "gdn_short_fwd")
    return out, final_state


def recurrent_fwd(q, k, v, g, beta, cu_seqlens, state_pool, token_slots, num_accepted=None, scale=None, eps=1e-6,
                  gk=None, update_rule="gated_delta", max_seqlen: int = 0, out=None, stream=None):
    """Token recurrence with the pool updated in place, one slot per token (``gdn_recurrent_fwd``).

    q, k [T, Nqk, Dk], v [T, Nv, Dv] with Dk 64 or 128 and Dv a multiple of 32, all bf16 (with an
    fp32 or bf16 pool) or all fp16 / fp32 (with an fp16 or fp32 pool, Dk = 128); ``out`` has their
    type; ``state_pool`` [P, Nv, Dk, Dv]; ``token_slots`` [T] int32 gives each token's
    slot; sequence b starts from the slot of its token ``num_accepted[b] - 1`` (its last token when
    ``num_accepted`` is None); ``gk`` [T, Nv, 128] fp32 is the optional key-dimension gate;
    ``update_rule`` is one of gated_delta, delta, gated, linear (g and gk are not needed by
    delta and linear, beta not by gated and linear: pass None).
    Returns ``out``; ``state_pool`` holds the updated states afterwards."""
    if state_pool is None or token_slots is None:
        raise ValueError("recurrent_fwd needs a state pool and a slot per token")
    if state_pool.dtype not in DTYPES or q.dtype not in DTYPES:
        raise RuntimeError(f"q/k/v and state_pool must be float32, bfloat16 or float16 (got {q.dtype}, "
                           f"{state_pool.dtype})")
    adt = q.dtype
    if update_rule not in UPDATE_RULES:
        raise ValueError(f"update_rule must be one of {sorted(UPDATE_RULES)}")
    rule = UPDATE_RULES[update_rule]
    decay, delta = rule in (0, 2), rule in (0, 1)
    if not decay:
        g = gk = None
    if not delta:
        beta = None
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q/k must be [T, Nqk, Dk] and v [T, Nv, Dv]")
    T, Nqk, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[2]
    if Nv % Nqk != 0:
        raise ValueError(f"Nv ({Nv}) must be a multiple of Nqk ({Nqk})")
    B = cu_seqlens.shape[0] - 1
    dev = q.device
    _need(q, "q", adt, (T, Nqk, Dk), dev)
    _need(k, "k", adt, (T, Nqk, Dk), dev)
    _need(v, "v", adt, (T, Nv, Dv), dev)
    if g is not None:
        _need(g, "g", torch.float32, (T, Nv), dev)
    if beta is not None:
        _need(beta, "beta", torch.bfloat16, (T, Nv), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    P = state_pool.shape[0]
    _need(state_pool, "state_pool", state_pool.dtype, (P, Nv, Dk, Dv), dev)
    _need(token_slots, "token_slots", torch.int32, (T,), dev)
    if num_accepted is not None:
        _need(num_accepted, "num_accepted", torch.int32, (B,), dev)
    if gk is not None:
        _need(gk, "gk", torch.float32, (T, Nv, Dk), dev)
    if out is None:
        out = torch.empty(T, Nv, Dv, dtype=adt, device=dev)
    else:
        _need(out, "out", adt, (T, Nv, Dv), dev)
    sc = 0.0 if scale is None else float(scale)
    rc = lib().gdn_recurrent_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gk), _ptr(cu_seqlens),
                                 _ptr(state_pool), DTYPES[adt], DTYPES[state_pool.dtype], rule, _ptr(token_slots),
                                 _ptr(num_accepted), sc,
                                 float(eps), _ptr(out), T, B, Nqk, Nv, Dk, Dv, P, int(max_seqlen), _stream(stream))
    _check(rc, "gdn_recurrent_fwd")
    return out


def recurrent_window_fwd(q, k, v, g, beta, cu_seqlens, state_window, window, scale=None, eps=1e-6, gk=None,
                         update_rule="gated_delta", max_seqlen: int = 0, out=None, stream=None):
    """Token recurrence keeping the ``window`` most recent states (``gdn_recurrent_window_fwd``).

    ``state_window`` [max(window, 1), B, Nv, Dk, Dv] holds the past window on entry (entry window - 1
    the newest; zeros for an absent past) and the present window afterwards; every other argument
    as for ``recurrent_fwd``.  Returns ``out``."""
    if update_rule not in UPDATE_RULES:
        raise ValueError(f"update_rule must be one of {sorted(UPDATE_RULES)}")
    rule = UPDATE_RULES[update_rule]
    decay, delta = rule in (0, 2), rule in (0, 1)
    if not decay:
        g = gk = None
    if not delta:
        beta = None
    if state_window is None or state_window.dtype not in DTYPES or q.dtype not in DTYPES:
        raise RuntimeError("state_window and q/k/v must be float32, bfloat16 or float16 tensors")
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q/k must be [T, Nqk, Dk] and v [T, Nv, Dv]")
    T, Nqk, Dk = q.shape
    Nv, Dv = v.shape[1], v.shape[2]
    B = cu_seqlens.shape[0] - 1
    W = max(int(window), 1)
    dev = q.device
    adt = q.dtype
    _need(q, "q", adt, (T, Nqk, Dk), dev)
    _need(k, "k", adt, (T, Nqk, Dk), dev)
    _need(v, "v", adt, (T, Nv, Dv), dev)
    if g is not None:
        _need(g, "g", torch.float32, (T, Nv), dev)
    if beta is not None:
        _need(beta, "beta", torch.bfloat16, (T, Nv), dev)
    if gk is not None:
        _need(gk, "gk", torch.float32, (T, Nv, Dk), dev)
    _need(cu_seqlens, "cu_seqlens", torch.int32, (B + 1,), dev)
    _need(state_window, "state_window", state_window.dtype, (W, B, Nv, Dk, Dv), dev)
    if out is None:
        out = torch.empty(T, Nv, Dv, dtype=adt, device=dev)
    else:
        _need(out, "out", adt, (T, Nv, Dv), dev)
    sc = 0.0 if scale is None else float(scale)
    rc = lib().gdn_recurrent_window_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(gk), _ptr(cu_seqlens),
                                        _ptr(state_window), int(window), DTYPES[adt], DTYPES[state_window.dtype], rule,
                                        sc, float(eps), _ptr(out), T, B, Nqk, Nv, Dk, Dv, int(max_seqlen),
                                        _stream(stream))
    _check(rc, "gdn_recurrent_window_fwd")
    return out


class Stages:
    """The four kernels of the chunked path as separate calls on one workspace.

    After ``run_all`` (or the individual calls in order) the intermediates are
    readable through the typed views ``U``, ``W``, ``Mk``, ``Sc``, ``rq``,
    ``rk``, ``gcum``, ``betaf``, ``chunk_info`` and ``status`` (U, W, Mk, Sc
    in fp16)."""

    def __init__(self, T, B, Nqk, Nv, device):
        self.T, self.B, self.Nqk, self.Nv = int(T), int(B), int(Nqk), int(Nv)
        self.layout = workspace_layout(T, B, Nqk, Nv)
        self.ws = torch.zeros(self.layout["total"], dtype=torch.uint8, device=device)
        self.nbytes = self.layout["total"]
        self.NC = int(self.layout["max_chunks"])

    def _view(self, name, dtype, shape):
        off = self.layout[name]
        n = int(math.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        return self.ws[off:off + n].view(dtype).view(*shape)

    @property
    def U(self):
        return self._view("U", torch.float16, (self.NC, self.Nv, CHUNK, HEAD_DIM))

    @property
    def W(self):
        return self._view("W", torch.float16, (self.NC, self.Nv, CHUNK, HEAD_DIM))

    @property
    def Mk(self):
        return self._view("Mk", torch.float16, (self.NC, self.Nv, HEAD_DIM, HEAD_DIM))

    @property
    def Sc(self):
        return self._view("Sc", torch.float16, (self.NC, self.Nv, HEAD_DIM, HEAD_DIM))

    @property
    def rq(self):
        return self._view("rq", torch.float32, (self.Nqk, self.T))

    @property
    def rk(self):
        return self._view("rk", torch.float32, (self.Nqk, self.T))

    @property
    def gcum(self):
        return self._view("gcum", torch.float32, (self.Nv, self.T))

    @property
    def betaf(self):
        return self._view("betaf", torch.float32, (self.Nv, self.T))

    @property
    def chunk_info(self):
        return self._view("chunk_info", torch.int32, (self.NC, 4))

    @property
    def status(self):
        return self._view("status", torch.int32, (4,))

    def chunk_map(self, cu_seqlens, stream=None):
        _check(lib().gdn_stage_chunk_map(_ptr(cu_seqlens), self.T, self.B, self.Nqk, self.Nv, _ptr(self.ws),
                                         self.nbytes, _stream(stream)), "gdn_stage_chunk_map")

    def intra(self, k, v, g, beta, eps=1e-6, stream=None):
        _check(lib().gdn_stage_intra(_ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(eps), self.T, self.B, self.Nqk,
                                     self.Nv, _ptr(self.ws), self.nbytes, _stream(stream)), "gdn_stage_intra")

    def state(self, k, state_pool=None, state_indices=None, final_state=None, stream=None):
        P = 0 if state_pool is None else int(state_pool.shape[0])
        _check(lib().gdn_stage_state(_ptr(k), _ptr(state_pool), _ptr(state_indices), _ptr(final_state), self.T,
                                     self.B, self.Nqk, self.Nv, P, _ptr(self.ws), self.nbytes, _stream(stream)),
               "gdn_stage_state")

    def output(self, q, k, g, out, scale=None, eps=1e-6, stream=None):
        sc = 0.0 if scale is None else float(scale)
        _check(lib().gdn_stage_output(_ptr(q), _ptr(k), _ptr(g), sc, float(eps), _ptr(out), self.T, self.B, self.Nqk,
                                      self.Nv, _ptr(self.ws), self.nbytes, _stream(stream)), "gdn_stage_output")

    def run_all(self, q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None, eps=1e-6,
                out=None, final_state=None, stream=None):
        dev = q.device
        if out is None:
            out = torch.empty(self.T, self.Nv, HEAD_DIM, dtype=torch.bfloat16, device=dev)
        if final_state is None:
            final_state = torch.empty(self.B, self.Nv, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev)
        self.chunk_map(cu_seqlens, stream)
        self.intra(k, v, g, beta, eps, stream)
        self.state(k, state_pool, state_indices, final_state, stream)
        self.output(q, k, g, out, scale, eps, stream)
        return out, final_state


def _host_tensor(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise RuntimeError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def host_plan(cu_seqlens, segments=0):
    """The cut of ``gdn_chunk_fwd_host`` into pieces (``gdn_testing_host_plan``): rows of (segment, first
    sequence, sequences, first token, end token, initial-state source, final-state target)."""
    cu = cu_seqlens.to(torch.int32).contiguous()
    B = cu.shape[0] - 1
    cap = 4 * (B + 64) + 8 * max(segments, 8)
    rows = torch.zeros(cap, 7, dtype=torch.int32)
    n = lib().gdn_testing_host_plan(_ptr(cu), int(cu[-1]), B, int(segments), _ptr(rows), cap)
    if n < 0:
        raise ValueError("invalid cu_seqlens for gdn_chunk_fwd_host")
    return rows[:n].tolist()


def host_buffer_bytes(cu_seqlens, Nqk, Nv, with_pool, segments=0) -> int:
    cu = cu_seqlens.to(torch.int32).contiguous()
    return int(lib().gdn_chunk_fwd_host_bytes(_ptr(cu), int(cu[-1]), cu.shape[0] - 1, Nqk, Nv, int(bool(with_pool)),
                                              int(segments)))


def chunk_fwd_host(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None, eps=1e-6,
                   device="cuda", out_host=None, final_host=None, device_buffer=None, segments=0, stream=None,
                   check_status=False):
    """End-to-end forward from host tensors through ``gdn_chunk_fwd_host``: the library streams the
    batch through the GPU in pieces, its uploads and downloads overlapped with the compute, and writes
    out and final_state into host tensors (pinned ones keep the copies asynchronous).  ``device_buffer``
    (uint8 on ``device``, at least ``host_buffer_bytes`` long) is allocated here when not given.
    Returns (out_host, final_host, h2d_bytes, d2h_bytes); the host tensors are complete once the
    stream has reached the end of the call (the stream is synchronised here).  The call's device status
    words, folded over its pieces, sit at the start of ``device_buffer`` (``read_status(device_buffer)``);
    ``check_status`` raises RuntimeError when they report a problem."""
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q/k must be [T, Nqk, 128] and v [T, Nv, 128]")
    T, Nqk, _ = q.shape
    Nv = v.shape[1]
    Bn = cu_seqlens.shape[0] - 1
    _host_tensor(q, "q", torch.bfloat16, (T, Nqk, HEAD_DIM))
    _host_tensor(k, "k", torch.bfloat16, (T, Nqk, HEAD_DIM))
    _host_tensor(v, "v", torch.bfloat16, (T, Nv, HEAD_DIM))
    _host_tensor(g, "g", torch.float32, (T, Nv))
    _host_tensor(beta, "beta", torch.bfloat16, (T, Nv))
    _host_tensor(cu_seqlens, "cu_seqlens", torch.int32, (Bn + 1,))
    P = 0
    if state_pool is not None:
        P = state_pool.shape[0]
        _host_tensor(state_pool, "state_pool", torch.float32, (P, Nv, HEAD_DIM, HEAD_DIM))
    if state_indices is not None:
        _host_tensor(state_indices, "state_indices", torch.int32, (Bn,))
    if out_host is None:
        out_host = torch.empty(T, Nv, HEAD_DIM, dtype=torch.bfloat16, pin_memory=True)
    if final_host is None:
        final_host = torch.empty(Bn, Nv, HEAD_DIM, HEAD_DIM, dtype=torch.float32, pin_memory=True)
    _host_tensor(out_host, "out_host", torch.bfloat16, (T, Nv, HEAD_DIM))
    _host_tensor(final_host, "final_host", torch.float32, (Bn, Nv, HEAD_DIM, HEAD_DIM))
    need = host_buffer_bytes(cu_seqlens, Nqk, Nv, state_pool is not None, segments)
    if device_buffer is None or device_buffer.numel() < need:
        device_buffer = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream(device_buffer.device) if stream is None else stream
    sc = 0.0 if scale is None else float(scale)
    rc = lib().gdn_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(cu_seqlens),
                                  _ptr(state_pool), _ptr(state_indices), sc, float(eps), _ptr(out_host),
                                  _ptr(final_host), T, Bn, Nqk, Nv, P, int(segments), _ptr(device_buffer),
                                  device_buffer.numel(), _stream(st))
    _check(rc, "gdn_chunk_fwd_host")
    st.synchronize()
    if check_status:
        found = decode_status(read_status(device_buffer, st))
        if found:
            raise RuntimeError("gdn_chunk_fwd_host: " + "; ".join(found))
    sbytes = Nv * HEAD_DIM * HEAD_DIM * 4
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v, g, beta, cu_seqlens)) + \
        (Bn * sbytes if state_pool is not None else 0)
    d2h = out_host.numel() * out_host.element_size() + final_host.numel() * final_host.element_size()
    return out_host, final_host, h2d, d2h
