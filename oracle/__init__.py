"""fp64 CPU oracle of the Gated Delta Rule forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA path never
imports this package and this package never imports the CUDA path.

Independent statements of the computation live here:

* ``recurrent``   -- the token recurrence (C, fp64), the definition that the
  GPU is compared against ("lite_boost.ops.recurrent_gated_delta_rule",
  algorithm flow; "Qwen3Next Samples", equation "L2 Normalization").
* ``chunked``     -- the chunked form of "Qwen3Next Samples"
  (chunk_gated_delta_rule, "Mathematical Formulas") in numpy fp64, with the
  chunk size as a parameter, exposing its per-chunk intermediates.
* ``transition``  -- brute-force affine transition matrices for tiny shapes.
* ``pool``, ``window`` -- the token loop with per-token pool slots (decode page)
  and with a window of recent states (LinearAttention page, state_window).
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

from . import build as _build
from .chunked import chunked, chunk_intermediates, inverse_by_block_merge, forward_substitution_inverse
from .transition import transition

__all__ = ["recurrent", "chunked", "chunk_intermediates", "transition", "inverse_by_block_merge",
           "forward_substitution_inverse", "as_numpy_exact", "load"]

_F64, _F32, _BF16 = 0, 1, 2
_lib = None


def load(path: str | None = None):
    """Load (building if needed) the C oracle shared library."""
    global _lib
    if path is not None:
        lib = ctypes.CDLL(path)
        _declare(lib)
        return lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        _declare(_lib)
    return _lib


def _declare(lib):
    p, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.gdn_oracle_recurrent.restype = ctypes.c_int
    lib.gdn_oracle_recurrent.argtypes = [
        p, ctypes.c_int, p, ctypes.c_int, p, ctypes.c_int, p, ctypes.c_int, p, ctypes.c_int,
        p, p, ctypes.c_int, p, i32, i32, i32, i32, i32, i32, ctypes.c_double, ctypes.c_double,
        p, p, p, i32, i32]


def _typed(x):
    """Return (contiguous numpy array, dtype tag) without changing any value.

    bf16 torch tensors are passed as their raw 16-bit patterns (the oracle
    widens them exactly); fp32 and fp64 pass through unchanged."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), _BF16
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, _F64
    if x.dtype == np.float32:
        return x, _F32
    if x.dtype == np.uint16:
        return x, _BF16
    raise TypeError(f"oracle input dtype {x.dtype} is not float64, float32 or bf16")


def as_numpy_exact(x) -> np.ndarray:
    """Widen a tensor/array exactly to float64 (bf16, fp16 and fp32 values are representable)."""
    try:
        import torch
        if isinstance(x, torch.Tensor) and x.dtype == torch.float16:
            return x.detach().cpu().numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    if isinstance(x, np.ndarray) and x.dtype == np.float16:
        return x.astype(np.float64)
    a, tag = _typed(x)
    if tag == _BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def recurrent(q, k, v, g, beta, cu_seqlens, state_pool=None, state_indices=None, scale=None,
              eps=1e-6, heads=None, nthreads=0, lib=None, return_threads=False):
    """Token recurrence in fp64.

    Shapes: q, k [T, Nqk, Dk]; v [T, Nv, Dv]; g, beta [T, Nv]; cu_seqlens [B+1];
    state_pool [P, Nv, Dk, Dv] or None (zero initial state); state_indices [B]
    or None (slot b).  ``scale`` None or <= 0 selects 1/sqrt(Dk), the default
    that the LinearAttention operator page gives for a zero scale.
    Returns (out [T, Nv|len(heads), Dv], final_state [B, Nv|len(heads), Dk, Dv]) as float64.
    """
    lib = lib or load()
    qa, tq = _typed(q)
    ka, tk = _typed(k)
    va, tv = _typed(v)
    ga, tg = _typed(g)
    ba, tb = _typed(beta)
    T, Nqk, Dk = qa.shape
    Nv, Dv = va.shape[1], va.shape[2]
    assert ka.shape == qa.shape and va.shape[0] == T and ga.shape == (T, Nv) and ba.shape == (T, Nv)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens if not hasattr(cu_seqlens, "numpy")
                                         else cu_seqlens.cpu().numpy(), dtype=np.int32))
    B = cu.shape[0] - 1
    if state_pool is not None:
        pa, tp = _typed(state_pool)
        P = pa.shape[0]
    else:
        pa, tp, P = None, _F64, 0
    idx = None
    if state_indices is not None:
        idx = np.ascontiguousarray(np.asarray(state_indices if not hasattr(state_indices, "numpy")
                                              else state_indices.cpu().numpy(), dtype=np.int32))
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(Dk)
    hl = None
    nh = Nv
    if heads is not None:
        hl = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
        nh = hl.shape[0]
    out = np.zeros((T, nh, Dv), dtype=np.float64)
    fin = np.zeros((B, nh, Dk, Dv), dtype=np.float64)
    rc = lib.gdn_oracle_recurrent(
        _ptr(qa), tq, _ptr(ka), tk, _ptr(va), tv, _ptr(ga), tg, _ptr(ba), tb, _ptr(cu),
        _ptr(pa), tp, _ptr(idx), B, Nqk, Nv, Dk, Dv, P, float(scale), float(eps),
        _ptr(out), _ptr(fin), _ptr(hl), nh if hl is not None else 0, int(nthreads))
    if rc < 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    if return_threads:
        return out, fin, rc
    return out, fin
