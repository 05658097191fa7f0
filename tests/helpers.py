"""Helpers shared by the tests: tolerance checks and oracle runs on seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerance of the GPU path against the fp64 oracle (bf16 inputs and outputs,
# fp32 accumulation and state): per tensor, relative L2 error <= 1e-2 and
# max-abs error <= 2e-2 * RMS(reference).  For a bf16 result the bound on each
# element also includes that element's own bf16 rounding, half an ulp
# (<= 2^-8 |ref|): bf16 keeps 8 significant bits, so an output element larger
# than ~5 RMS cannot be stored closer than 2e-2 RMS to the exact value.
REL_L2 = 1e-2
MAX_ABS_RMS = 2e-2
BF16_HALF_ULP = 2.0 ** -8
FP16_HALF_ULP = 2.0 ** -11   # for fp16 intermediates (11 significant bits)


def errors(got, ref, ulp_rel=0.0):
    """(relative L2 error, max over elements of |got - ref| - ulp_rel |ref|, RMS(ref))."""
    got = got.detach().cpu().double().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    d = got - ref
    nref = np.linalg.norm(ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    rel = float(np.linalg.norm(d) / nref) if nref > 0 else float(np.linalg.norm(d))
    mx = float(np.max(np.abs(d) - ulp_rel * np.abs(ref))) if d.size else 0.0
    return rel, mx, rms


def assert_close(got, ref, what, rel_l2=REL_L2, max_abs_rms=MAX_ABS_RMS, ulp=None):
    """Tolerance check; a bf16 (fp16) tensor gets its own half-ulp added per element."""
    if ulp is None:
        dt = got.dtype if isinstance(got, torch.Tensor) else None
        ulp = BF16_HALF_ULP if dt == torch.bfloat16 else FP16_HALF_ULP if dt == torch.float16 else 0.0
    rel, mx, rms = errors(got, ref, ulp)
    if rms == 0.0:
        assert mx <= 0.0, f"{what}: reference is zero, max abs {mx:.3e}"
        return rel, mx
    assert rel <= rel_l2, f"{what}: rel L2 {rel:.3e} > {rel_l2:.1e} (max abs {mx:.3e}, rms {rms:.3e})"
    assert mx <= max_abs_rms * rms, (f"{what}: max abs (beyond the storage half-ulp) {mx:.3e} > {max_abs_rms:.1e}"
                                     f" * rms {rms:.3e} (rel L2 {rel:.3e})")
    return rel, mx


def run_oracle(inp, heads=None, nthreads=0):
    """fp64 oracle on a GdnInputs batch (CPU tensors), optionally on a subset of v-heads."""
    return oracle.recurrent(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.state_pool,
                            inp.state_indices, scale=inp.scale, eps=inp.eps, heads=heads, nthreads=nthreads)
