"""Shared pieces of the GPU parity tests: run the library through its C ABI, run the
fp64 oracle on the same bf16 inputs, and measure the errors the accuracy bounds name."""
from __future__ import annotations

import numpy as np
import torch

import oracle  # noqa: F401  (re-exported for the tests)
from exact_attention_126_b200 import build, fa, synth

# Accuracy bounds: relative Frobenius error of O <= 5e-3, max |LSE error| <= 1e-3,
# relative Frobenius error of dQ, dK, dV <= 1e-2 (over the whole tensor compared).
TOL_O = 5e-3
TOL_LSE = 1e-3
TOL_GRAD = 1e-2

_built = False


def ensure_built():
    global _built
    if not _built:
        build.build()
        _built = True


def rel_frob(x: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def run_library(inp: dict, scale: float, causal: bool, window, backward: bool = True,
                alibi=None) -> dict:
    """Runs fa_fwd (and fa_bwd) on cuda:0, or their ALiBi forms when `alibi` (H slopes) is
    given; returns host tensors."""
    ensure_built()
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    slopes = None if alibi is None else torch.tensor(alibi, dtype=torch.float32, device=dev)
    o, lse = fa.attention_forward(q, k, v, scale, causal, window, alibi_slopes=slopes)
    out = {"o": o, "lse": lse}
    if backward:
        do = inp["do"].to(dev)
        dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window,
                                           alibi_slopes=slopes)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    return {n: t.cpu() for n, t in out.items()}


def compare(inp: dict, out: dict, scale: float, causal: bool, window, heads=None,
            backward: bool = True, alibi=None) -> dict:
    """Errors of the library's outputs against the oracle, on all heads or on the listed
    (b, h) pairs (each head is an independent problem, so a subset is exact); `alibi`: the
    H slopes the library ran with, if any."""
    def pick(t):
        a = synth.to_f64(t) if t.dtype == torch.bfloat16 else t.double().numpy()
        if heads is None:
            return a
        return np.stack([a[b, h] for b, h in heads])[None]

    q, k, v = (pick(inp[n]) for n in ("q", "k", "v"))
    slopes = None
    if alibi is not None:
        slopes = list(alibi) if heads is None else [alibi[h] for _, h in heads]
    o_ref, lse_ref = oracle.fwd(q, k, v, scale, causal, window, slopes)
    errs = {
        "o": rel_frob(pick(out["o"]), o_ref),
        "lse": float(np.abs(pick(out["lse"]) - lse_ref).max()),
    }
    if backward:
        do = pick(inp["do"])
        dq_ref, dk_ref, dv_ref = oracle.bwd(q, k, v, do, scale, causal, window, slopes)
        errs["dq"] = rel_frob(pick(out["dq"]), dq_ref)
        errs["dk"] = rel_frob(pick(out["dk"]), dk_ref)
        errs["dv"] = rel_frob(pick(out["dv"]), dv_ref)
    return errs


def assert_within_bounds(errs: dict, context=""):
    assert errs["o"] <= TOL_O, (context, errs)
    assert errs["lse"] <= TOL_LSE, (context, errs)
    for g in ("dq", "dk", "dv"):
        if g in errs:
            assert errs[g] <= TOL_GRAD, (context, errs)
    for x in errs.values():
        assert np.isfinite(x), (context, errs)
