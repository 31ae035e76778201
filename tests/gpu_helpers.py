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


# The e4m3 forward's bound on relFrob(O), derived from the arithmetic (e4m3 keeps 3 mantissa
# bits; fp64 emulation of the kernel's rounding gives 2-2.5% on these inputs).
TOL_O_FP8 = 5e-2


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
                alibi=None, key_padding=None, residual: bool = True, dropout=None,
                fused: bool = False, lengths=None) -> dict:
    """Runs the forward (and backward) on cuda:0 through the C ABI and returns host tensors.
    `alibi`: H slopes; `key_padding`: a (B, N) bool host tensor (True = padded key);
    `residual`: the forward keeps O - bf16(O) for the backward's delta (the training path
    the benchmark times); False runs plain fa_fwd / fa_bwd; `dropout`: (p, seed, offset);
    `fused`: the fused backward (head_dim 64); `lengths`: B real lengths of a
    variable-length batch."""
    ensure_built()
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    slopes = None if alibi is None else torch.tensor(alibi, dtype=torch.float32, device=dev)
    kpad = None if key_padding is None else key_padding.to(dev)
    lens = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device=dev)
    res = fa.attention_forward(q, k, v, scale, causal, window, alibi_slopes=slopes,
                               key_padding=kpad, keep_residual=residual and backward,
                               dropout=dropout, seq_lengths=lens)
    o, lse = res[0], res[1]
    o_low = res[2] if len(res) > 2 else None
    out = {"o": o, "lse": lse}
    if backward:
        do = inp["do"].to(dev)
        dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window,
                                           alibi_slopes=slopes, key_padding=kpad, o_low=o_low,
                                           dropout=dropout, fused=fused,
                                           seq_lengths=lens)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    return {n: t.cpu() for n, t in out.items()}


def pack_rows(t, lens):
    """(B, H, N, d) -> (total, H, d): the first lens[b] rows of entry b, back to back."""
    return torch.cat([t[b, :, :L].transpose(0, 1) for b, L in enumerate(lens)], 0).contiguous()


def cumulative(lens):
    return [0] + list(np.cumsum(lens).astype(int))


def run_library_packed(inp, lens, scale, causal, window, **kw):
    """The same problem as a packed batch (fa_options_t.cu_seqlens) through the public calls;
    returns the outputs in the padded layout's shape for the rows < length (the rest 0 and
    LSE -inf, as the padded path writes them)."""
    ensure_built()
    dev = torch.device("cuda:0")
    B, H, N, d = inp["q"].shape
    q, k, v, do = (pack_rows(inp[n], lens).to(dev) for n in ("q", "k", "v", "do"))
    cu = torch.tensor(cumulative(lens), dtype=torch.int32, device=dev)
    o, lse, o_low = fa.attention_forward(q, k, v, scale, causal, window, keep_residual=True,
                                         cu_seqlens=cu, max_seqlen=N, **kw)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window, o_low=o_low,
                                       cu_seqlens=cu, max_seqlen=N, **kw)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    out = {}
    c = cumulative(lens)
    for n, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        full = torch.zeros((B, H, N, d), dtype=torch.bfloat16)
        t = t.cpu()
        for b, L in enumerate(lens):
            full[b, :, :L] = t[c[b]:c[b] + L].transpose(0, 1)
        out[n] = full
    full = torch.full((B, H, N), float("-inf"), dtype=torch.float32)
    lse = lse.cpu()
    for b, L in enumerate(lens):
        full[b, :, :L] = lse[:, c[b]:c[b] + L]
    out["lse"] = full
    return out


def compare(inp: dict, out: dict, scale: float, causal: bool, window, heads=None,
            backward: bool = True, alibi=None, key_padding=None, dropout=None,
            lengths=None) -> dict:
    """Errors of the library's outputs against the oracle, on all heads or on the listed
    (b, h) pairs (each head is an independent problem, so a subset is exact); `alibi`: the
    H slopes the library ran with, if any; `key_padding`: its (B, N) flags, if any.
    Rows the oracle leaves with no visible key (LSE = -inf) must have LSE = -inf exactly;
    the LSE error is taken over the other rows."""
    def pick(t):
        a = synth.to_f64(t) if t.dtype == torch.bfloat16 else t.double().numpy()
        if heads is None:
            return a
        return np.stack([a[b, h] for b, h in heads])[None]

    q, k, v = (pick(inp[n]) for n in ("q", "k", "v"))
    slopes = None
    if alibi is not None:
        slopes = list(alibi) if heads is None else [alibi[h] for _, h in heads]
    kp = None
    if key_padding is not None:
        kp = key_padding.numpy().astype(np.uint8)
        if heads is not None:
            # one batch entry per sampled head, in the layout pick() gives: (1, n, N, d)
            # tensors need (1, N) flags per head, so compare head by head instead
            raise ValueError("sampled heads with key padding are not supported")
    if dropout is not None and heads is not None:
        # the keep flags depend on the (batch, head) index, which sampling renumbers
        raise ValueError("sampled heads with dropout are not supported")
    if lengths is not None and heads is not None:
        # pick() stacks the sampled heads as the heads of one batch entry: they must share
        # a batch entry, whose real length then applies to all of them
        if len({b for b, _ in heads}) != 1:
            raise ValueError("sampled heads of a variable-length batch: one entry at a time")
        lengths = [lengths[heads[0][0]]]
    o_ref, lse_ref = oracle.fwd(q, k, v, scale, causal, window, slopes, kp, dropout, lengths)
    lse = pick(out["lse"])
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), "rows with no visible key differ"
    errs = {
        "o": rel_frob(pick(out["o"]), o_ref),
        "lse": float(np.abs(lse[~dead] - lse_ref[~dead]).max()) if (~dead).any() else 0.0,
    }
    if backward:
        do = pick(inp["do"])
        dq_ref, dk_ref, dv_ref = oracle.bwd(q, k, v, do, scale, causal, window, slopes, kp,
                                            dropout, lengths)
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
