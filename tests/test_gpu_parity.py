"""The CUDA path against the fp64 oracle, element by element, on the same seeded bf16
inputs: small and ragged shapes in every mask mode, the five workloads at full size (all
heads where the oracle is quick, sampled heads otherwise), inputs that drive the online
softmax's rescaling, and degenerate inputs."""
import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth
from exact_attention_126_b200.workloads import WORKLOADS, alibi_slopes

pytestmark = pytest.mark.gpu

MODES = {
    "none": (False, (-1, -1)),
    "causal": (True, (-1, -1)),
    "win64_0": (False, (64, 0)),
    "win100_30": (False, (100, 30)),
    "causal_win200": (True, (200, -1)),
}


def inputs(B, H, N, d, seed_index):
    return synth.attention_inputs(B, H, N, d, seed_index)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300])
@pytest.mark.parametrize("mode", list(MODES))
def test_small_and_ragged(N, d, mode):
    causal, window = MODES[mode]
    inp = inputs(2, 2, N, d, 100 + N + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, causal, window)
    errs = G.compare(inp, out, scale, causal, window)
    G.assert_within_bounds(errs, (N, d, mode))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["none", "causal", "win100_30"])
def test_many_items_per_cta(d, mode):
    """More (head, tile) work items than SMs, so every persistent CTA runs several items
    back to back (the stationary tiles, accumulators and barrier phases carry over)."""
    causal, window = MODES[mode]
    B, H, N = 4, 64, 384  # 256 heads x 3 tiles = 768 items per kernel
    inp = inputs(B, H, N, d, 800 + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, causal, window)
    heads = [(0, 0), (1, 17), (2, 40), (3, 63)]
    errs = G.compare(inp, out, scale, causal, window, heads)
    G.assert_within_bounds(errs, (d, mode))
    for n in ("o", "dq", "dk", "dv"):
        assert torch.isfinite(out[n].float()).all(), n


def _sampled_heads(w, count=4):
    rng = np.random.default_rng(w.seed_index)
    BH = w.B * w.H
    picks = {0, BH - 1}
    while len(picks) < min(count, BH):
        picks.add(int(rng.integers(0, BH)))
    return [(p // w.H, p % w.H) for p in sorted(picks)]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_full_size(name):
    """The launch configuration the benchmark times, checked on all heads (c1..c3) or on
    the first, the last and two seeded random (batch, head) pairs (c4, c5)."""
    w = WORKLOADS[name]
    inp = inputs(w.B, w.H, w.N, w.d, w.seed_index)
    heads = None if w.B * w.H * w.N <= 2 * 8 * 4096 else _sampled_heads(w)
    if w.fp8:
        # the e4m3 forward on the seeded inputs rounded to e4m3 (descales 1), against the
        # oracle on exactly those values, at the FP8 bound on O
        G.ensure_built()
        dev = torch.device("cuda:0")
        x8 = {n: inp[n].float().to(torch.float8_e4m3fn) for n in ("q", "k", "v")}
        o, lse = fa.attention_forward_fp8(x8["q"].to(dev), x8["k"].to(dev), x8["v"].to(dev),
                                          scale=w.softmax_scale, causal=w.causal,
                                          window=w.window)
        torch.cuda.synchronize()
        assert fa.fa_debug_status() == 0
        ref = {n: x8[n].to(torch.float64).numpy() for n in ("q", "k", "v")}
        pick = lambda a: np.stack([a[b, h] for b, h in heads])[None]
        o_ref, lse_ref = G.oracle.fwd(pick(ref["q"]), pick(ref["k"]), pick(ref["v"]),
                                      w.softmax_scale, w.causal, w.window)
        err_o = G.rel_frob(pick(synth.to_f64(o.cpu())), o_ref)
        err_l = float(np.abs(pick(lse.cpu().double().numpy()) - lse_ref).max())
        print(name, {"o": err_o, "lse": err_l})
        assert err_o <= G.TOL_O_FP8 and err_l <= G.TOL_LSE, (err_o, err_l)
        return
    slopes = alibi_slopes(w.H) if w.alibi else None
    lengths = w.seq_lengths() if w.varlen else None
    out = G.run_library(inp, w.softmax_scale, w.causal, w.window, w.backward, slopes,
                        lengths=lengths)
    if w.packed:
        # the packed batch: bit-identical to the padded one on every real row (checked
        # against the oracle below)
        packed = G.run_library_packed(inp, lengths, w.softmax_scale, w.causal, w.window)
        for n in out:
            assert torch.equal(packed[n], out[n]), n
        out = packed
    if lengths is not None and heads is not None:
        # one sampled head at a time, each with its batch entry's real length
        per = [G.compare(inp, out, w.softmax_scale, w.causal, w.window, [bh], w.backward,
                         slopes, lengths=lengths) for bh in heads]
        errs = {key: max(e[key] for e in per) for key in per[0]}
    else:
        errs = G.compare(inp, out, w.softmax_scale, w.causal, w.window, heads, w.backward,
                         slopes)
    print(name, errs)
    G.assert_within_bounds(errs, name)


def _rescale_inputs(N, d, alternate):
    """Inputs whose scores climb along the sequence, so that the running maximum of a row
    keeps growing from key tile to key tile and the forward must rescale O and l.

    q_i = 32 u (u a unit vector) and k_j = c j u + n_j with n_j ~ N(0, 1) and c chosen so
    that the scores rise by about 6 nats per 128 keys, on top of noise of 4 nats (d = 64).
    The large factor sits in Q, so K has no large common offset and dQ = scale dS K stays
    well conditioned in bf16 (rounding dS to bf16 alone costs about 0.3%). With
    `alternate`, odd rows get q_i = -32 u and see falling scores, so the rows of one warp
    disagree on whether to rescale."""
    g = torch.Generator().manual_seed(7)
    u = torch.ones(d) / np.sqrt(d)
    q = (32.0 * u).repeat(N, 1)
    if alternate:
        q[1::2] *= -1
    slope = 6.0 / (128 * (1.0 / np.sqrt(d)) * 32.0)
    k = torch.arange(N, dtype=torch.float32)[:, None] * slope * u[None]
    k = k + torch.randn(N, d, generator=g)
    v = torch.randn(N, d, generator=g)
    do = torch.randn(N, d, generator=g)
    cast = lambda t: t.to(torch.bfloat16).reshape(1, 1, N, d).contiguous()
    return {"q": cast(q), "k": cast(k), "v": cast(v), "do": cast(do)}


def _rescale_events(inp, scale, causal):
    """How many (row, key tile) steps raise a row's running maximum by more than 2^8
    (8 in base-2 units), the threshold past which the forward rescales."""
    q = synth.to_f64(inp["q"])[0, 0]
    k = synth.to_f64(inp["k"])[0, 0]
    s = (q @ k.T) * scale / np.log(2.0)
    N = s.shape[0]
    if causal:
        s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
    tiles = [s[:, t:t + 128].max(axis=1) for t in range(0, N, 128)]
    run = tiles[0]
    events = 0
    for tmax in tiles[1:]:
        events += int(np.sum(tmax > run + 8.0))
        run = np.maximum(run, tmax)
    return events


@pytest.mark.parametrize("alternate", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_running_max_rescale(d, alternate):
    N = 1024
    inp = _rescale_inputs(N, d, alternate)
    scale = 1.0 / np.sqrt(d)
    for causal in (False, True):
        assert _rescale_events(inp, scale, causal) >= 256  # the path is really taken
        out = G.run_library(inp, scale, causal, (-1, -1))
        errs = G.compare(inp, out, scale, causal, (-1, -1))
        G.assert_within_bounds(errs, (d, alternate, causal))


@pytest.mark.parametrize("d", [64, 128])
def test_large_scale_peaked_softmax(d):
    """scale = 1 on N(0,1) inputs: scores of standard deviation sqrt(d), near one-hot rows."""
    inp = inputs(1, 2, 640, d, 300 + d)
    out = G.run_library(inp, 1.0, False, (-1, -1))
    errs = G.compare(inp, out, 1.0, False, (-1, -1))
    G.assert_within_bounds(errs, d)


@pytest.mark.parametrize("d", [64, 128])
def test_self_similar_inputs(d):
    """k = v = q (the comparison input of page "显存神技：必学FlashAttention！").

    Each row's own key dominates its softmax here (P_ii ~ 0.77 at d = 64, 0.98 at d = 128),
    so dS = P o (dP - delta) cancels almost to zero on the diagonal and delta must be
    formed from O to better than bf16: the training path keeps O - bf16(O) from the
    forward for that. Every output is held to the plain bounds."""
    base = inputs(1, 2, 384, d, 400 + d)
    inp = {"q": base["q"], "k": base["q"].clone(), "v": base["q"].clone(), "do": base["do"]}
    scale = 1.0 / np.sqrt(d)
    for causal in (False, True):
        out = G.run_library(inp, scale, causal, (-1, -1))
        errs = G.compare(inp, out, scale, causal, (-1, -1))
        print(d, causal, errs)
        G.assert_within_bounds(errs, (d, causal))


@pytest.mark.parametrize("d", [64, 128])
def test_self_similar_inputs_without_residual(d):
    """The same input through plain fa_fwd / fa_bwd, whose delta is formed from the bf16 O:
    O, LSE and dV keep the plain bounds, while dQ and dK carry the rounding of O amplified
    by the cancellation in dS (measured here, not bounded by the target's 1e-2: fp64
    emulation puts it near 1.2% at d = 64 and 11% at d = 128). The test pins that the
    residual is what removes it: with it, the same run is within 1e-2 (test above)."""
    base = inputs(1, 2, 384, d, 400 + d)
    inp = {"q": base["q"], "k": base["q"].clone(), "v": base["q"].clone(), "do": base["do"]}
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, False, (-1, -1), residual=False)
    errs = G.compare(inp, out, scale, False, (-1, -1))
    print(d, errs)
    assert errs["o"] <= G.TOL_O and errs["lse"] <= G.TOL_LSE and errs["dv"] <= G.TOL_GRAD
    assert errs["dq"] > G.TOL_GRAD / 4 and errs["dk"] > G.TOL_GRAD / 4, errs


@pytest.mark.parametrize("name", ["c1", "c3", "c4", "c5w"])
def test_plain_path_without_residual(name):
    """fa_fwd / fa_bwd as the target names them (delta from the bf16 O) on i.i.d. inputs:
    within the plain bounds on the full-size workloads."""
    w = WORKLOADS[name]
    inp = inputs(w.B, w.H, w.N, w.d, w.seed_index)
    out = G.run_library(inp, w.softmax_scale, w.causal, w.window, w.backward, residual=False)
    heads = None if w.B * w.H * w.N <= 2 * 8 * 4096 else _sampled_heads(w)
    errs = G.compare(inp, out, w.softmax_scale, w.causal, w.window, heads, w.backward)
    print(name, errs)
    G.assert_within_bounds(errs, name)


def test_zero_queries_closed_form():
    """Q = 0: O is the running mean of V (causal) and LSE = ln(i + 1), on the GPU."""
    N, d = 300, 64
    base = inputs(1, 1, N, d, 500)
    inp = dict(base, q=torch.zeros_like(base["q"]))
    out = G.run_library(inp, 0.125, True, (-1, -1))
    v = synth.to_f64(inp["v"])[0, 0]
    mean = np.cumsum(v, axis=0) / np.arange(1, N + 1)[:, None]
    o = synth.to_f64(out["o"])[0, 0]
    assert G.rel_frob(o, mean) < G.TOL_O
    np.testing.assert_allclose(out["lse"][0, 0].double().numpy(), np.log(np.arange(1, N + 1)),
                               atol=G.TOL_LSE)


def test_deterministic():
    """Two runs give bit-identical O, LSE, dQ, dK and dV (no atomics on the default path)."""
    w = WORKLOADS["c3"]
    inp = inputs(w.B, w.H, w.N, w.d, w.seed_index)
    a = G.run_library(inp, w.softmax_scale, True, (-1, -1))
    b = G.run_library(inp, w.softmax_scale, True, (-1, -1))
    for n in a:
        assert torch.equal(a[n], b[n]), n


def test_fused_backward_run_to_run():
    """The fused backward (FA_BWD_FUSED, head_dim 64): O, LSE, dK and dV are bit-identical
    from run to run; dQ, added up in fp32 in no fixed order, differs by fp32 rounding only
    (far below bf16's resolution), and both runs agree with the default backward within the
    bounds."""
    w = WORKLOADS["c3"]
    inp = inputs(w.B, w.H, w.N, w.d, w.seed_index)
    a = G.run_library(inp, w.softmax_scale, True, (-1, -1), fused=True)
    b = G.run_library(inp, w.softmax_scale, True, (-1, -1), fused=True)
    c = G.run_library(inp, w.softmax_scale, True, (-1, -1))
    for n in ("o", "lse", "dk", "dv"):
        assert torch.equal(a[n], b[n]), n
    spread = G.rel_frob(synth.to_f64(a["dq"]), synth.to_f64(b["dq"]))
    to_det = G.rel_frob(synth.to_f64(a["dq"]), synth.to_f64(c["dq"]))
    print("fused dQ run-to-run relative spread %.3g, vs the default path %.3g" % (spread, to_det))
    assert spread <= 1e-3 and to_det <= 2e-3
    errs = G.compare(inp, a, w.softmax_scale, True, (-1, -1))
    G.assert_within_bounds(errs, "fused")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["none", "causal", "win100_30"])
def test_fused_path_small_and_ragged(d, mode):
    """The fused backward against the oracle (at head_dim 128 the flag selects the same
    separate passes)."""
    causal, window = MODES[mode]
    for N in (17, 300):
        inp = inputs(2, 2, N, d, 150 + N + d)
        scale = 1.0 / np.sqrt(d)
        out = G.run_library(inp, scale, causal, window, fused=True)
        errs = G.compare(inp, out, scale, causal, window)
        G.assert_within_bounds(errs, (N, d, mode))


@pytest.mark.parametrize("name", ["c3", "c4"])
def test_fused_path_full_size(name):
    w = WORKLOADS[name]
    inp = inputs(w.B, w.H, w.N, w.d, w.seed_index)
    out = G.run_library(inp, w.softmax_scale, w.causal, w.window, fused=True)
    heads = None if w.B * w.H * w.N <= 2 * 8 * 4096 else _sampled_heads(w)
    errs = G.compare(inp, out, w.softmax_scale, w.causal, w.window, heads)
    G.assert_within_bounds(errs, name)


@pytest.mark.parametrize("d", [64, 128])
def test_outputs_stay_in_bounds(d):
    """Every output is written only inside its own extent: sentinels around each output
    buffer survive the calls."""
    B, H, N = 1, 3, 200
    inp = inputs(B, H, N, d, 600 + d)
    dev = torch.device("cuda:0")
    G.ensure_built()
    n = B * H * N * d
    pad = 4096
    q, k, v, do = (inp[x].to(dev) for x in ("q", "k", "v", "do"))

    def guarded(count, dtype):
        buf = torch.full((count + 2 * pad,), 7.0, dtype=dtype, device=dev)
        return buf, buf[pad:pad + count]

    ob, o = guarded(n, torch.bfloat16)
    lb, lse = guarded(B * H * N, torch.float32)
    fa.fa_fwd(q, k, v, o.view(B, H, N, d), lse.view(B, H, N), None, True, (-1, -1))
    gb = [guarded(n, torch.bfloat16) for _ in range(3)]
    wb, ws = guarded(fa.fa_bwd_workspace_bytes(B, H, N, d) // 4, torch.float32)
    fa.fa_bwd(q, k, v, o.view(B, H, N, d), do, lse.view(B, H, N),
              *(g[1].view(B, H, N, d) for g in gb), ws, None, True, (-1, -1))
    torch.cuda.synchronize()
    for buf, _ in [(ob, o), (lb, lse), (wb, ws)] + gb:
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
    for t in [o, lse] + [g[1] for g in gb]:
        assert torch.isfinite(t.float()).all()


def test_empty_problem_launches_nothing():
    G.ensure_built()
    z = torch.empty((1, 1, 0, 64), dtype=torch.bfloat16, device="cuda:0")
    o, lse = fa.attention_forward(z, z, z)
    assert o.shape == z.shape and lse.shape == (1, 1, 0)
