"""The e4m3 forward (fa_fwd_fp8: the FP8 support page "告别OOM和训练慢…(含A100环境配置)" §6
names as a next step) against the fp64 oracle on the descaled values of the same e4m3 inputs.

Tolerance, derived from the arithmetic: P is rounded to e4m3 (3-bit mantissa, relative RMS
2^-4/sqrt(3) ~ 3.6% per weight) for the P V product, which moves O by about 2-2.5% relative
Frobenius on i.i.d. N(0, 1) inputs at head_dim 128 (fp64 emulation at N = 1024..8192, causal
and not); O is held to 5e-2, twice that. LSE comes from fp32 scores of the exact e4m3 values
and keeps the bf16 path's bound of 1e-3."""
import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth

pytestmark = pytest.mark.gpu

TOL_O_FP8 = G.TOL_O_FP8

MODES = {
    "none": (False, (-1, -1)),
    "causal": (True, (-1, -1)),
    "win100_30": (False, (100, 30)),
    "causal_win1024": (True, (1024, -1)),
}


def fp8_inputs(B, H, N, seed, scales=(1.0, 1.0, 1.0)):
    """e4m3 tensors of the seeded N(0, 1) inputs divided by their descales (so that
    x8 * scale ~ N(0, 1)), and the exact descaled values in fp64."""
    inp = synth.attention_inputs(B, H, N, 128, seed, with_grad=False)
    out8, ref = {}, {}
    for (n, t), sc in zip(((n, inp[n]) for n in ("q", "k", "v")), scales):
        x8 = (t.float() / sc).to(torch.float8_e4m3fn)
        out8[n] = x8
        ref[n] = x8.to(torch.float64).numpy() * sc
    return out8, ref


def run_fp8(x8, scales, scale, causal, window):
    G.ensure_built()
    dev = torch.device("cuda:0")
    q, k, v = (x8[n].to(dev) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward_fp8(q, k, v, *scales, scale=scale, causal=causal,
                                      window=window)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    return o.cpu(), lse.cpu()


def check(o, lse, ref, scale, causal, window, heads=None):
    def pick(a):
        return a if heads is None else np.stack([a[b, h] for b, h in heads])[None]

    o_ref, lse_ref = G.oracle.fwd(pick(ref["q"]), pick(ref["k"]), pick(ref["v"]), scale, causal,
                                  window)
    err_o = G.rel_frob(pick(synth.to_f64(o)), o_ref)
    err_l = float(np.abs(pick(lse.double().numpy()) - lse_ref).max())
    assert err_o <= TOL_O_FP8, err_o
    assert err_l <= G.TOL_LSE, err_l
    return err_o, err_l


@pytest.mark.parametrize("N", [17, 129, 300, 1024])
@pytest.mark.parametrize("mode", list(MODES))
def test_fp8_small_and_ragged(N, mode):
    causal, window = MODES[mode]
    x8, ref = fp8_inputs(2, 3, N, 3000 + N)
    scale = 1.0 / np.sqrt(128)
    o, lse = run_fp8(x8, (1.0, 1.0, 1.0), scale, causal, window)
    print(N, mode, check(o, lse, ref, scale, causal, window))


def test_fp8_descales():
    """Per-tensor descales (powers of two and not) are applied to Q, K (in the scores) and V
    (in O)."""
    scales = (0.5, 0.3, 2.0)
    x8, ref = fp8_inputs(1, 4, 384, 3100, scales)
    scale = 1.0 / np.sqrt(128)
    o, lse = run_fp8(x8, scales, scale, True, (-1, -1))
    check(o, lse, ref, scale, True, (-1, -1))


def test_fp8_many_items_per_cta():
    x8, ref = fp8_inputs(4, 40, 384, 3200)
    scale = 1.0 / np.sqrt(128)
    o, lse = run_fp8(x8, (1.0, 1.0, 1.0), scale, True, (-1, -1))
    check(o, lse, ref, scale, True, (-1, -1), heads=[(0, 0), (1, 17), (3, 39)])


def test_fp8_long_sequence_sampled_heads():
    """The long-sequence shape (N = 8192, causal) on sampled heads."""
    x8, ref = fp8_inputs(1, 4, 8192, 3300)
    scale = 1.0 / np.sqrt(128)
    o, lse = run_fp8(x8, (1.0, 1.0, 1.0), scale, True, (-1, -1))
    print(check(o, lse, ref, scale, True, (-1, -1), heads=[(0, 0), (0, 3)]))


def test_fp8_matches_bf16_path_on_the_same_values():
    """The e4m3 forward against the bf16 forward on the descaled values (exact in bf16: e4m3
    values with power-of-two descales are bf16 numbers): same LSE to 1e-3, O within the FP8
    bound."""
    x8, ref = fp8_inputs(2, 2, 640, 3400, (0.5, 1.0, 0.25))
    scale = 1.0 / np.sqrt(128)
    o8, lse8 = run_fp8(x8, (0.5, 1.0, 0.25), scale, True, (-1, -1))
    dev = torch.device("cuda:0")
    q, k, v = (torch.from_numpy(ref[n]).to(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, scale, True)
    torch.cuda.synchronize()
    assert G.rel_frob(synth.to_f64(o8), synth.to_f64(o.cpu())) <= TOL_O_FP8
    assert float((lse8 - lse.cpu()).abs().max()) <= G.TOL_LSE
