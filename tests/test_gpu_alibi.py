"""ALiBi (fa_fwd_alibi, fa_bwd_alibi) against the fp64 oracle with the same slopes: the
linear bias -m_h |i - j| of the `alibi_slopes` parameter (page "告别OOM和训练慢…(含A100环境
配置)" §4.2), on small and ragged shapes in every mask mode, with many work items per
persistent CTA, with slopes steep enough that each row sees little but itself, and with
zero slopes."""
import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth
from exact_attention_126_b200.workloads import alibi_slopes

pytestmark = pytest.mark.gpu

MODES = {
    "none": (False, (-1, -1)),
    "causal": (True, (-1, -1)),
    "win64_0": (False, (64, 0)),
    "win100_30": (False, (100, 30)),
}


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 129, 300])
@pytest.mark.parametrize("mode", list(MODES))
def test_alibi_small_and_ragged(N, d, mode):
    causal, window = MODES[mode]
    H = 3
    inp = synth.attention_inputs(2, H, N, d, 300 + N + d)
    scale = 1.0 / np.sqrt(d)
    slopes = alibi_slopes(H)
    out = G.run_library(inp, scale, causal, window, True, slopes)
    errs = G.compare(inp, out, scale, causal, window, None, True, slopes)
    G.assert_within_bounds(errs, (N, d, mode))


@pytest.mark.parametrize("d", [64, 128])
def test_alibi_many_items_per_cta(d):
    """256 heads of 3 tiles each: every persistent CTA runs several items, each with its
    head's own slope."""
    B, H, N = 4, 64, 384
    inp = synth.attention_inputs(B, H, N, d, 900 + d)
    scale = 1.0 / np.sqrt(d)
    slopes = alibi_slopes(H)
    out = G.run_library(inp, scale, True, (-1, -1), True, slopes)
    heads = [(0, 0), (1, 17), (2, 40), (3, 63)]
    errs = G.compare(inp, out, scale, True, (-1, -1), heads, True, slopes)
    G.assert_within_bounds(errs, d)


@pytest.mark.parametrize("d", [64, 128])
def test_alibi_steep_slopes(d):
    """Slopes of 2 to 8 per position: a row's weight falls by e^-2 or more per key of
    distance, so O is dominated by a few neighbours of the diagonal, across tile borders."""
    H, N = 2, 260
    inp = synth.attention_inputs(1, H, N, d, 950 + d)
    scale = 1.0 / np.sqrt(d)
    slopes = [2.0, 8.0]
    for causal, window in MODES.values():
        out = G.run_library(inp, scale, causal, window, True, slopes)
        errs = G.compare(inp, out, scale, causal, window, None, True, slopes)
        G.assert_within_bounds(errs, (d, causal, window))


def test_alibi_zero_slopes_match_plain_attention():
    """Zero slopes are no bias: the ALiBi kernels agree with the oracle without a bias."""
    d, N, H = 64, 200, 2
    inp = synth.attention_inputs(1, H, N, d, 990)
    scale = 0.125
    out = G.run_library(inp, scale, True, (-1, -1), True, [0.0, 0.0])
    errs = G.compare(inp, out, scale, True, (-1, -1))
    G.assert_within_bounds(errs, "zero slopes")


def test_alibi_slopes_are_per_head():
    """Swapping two heads' slopes swaps exactly those heads' outputs."""
    G.ensure_built()
    dev = torch.device("cuda:0")
    d, N, H = 64, 256, 2
    x = synth.attention_inputs(1, H, N, d, 995)
    q = x["q"][:, :1].repeat(1, H, 1, 1).to(dev)
    k = x["k"][:, :1].repeat(1, H, 1, 1).to(dev)
    v = x["v"][:, :1].repeat(1, H, 1, 1).to(dev)
    a = torch.tensor([0.5, 0.05], device=dev)
    o1, l1 = fa.attention_forward(q, k, v, 0.125, True, (-1, -1), alibi_slopes=a)
    o2, l2 = fa.attention_forward(q, k, v, 0.125, True, (-1, -1), alibi_slopes=a.flip(0).contiguous())
    torch.cuda.synchronize()
    assert torch.equal(o1[:, 0], o2[:, 1]) and torch.equal(o1[:, 1], o2[:, 0])
    assert torch.equal(l1[:, 0], l2[:, 1])
    assert not torch.equal(o1[:, 0], o1[:, 1])
