"""Dropout on the attention weights (fa_options_t.dropout_p, with its seed and offset)
against the fp64 oracle with the same Philox4x32-10 keep flags: `dropout_p` of page
"告别OOM和训练慢…(含A100环境配置)" §4.2, applied after the softmax and before the product with V
as in the reference layer of page "Flash Attention 3.7 核心原理与实战" §4.2. Forward and
backward, every mask mode, both head sizes, ragged lengths, several probabilities, with key
padding and ALiBi, and with many work items per persistent CTA; p = 0 is no dropout at all,
and the same seed and offset give bit-identical results."""
import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import synth
from exact_attention_126_b200.workloads import alibi_slopes

pytestmark = pytest.mark.gpu

MODES = {
    "none": (False, (-1, -1)),
    "causal": (True, (-1, -1)),
    "win100_30": (False, (100, 30)),
}


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [17, 129, 300])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_small_and_ragged(N, d, mode, p):
    causal, window = MODES[mode]
    inp = synth.attention_inputs(2, 3, N, d, 1500 + N + d)
    scale = 1.0 / np.sqrt(d)
    drop = (p, 0x9E3779B97F4A7C15 + N, 17)
    out = G.run_library(inp, scale, causal, window, dropout=drop)
    errs = G.compare(inp, out, scale, causal, window, dropout=drop)
    G.assert_within_bounds(errs, (N, d, mode, p))


@pytest.mark.parametrize("d", [64, 128])
def test_dropout_many_items_per_cta(d):
    """More (head, tile) items than SMs: the flags follow each item's (batch, head)."""
    B, H, N = 4, 40, 384
    inp = synth.attention_inputs(B, H, N, d, 1600 + d)
    scale = 1.0 / np.sqrt(d)
    drop = (0.15, 2024, 3)
    out = G.run_library(inp, scale, True, (-1, -1), dropout=drop)
    errs = G.compare(inp, out, scale, True, (-1, -1), dropout=drop)
    G.assert_within_bounds(errs, d)


@pytest.mark.parametrize("d", [64, 128])
def test_dropout_with_padding_and_alibi(d):
    B, H, N = 3, 2, 260
    inp = synth.attention_inputs(B, H, N, d, 1700 + d)
    flags = np.zeros((B, N), dtype=bool)
    flags[1, 200:] = True
    flags[2, ::5] = True
    kp = torch.from_numpy(flags)
    slopes = alibi_slopes(H)
    scale = 1.0 / np.sqrt(d)
    drop = (0.25, 77, 1)
    out = G.run_library(inp, scale, True, (-1, -1), alibi=slopes, key_padding=kp, dropout=drop)
    errs = G.compare(inp, out, scale, True, (-1, -1), alibi=slopes, key_padding=kp,
                     dropout=drop)
    G.assert_within_bounds(errs, d)


def test_dropout_zero_is_no_dropout():
    """p = 0 selects the kernels without dropout: bit-identical to a call without it."""
    inp = synth.attention_inputs(1, 2, 300, 64, 1800)
    a = G.run_library(inp, 0.125, True, (-1, -1), dropout=(0.0, 5, 0))
    b = G.run_library(inp, 0.125, True, (-1, -1))
    for n in a:
        assert torch.equal(a[n], b[n]), n


def test_dropout_is_reproducible_and_follows_the_offset():
    """The same (seed, offset) gives bit-identical results; another offset or seed gives
    another draw (and its own match with the oracle)."""
    inp = synth.attention_inputs(1, 2, 256, 64, 1900)
    a = G.run_library(inp, 0.125, False, (-1, -1), dropout=(0.2, 11, 0))
    b = G.run_library(inp, 0.125, False, (-1, -1), dropout=(0.2, 11, 0))
    c = G.run_library(inp, 0.125, False, (-1, -1), dropout=(0.2, 11, 1))
    for n in a:
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["o"], c["o"])
    assert torch.equal(a["lse"], c["lse"])  # the normalisation comes before dropout
    errs = G.compare(inp, c, 0.125, False, (-1, -1), dropout=(0.2, 11, 1))
    G.assert_within_bounds(errs, "offset 1")
