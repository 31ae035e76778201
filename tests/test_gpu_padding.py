"""Key padding (fa_options_t.key_padding) against the fp64 oracle with the same flags: the
`key_padding_mask` (True = padded key) of page "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升训练
速度", applied with masked_fill(-inf) on every head and query as in the reference layer of page
"Flash Attention 3.7 核心原理与实战" §4.2, forward and backward, on suffix padding
of different lengths per batch entry (one entry fully padded), random flags, whole padded
key tiles in the middle of a sequence, every mask mode, both head sizes, with ALiBi, and
with many work items per persistent CTA."""
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
    "win64_0": (False, (64, 0)),
    "win100_30": (False, (100, 30)),
}


def suffix_padding(B, N, seed):
    """Batch entry b keeps its first len_b keys: lengths N, 1, 0 (fully padded) and random."""
    rng = np.random.default_rng(seed)
    lens = [N, 1, 0] + [int(rng.integers(1, N + 1)) for _ in range(max(0, B - 3))]
    flags = np.zeros((B, N), dtype=bool)
    for b in range(B):
        flags[b, lens[b % len(lens)]:] = True
    return torch.from_numpy(flags)


def random_padding(B, N, seed, p=0.3):
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.random((B, N)) < p)


def tile_padding(B, N):
    """Keys 128..255 (a whole key tile) and every 7th key padded."""
    flags = np.zeros((B, N), dtype=bool)
    flags[:, 128:256] = True
    flags[:, ::7] = True
    return torch.from_numpy(flags)


def check_dead_rows(out, kp, causal, window):
    """Rows with no visible unpadded key: O = 0, LSE = -inf and dQ = 0 exactly; padded
    keys: dK = dV = 0 exactly."""
    lse = out["lse"].double().numpy()
    dead = np.isneginf(lse)
    o = out["o"].float().numpy()
    assert np.all(o[dead] == 0.0)
    if "dq" in out:
        dq = out["dq"].float().numpy()
        assert np.all(dq[dead] == 0.0)
        flags = kp.numpy()
        for b in range(flags.shape[0]):
            for g in ("dk", "dv"):
                x = out[g].float().numpy()[b]
                assert np.all(x[:, flags[b]] == 0.0), g


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [17, 129, 300])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("pattern", ["suffix", "random"])
def test_padding_small_and_ragged(N, d, mode, pattern):
    causal, window = MODES[mode]
    B, H = 4, 2
    inp = synth.attention_inputs(B, H, N, d, 1000 + N + d)
    kp = suffix_padding(B, N, N) if pattern == "suffix" else random_padding(B, N, N + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, causal, window, key_padding=kp)
    errs = G.compare(inp, out, scale, causal, window, key_padding=kp)
    G.assert_within_bounds(errs, (N, d, mode, pattern))
    check_dead_rows(out, kp, causal, window)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", ["none", "causal", "win100_30"])
def test_padded_key_tile(d, mode):
    """A whole key tile padded (every row sees a tile of -inf scores) plus every 7th key."""
    causal, window = MODES[mode]
    B, H, N = 2, 3, 520
    inp = synth.attention_inputs(B, H, N, d, 1100 + d)
    kp = tile_padding(B, N)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, causal, window, key_padding=kp)
    errs = G.compare(inp, out, scale, causal, window, key_padding=kp)
    G.assert_within_bounds(errs, (d, mode))
    check_dead_rows(out, kp, causal, window)


@pytest.mark.parametrize("d", [64, 128])
def test_padding_with_alibi(d):
    B, H, N = 3, 4, 300
    inp = synth.attention_inputs(B, H, N, d, 1200 + d)
    kp = suffix_padding(B, N, 5)
    slopes = alibi_slopes(H)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, True, (-1, -1), alibi=slopes, key_padding=kp)
    errs = G.compare(inp, out, scale, True, (-1, -1), alibi=slopes, key_padding=kp)
    G.assert_within_bounds(errs, d)
    check_dead_rows(out, kp, True, (-1, -1))


@pytest.mark.parametrize("d", [64, 128])
def test_padding_many_items_per_cta(d):
    """More (head, tile) items than SMs, each batch entry with its own padding."""
    B, H, N = 8, 16, 384
    inp = synth.attention_inputs(B, H, N, d, 1300 + d)
    kp = suffix_padding(B, N, 11)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, True, (-1, -1), key_padding=kp)
    errs = G.compare(inp, out, scale, True, (-1, -1), key_padding=kp)
    G.assert_within_bounds(errs, d)
    check_dead_rows(out, kp, True, (-1, -1))


def test_no_flags_set_is_identical_to_no_padding():
    """All-false flags give bit-identical outputs to a call without key padding."""
    B, H, N, d = 2, 2, 300, 64
    inp = synth.attention_inputs(B, H, N, d, 1400)
    kp = torch.zeros((B, N), dtype=torch.bool)
    a = G.run_library(inp, 0.125, True, (-1, -1), key_padding=kp)
    b = G.run_library(inp, 0.125, True, (-1, -1))
    for n in a:
        assert torch.equal(a[n], b[n]), n
