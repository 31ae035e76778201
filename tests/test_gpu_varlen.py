"""Variable-length batches (fa_options_t.seq_lengths: each sample's real length, the
`lengths` of the dynamic batching of page "告别OOM和训练慢…(含A100环境配置)" §6) against the
fp64 oracle with the same lengths, forward and backward (separate and fused dQ), in every
mask mode, both head sizes, with lengths that end inside a tile, on a tile boundary, at 1,
at 0 and at N; with key padding, ALiBi and dropout on top; with many items per CTA. Rows
past a length must be exactly zero (LSE -inf), and the tiles past it are not computed."""
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


def _lengths(B, N, seed):
    rng = np.random.default_rng(seed)
    base = [N, 0, 1, 128 if N > 128 else N, N - 1]
    return [base[b] if b < len(base) else int(rng.integers(1, N + 1)) for b in range(B)]


def check_past_length(out, lengths):
    for b, L in enumerate(lengths):
        assert np.all(out["o"][b, :, L:].float().numpy() == 0.0)
        assert np.all(np.isneginf(out["lse"][b, :, L:].numpy()))
        for g in ("dq", "dk", "dv"):
            if g in out:
                assert np.all(out[g][b, :, L:].float().numpy() == 0.0), g


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [129, 300, 520])
@pytest.mark.parametrize("mode", list(MODES))
def test_varlen_small_and_ragged(N, d, mode):
    causal, window = MODES[mode]
    B, H = 6, 2
    lens = _lengths(B, N, N + d)
    inp = synth.attention_inputs(B, H, N, d, 2000 + N + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, causal, window, lengths=lens)
    errs = G.compare(inp, out, scale, causal, window, lengths=lens)
    G.assert_within_bounds(errs, (N, d, mode, lens))
    check_past_length(out, lens)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_fused_backward(d):
    B, H, N = 5, 3, 400
    lens = _lengths(B, N, 7)
    inp = synth.attention_inputs(B, H, N, d, 2100 + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, True, (-1, -1), lengths=lens, fused=True)
    errs = G.compare(inp, out, scale, True, (-1, -1), lengths=lens)
    G.assert_within_bounds(errs, d)
    check_past_length(out, lens)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_with_padding_alibi_dropout(d):
    B, H, N = 4, 2, 300
    lens = [300, 170, 5, 129]
    inp = synth.attention_inputs(B, H, N, d, 2200 + d)
    flags = np.zeros((B, N), dtype=bool)
    flags[0, 250:] = True
    flags[1, ::4] = True
    kp = torch.from_numpy(flags)
    slopes = alibi_slopes(H)
    scale = 1.0 / np.sqrt(d)
    drop = (0.2, 99, 4)
    out = G.run_library(inp, scale, True, (-1, -1), alibi=slopes, key_padding=kp, dropout=drop,
                        lengths=lens)
    errs = G.compare(inp, out, scale, True, (-1, -1), alibi=slopes, key_padding=kp,
                     dropout=drop, lengths=lens)
    G.assert_within_bounds(errs, d)
    check_past_length(out, lens)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_many_items_per_cta(d):
    """More items than SMs, most of them past their entry's length (skipped by every role)."""
    B, H, N = 8, 16, 640
    lens = [640, 1, 300, 0, 129, 512, 77, 640]
    inp = synth.attention_inputs(B, H, N, d, 2300 + d)
    scale = 1.0 / np.sqrt(d)
    out = G.run_library(inp, scale, True, (-1, -1), lengths=lens)
    errs = G.compare(inp, out, scale, True, (-1, -1), lengths=lens)
    G.assert_within_bounds(errs, d)
    check_past_length(out, lens)


def test_full_lengths_are_no_restriction():
    """seq_lengths = N everywhere: bit-identical to a call without lengths."""
    B, H, N, d = 2, 2, 300, 64
    inp = synth.attention_inputs(B, H, N, d, 2400)
    a = G.run_library(inp, 0.125, True, (-1, -1), lengths=[N, N])
    b = G.run_library(inp, 0.125, True, (-1, -1))
    for n in a:
        assert torch.equal(a[n], b[n]), n


@pytest.mark.parametrize("d", [64])
def test_varlen_schedules_agree(d):
    """Items are scheduled by their tile's distance from the start or end of the sequence
    for batches of up to 8192 entries (tables built on the GPU), by the chunked order
    beyond. Every item's result is independent of the CTA that computes it, so the first
    entries of an 8200-entry batch (chunked order) must equal, bit for bit, the same entries
    run as a batch of their own (the sorted order); sampled entries are also checked against
    the oracle, and every row past a length must be zero."""
    B, H, N = 8200, 1, 130
    rng = np.random.default_rng(2500)
    lens = [int(x) for x in rng.integers(0, N + 1, size=B)]
    lens[:6] = [N, 0, 1, 128, 129, 64]
    inp = synth.attention_inputs(B, H, N, d, 2500)
    scale = 1.0 / np.sqrt(d)
    big = G.run_library(inp, scale, True, (-1, -1), lengths=lens)
    small_inp = {n: t[:16].clone() for n, t in inp.items()}
    small = G.run_library(small_inp, scale, True, (-1, -1), lengths=lens[:16])
    for n in small:
        assert torch.equal(big[n][:16], small[n]), n
    for b in (0, 2, 3, 4, 5, 4097, B - 1):
        errs = G.compare(inp, big, scale, True, (-1, -1), heads=[(b, 0)], lengths=lens)
        G.assert_within_bounds(errs, (b, lens[b]))
    check_past_length(big, lens)


def _pack(t, lens):
    """(B, H, N, d) -> (total, H, d): the first lens[b] rows of entry b, back to back."""
    return torch.cat([t[b, :, :L].transpose(0, 1) for b, L in enumerate(lens)], 0).contiguous()


def _cu(lens):
    return [0] + list(np.cumsum(lens).astype(int))


def _run_packed(inp, lens, scale, causal, window, d, **kw):
    """The same problem as a packed batch (fa_options_t.cu_seqlens) through the public calls;
    returns the outputs in the padded layout's shape for the rows < length (the rest 0 and
    LSE -inf, as the padded path writes them)."""
    G.ensure_built()
    from exact_attention_126_b200 import fa
    dev = torch.device("cuda:0")
    B, H, N, _ = inp["q"].shape
    q, k, v, do = (_pack(inp[n], lens).to(dev) for n in ("q", "k", "v", "do"))
    cu = torch.tensor(_cu(lens), dtype=torch.int32, device=dev)
    o, lse, o_low = fa.attention_forward(q, k, v, scale, causal, window, keep_residual=True,
                                         cu_seqlens=cu, max_seqlen=N, **kw)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window, o_low=o_low,
                                       cu_seqlens=cu, max_seqlen=N, **kw)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    out = {}
    c = _cu(lens)
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


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mode", list(MODES))
def test_packed_batch_matches_padded(d, mode):
    """cu_seqlens: the sequences stored back to back with no padding (the page's dynamic
    batching avoids padding waste). Every real row of every output is bit-identical to the
    padded layout with seq_lengths (the same arithmetic per tile; a tile that runs into the
    next sequence only sees masked keys and unwritten rows there), and matches the oracle."""
    causal, window = MODES[mode]
    B, H, N = 7, 2, 300
    lens = _lengths(B, N, 31 + d)
    lens[5] = 200
    inp = synth.attention_inputs(B, H, N, d, 2600 + d)
    scale = 1.0 / np.sqrt(d)
    padded = G.run_library(inp, scale, causal, window, lengths=lens)
    packed = _run_packed(inp, lens, scale, causal, window, d)
    for n in padded:
        assert torch.equal(packed[n], padded[n]), (n, mode, d)
    errs = G.compare(inp, packed, scale, causal, window, lengths=lens)
    G.assert_within_bounds(errs, (d, mode, lens))


def test_packed_batch_with_alibi_padding_dropout():
    """The options that act per sequence (ALiBi, key padding by position, dropout by
    (batch, head, position)) give the packed batch the padded batch's results."""
    B, H, N, d = 5, 3, 260, 64
    lens = [260, 0, 129, 1, 200]
    inp = synth.attention_inputs(B, H, N, d, 2700)
    scale = 1.0 / np.sqrt(d)
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(2700)
    kpad = torch.tensor(rng.random((B, N)) < 0.2)
    slopes = alibi_slopes(H)
    kw = dict(alibi_slopes=torch.tensor(slopes, dtype=torch.float32, device=dev),
              key_padding=kpad.to(dev), dropout=(0.1, 1234, 5))
    padded = G.run_library(inp, scale, True, (-1, -1), lengths=lens, alibi=slopes,
                           key_padding=kpad, dropout=(0.1, 1234, 5))
    packed = _run_packed(inp, lens, scale, True, (-1, -1), d, **kw)
    for n in padded:
        assert torch.equal(packed[n], padded[n]), n

