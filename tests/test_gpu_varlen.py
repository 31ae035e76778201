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
    packed = G.run_library_packed(inp, lens, scale, causal, window)
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
    packed = G.run_library_packed(inp, lens, scale, True, (-1, -1), **kw)
    for n in padded:
        assert torch.equal(packed[n], padded[n]), n


@pytest.mark.parametrize("d", [64, 128])
def test_packed_outputs_stay_in_bounds(d):
    """A packed batch writes only its sequences' tokens: sentinels in guard bands around
    every output and workspace, and in the tokens before the first and after the last
    sequence (which no sequence covers), survive the forward and the backward."""
    from exact_attention_126_b200 import fa
    G.ensure_built()
    dev = torch.device("cuda:0")
    B, H, N = 3, 2, 300
    lens = [300, 5, 129]
    lead, extra = 7, 40  # tokens before the first sequence and after the last
    total = lead + sum(lens) + extra
    g = torch.Generator(device=dev).manual_seed(2800 + d)
    q, k, v, do = (torch.randn((total, H, d), generator=g, device=dev).to(torch.bfloat16)
                   for _ in range(4))
    pad = 4096

    def guarded(count, dtype):
        buf = torch.full((count + 2 * pad,), 7.0, dtype=dtype, device=dev)
        return buf, buf[pad:pad + count]

    n = total * H * d
    ob, o = guarded(n, torch.bfloat16)
    olb, o_low = guarded(n, torch.bfloat16)
    lb, lse = guarded(H * total, torch.float32)
    cu = torch.tensor([lead + c for c in G.cumulative(lens)], dtype=torch.int32, device=dev)
    dims = (B, H, N, d)
    opt = fa.options(o_low=o_low, cu_seqlens=cu, total_tokens=total)
    fa.fa_fwd_ex(q, k, v, o.view(total, H, d), lse.view(H, total), opt, None, True, (-1, -1),
                 dims=dims)
    gb = [guarded(n, torch.bfloat16) for _ in range(3)]
    wb, ws = guarded(fa.fa_bwd_workspace_bytes_ex(B, H, N, d, opt) // 4, torch.float32)
    fa.fa_bwd_ex(q, k, v, o.view(total, H, d), do, lse.view(H, total),
                 *(x[1].view(total, H, d) for x in gb), ws, opt, None, True, (-1, -1),
                 dims=dims)
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    for buf, _ in [(ob, o), (olb, o_low), (lb, lse), (wb, ws)] + gb:
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
    end = lead + sum(lens)
    for t in [o, o_low] + [x[1] for x in gb]:
        rows = t.view(total, H, d)
        # nobody's tokens, before the first sequence and after the last: untouched
        assert torch.all(rows[:lead] == 7.0) and torch.all(rows[end:] == 7.0)
        assert torch.isfinite(rows[lead:end].float()).all()
    lse_rows = lse.view(H, total)
    assert torch.all(lse_rows[:, :lead] == 7.0) and torch.all(lse_rows[:, end:] == 7.0)


def test_packed_sequence_longer_than_n_is_cut():
    """A sequence longer than N (the longest length the call handles) is cut at N: its
    first N tokens get the results of an N-token sequence and the tokens past N are not
    written (their sentinels survive)."""
    from exact_attention_126_b200 import fa
    G.ensure_built()
    dev = torch.device("cuda:0")
    H, d, N = 2, 64, 256
    lens = [300, 129]
    total = sum(lens)
    g = torch.Generator(device=dev).manual_seed(2900)
    q, k, v, do = (torch.randn((total, H, d), generator=g, device=dev).to(torch.bfloat16)
                   for _ in range(4))
    cu = torch.tensor(G.cumulative(lens), dtype=torch.int32, device=dev)
    o = torch.full((total, H, d), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((H, total), 7.0, dtype=torch.float32, device=dev)
    opt = fa.options(cu_seqlens=cu, total_tokens=total)
    fa.fa_fwd_ex(q, k, v, o, lse, opt, None, True, (-1, -1), dims=(2, H, N, d))
    # the same first sequence cut to N tokens, as a batch of its own
    cu1 = torch.tensor([0, N], dtype=torch.int32, device=dev)
    o1 = torch.empty((N, H, d), dtype=torch.bfloat16, device=dev)
    lse1 = torch.empty((H, N), dtype=torch.float32, device=dev)
    fa.fa_fwd_ex(q[:N].contiguous(), k[:N].contiguous(), v[:N].contiguous(), o1, lse1,
                 fa.options(cu_seqlens=cu1, total_tokens=N), None, True, (-1, -1),
                 dims=(1, H, N, d))
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    assert torch.equal(o[:N], o1) and torch.equal(lse[:, :N], lse1)
    assert torch.all(o[N:300] == 7.0) and torch.all(lse[:, N:300] == 7.0)
    assert torch.isfinite(o[300:].float()).all()

