"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (an engine
that reserved all of its memory up front, a plugin whose enqueue step may not call
cudaMalloc). It must give what fa_bwd gives, call after call, using the library's own
fixed device array instead of a caller workspace. The two run the same deterministic
kernels on the same statistics, so their outputs must be bit-identical.

This file is collected last on purpose: should it fail, a run that stops at the first
failure has run every other test already. It passes alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 8 << 20  # the fixed device array (include/fa.h)
ROWS_MAX = NOALLOC_BYTES // 8  # B * H * Np fp32 pairs that fit


def _problem(B, H, N, d, causal, window, seed):
    G.ensure_built()
    dev = torch.device("cuda:0")
    inp = synth.attention_inputs(B, H, N, d, seed)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale, causal, window)
    ref = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window)
    return (q, k, v, o, do, lse, scale), ref


def _noalloc(args, causal, window):
    q, k, v, o, do, lse, scale = args
    dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
    fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale, causal, window)
    return dq, dk, dv


def _assert_identical(got, want):
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert torch.equal(g, w), name


@pytest.mark.parametrize("B,H,N,d,causal,window", [
    (2, 3, 300, 64, True, (-1, -1)),
    (1, 4, 1024, 128, True, (200, -1)),
    (2, 2, 129, 128, False, (-1, -1)),
])
def test_noalloc_matches_fa_bwd(B, H, N, d, causal, window):
    """Two calls in a row share the array: both bit-identical to fa_bwd."""
    args, ref = _problem(B, H, N, d, causal, window, 700 + N + d)
    for _ in range(2):
        _assert_identical(_noalloc(args, causal, window), ref)


def test_noalloc_at_its_limit_then_a_smaller_problem():
    """B * H * Np exactly at the array's capacity is accepted and right; a smaller problem
    after it (whose statistics cover only the start of the array, over the larger call's
    leftovers) is right too."""
    N = 2048
    B, H = 2, ROWS_MAX // (2 * N)
    assert B * H * N == ROWS_MAX
    big_args, big_ref = _problem(B, H, N, 64, True, (-1, -1), 710)
    _assert_identical(_noalloc(big_args, True, (-1, -1)), big_ref)
    small_args, small_ref = _problem(1, 2, 200, 64, False, (-1, -1), 711)
    _assert_identical(_noalloc(small_args, False, (-1, -1)), small_ref)


def test_noalloc_rejects_problems_beyond_its_array():
    """One row past the capacity returns FA_ERR_WORKSPACE before anything is launched."""
    lib = fa.library()
    W = fa.fa_window_t(-1, -1)
    A = 0x10000  # never dereferenced: the size check comes first
    B, H, N = 1, ROWS_MAX // 1024 + 1, 1024
    assert B * H * N > ROWS_MAX
    assert lib.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, B, H, N, 64, 0.125, 0, W, None) == 4
