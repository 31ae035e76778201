"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (an engine
that reserved all of its memory up front, a plugin whose enqueue step may not call
cudaMalloc). It must give what fa_bwd gives, call after call, using the library's own
fixed device array instead of a caller workspace.

This file is collected last on purpose: should it fail, a run that stops at the first
failure has run every other test already. It passes alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 8 << 20  # the fixed device array (include/fa.h)


def _run_both(B, H, N, d, causal, window, seed):
    G.ensure_built()
    dev = torch.device("cuda:0")
    inp = synth.attention_inputs(B, H, N, d, seed)
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_forward(q, k, v, scale, causal, window)
    ref = fa.attention_backward(q, k, v, o, lse, do, scale, causal, window)
    outs = []
    for _ in range(2):  # two calls in a row share the array
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale, causal, window)
        outs.append((dq, dk, dv))
    torch.cuda.synchronize()
    assert fa.fa_debug_status() == 0
    return ref, outs


@pytest.mark.parametrize("B,H,N,d,causal,window", [
    (2, 3, 300, 64, True, (-1, -1)),
    (1, 4, 1024, 128, True, (200, -1)),
    (2, 2, 129, 128, False, (-1, -1)),
])
def test_noalloc_matches_fa_bwd(B, H, N, d, causal, window):
    ref, outs = _run_both(B, H, N, d, causal, window, 700 + N + d)
    for call in outs:
        for name, got, want in zip(("dq", "dk", "dv"), call, ref):
            err = G.rel_frob(synth.to_f64(got.cpu()), synth.to_f64(want.cpu()))
            assert err <= G.TOL_GRAD, (name, err)


def test_noalloc_rejects_problems_beyond_its_array():
    """2 * B * H * Np * 4 bytes must fit in the array; beyond it nothing is launched."""
    lib = fa.library()
    W = fa.fa_window_t(-1, -1)
    A = 0x10000  # never dereferenced: the size check comes first
    rows_max = NOALLOC_BYTES // 8
    B, H, N = 1, rows_max // 1024 + 1, 1024
    assert B * H * N > rows_max
    assert lib.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, B, H, N, 64, 0.125, 0, W, None) == 4
    B, H, N = 1, rows_max // 1024, 1024
    assert B * H * N <= rows_max
