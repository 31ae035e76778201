"""Failure detection without a GPU fault: a host-set test hook makes the forward's copy
warp skip every V tile, so the kernel's bounded wait for V runs out (about two seconds);
the kernel must exit on its own, report FA_ERR_TIMEOUT, and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import gpu_helpers as G
from exact_attention_126_b200 import fa, synth

pytestmark = pytest.mark.gpu


def test_timeout_is_reported_and_the_context_survives():
    G.ensure_built()
    inp = synth.attention_inputs(1, 1, 256, 64, 900, with_grad=False)
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    assert fa.fa_debug_status() == 0
    fa.fa_debug_set_fault(1)
    try:
        t0 = time.time()
        fa.attention_forward(q, k, v, 0.125, True)
        status = fa.fa_debug_status()  # synchronises the stream
        waited = time.time() - t0
    finally:
        fa.fa_debug_set_fault(0)
    assert status == 6, status  # FA_ERR_TIMEOUT
    assert waited < 30.0
    assert fa.fa_debug_status() == 0  # reading cleared it
    out = G.run_library(inp, 0.125, True, (-1, -1), backward=False)
    errs = G.compare(inp, out, 0.125, True, (-1, -1), backward=False)
    G.assert_within_bounds(errs, "after the timeout")


def test_fault_hook_rejects_unknown_values():
    lib = fa.library()
    assert lib.fa_debug_set_fault(7) == 1
    assert lib.fa_debug_set_fault(-1) == 1
    assert lib.fa_debug_set_fault(0) == 0
