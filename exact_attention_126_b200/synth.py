"""Seeded synthetic inputs for exact attention: the one module both the CUDA path's
callers and the CPU oracle's callers draw their inputs from.

It holds no attention arithmetic: it only turns (seed, element index) into i.i.d.
N(0, 1) values rounded to bf16, so that the GPU kernels and the oracle see the very
same bits.

Generator (all steps are published algorithms, restated here):
  * SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) used in counter mode: the n-th output of a
    SplitMix64 stream seeded with ``s`` is ``mix64(s + (n + 1) * GOLDEN)``,
    so any element can be produced independently of the others.
  * 53-bit uniforms in the open interval (0, 1): ``((x >> 11) + 0.5) * 2**-53``.
  * Box-Muller (Box & Muller 1958): the pair (u1, u2) at indices (2p, 2p+1)
    gives ``sqrt(-2 ln u1) * cos(2 pi u2)`` and ``sqrt(-2 ln u1) * sin(2 pi u2)``.
  * fp64 -> fp32 (round to nearest) -> bf16 (round to nearest even, by torch).

The pages' workloads use i.i.d. normal Q, K, V (and dO for the backward) in the
(batch, heads, seq_len, head_dim) layout; see the page "Flash Attention 3.7 核心原理与实战"
§3.2 for the layout and the page "显存神技：必学FlashAttention！" §三 for the shapes.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

#: tensor ids used in the per-tensor seed
TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}

#: base of the per-config seeds
SEED_BASE = 0x5EED0000


def config_seed(cfg_index: int, tensor: str) -> int:
    """Seed for tensor ``tensor`` of workload ``cfg_index``: 0x5EED0000 + 16*cfg + id."""
    return SEED_BASE + 16 * int(cfg_index) + TENSOR_IDS[tensor]


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 stream seeded with ``seed``."""
    n = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + n * GOLDEN)


def uniform_open(seed: int, start: int, count: int) -> np.ndarray:
    """53-bit uniforms in (0, 1) from the SplitMix64 stream."""
    x = splitmix64(seed, start, count)
    return ((x >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal_f64(seed: int, count: int) -> np.ndarray:
    """``count`` i.i.d. N(0,1) fp64 values (Box-Muller on consecutive uniform pairs)."""
    return _normal_range(seed, 0, count)


def normal_bf16(seed: int, shape, chunk: int = 1 << 21, pin: bool = False) -> torch.Tensor:
    """A host bf16 tensor of i.i.d. N(0,1) values with the given shape (optionally in
    pinned memory). Chunks are generated on a thread pool; the values do not depend on
    the chunking."""
    count = int(np.prod(shape))
    out = torch.empty(count, dtype=torch.bfloat16, pin_memory=pin)
    step = max(2, chunk - chunk % 2)

    def fill(lo):
        # each chunk starts on an even element, so Box-Muller pairs never straddle chunks
        hi = min(count, lo + step)
        vals = _normal_range(seed, lo, hi)
        out[lo:hi] = torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)

    starts = list(range(0, count, step))
    if len(starts) > 1:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    elif starts:
        fill(0)
    return out.view(*shape)


def _normal_range(seed: int, lo: int, hi: int) -> np.ndarray:
    """Elements ``lo .. hi-1`` (lo even) of the normal sequence of ``seed``."""
    assert lo % 2 == 0
    p0, p1 = lo // 2, (hi + 1) // 2
    u = uniform_open(seed, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    t = 2.0 * np.pi * u[:, 1]
    z = np.empty(2 * (p1 - p0), dtype=np.float64)
    z[0::2] = r * np.cos(t)
    z[1::2] = r * np.sin(t)
    return z[: hi - lo]


def normal_bf16_range(seed: int, start: int, count: int) -> torch.Tensor:
    """Elements ``start .. start+count-1`` of the tensor ``normal_bf16(seed, ...)`` would
    produce (``start`` even), as a flat host bf16 tensor."""
    vals = _normal_range(seed, start, start + count)
    return torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16)


def head_inputs(B: int, H: int, N: int, d: int, cfg_index: int, b: int, h: int,
                names=("q", "k", "v", "do")) -> dict:
    """The (N, d) slice of (batch b, head h) of each tensor of ``attention_inputs``,
    without generating the other heads (N * d must be even)."""
    start = (b * H + h) * N * d
    return {n: normal_bf16_range(config_seed(cfg_index, n), start, N * d).view(1, 1, N, d)
            for n in names}


def attention_inputs(B: int, H: int, N: int, d: int, cfg_index: int,
                     with_grad: bool = True, pin: bool = False) -> dict:
    """Host bf16 tensors q, k, v (and do) of shape (B, H, N, d), seeded per workload."""
    names = ["q", "k", "v"] + (["do"] if with_grad else [])
    return {n: normal_bf16(config_seed(cfg_index, n), (B, H, N, d), pin=pin) for n in names}


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16 tensor to a contiguous fp64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).contiguous().numpy()
